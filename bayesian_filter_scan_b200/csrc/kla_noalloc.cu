// kla_noalloc.cu -- kla_forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// code inside a custom allocator or memory-pool callback, plug-ins whose host
// framework owns every device allocation, or tightly budgeted inference
// processes that must not grow their footprint after start-up. They still own
// their inputs and outputs, but cannot provide the workspace that long rows
// split into segments need. This entry point takes that workspace from a
// file-scope device array instead, reserved once per GPU when the library's
// device code for this file is loaded and held until the process exits.
#include "kla_internal.cuh"
#include "../../include/kla.h"

namespace {

// The fixed scratch area (32 MiB per device).
__device__ __align__(256) unsigned char g_noalloc_scratch[KLA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array, looked up once per device. In host code
// the array's name is only a host-side stand-in, so its device address must be
// taken with cudaGetSymbolAddress while that device is current.
void *scratch_address() {
    static kla::PerDevice<void *> addr;
    const int dev = kla::current_device();
    if (dev < 0) return nullptr;
    void *p = addr.v[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr.v[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" kla_status kla_forward_noalloc(const kla_desc *desc, const void *q, const void *k, const void *v,
                                          const float *a, const float *qn, const float *beta,
                                          const float *lambda0, const float *eta0, void *out,
                                          float *final_lambda, float *final_eta, cudaStream_t stream) {
    if (!desc) return KLA_ERR_INVALID_ARG;
    const size_t need = kla_workspace_bytes(desc);
    if (need > (size_t)KLA_NOALLOC_SCRATCH_BYTES) return KLA_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        ws = scratch_address();
        if (!ws) return KLA_ERR_CUDA;
    }
    return kla_forward(desc, q, k, v, a, qn, beta, lambda0, eta0, out, final_lambda, final_eta, ws,
                       (size_t)KLA_NOALLOC_SCRATCH_BYTES, stream);
}
