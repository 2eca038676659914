// kla_internal.cuh -- shared definitions of the libkla CUDA sources (sm_100a).
//
// Indexing conventions (all row-major, tokens flattened over the batch):
//   token-head index  th = tok * H + h
//   q, k  [th * dk + i]      v, out [th * dv + j]
//   a, qn [th * dk + i]  (iso: [th])      beta [th]
//   per-unit state: unit u = n * H + h  (n = batch row or packed sequence)
//
// A "segment" is a contiguous run of tokens of one (row, head) that one CTA
// walks; a "block" is the granule of the Moebius reduction (Lb tokens). Both
// start at row starts; segments are whole numbers of blocks.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace kla {

constexpr int kBlockTokens = 64;   // Lb: tokens per Moebius-reduction block (one chunk)
constexpr int kChunk = 64;         // C: tokens per chunk of the chunked form
constexpr int kMaxOrderSeqs = 1024; // packed sequences ranked by length for the launch order
constexpr int kInlineCarryBlocks = 64; // at most this many blocks before a segment: carry in the walk kernel
constexpr int kQuarters = 4;       // pass quarters per chunk: the chunk kernel's finest reference granularity
                                   // (16 tokens, the token step of its tensor-core contractions)
constexpr int kMaxDevices = 64;

// Host state kept once per device (symbol addresses, function attributes).
// Entries are atomics, so first calls that race from several host threads
// store the same value without a data race.
template <typename T>
struct PerDevice {
    std::atomic<T> v[kMaxDevices];
    PerDevice() {
        for (auto &x : v) x.store(T{}, std::memory_order_relaxed);
    }
};

// The current device, or -1 if there is none or its index is out of range.
inline int current_device() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
    return d;
}

// Sets the dynamic shared-memory limit of `kern` once per device.
template <typename K>
inline cudaError_t ensure_smem_attr(PerDevice<bool> &done, K kern, int bytes) {
    const int dev = current_device();
    if (dev >= 0 && done.v[dev].load(std::memory_order_acquire)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0) done.v[dev].store(true, std::memory_order_release);
    return e;
}

// Bits of the library's device status word (kla_check reads and clears it);
// kernels that can detect an error receive its address and OR a bit into it.
enum : int { kStatusRange = 1, kStatusTimeout = 2 };

struct Plan {
    int N;          // rows (or packed sequences)
    int H, dk, dv;
    int nl;         // precisions per (row, head): dk (diag) or 1 (iso)
    bool iso, varlen, bf16;
    long long T;    // tokens per row (non-varlen)
    long long ntok; // tokens in the flattened axis (B*T)
    int NB;         // Moebius blocks per row (non-varlen)
    int P;          // segments per row (1 for varlen)
    int seg_blocks; // blocks per segment
    int sms;        // SMs of the current device
    long long Lseg; // tokens per segment (seg_blocks * kBlockTokens)
    // workspace layout (byte offsets; all 256-byte aligned)
    size_t off_agg, off_lam, off_dS, off_decay, bytes;
    // packed sequences: longest-first launch order (int per sequence, in the
    // workspace at off_perm) when `order`; perm is its device address once the
    // workspace is known, else nullptr (launch in sequence order)
    bool order;
    size_t off_perm;
    const int *perm;
    // segment-start precision composed inside the walk kernel from the block
    // aggregates at agg (short segments), instead of a separate carry launch
    bool inline_carry;
    const float4 *agg;
    // split rows on the tensor-core path: segments walk from a zero state and a
    // correction pass adds the carried state; the walk exports its folded q
    // tiles (qbuf [Ntok, H, dk] bf16) and the log2 reference of every pass
    // quarter of every chunk (rlog [N*H][NB][kQuarters][dk] fp32), in the
    // workspace at off_qbuf / off_rlog
    bool local;
    size_t off_qbuf, off_rlog;
    void *qbuf;
    float *rlog;
};

__device__ __forceinline__ float ld_in(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ void st_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Four consecutive input values as float (16-byte fp32 or 8-byte bf16 loads).
__device__ __forceinline__ float4 ld4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
    uint2 r = __ldg(reinterpret_cast<const uint2 *>(p));
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&r.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&r.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

// 3-D TMA tensor map over [ntok][H][inner] (inner contiguous) with box
// (box_inner, 1, box_rows); false if the driver entry point or the encoding fails.
bool make_tma_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int inner, int H,
                  long long ntok, int box_inner, int box_rows, bool swizzle);

// 2x2 Moebius matrix (m00, m01, m10, m11) acting as x -> (m00 x + m01)/(m10 x + m11).
struct Mob { float m00, m01, m10, m11; };

// One predict+update step: lambda' = lambda/(a^2 + qn*lambda) + b
//   = ((1 + b qn) lambda + b a^2) / (qn lambda + a^2).
__device__ __forceinline__ Mob mob_step(float a, float qn, float b) {
    float a2 = a * a;
    return Mob{fmaf(b, qn, 1.0f), b * a2, qn, a2};
}

// L * R : apply R first, then L.
__device__ __forceinline__ Mob mob_mul(const Mob &L, const Mob &R) {
    return Mob{fmaf(L.m00, R.m00, L.m01 * R.m10), fmaf(L.m00, R.m01, L.m01 * R.m11),
               fmaf(L.m10, R.m00, L.m11 * R.m10), fmaf(L.m10, R.m01, L.m11 * R.m11)};
}

// Rescale by an exact power of two so the largest entry is in [1, 2): the map is
// projective, so this changes nothing but keeps the entries inside fp32 range.
__device__ __forceinline__ Mob mob_norm(const Mob &M) {
    float mx = fmaxf(fmaxf(M.m00, M.m01), fmaxf(M.m10, M.m11));
    int e = ((__float_as_int(mx) >> 23) & 0xff) - 127;
    e = max(-126, min(126, e));
    float s = __int_as_float((127 - e) << 23);
    return Mob{M.m00 * s, M.m01 * s, M.m10 * s, M.m11 * s};
}

__device__ __forceinline__ float mob_apply(const Mob &M, float x) {
    return fmaf(M.m00, x, M.m01) / fmaf(M.m10, x, M.m11);
}

// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialization, so it may start while the kernel before
// it in the stream is still running. Each kernel therefore
//  * calls pdl_wait() before its first global-memory access (read or write):
//    it returns once the preceding grid has completed and its writes are
//    visible, so the data dependences are those of plain stream order;
//  * calls pdl_release() once it holds every on-chip resource it will take
//    (after its tensor-memory allocation): the next kernel's CTAs may become
//    resident from then on and run their prologue (barrier setup, tensor-map
//    prefetch, tensor-memory allocation) under this kernel's tail. Releasing
//    only after the allocation means a waiting dependent can never hold
//    tensor memory that a CTA of this grid still needs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches `kern` on `st` with programmatic stream serialization (see above).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace kla
