// kla_api.cu -- the C ABI of libkla (include/kla.h): descriptor validation,
// work planning, workspace layout and the launch sequence of the forward pass.
//
// Launch sequence of kla_forward for B rows of T tokens split into P segments
// per row (P = 1 when rows x heads already fill the GPU):
//   tensor-core path (bf16, dk and dv in {64, 128}):
//     P = 1:  chunk kernel walking whole rows                       (1 launch)
//     P > 1:  mobius_reduce [-> mobius_carry for long segments]      (lambda at
//             every segment start) -> chunk kernel walking every segment from a
//             zero state -> segment-start beliefs -> correction pass (4 or 5)
//   CUDA-core walk (fp32 inputs, other head dims):
//     P > 1:  mobius_reduce -> mobius_carry -> state walk of segments 0..P-2 ->
//             state carry -> output walk of every segment               (5)
//     P = 1:  output walk                                                (1)
// Packed variable-length sequences (cu_seqlens) are walked whole, longest
// first (one more launch ranks them by length). kla_kdn_forward and
// kla_prologue are one launch each; kla_backward is five (seven isotropic).
// Nothing allocates, nothing synchronises; all work goes on the caller's stream.
#include <cstdlib>
#include <cstring>
#include <cstdint>

#include "kla_internal.cuh"
#include "../../include/kla.h"

namespace kla {

__device__ int g_status = 0;

template <typename TIn>
cudaError_t launch_mobius_reduce(const Plan &, const void *, const float *, const float *,
                                 const float *, float4 *, int *, cudaStream_t);
cudaError_t launch_mobius_carry(const Plan &, const float4 *, const float *, float *, cudaStream_t);
template <typename TIn>
cudaError_t launch_mobius_emit(const Plan &, const int *, const void *, const float *, const float *,
                               const float *, const float *, const float *, float *, cudaStream_t);
cudaError_t launch_walk(const Plan &, const int *, int, const void *, const void *, const void *,
                        const float *, const float *, const float *, const float *, const float *,
                        const float *, float *, float *, void *, float *, float *, cudaStream_t);
cudaError_t launch_state_carry(const Plan &, const float *, const float *, float *, cudaStream_t);
cudaError_t launch_seq_order(const Plan &, const int *, int *, cudaStream_t);
cudaError_t launch_correct(const Plan &, const float *, const float *, void *, float *, int *, cudaStream_t);
bool chunk_tc_supported(const Plan &);
bool kdn_supported(int dk, int dv);
cudaError_t launch_prologue(int H, long long ntok, long long T, const int *cu, int nseq, int dk, int dv, bool iso,
                            bool bf16, int W, const void *xq, const void *xk, const void *xv, const float *xa,
                            const float *xqn, const float *xbeta, const float *wq, const float *wk,
                            const float *wv, const float *bq, const float *bk, const float *bv, void *q, void *k,
                            void *v, float *a, float *qn, float *beta, cudaStream_t st);
bool backward_supported(int dk, int dv);
size_t backward_workspace_bytes(long long ntok, int H, long long units, int dk, bool iso);
cudaError_t launch_backward(int H, long long T, long long ntok, long long units, int dk, int dv, bool iso, bool bf16,
                            const int *cu, const void *q, const void *k, const void *v, const float *a,
                            const float *qn, const float *beta, const float *lambda0, const float *eta0,
                            const void *dout, const float *dfinal_lambda, const float *dfinal_eta, float *dq,
                            float *dk_, float *dv_, float *da, float *dqn, float *dbeta, float *dlambda0,
                            float *deta0, void *ws, cudaStream_t st);
cudaError_t launch_kdn(int H, long long T, long long units, int dk, int dv, bool iso, bool bf16, const int *cu,
                       const void *q, const void *k, const void *v, const float *a, const float *qn,
                       const float *beta, const float *lambda0, const float *M0, void *out, float *final_lambda,
                       float *final_M, cudaStream_t st);
cudaError_t launch_chunk_tc(const Plan &, const int *, int, const void *, const void *, const void *,
                            const float *, const float *, const float *, const float *, const float *,
                            const float *, float *, float *, void *, float *, float *, int *,
                            cudaStream_t);

// Device address of the status word, looked up once per device.
static int *status_ptr() {
    static PerDevice<int *> ptrs;
    const int dev = current_device();
    if (dev < 0) return nullptr;
    int *p = ptrs.v[dev].load(std::memory_order_acquire);
    if (!p) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_status) != cudaSuccess) return nullptr;
        p = (int *)a;
        ptrs.v[dev].store(p, std::memory_order_release);
    }
    return p;
}

static int sm_count() {
    static PerDevice<int> counts;
    const int dev = current_device();
    if (dev < 0) return 148;
    int c = counts.v[dev].load(std::memory_order_acquire);
    if (!c) {
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        counts.v[dev].store(c, std::memory_order_release);
    }
    return c;
}

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static bool pow2_in(int x, int lo, int hi) {
    return x >= lo && x <= hi && (x & (x - 1)) == 0;
}

// Segments per row. The walk kernel keeps one segment per CTA and
// `per_sm` CTAs fit on an SM, so the segment count is the largest that keeps
// every (row, head, segment) unit in one wave: more units would add a partial
// wave, fewer would leave SMs idle. Rows x heads that already occupy half the
// SMs are not split (the Moebius reduce and the correction pass would cost more
// than they gain). KLA_SEGMENTS overrides (tuning only; the result does not depend
// on it beyond rounding).
static int choose_segments(long long units, int NB, int per_sm) {
    const char *env = getenv("KLA_SEGMENTS");
    if (env && *env) {
        int P = atoi(env);
        return P < 1 ? 1 : (P > NB ? NB : P);
    }
    const long long cap = (long long)sm_count() * per_sm;
    if (2 * units >= cap) return 1;
    const long long P = cap / units;
    return (int)(P > NB ? NB : P);
}

// Validates the descriptor and fills the plan. Returns KLA_OK or an error.
static kla_status make_plan(const kla_desc *d, Plan &p, bool precision_only) {
    if (!d) return KLA_ERR_INVALID_ARG;
    if (d->B < 0 || d->T < 0 || d->H <= 0) return KLA_ERR_INVALID_ARG;
    if (!pow2_in(d->dk, 16, 128) || !pow2_in(d->dv, 16, 256)) return KLA_ERR_INVALID_ARG;
    if (d->dtype != KLA_BF16 && d->dtype != KLA_FP32) return KLA_ERR_INVALID_ARG;
    if (d->mode != KLA_DIAG && d->mode != KLA_ISO) return KLA_ERR_INVALID_ARG;
    if (d->cu_seqlens && d->num_seqs < 1) return KLA_ERR_INVALID_ARG;
    std::memset(&p, 0, sizeof(p));
    p.varlen = d->cu_seqlens != nullptr;
    p.N = p.varlen ? d->num_seqs : d->B;
    p.H = d->H; p.dk = d->dk; p.dv = d->dv;
    p.iso = d->mode == KLA_ISO;
    p.nl = p.iso ? 1 : d->dk;
    p.bf16 = d->dtype == KLA_BF16;
    p.T = d->T;
    p.ntok = (long long)d->B * d->T;
    p.sms = sm_count();
    if (p.varlen) {
        p.NB = 1; p.P = 1; p.seg_blocks = 1; p.Lseg = 0;
    } else {
        p.NB = (int)((p.T + kBlockTokens - 1) / kBlockTokens);
        if (p.NB < 1) p.NB = 1;
        // resident walk CTAs per SM: two for the tensor-core walk at dk = dv = 64
        // (its shared memory, TMEM columns and registers fit twice), else one
        const int per_sm = (chunk_tc_supported(p) && p.dk == 64 && p.dv == 64) ? 2 : 1;
        int P = precision_only ? p.NB : choose_segments((long long)p.N * p.H, p.NB, per_sm);
        p.seg_blocks = (p.NB + P - 1) / P;
        p.P = (p.NB + p.seg_blocks - 1) / p.seg_blocks;
        p.Lseg = (long long)p.seg_blocks * kBlockTokens;
    }
    size_t units = (size_t)p.N * p.H;
    size_t off = 0;
    bool scan = !p.varlen && (precision_only || p.P > 1);
    p.off_agg = off;
    if (scan) off += align256(units * p.NB * p.nl * sizeof(float4));
    p.off_lam = off;
    if (scan) off += align256(units * p.NB * p.nl * sizeof(float));
    p.off_dS = off;
    p.off_decay = off;
    if (!precision_only && p.P > 1) {
        off += align256(units * p.P * p.dk * p.dv * sizeof(float));
        p.off_decay = off;
        off += align256(units * p.P * p.nl * sizeof(float));
    }
    // split rows on the tensor-core path: the walk's folded q tiles and the
    // per-chunk factors for the correction pass
    p.local = !precision_only && p.P > 1 && chunk_tc_supported(p);
    p.off_qbuf = off;
    if (p.local) off += align256((size_t)p.ntok * p.H * p.dk * 2);
    p.off_rlog = off;
    if (p.local) off += align256(units * p.NB * kQuarters * p.dk * sizeof(float));
    p.qbuf = nullptr;
    p.rlog = nullptr;
    // longest-first launch order of packed sequences (list scheduling of the
    // walks: the long ones start first, the short ones fill in behind them)
    p.order = !precision_only && p.varlen && p.N >= 2 && p.N <= kMaxOrderSeqs;
    p.off_perm = off;
    if (p.order) off += align256((size_t)p.N * sizeof(int));
    p.perm = nullptr;
    p.inline_carry = false;
    p.agg = nullptr;
    p.bytes = off;
    return KLA_OK;
}

static bool aligned16(const void *x) { return ((uintptr_t)x & 15) == 0; }
static bool aligned4(const void *x) { return ((uintptr_t)x & 3) == 0; }
static bool ok_opt(const void *x) { return x == nullptr || aligned16(x); }
static bool ok_opt4(const void *x) { return x == nullptr || aligned4(x); }

static kla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA; }

}  // namespace kla

using namespace kla;

extern "C" {

const char *kla_status_string(kla_status s) {
    switch (s) {
        case KLA_OK: return "ok";
        case KLA_ERR_INVALID_ARG: return "invalid argument (shape, null or misaligned pointer, workspace)";
        case KLA_ERR_UNSUPPORTED: return "unsupported configuration";
        case KLA_ERR_CUDA: return "CUDA error";
        case KLA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case KLA_ERR_RANGE: return "in-chunk log-gate span exceeded the representable range";
    }
    return "unknown status";
}

int kla_version(void) { return 100; }

size_t kla_workspace_bytes(const kla_desc *d) {
    Plan p;
    if (make_plan(d, p, false) != KLA_OK) return 0;
    return p.bytes;
}

size_t kla_precision_workspace_bytes(const kla_desc *d) {
    Plan p;
    if (make_plan(d, p, true) != KLA_OK) return 0;
    return p.bytes;
}

static kla_status forward_impl(const kla_desc *d, const void *q, const void *k, const void *v,
                               const float *a, const float *qn, const float *beta,
                               const float *lambda0, const float *eta0, void *out,
                               float *final_lambda, float *final_eta, void *ws, size_t ws_bytes,
                               cudaStream_t st, cudaEvent_t *ev) {
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    long long ntok = (long long)d->B * d->T;
    if (ntok == 0 && !p.varlen) return KLA_OK;
    if (!q || !k || !v || !a || !qn || !beta || !out) return KLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(qn) ||
        !aligned4(beta) || !aligned16(out) || !ok_opt4(lambda0) || !ok_opt(eta0) ||
        !ok_opt4(final_lambda) || !ok_opt(final_eta))
        return KLA_ERR_INVALID_ARG;
    if (p.bytes > 0 && (!ws || ((uintptr_t)ws & 255) || ws_bytes < p.bytes)) return KLA_ERR_INVALID_ARG;
    char *w = (char *)ws;
    float4 *agg = (float4 *)(w + p.off_agg);
    float *lam_blk = (float *)(w + p.off_lam);
    float *S_io = (float *)(w + p.off_dS);
    float *decay = (float *)(w + p.off_decay);
    const int *cu = d->cu_seqlens;
    int *status = status_ptr();
    if (!status) return KLA_ERR_CUDA;
    const bool tc = chunk_tc_supported(p);
    cudaError_t e = cudaSuccess;
    auto mark = [&](int i) {
        if (ev && e == cudaSuccess) e = cudaEventRecord(ev[i], st);
    };
    mark(0);
    if (p.order) {
        int *perm = (int *)(w + p.off_perm);
        e = launch_seq_order(p, cu, perm, st);
        p.perm = perm;
    }
    if (e == cudaSuccess && p.P > 1) {
        e = p.bf16 ? launch_mobius_reduce<__nv_bfloat16>(p, k, a, qn, beta, agg, status, st)
                   : launch_mobius_reduce<float>(p, k, a, qn, beta, agg, status, st);
        mark(1);
        // short segments: the tensor-core kernel composes the block aggregates itself
        p.inline_carry = tc && (long long)(p.P - 1) * p.seg_blocks <= kInlineCarryBlocks;
        p.agg = agg;
        if (e == cudaSuccess && !p.inline_carry) e = launch_mobius_carry(p, agg, lambda0, lam_blk, st);
        mark(2);
        if (p.local) {
            // tensor-core path: every segment walks from a zero state (segment 0
            // from eta0) and exports its transfer, gate product, folded q tiles
            // and chunk factors; the correction pass then adds the carried state
            p.qbuf = w + p.off_qbuf;
            p.rlog = (float *)(w + p.off_rlog);
            mark(3);
            mark(4);
            if (e == cudaSuccess)
                e = launch_chunk_tc(p, cu, 2, q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay, out,
                                    final_lambda, final_eta, status, st);
            mark(5);
            if (e == cudaSuccess) e = launch_correct(p, S_io, decay, out, final_eta, status, st);
            mark(6);
            return cuda_status(e);
        }
        if (e == cudaSuccess)
            e = launch_walk(p, cu, 1, q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay, out, final_lambda,
                            final_eta, st);
        mark(3);
        if (e == cudaSuccess) e = launch_state_carry(p, eta0, decay, S_io, st);
        mark(4);
    } else {
        mark(1); mark(2); mark(3); mark(4);
    }
    if (e == cudaSuccess)
        e = tc ? launch_chunk_tc(p, cu, 0, q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay,
                                 out, final_lambda, final_eta, status, st)
               : launch_walk(p, cu, 0, q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay,
                             out, final_lambda, final_eta, st);
    mark(5);
    mark(6);
    return cuda_status(e);
}

kla_status kla_forward(const kla_desc *d, const void *q, const void *k, const void *v,
                       const float *a, const float *qn, const float *beta,
                       const float *lambda0, const float *eta0, void *out,
                       float *final_lambda, float *final_eta, void *ws, size_t ws_bytes,
                       cudaStream_t st) {
    return forward_impl(d, q, k, v, a, qn, beta, lambda0, eta0, out, final_lambda, final_eta, ws,
                        ws_bytes, st, nullptr);
}

kla_status kla_forward_profiled(const kla_desc *d, const void *q, const void *k, const void *v,
                                const float *a, const float *qn, const float *beta,
                                const float *lambda0, const float *eta0, void *out,
                                float *final_lambda, float *final_eta, void *ws, size_t ws_bytes,
                                cudaStream_t st, cudaEvent_t *events) {
    if (!events) return KLA_ERR_INVALID_ARG;
    for (int i = 0; i < 7; ++i)
        if (!events[i]) return KLA_ERR_INVALID_ARG;
    return forward_impl(d, q, k, v, a, qn, beta, lambda0, eta0, out, final_lambda, final_eta, ws,
                        ws_bytes, st, events);
}

kla_status kla_kdn_forward(const kla_desc *d, const void *q, const void *k, const void *v,
                           const float *a, const float *qn, const float *beta, const float *lambda0,
                           const float *M0, void *out, float *final_lambda, float *final_M,
                           cudaStream_t st) {
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    if (!kdn_supported(p.dk, p.dv)) return KLA_ERR_UNSUPPORTED;
    if (p.ntok == 0 && !p.varlen) return KLA_OK;
    if (!q || !k || !v || !a || !qn || !beta || !out) return KLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(qn) ||
        !aligned4(beta) || !aligned16(out) || !aligned4(lambda0) || !aligned16(M0) ||
        !aligned4(final_lambda) || !aligned16(final_M))
        return KLA_ERR_INVALID_ARG;
    return cuda_status(launch_kdn(p.H, p.T, (long long)p.N * p.H, p.dk, p.dv, p.iso, p.bf16,
                                  p.varlen ? d->cu_seqlens : nullptr, q, k, v, a, qn, beta, lambda0, M0,
                                  out, final_lambda, final_M, st));
}

kla_status kla_prologue(const kla_desc *d, int conv_width, const void *xq, const void *xk, const void *xv,
                        const float *xa, const float *xqn, const float *xbeta, const float *wq,
                        const float *wk, const float *wv, const float *bq, const float *bk, const float *bv,
                        void *q, void *k, void *v, float *a, float *qn, float *beta, cudaStream_t st) {
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    if (conv_width < 1 || conv_width > 4) return KLA_ERR_INVALID_ARG;
    if (!wq || !wk || !wv) return KLA_ERR_INVALID_ARG;
    if (p.ntok == 0 && !p.varlen) return KLA_OK;
    if (!xq || !xk || !xv || !xa || !xqn || !xbeta || !q || !k || !v || !a || !qn || !beta)
        return KLA_ERR_INVALID_ARG;
    // rows move as vectors: 16-byte aligned tensors; weights, biases and beta 4-byte
    const void *vec[] = {xq, xk, xv, xa, xqn, q, k, v, a, qn};
    for (const void *x : vec)
        if (!aligned16(x)) return KLA_ERR_INVALID_ARG;
    const void *sca[] = {xbeta, beta, wq, wk, wv, bq, bk, bv};
    for (const void *x : sca)
        if (!aligned4(x)) return KLA_ERR_INVALID_ARG;
    const long long ntok = p.varlen ? -1 : p.ntok;
    return cuda_status(launch_prologue(p.H, ntok < 0 ? (long long)d->B * d->T : ntok, p.T,
                                       p.varlen ? d->cu_seqlens : nullptr, p.N, p.dk, p.dv, p.iso, p.bf16,
                                       conv_width, xq, xk, xv, xa, xqn, xbeta, wq, wk, wv, bq, bk, bv, q, k, v, a,
                                       qn, beta, st));
}

size_t kla_backward_workspace_bytes(const kla_desc *d) {
    Plan p;
    if (make_plan(d, p, false) != KLA_OK || !backward_supported(p.dk, p.dv)) return 0;
    return backward_workspace_bytes((long long)d->B * d->T, p.H, (long long)p.N * p.H, p.dk, p.iso);
}

kla_status kla_backward(const kla_desc *d, const void *q, const void *k, const void *v, const float *a,
                        const float *qn, const float *beta, const float *lambda0, const float *eta0,
                        const void *dout, const float *dfinal_lambda, const float *dfinal_eta, float *dq,
                        float *dk, float *dv, float *da, float *dqn, float *dbeta, float *dlambda0, float *deta0,
                        void *workspace, size_t workspace_bytes, cudaStream_t st) {
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    if (!backward_supported(p.dk, p.dv)) return KLA_ERR_UNSUPPORTED;
    const long long ntok = (long long)d->B * d->T;
    if (ntok == 0 && !p.varlen) return KLA_OK;
    if (!q || !k || !v || !a || !qn || !beta || !dout || !dq || !dk || !dv || !da || !dqn || !dbeta)
        return KLA_ERR_INVALID_ARG;
    // rows of q, k, v, dout move as 16-byte vectors; everything else is read per element
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(workspace))
        return KLA_ERR_INVALID_ARG;
    const void *sca[] = {a, qn, beta, lambda0, eta0, dfinal_lambda, dfinal_eta, dq, dk, dv, da, dqn, dbeta,
                         dlambda0, deta0};
    for (const void *x : sca)
        if (!aligned4(x)) return KLA_ERR_INVALID_ARG;
    const size_t need = backward_workspace_bytes(ntok, p.H, (long long)p.N * p.H, p.dk, p.iso);
    if (!workspace || workspace_bytes < need) return KLA_ERR_INVALID_ARG;
    return cuda_status(launch_backward(p.H, p.T, ntok, (long long)p.N * p.H, p.dk, p.dv, p.iso, p.bf16,
                                       p.varlen ? d->cu_seqlens : nullptr, q, k, v, a, qn, beta, lambda0, eta0,
                                       dout, dfinal_lambda, dfinal_eta, dq, dk, dv, da, dqn, dbeta, dlambda0, deta0,
                                       workspace, st));
}

kla_status kla_plan(const kla_desc *d, int *segments_per_row, int *launches, int *tensor_core) {
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    if (segments_per_row) *segments_per_row = p.P;
    int n = 1;
    if (p.P > 1) {
        const bool tc = chunk_tc_supported(p);
        // tensor cores: reduce, [carry], chunk kernel, segment starts, correction;
        // CUDA cores: reduce, carry, state walk, state carry, output walk
        n = tc ? ((long long)(p.P - 1) * p.seg_blocks <= kInlineCarryBlocks ? 4 : 5) : 5;
    }
    if (launches) *launches = n + (p.order ? 1 : 0);
    if (tensor_core) *tensor_core = chunk_tc_supported(p) ? 1 : 0;
    return KLA_OK;
}

kla_status kla_precision(const kla_desc *d, const void *k, const float *a, const float *qn,
                         const float *beta, const float *lambda0, float *lambda_out, void *ws,
                         size_t ws_bytes, cudaStream_t st) {
    Plan p;
    kla_status s = make_plan(d, p, true);
    if (s != KLA_OK) return s;
    long long ntok = (long long)d->B * d->T;
    if (ntok == 0 && !p.varlen) return KLA_OK;
    if (!k || !a || !qn || !beta || !lambda_out) return KLA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(a) || !aligned16(qn) || !aligned4(beta) ||
        !aligned16(lambda_out) || !ok_opt4(lambda0))
        return KLA_ERR_INVALID_ARG;
    if (p.bytes > 0 && (!ws || ((uintptr_t)ws & 255) || ws_bytes < p.bytes)) return KLA_ERR_INVALID_ARG;
    char *w = (char *)ws;
    float4 *agg = (float4 *)(w + p.off_agg);
    float *lam_blk = (float *)(w + p.off_lam);
    int *status = status_ptr();
    if (!status) return KLA_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (!p.varlen) {
        e = p.bf16 ? launch_mobius_reduce<__nv_bfloat16>(p, k, a, qn, beta, agg, status, st)
                   : launch_mobius_reduce<float>(p, k, a, qn, beta, agg, status, st);
        if (e == cudaSuccess) e = launch_mobius_carry(p, agg, lambda0, lam_blk, st);
    }
    if (e == cudaSuccess)
        e = p.bf16 ? launch_mobius_emit<__nv_bfloat16>(p, d->cu_seqlens, k, a, qn, beta, lam_blk, lambda0,
                                                       lambda_out, st)
                   : launch_mobius_emit<float>(p, d->cu_seqlens, k, a, qn, beta, lam_blk, lambda0,
                                               lambda_out, st);
    return cuda_status(e);
}

kla_status kla_decode_step(const kla_desc *d, const void *q, const void *k, const void *v,
                           const float *a, const float *qn, const float *beta, float *lambda,
                           float *eta, void *out, cudaStream_t st) {
    if (!d || d->T != 1 || d->cu_seqlens) return KLA_ERR_INVALID_ARG;
    if (!lambda || !eta) return KLA_ERR_INVALID_ARG;
    Plan p;
    kla_status s = make_plan(d, p, false);
    if (s != KLA_OK) return s;
    if (d->B == 0) return KLA_OK;
    if (!q || !k || !v || !a || !qn || !beta || !out) return KLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(qn) ||
        !aligned4(beta) || !aligned16(out) || !aligned4(lambda) || !aligned16(eta))
        return KLA_ERR_INVALID_ARG;
    // One token per row: a single segment; the walk reads the belief before it
    // writes it, so the state may be updated in place.
    return cuda_status(launch_walk(p, nullptr, 0, q, k, v, a, qn, beta, lambda, eta, nullptr, nullptr,
                                   nullptr, out, lambda, eta, st));
}

// ---- host-buffer variant ---------------------------------------------------

struct HostLayout {
    size_t q, k, v, a, qn, beta, lam0, eta0, cu, out, flam, feta, ws, total;
    size_t qk_b, v_b, ab, b_b, lam_b, eta_b, cu_b;
};

static bool host_layout(const kla_desc *d, HostLayout &L) {
    Plan p;
    if (make_plan(d, p, false) != KLA_OK) return false;
    size_t es = p.bf16 ? 2 : 4;
    size_t ntok = (size_t)d->B * d->T;
    size_t units = (size_t)p.N * p.H;
    L.qk_b = ntok * p.H * p.dk * es;
    L.v_b = ntok * p.H * p.dv * es;
    L.ab = ntok * p.H * p.nl * 4;
    L.b_b = ntok * p.H * 4;
    L.lam_b = units * p.nl * 4;
    L.eta_b = units * p.dk * p.dv * 4;
    L.cu_b = p.varlen ? (size_t)(p.N + 1) * 4 : 0;
    size_t off = 0;
    auto put = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
    L.q = put(L.qk_b); L.k = put(L.qk_b); L.v = put(L.v_b);
    L.a = put(L.ab); L.qn = put(L.ab); L.beta = put(L.b_b);
    L.lam0 = put(L.lam_b); L.eta0 = put(L.eta_b); L.cu = put(L.cu_b);
    L.out = put(L.v_b); L.flam = put(L.lam_b); L.feta = put(L.eta_b);
    L.ws = put(p.bytes);
    L.total = off;
    return true;
}

size_t kla_host_device_bytes(const kla_desc *d) {
    HostLayout L;
    return host_layout(d, L) ? L.total : 0;
}

kla_status kla_forward_host(const kla_desc *d, const void *q, const void *k, const void *v,
                            const float *a, const float *qn, const float *beta,
                            const float *lambda0, const float *eta0, void *out,
                            float *final_lambda, float *final_eta, void *dbuf, size_t dbytes,
                            cudaStream_t st) {
    HostLayout L;
    if (!host_layout(d, L)) return KLA_ERR_INVALID_ARG;
    if (!q || !k || !v || !a || !qn || !beta || !out) return KLA_ERR_INVALID_ARG;
    if (!dbuf || ((uintptr_t)dbuf & 255) || dbytes < L.total) return KLA_ERR_INVALID_ARG;
    char *b = (char *)dbuf;
    kla_desc dd = *d;
    cudaError_t e = cudaSuccess;
    auto h2d = [&](size_t off, const void *src, size_t n) {
        if (e == cudaSuccess && n) e = cudaMemcpyAsync(b + off, src, n, cudaMemcpyHostToDevice, st);
    };
    h2d(L.q, q, L.qk_b); h2d(L.k, k, L.qk_b); h2d(L.v, v, L.v_b);
    h2d(L.a, a, L.ab); h2d(L.qn, qn, L.ab); h2d(L.beta, beta, L.b_b);
    if (lambda0) h2d(L.lam0, lambda0, L.lam_b);
    if (eta0) h2d(L.eta0, eta0, L.eta_b);
    if (d->cu_seqlens) { h2d(L.cu, d->cu_seqlens, L.cu_b); dd.cu_seqlens = (const int *)(b + L.cu); }
    if (e != cudaSuccess) return KLA_ERR_CUDA;
    kla_status s = kla_forward(&dd, b + L.q, b + L.k, b + L.v, (const float *)(b + L.a),
                               (const float *)(b + L.qn), (const float *)(b + L.beta),
                               lambda0 ? (const float *)(b + L.lam0) : nullptr,
                               eta0 ? (const float *)(b + L.eta0) : nullptr, b + L.out,
                               final_lambda ? (float *)(b + L.flam) : nullptr,
                               final_eta ? (float *)(b + L.feta) : nullptr, b + L.ws,
                               dbytes - L.ws, st);
    if (s != KLA_OK) return s;
    auto d2h = [&](void *dst, size_t off, size_t n) {
        if (e == cudaSuccess && n) e = cudaMemcpyAsync(dst, b + off, n, cudaMemcpyDeviceToHost, st);
    };
    d2h(out, L.out, L.v_b);
    if (final_lambda) d2h(final_lambda, L.flam, L.lam_b);
    if (final_eta) d2h(final_eta, L.feta, L.eta_b);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}

kla_status kla_check(cudaStream_t st) {
    if (cudaStreamSynchronize(st) != cudaSuccess) return KLA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return KLA_ERR_CUDA;
    if (v) {
        int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return KLA_ERR_CUDA;
    }
    if (v & kStatusTimeout) return KLA_ERR_TIMEOUT;
    if (v & kStatusRange) return KLA_ERR_RANGE;
    return KLA_OK;
}

}  // extern "C"
