// kla_prologue.cu -- the mixer's input prologue, fused in one pass (sm_100a):
// a depthwise causal 1-D convolution and SiLU of the q, k, v pre-activations,
// the L2 norm of q and k over dk, and the sigmoid / softplus gate activations
// (Kalman Linear Attention, technical summary section 4: a Mamba-like block
// with a 1-D causal convolution and SiLU in front of the mixer):
//   q = l2norm(silu(conv(xq))), k = l2norm(silu(conv(xk))), v = silu(conv(xv)),
//   a = sigmoid(xa), qn = softplus(xqn), beta = sigmoid(xbeta),
//   conv: y[t,c] = b[c] + sum_{w<W} wgt[c,w] x[t-(W-1)+w, c], x = 0 before the
//   start of t's sequence; l2norm: y / sqrt(sum_c y^2 + 1e-6).
// The outputs are the forward pass's inputs in its layouts, so the mixer reads
// them without another conversion pass.
//
// CTA = 32 tokens of one head, 8 warps of 4 consecutive tokens; a lane covers
// dk / 32 (dv / 32) channels and keeps their conv taps in registers. Inputs are
// read once from HBM: the three earlier rows a token's taps reach are the rows
// the warp (or the warp before it) has just read, served from L1/L2.
#include "kla_internal.cuh"

namespace kla {

namespace {

constexpr int kProTok = 32;      // tokens per CTA
constexpr int kProMaxW = 4;      // widest convolution
constexpr float kProEps = 1e-6f;

struct ProArgs {
    int H, W;
    long long ntok, T;
    const int *cu;
    int nseq;
    const void *xq, *xk, *xv;
    const float *xa, *xqn, *xbeta;
    const float *wq, *wk, *wv, *bq, *bk, *bv;
    void *q, *k, *v;
    float *a, *qn, *beta;
};

template <typename T>
__device__ __forceinline__ float ld1(const T *p, long long i);
template <>
__device__ __forceinline__ float ld1<float>(const float *p, long long i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void st1(T *p, long long i, float x);
template <>
__device__ __forceinline__ void st1<float>(float *p, long long i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float silu(float y) { return y / (1.f + __expf(-y)); }
__device__ __forceinline__ float sigm(float y) { return 1.f / (1.f + __expf(-y)); }
__device__ __forceinline__ float softplus(float y) { return log1pf(__expf(-fabsf(y))) + fmaxf(y, 0.f); }

// First token of the sequence that holds token t.
__device__ __forceinline__ long long seq_start(const ProArgs &g, long long t) {
    if (!g.cu) return (t / g.T) * g.T;
    int lo = 0, hi = g.nseq;   // cu[lo] <= t < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (g.cu[mid] <= t) lo = mid; else hi = mid;
    }
    return g.cu[lo];
}

// conv + SiLU of the C channels of row (t, h) this lane covers (CPL per lane),
// optional L2 norm across the warp; writes the bf16 / fp32 outputs.
template <int D, bool NORM, typename T>
__device__ __forceinline__ void conv_row(const T *x, const float *wgt, const float *bias, T *y, const ProArgs &g,
                                         long long t, long long s0, int h, int lane) {
    constexpr int CPL = (D + 31) / 32;
    float acc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int ch = lane * CPL + c;
        acc[c] = (ch < D && bias) ? __ldg(bias + h * D + ch) : 0.f;
    }
#pragma unroll
    for (int w = 0; w < kProMaxW; ++w) {
        if (w >= g.W) break;
        const long long src = t - (g.W - 1) + w;
        if (src < s0) continue;
        const long long row = (src * g.H + h) * D;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int ch = lane * CPL + c;
            if (ch < D) acc[c] = fmaf(__ldg(wgt + ((long long)h * D + ch) * g.W + w), ld1<T>(x, row + ch), acc[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = silu(acc[c]);
    float scale = 1.f;
    if (NORM) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            if (lane * CPL + c < D) ss = fmaf(acc[c], acc[c], ss);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);
        scale = rsqrtf(ss + kProEps);
    }
    const long long orow = (t * g.H + h) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int ch = lane * CPL + c;
        if (ch < D) st1<T>(y, orow + ch, acc[c] * scale);
    }
}

template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(256) prologue_kernel(const ProArgs g) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const long long tbase = (long long)blockIdx.x * kProTok + warp * (kProTok / 8);
    for (int x = 0; x < kProTok / 8; ++x) {
        const long long t = tbase + x;
        if (t >= g.ntok) break;
        const long long s0 = seq_start(g, t);
        conv_row<DK, true, T>(static_cast<const T *>(g.xq), g.wq, g.bq, static_cast<T *>(g.q), g, t, s0, h, lane);
        conv_row<DK, true, T>(static_cast<const T *>(g.xk), g.wk, g.bk, static_cast<T *>(g.k), g, t, s0, h, lane);
        conv_row<DV, false, T>(static_cast<const T *>(g.xv), g.wv, g.bv, static_cast<T *>(g.v), g, t, s0, h, lane);
        const long long th = t * g.H + h;
        if (ISO) {
            if (lane == 0) {
                g.a[th] = sigm(__ldg(g.xa + th));
                g.qn[th] = softplus(__ldg(g.xqn + th));
            }
        } else {
            for (int c = lane; c < DK; c += 32) {
                g.a[th * DK + c] = sigm(__ldg(g.xa + th * DK + c));
                g.qn[th * DK + c] = softplus(__ldg(g.xqn + th * DK + c));
            }
        }
        if (lane == 0) g.beta[th] = sigm(__ldg(g.xbeta + th));
    }
}

template <int DK, int DV, bool ISO, typename T>
cudaError_t launch_pro_t(const ProArgs &g, cudaStream_t st) {
    dim3 grid((unsigned)((g.ntok + kProTok - 1) / kProTok), (unsigned)g.H);
    prologue_kernel<DK, DV, ISO, T><<<grid, 256, 0, st>>>(g);
    return cudaGetLastError();
}

template <int DK, int DV, typename T>
cudaError_t launch_pro_iso(bool iso, const ProArgs &g, cudaStream_t st) {
    return iso ? launch_pro_t<DK, DV, true, T>(g, st) : launch_pro_t<DK, DV, false, T>(g, st);
}

template <int DK, typename T>
cudaError_t launch_pro_dv(int dv, bool iso, const ProArgs &g, cudaStream_t st) {
    switch (dv) {
        case 16: return launch_pro_iso<DK, 16, T>(iso, g, st);
        case 32: return launch_pro_iso<DK, 32, T>(iso, g, st);
        case 64: return launch_pro_iso<DK, 64, T>(iso, g, st);
        case 128: return launch_pro_iso<DK, 128, T>(iso, g, st);
        case 256: return launch_pro_iso<DK, 256, T>(iso, g, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_pro_dk(int dk, int dv, bool iso, const ProArgs &g, cudaStream_t st) {
    switch (dk) {
        case 16: return launch_pro_dv<16, T>(dv, iso, g, st);
        case 32: return launch_pro_dv<32, T>(dv, iso, g, st);
        case 64: return launch_pro_dv<64, T>(dv, iso, g, st);
        case 128: return launch_pro_dv<128, T>(dv, iso, g, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_prologue(int H, long long ntok, long long T, const int *cu, int nseq, int dk, int dv, bool iso,
                            bool bf16, int W, const void *xq, const void *xk, const void *xv, const float *xa,
                            const float *xqn, const float *xbeta, const float *wq, const float *wk,
                            const float *wv, const float *bq, const float *bk, const float *bv, void *q, void *k,
                            void *v, float *a, float *qn, float *beta, cudaStream_t st) {
    if (ntok == 0) return cudaSuccess;
    ProArgs g;
    g.H = H; g.W = W; g.ntok = ntok; g.T = T; g.cu = cu; g.nseq = nseq;
    g.xq = xq; g.xk = xk; g.xv = xv; g.xa = xa; g.xqn = xqn; g.xbeta = xbeta;
    g.wq = wq; g.wk = wk; g.wv = wv; g.bq = bq; g.bk = bk; g.bv = bv;
    g.q = q; g.k = k; g.v = v; g.a = a; g.qn = qn; g.beta = beta;
    return bf16 ? launch_pro_dk<__nv_bfloat16>(dk, dv, iso, g, st) : launch_pro_dk<float>(dk, dv, iso, g, st);
}

}  // namespace kla
