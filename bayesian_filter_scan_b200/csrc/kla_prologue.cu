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
// CTA = 128 tokens of one head and one role (q, k, v, or the gates), 8 warps of
// 16 consecutive tokens; a lane covers dk / 32 (dv / 32) contiguous channels,
// keeps their conv taps in registers and slides a window of the last W - 1
// rows along its tokens, so every input row is read once (plus a 3-row halo per
// warp); a window is cleared where a new row or packed sequence starts. Rows
// move as one vector per lane and are loaded one token ahead.
#include "kla_internal.cuh"

namespace kla {

namespace {

constexpr int kProWarpTok = 16;  // tokens per warp
constexpr int kProTok = 8 * kProWarpTok;   // tokens per CTA
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

// N contiguous values (N = 1, 2, 4) as one vector access
template <int N, typename T>
__device__ __forceinline__ void ldv(const T *p, float (&x)[N]);
template <int N, typename T>
__device__ __forceinline__ void stv(T *p, const float (&x)[N]);
template <>
__device__ __forceinline__ void ldv<1, float>(const float *p, float (&x)[1]) { x[0] = __ldg(p); }
template <>
__device__ __forceinline__ void ldv<2, float>(const float *p, float (&x)[2]) {
    const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
    x[0] = v.x; x[1] = v.y;
}
template <>
__device__ __forceinline__ void ldv<4, float>(const float *p, float (&x)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
template <>
__device__ __forceinline__ void ldv<8, float>(const float *p, float (&x)[8]) {
    const float4 v = __ldg(reinterpret_cast<const float4 *>(p)), w = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
}
template <>
__device__ __forceinline__ void ldv<1, __nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[1]) {
    x[0] = __bfloat162float(*p);
}
template <>
__device__ __forceinline__ void ldv<2, __nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[2]) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
    x[0] = v.x; x[1] = v.y;
}
template <>
__device__ __forceinline__ void ldv<4, __nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[4]) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
template <>
__device__ __forceinline__ void ldv<8, __nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x; x[2 * i + 1] = f.y;
    }
}
template <>
__device__ __forceinline__ void stv<1, float>(float *p, const float (&x)[1]) { *p = x[0]; }
template <>
__device__ __forceinline__ void stv<2, float>(float *p, const float (&x)[2]) {
    *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void stv<4, float>(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <>
__device__ __forceinline__ void stv<8, float>(float *p, const float (&x)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ uint32_t pk2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
template <>
__device__ __forceinline__ void stv<1, __nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[1]) {
    *p = __float2bfloat16_rn(x[0]);
}
template <>
__device__ __forceinline__ void stv<2, __nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[2]) {
    *reinterpret_cast<uint32_t *>(p) = pk2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void stv<4, __nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[4]) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(pk2(x[0], x[1]), pk2(x[2], x[3]));
}
template <>
__device__ __forceinline__ void stv<8, __nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[8]) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(pk2(x[0], x[1]), pk2(x[2], x[3]), pk2(x[4], x[5]), pk2(x[6], x[7]));
}

__device__ __forceinline__ float silu(float y) { return y / (1.f + __expf(-y)); }
__device__ __forceinline__ float sigm(float y) { return 1.f / (1.f + __expf(-y)); }
__device__ __forceinline__ float softplus(float y) { return log1pf(__expf(-fabsf(y))) + fmaxf(y, 0.f); }

// The row or packed sequence that holds token t: its first token and the next
// sequence's first token (the end).
__device__ __forceinline__ void seq_bounds(const ProArgs &g, long long t, long long &s0, long long &s1) {
    if (!g.cu) {
        s0 = (t / g.T) * g.T;
        s1 = s0 + g.T;
        return;
    }
    int lo = 0, hi = g.nseq;   // cu[lo] <= t < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (g.cu[mid] <= t) lo = mid; else hi = mid;
    }
    s0 = g.cu[lo];
    s1 = g.cu[lo + 1];
}

// One convolved channel group of a lane: conv taps, bias, the last W - 1 rows.
template <int C>
struct ConvLane {
    float w[C][kProMaxW], b[C], hist[kProMaxW - 1][C];
};

template <int D, int C, typename T>
__device__ __forceinline__ void conv_init(ConvLane<C> &cl, const float *wgt, const float *bias, int W, int h,
                                          int lane, bool active) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const int ch = lane * C + c;
#pragma unroll
        for (int w = 0; w < kProMaxW; ++w) {
            // taps aligned to the right: tap kProMaxW-1 multiplies the current row
            const int src_w = w - (kProMaxW - W);
            cl.w[c][w] = (active && src_w >= 0) ? __ldg(wgt + ((long long)h * D + ch) * W + src_w) : 0.f;
        }
        cl.b[c] = (active && bias) ? __ldg(bias + h * D + ch) : 0.f;
#pragma unroll
        for (int r = 0; r < kProMaxW - 1; ++r) cl.hist[r][c] = 0.f;
    }
}

// y = conv of the current row x with the window; the window slides
template <int C>
__device__ __forceinline__ void conv_step(ConvLane<C> &cl, const float (&x)[C], float (&y)[C]) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
        float acc = fmaf(cl.w[c][kProMaxW - 1], x[c], cl.b[c]);
#pragma unroll
        for (int r = 0; r < kProMaxW - 1; ++r) acc = fmaf(cl.w[c][r], cl.hist[r][c], acc);
        y[c] = acc;
#pragma unroll
        for (int r = 0; r < kProMaxW - 2; ++r) cl.hist[r][c] = cl.hist[r + 1][c];
        cl.hist[kProMaxW - 2][c] = x[c];
    }
}

template <int C>
__device__ __forceinline__ void conv_clear(ConvLane<C> &cl) {
#pragma unroll
    for (int r = 0; r < kProMaxW - 1; ++r)
#pragma unroll
        for (int c = 0; c < C; ++c) cl.hist[r][c] = 0.f;
}

// One convolved tensor (q, k: with the L2 norm over its D channels; v: without)
// over a warp's tokens [t0, t1): the window slides along them, the rows are
// loaded one token ahead.
template <int D, bool NORM, typename T>
__device__ __forceinline__ void conv_tensor(const ProArgs &g, const T *x, const float *wgt, const float *bias, T *y,
                                            int h, int lane, long long t0, long long t1) {
    constexpr int C = (D + 31) / 32;
    const bool act = lane * C < D;
    ConvLane<C> cl;
    conv_init<D, C, T>(cl, wgt, bias, g.W, h, lane, act);
    long long s0, s1;
    seq_bounds(g, t0, s0, s1);
    float tmp[C];
    // the window before the warp's first token (rows of the same sequence)
    for (long long src = max(s0, t0 - (kProMaxW - 1)); src < t0; ++src) {
        float xr[C];
        if (act) ldv<C, T>(x + (src * g.H + h) * D + lane * C, xr);
        else
#pragma unroll
            for (int c = 0; c < C; ++c) xr[c] = 0.f;
        conv_step(cl, xr, tmp);
    }
    float nx[C];
    auto fetch = [&](long long t) {
        if (act) ldv<C, T>(x + (t * g.H + h) * D + lane * C, nx);
        else
#pragma unroll
            for (int c = 0; c < C; ++c) nx[c] = 0.f;
    };
    fetch(t0);
    for (long long t = t0; t < t1; ++t) {
        float xr[C], yr[C];
#pragma unroll
        for (int c = 0; c < C; ++c) xr[c] = nx[c];
        if (t + 1 < t1) fetch(t + 1);
        if (t == s1) {
            // a new row or packed sequence: its window starts empty
            long long a0;
            seq_bounds(g, t, a0, s1);
            conv_clear(cl);
        }
        conv_step(cl, xr, yr);
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            yr[c] = silu(yr[c]);
            if (act) ss = fmaf(yr[c], yr[c], ss);
        }
        if (NORM) {
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);
            const float sc = rsqrtf(ss + kProEps);
#pragma unroll
            for (int c = 0; c < C; ++c) yr[c] *= sc;
        }
        if (act) stv<C, T>(y + (t * g.H + h) * D + lane * C, yr);
    }
}

// The gate activations of a warp's tokens.
template <int DK, bool ISO>
__device__ __forceinline__ void gate_tokens(const ProArgs &g, int h, int lane, long long t0, long long t1) {
    constexpr int C = (DK + 31) / 32;
    for (long long t = t0; t < t1; ++t) {
        const long long th = t * g.H + h;
        if (ISO) {
            if (lane == 0) {
                g.a[th] = sigm(__ldg(g.xa + th));
                g.qn[th] = softplus(__ldg(g.xqn + th));
            }
        } else if (lane * C < DK) {
            float xa[C], xn[C];
            ldv<C, float>(g.xa + th * DK + lane * C, xa);
            ldv<C, float>(g.xqn + th * DK + lane * C, xn);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                xa[c] = sigm(xa[c]);
                xn[c] = softplus(xn[c]);
            }
            stv<C, float>(g.a + th * DK + lane * C, xa);
            stv<C, float>(g.qn + th * DK + lane * C, xn);
        }
        if (lane == 0) g.beta[th] = sigm(__ldg(g.xbeta + th));
    }
}

// CTA = (128 tokens, head, role): role 0 q, 1 k, 2 v, 3 the gates; each
// role holds only its own window and taps in registers.
template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(256) prologue_kernel(const ProArgs g) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, role = blockIdx.z;
    const long long t0 = (long long)blockIdx.x * kProTok + warp * kProWarpTok;
    if (t0 >= g.ntok) return;
    const long long t1 = min(t0 + kProWarpTok, g.ntok);
    if (role == 0)
        conv_tensor<DK, true, T>(g, static_cast<const T *>(g.xq), g.wq, g.bq, static_cast<T *>(g.q), h, lane, t0, t1);
    else if (role == 1)
        conv_tensor<DK, true, T>(g, static_cast<const T *>(g.xk), g.wk, g.bk, static_cast<T *>(g.k), h, lane, t0, t1);
    else if (role == 2)
        conv_tensor<DV, false, T>(g, static_cast<const T *>(g.xv), g.wv, g.bv, static_cast<T *>(g.v), h, lane, t0, t1);
    else
        gate_tokens<DK, ISO>(g, h, lane, t0, t1);
}

template <int DK, int DV, bool ISO, typename T>
cudaError_t launch_pro_t(const ProArgs &g, cudaStream_t st) {
    dim3 grid((unsigned)((g.ntok + kProTok - 1) / kProTok), (unsigned)g.H, 4u);
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
