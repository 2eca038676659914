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
// CTA = 8 warps x (tiles of 16 tokens per warp) of one head and one role (q, k,
// v, a with beta, or qn). A convolving warp walks its consecutive tiles in
// order: it copies a tile's rows (for the first, also the 3 before them) into
// shared memory, all copies in flight at once, and the next tile's copies fly
// while it convolves the current one; a lane covers dk / 32 (dv / 32)
// contiguous channels, keeps their conv taps in registers and slides a window
// of the last W - 1 rows along its tokens; a window is cleared where a new row
// or packed sequence starts. A gate CTA is elementwise, with 8 vector loads in
// flight per thread.
#include "kla_internal.cuh"

namespace kla {

namespace {

#ifndef KLA_PRO_TILES
#define KLA_PRO_TILES 1
#endif
constexpr int kProTileTok = 16;  // tokens per tile
constexpr int kProMaxW = 4;      // widest convolution
constexpr int kProRoles = 5;     // q, k, v, a and beta, qn
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

// N contiguous values as one vector access (loads: fp32, N = 1, 4)
template <int N, typename T>
__device__ __forceinline__ void ldv(const T *p, float (&x)[N]);
template <int N, typename T>
__device__ __forceinline__ void stv(T *p, const float (&x)[N]);
template <>
__device__ __forceinline__ void ldv<1, float>(const float *p, float (&x)[1]) { x[0] = __ldg(p); }
template <>
__device__ __forceinline__ void ldv<4, float>(const float *p, float (&x)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
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

// The tiling of one instantiation (DM = max(dk, dv) channels of type T): the
// tiles a warp walks in order (KLA_PRO_TILES, or 1 where two tile buffers per
// warp would not fit in shared memory), and the rows a warp holds in shared
// memory: one or two tile buffers, the first with the W - 1 rows before the
// warp's first token in front of it.
template <int DM, typename T>
struct ProShape {
    static constexpr int two_buf_bytes = 8 * (kProMaxW - 1 + 2 * kProTileTok) * DM * (int)sizeof(T);
    static constexpr int tiles = (KLA_PRO_TILES > 1 && two_buf_bytes <= 200 * 1024) ? KLA_PRO_TILES : 1;
    static constexpr int bufs = tiles > 1 ? 2 : 1;
    static constexpr int rows = kProMaxW - 1 + bufs * kProTileTok;   // rows per warp
    static constexpr int warp_tok = tiles * kProTileTok;              // tokens per warp
    static constexpr int cta_tok = 8 * warp_tok;                      // tokens per CTA
    static constexpr int smem = 8 * rows * DM * (int)sizeof(T);
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

// C contiguous values of a shared-memory row as floats
template <int C, typename T>
__device__ __forceinline__ void lds(const T *p, float (&x)[C]) {
    if constexpr (std::is_same<T, float>::value) {
#pragma unroll
        for (int c = 0; c < C; ++c) x[c] = p[c];
    } else if constexpr (C == 1) {
        x[0] = __bfloat162float(p[0]);
    } else {
#pragma unroll
        for (int c = 0; c < C; c += 2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p + c));
            x[c] = f.x;
            if (c + 1 < C) x[c + 1] = f.y;
        }
    }
}

// One convolved tensor (q, k: with the L2 norm over its D channels; v: without)
// over a warp's tokens [tw0, tw1), walked as tiles of 16 tokens. The rows of a
// tile (for the first, also the W - 1 rows before it) are copied into shared
// memory with asynchronous 16-byte copies, all in flight at once; the next
// tile's copies are in flight while the warp convolves the current one (two
// buffers). The window of the last W - 1 rows slides along the whole span in
// registers.
template <int D, bool NORM, int NT, typename T>
__device__ __forceinline__ void conv_tensor(const ProArgs &g, const T *x, const float *wgt, const float *bias, T *y,
                                            int h, int lane, long long tw0, long long tw1, T *rows) {
    constexpr int NB = NT > 1 ? 2 : 1;   // tile buffers
    constexpr int C = (D + 31) / 32;
    constexpr int CH = (D * (int)sizeof(T)) / 16;   // 16-byte pieces per row
    static_assert(CH * 16 == D * (int)sizeof(T), "rows are whole 16-byte pieces");
    constexpr int H0 = kProMaxW - 1;
    const bool act = lane * C < D;
    long long s0, s1;
    seq_bounds(g, tw0, s0, s1);
    const long long r0 = max(s0, tw0 - H0);   // first row the window needs
    const int off = (int)(r0 - (tw0 - H0));
    // tile i's first token sits at row slot tile_slot(i) of the warp's rows
    auto tile_slot = [](int i) { return H0 + (i % NB) * kProTileTok; };
    // copies of tile i: its rows (and for tile 0 the rows before it), one group
    auto issue = [&](int i) {
        const long long a = i == 0 ? r0 : tw0 + (long long)i * kProTileTok;
        const long long b = min(tw0 + (long long)(i + 1) * kProTileTok, tw1);
        const int slot0 = i == 0 ? off : tile_slot(i);
        const int n = a < b ? (int)(b - a) * CH : 0;
        for (int e = lane; e < n; e += 32) {
            const int r = e / CH, c = e - r * CH;
            cp_async16(reinterpret_cast<char *>(rows + (slot0 + r) * D) + 16 * c,
                       reinterpret_cast<const char *>(x + ((a + r) * g.H + h) * D) + 16 * c);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    issue(0);
    if (NT > 1) issue(1);
    ConvLane<C> cl;
    conv_init<D, C, T>(cl, wgt, bias, g.W, h, lane, act);
    float tmp[C];
#pragma unroll 1
    for (int i = 0; i < NT; ++i) {
        const long long t0 = tw0 + (long long)i * kProTileTok;
        // tile i's group is complete once at most the later one is pending
        if (i + 1 < NT) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncwarp();
        if (t0 >= tw1) break;
        if (i == 0) {
            // the window before the warp's first token (rows of the same sequence)
            for (int r = off; r < H0; ++r) {
                float xr[C];
                if (act) lds<C, T>(rows + r * D + lane * C, xr);
                else
#pragma unroll
                    for (int c = 0; c < C; ++c) xr[c] = 0.f;
                conv_step(cl, xr, tmp);
            }
        }
        const T *buf = rows + tile_slot(i) * D;
        const long long t1 = min(t0 + kProTileTok, tw1);
        for (long long t = t0; t < t1; ++t) {
            float xr[C], yr[C];
            if (act) lds<C, T>(buf + (int)(t - t0) * D + lane * C, xr);
            else
#pragma unroll
                for (int c = 0; c < C; ++c) xr[c] = 0.f;
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
        // every lane has read this buffer before it is refilled
        __syncwarp();
        if (i + 2 < NT) issue(i + 2);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// An elementwise gate over the CTA's tokens [tb, te): out = f(in) on NL values
// per (token, head); each thread loads a batch of vectors before it computes.
template <int NL, int F>
__device__ __forceinline__ void gate_tensor(const ProArgs &g, const float *in, float *out, int h, long long tb,
                                            long long te) {
    constexpr int V = NL % 4 == 0 ? 4 : 1;     // floats per access
    constexpr int PR = NL / V;                  // accesses per row
    constexpr int B = 8;                        // accesses in flight per thread
    const int n = (int)(te - tb) * PR;
    auto f = [](float y) { return F == 0 ? sigm(y) : softplus(y); };
    for (int e0 = threadIdx.x; e0 < n; e0 += B * blockDim.x) {
        float xv[B][V];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int e = e0 + j * blockDim.x;
            if (e < n) {
                const int r = e / PR, c = e - r * PR;
                ldv<V, float>(in + ((tb + r) * g.H + h) * NL + c * V, xv[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int e = e0 + j * blockDim.x;
            if (e < n) {
                const int r = e / PR, c = e - r * PR;
#pragma unroll
                for (int v = 0; v < V; ++v) xv[j][v] = f(xv[j][v]);
                stv<V, float>(out + ((tb + r) * g.H + h) * NL + c * V, xv[j]);
            }
        }
    }
}

// CTA = (role, token block, head); the roles of one token block are adjacent
// in the grid so that every SM runs a mix of them: 0 q, 1 k, 2 v (a warp per
// ProShape::warp_tok tokens, rows staged in shared memory), 3 a and beta, 4 qn
// (elementwise).
template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(256) prologue_kernel(const ProArgs g) {
    extern __shared__ __align__(16) unsigned char pro_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int DM = DK > DV ? DK : DV;
    using S = ProShape<DM, T>;
    const int h = blockIdx.y, role = (int)(blockIdx.x % kProRoles);
    const long long tb = (long long)(blockIdx.x / kProRoles) * S::cta_tok;
    const long long te = min(tb + S::cta_tok, g.ntok);
    if (role >= 3) {
        constexpr int NL = ISO ? 1 : DK;
        if (role == 3) {
            gate_tensor<NL, 0>(g, g.xa, g.a, h, tb, te);
            gate_tensor<1, 0>(g, g.xbeta, g.beta, h, tb, te);
        } else {
            gate_tensor<NL, 1>(g, g.xqn, g.qn, h, tb, te);
        }
        return;
    }
    const long long t0 = tb + (long long)warp * S::warp_tok;
    if (t0 >= g.ntok) return;
    const long long t1 = min(t0 + S::warp_tok, g.ntok);
    T *rows = reinterpret_cast<T *>(pro_smem) + (size_t)warp * S::rows * DM;
    if (role == 0)
        conv_tensor<DK, true, S::tiles, T>(g, static_cast<const T *>(g.xq), g.wq, g.bq, static_cast<T *>(g.q), h,
                                           lane, t0, t1, rows);
    else if (role == 1)
        conv_tensor<DK, true, S::tiles, T>(g, static_cast<const T *>(g.xk), g.wk, g.bk, static_cast<T *>(g.k), h,
                                           lane, t0, t1, rows);
    else
        conv_tensor<DV, false, S::tiles, T>(g, static_cast<const T *>(g.xv), g.wv, g.bv, static_cast<T *>(g.v), h,
                                            lane, t0, t1, rows);
}

template <int DK, int DV, bool ISO, typename T>
cudaError_t launch_pro_t(const ProArgs &g, cudaStream_t st) {
    static PerDevice<bool> attr;
    constexpr int DM = DK > DV ? DK : DV;
    using S = ProShape<DM, T>;
    const int smem = S::smem;
    auto kern = prologue_kernel<DK, DV, ISO, T>;
    cudaError_t e = ensure_smem_attr(attr, kern, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((g.ntok + S::cta_tok - 1) / S::cta_tok * kProRoles), (unsigned)g.H);
    kern<<<grid, 256, smem, st>>>(g);
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
