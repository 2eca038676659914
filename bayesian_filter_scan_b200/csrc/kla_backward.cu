// kla_backward.cu -- gradients of the KLA filter (sm_100a, CUDA cores, fp32).
//
// Kalman Linear Attention abstract: the layer is meant for efficient parallel
// training. Per (row or packed sequence, head), with q^ = q / lambda (lambda:
// the posterior precision after the token), k^ = beta k and the forget gate
// g = a / (a^2 + qn lambda_prev), the mean recursion is a gated linear one,
//   eta_t = g_t . eta_{t-1} + k^_t v_t^T,      out_t = eta_t^T q^_t,
// and the precision chain is scalar per key. The gradients come from three
// sweeps that never store a per-token state:
//   forward sweep    eta in registers:  dq^_t = eta_t do_t
//   reverse sweep    the adjoint d_t = g_{t+1} . d_{t+1} + q^_t do_t^T in
//                    registers:         dk^_t = d_t v_t, dv_t = d_t^T k^_t;
//                    the gate term G_t = g_t dL/dg_t (per key) by the identity
//                    G_t = G_{t+1} + q^_t dq^_t - k^_t dk^_t,
//                    G_{T+1} = <dfinal_eta, eta_T>, and dL/deta0 = g_1 . d_1
//   precision chain  in reverse, per key (per head in isotropic mode): the
//                    adjoint of lambda through q^, lambda's own update and the
//                    gate, giving da, dqn and dL/dlambda0;
// then one elementwise pass assembles dq, dk and dbeta. The row sweeps keep
// M's rows per thread (thread = key row x 32 value columns), the column sweep
// keeps its columns (thread = value column x 32 key rows), so every sum a
// sweep needs is a shuffle among at most four adjacent lanes. No atomics.
#include "kla_internal.cuh"

namespace kla {

namespace {

struct BwdArgs {
    int H;
    long long T;
    const int *cu;
    const void *q, *k, *v, *dout;
    const float *a, *qn, *beta, *lambda0, *eta0, *dfl, *dfe;
    float *dq, *dk, *dv, *da, *dqn, *dbeta, *dlambda0, *deta0;
    // workspace: per token-head (nl = dk, or 1 in isotropic mode)
    float *lam;    // posterior precision [Ntok,H,nl]
    float *gate;   // forget gate [Ntok,H,nl]
    float *dqh;    // dL/dq^ [Ntok,H,dk]
    float *dkh;    // dL/dk^ [Ntok,H,dk]
    float *G;      // g dL/dg per key [Ntok,H,dk]
    float *dlp;    // dL/dlambda (posterior, total) [Ntok,H,nl]
    float *ginit;  // <dfinal_eta, eta_T> per key [units,dk]
    float *ksq;    // |k|^2 [Ntok,H] (isotropic)
    float *giso;   // sum_i G [Ntok,H] (isotropic)
    float *siso;   // sum_i dq^ q [Ntok,H] (isotropic)
};

template <typename T>
__device__ __forceinline__ float ld1(const T *p, long long i);
template <>
__device__ __forceinline__ float ld1<float>(const float *p, long long i) {
    return __ldg(p + i);
}
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}

// N contiguous values (N a multiple of 8; 16-byte aligned) as vector loads
template <int N>
__device__ __forceinline__ void ldrow(const float *p, float (&x)[N]) {
#pragma unroll
    for (int c = 0; c < N; c += 4) {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(p + c));
        x[c] = f.x; x[c + 1] = f.y; x[c + 2] = f.z; x[c + 3] = f.w;
    }
}
template <int N>
__device__ __forceinline__ void ldrow(const __nv_bfloat16 *p, float (&x)[N]) {
#pragma unroll
    for (int c = 0; c < N; c += 8) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p + c));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
            x[c + 2 * e] = f.x; x[c + 2 * e + 1] = f.y;
        }
    }
}

__device__ __forceinline__ void unit_bounds(const BwdArgs &g, long long u, long long &tb, long long &te) {
    const long long n = u / g.H;
    if (g.cu) { tb = g.cu[n]; te = g.cu[n + 1]; }
    else { tb = n * g.T; te = tb + g.T; }
}

// Sum over groups of NG adjacent lanes (NG = 1, 2 or 4).
template <int NG>
__device__ __forceinline__ float group_sum(float x, unsigned mask) {
#pragma unroll
    for (int d = 1; d < NG; d <<= 1) x += __shfl_xor_sync(mask, x, d);
    return x;
}

template <int DK, int DV>
struct RowLayout {   // thread = (key row i, block of CW value columns)
    static constexpr int CW = DV < 32 ? DV : 32;
    static constexpr int NCB = DV / CW;
    static constexpr int NT = DK * NCB;
    static constexpr int THREADS = NT < 32 ? 32 : NT;
};
template <int DK, int DV>
struct ColLayout {   // thread = (value column j, block of RW key rows)
    static constexpr int RW = DK < 32 ? DK : 32;
    static constexpr int NRB = DK / RW;
    static constexpr int NT = DV * NRB;
    static constexpr int THREADS = NT < 32 ? 32 : NT;
};

// Isotropic: |k|^2 per token-head (mode 0), or sum_i G and sum_i dq^ q (mode 1).
// A warp per token-head.
template <int DK, typename T>
__global__ void __launch_bounds__(256) bwd_row_sums(const BwdArgs g, long long nth, int mode) {
    const long long th = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= nth) return;
    const T *q = static_cast<const T *>(g.q), *k = static_cast<const T *>(g.k);
    float s0 = 0.f, s1 = 0.f;
    for (int i = lane; i < DK; i += 32) {
        if (mode == 0) {
            const float x = ld1<T>(k, th * DK + i);
            s0 = fmaf(x, x, s0);
        } else {
            s0 += g.G[th * DK + i];
            s1 = fmaf(g.dqh[th * DK + i], ld1<T>(q, th * DK + i), s1);
        }
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, d);
        s1 += __shfl_xor_sync(0xffffffffu, s1, d);
    }
    if (lane == 0) {
        if (mode == 0) g.ksq[th] = s0;
        else { g.giso[th] = s0; g.siso[th] = s1; }
    }
}

// Forward sweep: the precision chain, the mean in registers, dq^ = eta do.
template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(RowLayout<DK, DV>::THREADS) bwd_forward_sweep(const BwdArgs g) {
    using L = RowLayout<DK, DV>;
    constexpr int CW = L::CW, NCB = L::NCB, NL = ISO ? 1 : DK;
    const int tid = threadIdx.x;
    if (tid >= L::NT) return;
    const unsigned mask = L::NT >= 32 ? 0xffffffffu : ((1u << L::NT) - 1u);
    const int i = tid / NCB, cb = tid % NCB, li = ISO ? 0 : i;
    const long long u = blockIdx.x;
    const int h = (int)(u % g.H);
    long long tb, te;
    unit_bounds(g, u, tb, te);
    const T *k = static_cast<const T *>(g.k), *v = static_cast<const T *>(g.v), *dout = static_cast<const T *>(g.dout);
    float eta[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) eta[c] = g.eta0 ? g.eta0[(u * DK + i) * DV + cb * CW + c] : 0.f;
    float lam = g.lambda0 ? g.lambda0[u * NL + li] : 1.f;
    for (long long t = tb; t < te; ++t) {
        const long long th = t * g.H + h;
        const float at = ISO ? __ldg(g.a + th) : __ldg(g.a + th * DK + i);
        const float qt = ISO ? __ldg(g.qn + th) : __ldg(g.qn + th * DK + i);
        const float bt = __ldg(g.beta + th), ki = ld1<T>(k, th * DK + i);
        const float den = fmaf(at, at, qt * lam);
        const float gt = at / den;
        lam = lam / den + (ISO ? bt * g.ksq[th] * (1.f / (float)DK) : bt * ki * ki);
        const float kh = bt * ki;
        float s = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += 8) {
            float vr[8], dr[8];
            ldrow<8>(v + th * DV + cb * CW + c0, vr);
            ldrow<8>(dout + th * DV + cb * CW + c0, dr);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                eta[c0 + c] = fmaf(gt, eta[c0 + c], kh * vr[c]);
                s = fmaf(eta[c0 + c], dr[c], s);
            }
        }
        s = group_sum<NCB>(s, mask);
        if (cb == 0) {
            g.dqh[th * DK + i] = s;
            if (!ISO || i == 0) {
                g.lam[th * NL + li] = lam;
                g.gate[th * NL + li] = gt;
            }
        }
    }
    float s = 0.f;
    if (g.dfe)
#pragma unroll
        for (int c = 0; c < CW; ++c) s = fmaf(g.dfe[(u * DK + i) * DV + cb * CW + c], eta[c], s);
    s = group_sum<NCB>(s, mask);
    if (cb == 0) g.ginit[u * DK + i] = s;
}

// Reverse sweep over key rows: the adjoint in registers, dk^, the gate term G,
// and dL/deta0.
template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(RowLayout<DK, DV>::THREADS) bwd_reverse_rows(const BwdArgs g) {
    using L = RowLayout<DK, DV>;
    constexpr int CW = L::CW, NCB = L::NCB, NL = ISO ? 1 : DK;
    const int tid = threadIdx.x;
    if (tid >= L::NT) return;
    const unsigned mask = L::NT >= 32 ? 0xffffffffu : ((1u << L::NT) - 1u);
    const int i = tid / NCB, cb = tid % NCB, li = ISO ? 0 : i;
    const long long u = blockIdx.x;
    const int h = (int)(u % g.H);
    long long tb, te;
    unit_bounds(g, u, tb, te);
    const T *q = static_cast<const T *>(g.q), *k = static_cast<const T *>(g.k), *v = static_cast<const T *>(g.v),
            *dout = static_cast<const T *>(g.dout);
    float d[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) d[c] = g.dfe ? g.dfe[(u * DK + i) * DV + cb * CW + c] : 0.f;
    float G = g.ginit[u * DK + i], Gc = 0.f;
    for (long long t = te - 1; t >= tb; --t) {
        const long long th = t * g.H + h;
        if (t + 1 < te) {
            const float g1 = g.gate[(th + g.H) * NL + li];
#pragma unroll
            for (int c = 0; c < CW; ++c) d[c] *= g1;
        }
        const float qh = ld1<T>(q, th * DK + i) / g.lam[th * NL + li];
        float p = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += 8) {
            float vr[8], dr[8];
            ldrow<8>(v + th * DV + cb * CW + c0, vr);
            ldrow<8>(dout + th * DV + cb * CW + c0, dr);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                d[c0 + c] = fmaf(qh, dr[c], d[c0 + c]);
                p = fmaf(d[c0 + c], vr[c], p);
            }
        }
        p = group_sum<NCB>(p, mask);
        const float kh = __ldg(g.beta + th) * ld1<T>(k, th * DK + i);
        // compensated running sum: the gate term sums over the rest of the sequence
        const float y = fmaf(qh, g.dqh[th * DK + i], -kh * p) - Gc;
        const float Gn = G + y;
        Gc = (Gn - G) - y;
        G = Gn;
        if (cb == 0) {
            g.dkh[th * DK + i] = p;
            g.G[th * DK + i] = G;
        }
    }
    if (g.deta0) {
        const float g0 = te > tb ? g.gate[(tb * g.H + h) * NL + li] : 1.f;
#pragma unroll
        for (int c = 0; c < CW; ++c) g.deta0[(u * DK + i) * DV + cb * CW + c] = g0 * d[c];
    }
}

// Reverse sweep over value columns: the same adjoint, dv = d^T k^.
template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(ColLayout<DK, DV>::THREADS) bwd_reverse_cols(const BwdArgs g) {
    using L = ColLayout<DK, DV>;
    constexpr int RW = L::RW, NRB = L::NRB;
    const int tid = threadIdx.x;
    if (tid >= L::NT) return;
    const unsigned mask = L::NT >= 32 ? 0xffffffffu : ((1u << L::NT) - 1u);
    const int j = tid / NRB, rb = tid % NRB, i0 = rb * RW;
    const long long u = blockIdx.x;
    const int h = (int)(u % g.H);
    long long tb, te;
    unit_bounds(g, u, tb, te);
    const T *q = static_cast<const T *>(g.q), *k = static_cast<const T *>(g.k), *dout = static_cast<const T *>(g.dout);
    float d[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) d[r] = g.dfe ? g.dfe[(u * DK + i0 + r) * DV + j] : 0.f;
    for (long long t = te - 1; t >= tb; --t) {
        const long long th = t * g.H + h;
        const bool more = t + 1 < te;
        const float dj = ld1<T>(dout, th * DV + j), bt = __ldg(g.beta + th);
        const float giso = ISO && more ? g.gate[th + g.H] : 1.f, liso = ISO ? g.lam[th] : 1.f;
        float p = 0.f;
#pragma unroll
        for (int r0 = 0; r0 < RW; r0 += 8) {
            float qr[8], kr[8], lr[8], g1[8];
            ldrow<8>(q + th * DK + i0 + r0, qr);
            ldrow<8>(k + th * DK + i0 + r0, kr);
            if (ISO) {
#pragma unroll
                for (int r = 0; r < 8; ++r) { lr[r] = liso; g1[r] = giso; }
            } else {
                ldrow<8>(g.lam + th * DK + i0 + r0, lr);
                if (more) ldrow<8>(g.gate + (th + g.H) * DK + i0 + r0, g1);
                else
#pragma unroll
                    for (int r = 0; r < 8; ++r) g1[r] = 1.f;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                d[r0 + r] = fmaf(qr[r] / lr[r], dj, d[r0 + r] * g1[r]);
                p = fmaf(kr[r], d[r0 + r], p);
            }
        }
        p = group_sum<NRB>(p, mask) * bt;
        if (rb == 0) g.dv[th * DV + j] = p;
    }
}

// The precision chain in reverse: a thread per (unit, key), or per unit in
// isotropic mode.
template <int DK, bool ISO, typename T>
__global__ void __launch_bounds__(128) bwd_precision_chain(const BwdArgs g, long long units) {
    constexpr int NL = ISO ? 1 : DK;
    const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= units * NL) return;
    const long long u = x / NL;
    const int i = (int)(x % NL);
    const int h = (int)(u % g.H);
    long long tb, te;
    unit_bounds(g, u, tb, te);
    const T *q = static_cast<const T *>(g.q);
    const float lam0 = g.lambda0 ? g.lambda0[u * NL + i] : 1.f;
    float dl = g.dfl ? g.dfl[u * NL + i] : 0.f;
    for (long long t = te - 1; t >= tb; --t) {
        const long long th = t * g.H + h;
        const float lt = g.lam[th * NL + i];
        const float lp = t > tb ? g.lam[(th - g.H) * NL + i] : lam0;
        const float at = g.a[th * NL + i], qt = g.qn[th * NL + i];
        float sq, Gt;
        if (ISO) { sq = g.siso[th]; Gt = g.giso[th]; }
        else { sq = g.dqh[th * DK + i] * ld1<T>(q, th * DK + i); Gt = g.G[th * DK + i]; }
        const float dlt = dl - sq / (lt * lt);   // adjoint of the posterior precision
        g.dlp[th * NL + i] = dlt;
        const float den = fmaf(at, at, qt * lp);
        const float dg = Gt * den / at;          // dL/dg = G / g
        const float dden = -(dlt * lp + dg * at) / (den * den);
        g.da[th * NL + i] = dg / den + 2.f * at * dden;
        g.dqn[th * NL + i] = lp * dden;
        dl = dlt / den + qt * dden;
    }
    if (g.dlambda0) g.dlambda0[u * NL + i] = dl;
}

// dq = dq^ / lambda, dk = beta dk^ + 2 beta k dL/dlambda (iso: / dk),
// dbeta = sum_i k dk^ + k^2 dL/dlambda: a warp per token-head.
template <int DK, bool ISO, typename T>
__global__ void __launch_bounds__(256) bwd_assemble(const BwdArgs g, long long nth) {
    const long long th = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (th >= nth) return;
    const T *k = static_cast<const T *>(g.k);
    const float bt = __ldg(g.beta + th);
    float s = 0.f;
    for (int i = lane; i < DK; i += 32) {
        const long long e = th * DK + i;
        const float ki = ld1<T>(k, e), dkh = g.dkh[e];
        const float lt = ISO ? g.lam[th] : g.lam[e];
        const float dlt = ISO ? g.dlp[th] * (1.f / (float)DK) : g.dlp[e];
        g.dq[e] = g.dqh[e] / lt;
        g.dk[e] = bt * dkh + 2.f * bt * ki * dlt;
        s = fmaf(ki, dkh + ki * dlt, s);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
    if (lane == 0) g.dbeta[th] = s;
}

template <int DK, int DV, bool ISO, typename T>
cudaError_t launch_bwd_t(long long units, long long nth, const BwdArgs &g, cudaStream_t st) {
    const unsigned rows = (unsigned)((nth + 7) / 8);
    if (ISO) {
        bwd_row_sums<DK, T><<<rows, 256, 0, st>>>(g, nth, 0);
    }
    bwd_forward_sweep<DK, DV, ISO, T><<<(unsigned)units, RowLayout<DK, DV>::THREADS, 0, st>>>(g);
    bwd_reverse_rows<DK, DV, ISO, T><<<(unsigned)units, RowLayout<DK, DV>::THREADS, 0, st>>>(g);
    bwd_reverse_cols<DK, DV, ISO, T><<<(unsigned)units, ColLayout<DK, DV>::THREADS, 0, st>>>(g);
    if (ISO) {
        bwd_row_sums<DK, T><<<rows, 256, 0, st>>>(g, nth, 1);
    }
    const long long chains = units * (ISO ? 1 : DK);
    bwd_precision_chain<DK, ISO, T><<<(unsigned)((chains + 127) / 128), 128, 0, st>>>(g, units);
    bwd_assemble<DK, ISO, T><<<rows, 256, 0, st>>>(g, nth);
    return cudaGetLastError();
}

template <int DK, int DV, typename T>
cudaError_t launch_bwd_iso(bool iso, long long units, long long nth, const BwdArgs &g, cudaStream_t st) {
    return iso ? launch_bwd_t<DK, DV, true, T>(units, nth, g, st) : launch_bwd_t<DK, DV, false, T>(units, nth, g, st);
}

template <int DK, typename T>
cudaError_t launch_bwd_dv(int dv, bool iso, long long units, long long nth, const BwdArgs &g, cudaStream_t st) {
    switch (dv) {
        case 16: return launch_bwd_iso<DK, 16, T>(iso, units, nth, g, st);
        case 32: return launch_bwd_iso<DK, 32, T>(iso, units, nth, g, st);
        case 64: return launch_bwd_iso<DK, 64, T>(iso, units, nth, g, st);
        case 128: return launch_bwd_iso<DK, 128, T>(iso, units, nth, g, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_bwd_dk(int dk, int dv, bool iso, long long units, long long nth, const BwdArgs &g,
                          cudaStream_t st) {
    switch (dk) {
        case 16: return launch_bwd_dv<16, T>(dv, iso, units, nth, g, st);
        case 32: return launch_bwd_dv<32, T>(dv, iso, units, nth, g, st);
        case 64: return launch_bwd_dv<64, T>(dv, iso, units, nth, g, st);
        case 128: return launch_bwd_dv<128, T>(dv, iso, units, nth, g, st);
        default: return cudaErrorInvalidValue;
    }
}

constexpr size_t kBwdAlign = 256;
size_t bwd_round(size_t x) { return (x + kBwdAlign - 1) / kBwdAlign * kBwdAlign; }

}  // namespace

bool backward_supported(int dk, int dv) {
    auto ok = [](int x) { return x == 16 || x == 32 || x == 64 || x == 128; };
    return ok(dk) && ok(dv);
}

size_t backward_workspace_bytes(long long ntok, int H, long long units, int dk, bool iso) {
    const size_t nth = (size_t)ntok * H, nl = iso ? 1 : (size_t)dk;
    return 3 * bwd_round(nth * nl * 4) + 3 * bwd_round(nth * dk * 4) + bwd_round((size_t)units * dk * 4) +
           3 * bwd_round(nth * 4);
}

cudaError_t launch_backward(int H, long long T, long long ntok, long long units, int dk, int dv, bool iso, bool bf16,
                            const int *cu, const void *q, const void *k, const void *v, const float *a,
                            const float *qn, const float *beta, const float *lambda0, const float *eta0,
                            const void *dout, const float *dfinal_lambda, const float *dfinal_eta, float *dq,
                            float *dk_, float *dv_, float *da, float *dqn, float *dbeta, float *dlambda0,
                            float *deta0, void *ws, cudaStream_t st) {
    if (units == 0) return cudaSuccess;
    BwdArgs g;
    g.H = H; g.T = T; g.cu = cu;
    g.q = q; g.k = k; g.v = v; g.dout = dout;
    g.a = a; g.qn = qn; g.beta = beta; g.lambda0 = lambda0; g.eta0 = eta0;
    g.dfl = dfinal_lambda; g.dfe = dfinal_eta;
    g.dq = dq; g.dk = dk_; g.dv = dv_; g.da = da; g.dqn = dqn; g.dbeta = dbeta;
    g.dlambda0 = dlambda0; g.deta0 = deta0;
    const size_t nth = (size_t)ntok * H, nl = iso ? 1 : (size_t)dk;
    char *p = static_cast<char *>(ws);
    auto take = [&](size_t bytes) { float *r = reinterpret_cast<float *>(p); p += bwd_round(bytes); return r; };
    g.lam = take(nth * nl * 4);
    g.gate = take(nth * nl * 4);
    g.dlp = take(nth * nl * 4);
    g.dqh = take(nth * dk * 4);
    g.dkh = take(nth * dk * 4);
    g.G = take(nth * dk * 4);
    g.ginit = take((size_t)units * dk * 4);
    g.ksq = take(nth * 4);
    g.giso = take(nth * 4);
    g.siso = take(nth * 4);
    return bf16 ? launch_bwd_dk<__nv_bfloat16>(dk, dv, iso, units, (long long)nth, g, st)
                : launch_bwd_dk<float>(dk, dv, iso, units, (long long)nth, g, st);
}

}  // namespace kla
