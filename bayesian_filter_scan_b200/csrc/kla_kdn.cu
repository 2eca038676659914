// kla_kdn.cu -- the Kalman Delta Network forward with the Kalman-gain residual
// write (sm_100a, CUDA cores). One CTA per (row or packed sequence, head, block
// of value columns) walks its tokens in order; its part of the mean state lives
// in registers for the whole walk.
//
// Kalman Delta Networks abstract: the memory is the state of a linear-Gaussian
// model whose transition propagates the mean and its uncertainty, the Kalman
// gain weights each residual write, diagonal KDN projects each one-step
// posterior onto diagonal Gaussians and isotropic KDN keeps one uncertainty
// scalar per head. Read as (per token; precision lambda per key, mean M[dk][dv]):
//   lambda~ = lambda / (a^2 + qn lambda)       the KLA filter's predict step
//   w       = k / lambda~                       predictive covariance times k
//   gamma   = beta / (1 + beta k.w)             reciprocal innovation variance
//   r       = v - (a M)^T k                     innovation, per value column
//   M       = a M + gamma w r^T                 the Kalman mean update
//   lambda  = lambda~ + beta k^2                diagonal of the posterior precision
//   o       = M^T q = (a M)^T q + gamma (q.w) r  readout of the posterior mean
// (isotropic: a, qn and lambda are scalars per head, lambda += beta |k|^2 / dk).
//
// The value columns of M evolve independently given the key-side quantities
// (a, k, w, gamma), so a (row, head) is split over CTAs by blocks of DVB value
// columns; each CTA repeats the cheap key-side step. Thread layout inside a
// CTA: thread t owns column j = cb * DVB + t % DVB and rows
// [rg * dk/RG, (rg + 1) * dk/RG) of M, rg = t / DVB, RG = 256 / DVB; threads
// t < dk prepare key t's precision step and gain. Per token: the key threads
// stage (a, k, q, w) and per-warp partial sums (k.w, q.w, |k|^2) in shared
// memory; every thread decays its rows and forms its partial dot products with
// k and q; the column's partials are summed, and the rows take the rank-1
// write. Two barriers per token: the staging is double-buffered by token
// parity, so the next token's staging never overwrites what a slower thread
// still reads. Inputs are loaded one token ahead.
#include "kla_internal.cuh"

namespace kla {

namespace {

constexpr int kKdnThreads = 256;

struct KdnArgs {
    int H;
    long long T;
    const int *cu;
    const void *q, *k, *v;
    const float *a, *qn, *beta;
    const float *lambda0, *M0;
    void *out;
    float *final_lambda, *final_M;
};

template <typename T>
__device__ __forceinline__ float ldx(const T *p, long long i);
template <>
__device__ __forceinline__ float ldx<float>(const float *p, long long i) {
    return __ldg(p + i);
}
template <>
__device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void stx(T *p, long long i, float x);
template <>
__device__ __forceinline__ void stx<float>(float *p, long long i, float x) {
    p[i] = x;
}
template <>
__device__ __forceinline__ void stx<__nv_bfloat16>(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) x += __shfl_xor_sync(0xffffffffu, x, d);
    return x;
}

// Value columns per CTA: 32, or dv when it is smaller.
template <int DV>
constexpr int kdn_dvb() { return DV < 32 ? DV : 32; }

template <int DK, int DV, bool ISO, typename T>
__global__ void __launch_bounds__(kKdnThreads) kdn_walk_kernel(const KdnArgs g) {
    constexpr int DVB = kdn_dvb<DV>();     // value columns of this CTA
    constexpr int RG = kKdnThreads / DVB;  // row groups
    constexpr int RPT = DK / RG;           // rows of M per thread
    constexpr int NWK = (DK + 31) / 32;    // warps holding keys
    static_assert(RPT >= 1 && RPT * RG == DK, "thread layout");
    __shared__ float s_a[2][DK], s_k[2][DK], s_q[2][DK], s_w[2][DK], s_v[2][DVB];
    __shared__ float s_pk[2][RG][DVB], s_pq[2][RG][DVB];
    __shared__ float s_red[2][NWK][3];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int jl = tid % DVB, rg = tid / DVB, i0 = rg * RPT;
    const int cb = (int)blockIdx.y, j = cb * DVB + jl;   // local and global column
    const long long u = blockIdx.x;
    const int h = (int)(u % g.H);
    const long long n = u / g.H;
    long long tb, te;
    if (g.cu) { tb = g.cu[n]; te = g.cu[n + 1]; }
    else { tb = n * g.T; te = tb + g.T; }
    const T *q = static_cast<const T *>(g.q), *k = static_cast<const T *>(g.k), *v = static_cast<const T *>(g.v);
    T *out = static_cast<T *>(g.out);

    float m[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) m[r] = g.M0 ? g.M0[(u * DK + i0 + r) * DV + j] : 0.f;
    // precision: key threads (diagonal) or every thread (isotropic)
    float lam = 1.f;
    if (ISO) lam = g.lambda0 ? g.lambda0[u] : 1.f;
    else if (tid < DK) lam = g.lambda0 ? g.lambda0[u * DK + tid] : 1.f;

    // inputs of token t, loaded one token ahead
    float nk = 0.f, nq = 0.f, na = 1.f, nqn = 0.f, nv = 0.f, nb = 0.f;
    auto fetch = [&](long long t) {
        const long long th = t * g.H + h;
        if (tid < DK) {
            nk = ldx<T>(k, th * DK + tid);
            nq = ldx<T>(q, th * DK + tid);
            if (!ISO) {
                na = __ldg(g.a + th * DK + tid);
                nqn = __ldg(g.qn + th * DK + tid);
            }
        }
        if (ISO) {
            na = __ldg(g.a + th);
            nqn = __ldg(g.qn + th);
        }
        if (tid < DVB) nv = ldx<T>(v, th * DV + cb * DVB + tid);
        nb = __ldg(g.beta + th);
    };
    if (te > tb) fetch(tb);

    for (long long t = tb; t < te; ++t) {
        const int buf = (int)((t - tb) & 1);
        const float ck = nk, cq = nq, ca = na, cqn = nqn, cv = nv, cb = nb;
        if (t + 1 < te) fetch(t + 1);
        // ---- key threads: the precision step and the gain direction
        const float lt_iso = ISO ? lam / fmaf(ca, ca, cqn * lam) : 0.f;
        float kw = 0.f, qw = 0.f, kk = 0.f;
        if (tid < DK) {
            const float lt = ISO ? lt_iso : lam / fmaf(ca, ca, cqn * lam);
            const float w = ck / lt;
            if (!ISO) lam = fmaf(cb * ck, ck, lt);
            s_a[buf][tid] = ca;
            s_k[buf][tid] = ck;
            s_q[buf][tid] = cq;
            s_w[buf][tid] = w;
            kw = ck * w;
            qw = cq * w;
            kk = ck * ck;
        }
        if (tid < DVB) s_v[buf][tid] = cv;
        if (wid < NWK) {
            kw = warp_sum(kw);
            qw = warp_sum(qw);
            kk = warp_sum(kk);
            if (lane == 0) {
                s_red[buf][wid][0] = kw;
                s_red[buf][wid][1] = qw;
                s_red[buf][wid][2] = kk;
            }
        }
        __syncthreads();
        // ---- every thread: decay its rows, partial dot products with k and q
        float s = 0.f, gq = 0.f, ksq = 0.f;
#pragma unroll
        for (int x = 0; x < NWK; ++x) {
            s += s_red[buf][x][0];
            gq += s_red[buf][x][1];
            ksq += s_red[buf][x][2];
        }
        const float gam = cb / fmaf(cb, s, 1.f);
        if (ISO) lam = fmaf(cb, ksq * (1.f / (float)DK), lt_iso);
        float ak = 0.f, aq = 0.f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = i0 + r;
            m[r] *= ISO ? ca : s_a[buf][i];
            ak = fmaf(s_k[buf][i], m[r], ak);
            aq = fmaf(s_q[buf][i], m[r], aq);
        }
        s_pk[buf][rg][jl] = ak;
        s_pq[buf][rg][jl] = aq;
        __syncthreads();
        // ---- the column's innovation, the rank-1 write, the readout
        float mk = 0.f, mq = 0.f;
#pragma unroll
        for (int x = 0; x < RG; ++x) {
            mk += s_pk[buf][x][jl];
            mq += s_pq[buf][x][jl];
        }
        const float rj = s_v[buf][jl] - mk;
        const float gr = gam * rj;
#pragma unroll
        for (int r = 0; r < RPT; ++r) m[r] = fmaf(s_w[buf][i0 + r], gr, m[r]);
        if (rg == 0) stx<T>(out, (t * g.H + h) * DV + j, fmaf(gq, gr, mq));
    }
    if (g.final_lambda && cb == 0) {
        if (ISO) { if (tid == 0) g.final_lambda[u] = lam; }
        else if (tid < DK) g.final_lambda[u * DK + tid] = lam;
    }
    if (g.final_M) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) g.final_M[(u * DK + i0 + r) * DV + j] = m[r];
    }
}

template <int DK, int DV, bool ISO, typename T>
cudaError_t launch_kdn_t(long long units, const KdnArgs &g, cudaStream_t st) {
    const dim3 grid((unsigned)units, (unsigned)(DV / kdn_dvb<DV>()));
    kdn_walk_kernel<DK, DV, ISO, T><<<grid, kKdnThreads, 0, st>>>(g);
    return cudaGetLastError();
}

template <int DK, int DV, typename T>
cudaError_t launch_kdn_iso(bool iso, long long units, const KdnArgs &g, cudaStream_t st) {
    return iso ? launch_kdn_t<DK, DV, true, T>(units, g, st) : launch_kdn_t<DK, DV, false, T>(units, g, st);
}

template <int DK, typename T>
cudaError_t launch_kdn_dv(int dv, bool iso, long long units, const KdnArgs &g, cudaStream_t st) {
    switch (dv) {
        case 16: return launch_kdn_iso<DK, 16, T>(iso, units, g, st);
        case 32: return launch_kdn_iso<DK, 32, T>(iso, units, g, st);
        case 64: return launch_kdn_iso<DK, 64, T>(iso, units, g, st);
        case 128: return launch_kdn_iso<DK, 128, T>(iso, units, g, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_kdn_dk(int dk, int dv, bool iso, long long units, const KdnArgs &g, cudaStream_t st) {
    switch (dk) {
        case 16: return launch_kdn_dv<16, T>(dv, iso, units, g, st);
        case 32: return launch_kdn_dv<32, T>(dv, iso, units, g, st);
        case 64: return launch_kdn_dv<64, T>(dv, iso, units, g, st);
        case 128: return launch_kdn_dv<128, T>(dv, iso, units, g, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool kdn_supported(int dk, int dv) {
    auto ok = [](int x) { return x == 16 || x == 32 || x == 64 || x == 128; };
    return ok(dk) && ok(dv);
}

cudaError_t launch_kdn(int H, long long T, long long units, int dk, int dv, bool iso, bool bf16, const int *cu,
                       const void *q, const void *k, const void *v, const float *a, const float *qn,
                       const float *beta, const float *lambda0, const float *M0, void *out, float *final_lambda,
                       float *final_M, cudaStream_t st) {
    if (units == 0) return cudaSuccess;
    KdnArgs g;
    g.H = H; g.T = T; g.cu = cu;
    g.q = q; g.k = k; g.v = v; g.a = a; g.qn = qn; g.beta = beta;
    g.lambda0 = lambda0; g.M0 = M0; g.out = out; g.final_lambda = final_lambda; g.final_M = final_M;
    return bf16 ? launch_kdn_dk<__nv_bfloat16>(dk, dv, iso, units, g, st)
                : launch_kdn_dk<float>(dk, dv, iso, units, g, st);
}

}  // namespace kla
