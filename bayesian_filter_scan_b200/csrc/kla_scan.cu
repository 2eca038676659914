// kla_scan.cu -- the precision path: a parallel scan of the Moebius maps that
// one predict+update step applies to the precision lambda (Kalman Linear
// Attention, technical summary section 2: the posterior precision is a
// fractional-linear function of the previous one, such maps compose
// associatively, so lambda_1..T comes from a prefix scan).
//
// Three kernels, no inter-CTA waiting (reduce, then scan, then re-walk):
//   mobius_reduce : per (row, head, block of Lb tokens, key) the composed 2x2
//                   matrix of the block (normalised by powers of two); one CTA
//                   per block, sub-blocks of dk tokens per thread, composed in
//                   shared memory.
//   mobius_carry  : per (row, head, key) one warp: the product of each
//                   segment's blocks, a shuffle scan over segments, applied to
//                   lambda0: lambda at every segment start.
//   mobius_emit   : per (row/sequence, head, block, key) re-walks the block
//                   from its start lambda and writes lambda after every token
//                   (the kla_precision output; there segments are blocks).
#include "kla_internal.cuh"

namespace kla {

struct ScanArgs {
    int N, H, dk;
    long long T;      // tokens per row (non-varlen)
    int NB;           // blocks per row
    const int *cu;    // packed sequence offsets (emit only) or nullptr
};

// ---- reduce --------------------------------------------------------------

// CTA = one (row, head, block of Lb tokens); dk threads = 4 sub-blocks of
// Lb/4 tokens x dk/4 quads of keys. A thread walks its sub-block for 4
// consecutive keys (16-byte loads of a and qn, 8-byte loads of bf16 k). The
// block matrix is carried as its two columns, the images of (1, 0) and (0, 1):
// each step is the projective chain d <- a^2 d + qn n, n <- n + b d on both
// columns (b = beta k^2), three fp32 operations per column. The four sub-block
// products are composed in shared memory. CTAs run head-fastest, so that the
// heads of one token range (adjacent in memory) are read together.
template <typename TIn>
__global__ void __launch_bounds__(128)
mobius_reduce_diag(ScanArgs s, const TIn *__restrict__ k, const float *__restrict__ a,
                   const float *__restrict__ qn, const float *__restrict__ beta,
                   float4 *__restrict__ agg) {
    constexpr int kSub = 4, kLen = kBlockTokens / kSub;
    __shared__ float4 part[kSub][128];
    const int dk = s.dk, nq = dk / 4;
    const int quad = threadIdx.x % nq, sub = threadIdx.x / nq;
    const long long units = (long long)s.N * s.H;
    const long long u = blockIdx.x % units;
    const int blk = (int)(blockIdx.x / units);
    const int n = (int)(u / s.H), h = (int)(u % s.H);
    const long long t0 = (long long)blk * kBlockTokens + (long long)sub * kLen;
    const int len = (int)max(0LL, min((long long)kLen, s.T - t0));
    float n1[4], d1[4], n2[4], d2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) { n1[c] = 1.f; d1[c] = 0.f; n2[c] = 0.f; d2[c] = 1.f; }
#pragma unroll
    for (int half = 0; half < kLen; half += 8) {
        float4 av[8], qv[8], kv[8];
        float bv[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            av[r] = make_float4(1.f, 1.f, 1.f, 1.f);
            qv[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            kv[r] = qv[r];
            bv[r] = 0.f;
            if (half + r < len) {
                const long long th = ((long long)n * s.T + t0 + half + r) * s.H + h;
                av[r] = ld4(a + th * dk + 4 * quad);
                qv[r] = ld4(qn + th * dk + 4 * quad);
                kv[r] = ld4(k + th * dk + 4 * quad);
                bv[r] = __ldg(beta + th);
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const float *ap = &av[r].x, *qp = &qv[r].x, *kp = &kv[r].x;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float a2 = ap[c] * ap[c], b = bv[r] * kp[c] * kp[c];
                d1[c] = fmaf(a2, d1[c], qp[c] * n1[c]);
                n1[c] = fmaf(b, d1[c], n1[c]);
                d2[c] = fmaf(a2, d2[c], qp[c] * n2[c]);
                n2[c] = fmaf(b, d2[c], n2[c]);
            }
        }
        // exact power-of-two rescale of each key's matrix (entries are >= 0)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const Mob m = mob_norm(Mob{n1[c], n2[c], d1[c], d2[c]});
            n1[c] = m.m00; n2[c] = m.m01; d1[c] = m.m10; d2[c] = m.m11;
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) part[sub][4 * quad + c] = make_float4(n1[c], n2[c], d1[c], d2[c]);
    __syncthreads();
    if (sub == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = 4 * quad + c;
            Mob acc{n1[c], n2[c], d1[c], d2[c]};
#pragma unroll
            for (int b = 1; b < kSub; ++b) {
                const float4 m = part[b][i];
                acc = mob_norm(mob_mul(Mob{m.x, m.y, m.z, m.w}, acc));
            }
            agg[(u * s.NB + blk) * dk + i] = make_float4(acc.m00, acc.m01, acc.m10, acc.m11);
        }
    }
}

// Isotropic: one precision per head; increment beta*|k|^2/dk.
template <typename TIn>
__device__ __forceinline__ float ksq_row(const TIn *kr, int dk) {
    float s = 0.f;
    for (int i = 0; i < dk; i += 4) {
        float4 x = ld4(kr + i);
        s = fmaf(x.x, x.x, s); s = fmaf(x.y, x.y, s);
        s = fmaf(x.z, x.z, s); s = fmaf(x.w, x.w, s);
    }
    return s;
}

template <typename TIn>
__global__ void __launch_bounds__(128)
mobius_reduce_iso(ScanArgs s, const TIn *__restrict__ k, const float *__restrict__ a,
                  const float *__restrict__ qn, const float *__restrict__ beta,
                  float4 *__restrict__ agg) {
    long long pair = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (pair >= (long long)s.N * s.H * s.NB) return;
    int blk = (int)(pair % s.NB);
    long long u = pair / s.NB;
    int n = (int)(u / s.H), h = (int)(u % s.H);
    long long t0 = (long long)blk * kBlockTokens;
    long long t1 = min(t0 + kBlockTokens, s.T);
    const float inv_dk = 1.0f / (float)s.dk;
    Mob P{1.f, 0.f, 0.f, 1.f};
    for (long long t = t0; t < t1; ++t) {
        long long th = ((long long)n * s.T + t) * s.H + h;
        float b = __ldg(beta + th) * ksq_row(k + th * s.dk, s.dk) * inv_dk;
        P = mob_mul(mob_step(__ldg(a + th), __ldg(qn + th), b), P);
        if (((t - t0) & 7) == 7) P = mob_norm(P);
    }
    P = mob_norm(P);
    agg[pair] = make_float4(P.m00, P.m01, P.m10, P.m11);
}

// ---- carry ---------------------------------------------------------------

// lam_blk[(u*NB + p*seg_blocks)*nl + i] = (all blocks before segment p)(lambda0):
// lambda at every segment start (every block start when segments are blocks).
// One warp per (row, head, key): lane l composes the blocks of segments l,
// l+32, ..., then a warp-shuffle scan of the 2x2 maps gives the exclusive
// prefixes, carried across groups of 32 segments.
__device__ __forceinline__ Mob shfl_up_m(const Mob &m, int d) {
    return Mob{__shfl_up_sync(0xffffffffu, m.m00, d), __shfl_up_sync(0xffffffffu, m.m01, d),
               __shfl_up_sync(0xffffffffu, m.m10, d), __shfl_up_sync(0xffffffffu, m.m11, d)};
}
__device__ __forceinline__ Mob shfl_m(const Mob &m, int src) {
    return Mob{__shfl_sync(0xffffffffu, m.m00, src), __shfl_sync(0xffffffffu, m.m01, src),
               __shfl_sync(0xffffffffu, m.m10, src), __shfl_sync(0xffffffffu, m.m11, src)};
}

__global__ void __launch_bounds__(128)
mobius_carry(ScanArgs s, int nl, int P, int seg_blocks, const float4 *__restrict__ agg,
             const float *__restrict__ lambda0, float *__restrict__ lam_blk) {
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (long long)s.N * s.H * nl) return;
    const long long u = gw / nl;
    const int i = (int)(gw % nl);
    const float l0 = lambda0 ? __ldg(lambda0 + gw) : 1.0f;
    const float4 *src = agg + u * s.NB * nl + i;
    Mob carry{1.f, 0.f, 0.f, 1.f};
    for (int base = 0; base < P; base += 32) {
        const int p = base + lane;
        Mob S{1.f, 0.f, 0.f, 1.f};
        if (p < P) {
            const int b0 = p * seg_blocks, b1 = min(b0 + seg_blocks, s.NB);
            for (int b = b0; b < b1; b += 8) {
                float4 m[8];
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (b + r < b1) m[r] = __ldg(src + (long long)(b + r) * nl);
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (b + r < b1) S = mob_norm(mob_mul(Mob{m[r].x, m[r].y, m[r].z, m[r].w}, S));
            }
        }
        Mob incl = S;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const Mob o = shfl_up_m(incl, d);
            if (lane >= d) incl = mob_norm(mob_mul(incl, o));
        }
        Mob excl = shfl_up_m(incl, 1);
        if (lane == 0) excl = Mob{1.f, 0.f, 0.f, 1.f};
        if (p < P) lam_blk[(u * s.NB + (long long)p * seg_blocks) * nl + i] = mob_apply(mob_mul(excl, carry), l0);
        carry = mob_norm(mob_mul(shfl_m(incl, 31), carry));
    }
}

// ---- emit ----------------------------------------------------------------

// Token range and start precision of a (pair, key) walk. Non-varlen: pair =
// (u, blk), start from lam_blk. Varlen: pair = u (whole packed sequence), start
// from lambda0.
__device__ __forceinline__ void emit_range(const ScanArgs &s, long long pair, long long &u,
                                           long long &tb, long long &te) {
    if (s.cu) {
        u = pair;
        int n = (int)(u / s.H);
        tb = s.cu[n];
        te = s.cu[n + 1];
    } else {
        int blk = (int)(pair % s.NB);
        u = pair / s.NB;
        int n = (int)(u / s.H);
        tb = (long long)n * s.T + (long long)blk * kBlockTokens;
        te = (long long)n * s.T + min((long long)(blk + 1) * kBlockTokens, s.T);
    }
}

template <typename TIn>
__global__ void __launch_bounds__(128)
mobius_emit_diag(ScanArgs s, const TIn *__restrict__ k, const float *__restrict__ a,
                 const float *__restrict__ qn, const float *__restrict__ beta,
                 const float *__restrict__ lam_start, const float *__restrict__ lambda0,
                 float *__restrict__ lam_out) {
    const int nkq = s.dk / 4;
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long pair = gid / nkq;
    int kq = (int)(gid % nkq);
    long long npairs = s.cu ? (long long)s.N * s.H : (long long)s.N * s.H * s.NB;
    if (pair >= npairs) return;
    long long u, tb, te;
    emit_range(s, pair, u, tb, te);
    int h = (int)(u % s.H);
    float lam[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (s.cu) lam[c] = lambda0 ? __ldg(lambda0 + u * s.dk + 4 * kq + c) : 1.0f;
        else lam[c] = __ldg(lam_start + pair * s.dk + 4 * kq + c);
    }
    for (long long t = tb; t < te; t += 8) {
        float4 av[8], qv[8], kv[8];
        float bv[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            if (t + r < te) {
                long long th = (t + r) * s.H + h;
                av[r] = ld4(a + th * s.dk + 4 * kq);
                qv[r] = ld4(qn + th * s.dk + 4 * kq);
                kv[r] = ld4(k + th * s.dk + 4 * kq);
                bv[r] = __ldg(beta + th);
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            if (t + r < te) {
                const float *ap = &av[r].x, *qp = &qv[r].x, *kp = &kv[r].x;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float den = fmaf(ap[c], ap[c], qp[c] * lam[c]);
                    lam[c] = fmaf(bv[r] * kp[c], kp[c], lam[c] / den);
                }
                long long th = (t + r) * s.H + h;
                *reinterpret_cast<float4 *>(lam_out + th * s.dk + 4 * kq) =
                    make_float4(lam[0], lam[1], lam[2], lam[3]);
            }
        }
    }
}

template <typename TIn>
__global__ void __launch_bounds__(128)
mobius_emit_iso(ScanArgs s, const TIn *__restrict__ k, const float *__restrict__ a,
                const float *__restrict__ qn, const float *__restrict__ beta,
                const float *__restrict__ lam_start, const float *__restrict__ lambda0,
                float *__restrict__ lam_out) {
    long long pair = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long npairs = s.cu ? (long long)s.N * s.H : (long long)s.N * s.H * s.NB;
    if (pair >= npairs) return;
    long long u, tb, te;
    emit_range(s, pair, u, tb, te);
    int h = (int)(u % s.H);
    float lam = s.cu ? (lambda0 ? __ldg(lambda0 + u) : 1.0f) : __ldg(lam_start + pair);
    const float inv_dk = 1.0f / (float)s.dk;
    for (long long t = tb; t < te; ++t) {
        long long th = t * s.H + h;
        float at = __ldg(a + th);
        float den = fmaf(at, at, __ldg(qn + th) * lam);
        lam = fmaf(__ldg(beta + th) * ksq_row(k + th * s.dk, s.dk), inv_dk, lam / den);
        lam_out[th] = lam;
    }
}

// ---- host launchers ------------------------------------------------------

static inline unsigned blocks_for(long long threads, int per) {
    return (unsigned)((threads + per - 1) / per);
}

template <typename TIn>
cudaError_t launch_mobius_reduce(const Plan &p, const void *k, const float *a, const float *qn,
                                 const float *beta, float4 *agg, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, nullptr};
    long long pairs = (long long)p.N * p.H * p.NB;
    if (p.iso)
        mobius_reduce_iso<TIn><<<blocks_for(pairs, 128), 128, 0, st>>>(
            s, (const TIn *)k, a, qn, beta, agg);
    else
        mobius_reduce_diag<TIn><<<(unsigned)pairs, p.dk, 0, st>>>(s, (const TIn *)k, a, qn, beta, agg);
    return cudaGetLastError();
}

cudaError_t launch_mobius_carry(const Plan &p, const float4 *agg, const float *lambda0,
                                float *lam_blk, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, nullptr};
    long long thr = (long long)p.N * p.H * p.nl * 32;
    mobius_carry<<<blocks_for(thr, 128), 128, 0, st>>>(s, p.nl, p.P, p.seg_blocks, agg, lambda0, lam_blk);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_mobius_emit(const Plan &p, const int *cu, const void *k, const float *a,
                               const float *qn, const float *beta, const float *lam_blk,
                               const float *lambda0, float *lam_out, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, cu};
    long long pairs = cu ? (long long)p.N * p.H : (long long)p.N * p.H * p.NB;
    if (p.iso)
        mobius_emit_iso<TIn><<<blocks_for(pairs, 128), 128, 0, st>>>(
            s, (const TIn *)k, a, qn, beta, lam_blk, lambda0, lam_out);
    else
        mobius_emit_diag<TIn><<<blocks_for(pairs * (p.dk / 4), 128), 128, 0, st>>>(
            s, (const TIn *)k, a, qn, beta, lam_blk, lambda0, lam_out);
    return cudaGetLastError();
}

template cudaError_t launch_mobius_reduce<float>(const Plan &, const void *, const float *,
                                                 const float *, const float *, float4 *, cudaStream_t);
template cudaError_t launch_mobius_reduce<__nv_bfloat16>(const Plan &, const void *, const float *,
                                                         const float *, const float *, float4 *,
                                                         cudaStream_t);
template cudaError_t launch_mobius_emit<float>(const Plan &, const int *, const void *, const float *,
                                               const float *, const float *, const float *,
                                               const float *, float *, cudaStream_t);
template cudaError_t launch_mobius_emit<__nv_bfloat16>(const Plan &, const int *, const void *,
                                                       const float *, const float *, const float *,
                                                       const float *, const float *, float *,
                                                       cudaStream_t);

}  // namespace kla
