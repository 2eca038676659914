// kla_scan.cu -- the precision path: a parallel scan of the Moebius maps that
// one predict+update step applies to the precision lambda (Kalman Linear
// Attention, technical summary section 2: the posterior precision is a
// fractional-linear function of the previous one, such maps compose
// associatively, so lambda_1..T comes from a prefix scan).
//
// Three kernels, no inter-CTA waiting (reduce, then scan, then re-walk):
//   mobius_reduce : per (row, head, block of Lb tokens, key) the composed 2x2
//                   matrix of the block (normalised by powers of two); diagonal
//                   mode streams a, qn, k through a TMA-fed shared-memory ring
//                   in persistent CTAs, eight 8-token sub-blocks per block
//                   composed by a tree in shared memory.
//   mobius_carry  : per (row, head, key) one warp: each segment's product
//                   (lanes compose slices, a shuffle tree joins them), carried
//                   in order and applied to lambda0: lambda at every segment
//                   start.
//   mobius_emit   : per (row/sequence, head, block, key) re-walks the block
//                   from its start lambda and writes lambda after every token
//                   (the kla_precision output; there segments are blocks).
#include <algorithm>

#include "kla_internal.cuh"
#include "kla_tc_ptx.cuh"

namespace kla {

struct ScanArgs {
    int N, H, dk;
    long long T;      // tokens per row (non-varlen)
    int NB;           // blocks per row
    const int *cu;    // packed sequence offsets (emit only) or nullptr
};

// ---- reduce --------------------------------------------------------------

// Diagonal: per (row, head, block of Lb tokens, key) the composed block
// matrix, carried as its two columns, the images of (1, 0) and (0, 1): each
// step is the projective chain d <- a^2 d + qn n, n <- n + b d on both columns
// (b = beta k^2), three fp32 operations per column. Persistent and TMA-fed:
// work item = (block of Lb
// tokens, row x head, half of the keys: min(dk, 64) keys), head-fastest. A CTA
// of 8 sub-blocks x (keys/4) quads streams its items through a 2-stage
// shared-memory ring filled by TMA (a, qn fp32 and k tiles of Lb rows), so the
// loads in flight do not occupy registers; beta of the next item is loaded
// into registers while the current one is composed. Thread 0 issues the
// copies; every wait is bounded (on timeout the status bit is set and the CTA
// stops after its copies in flight have landed).
constexpr int kRedStages = 2;
constexpr int kRedSub = 8, kRedLen = kBlockTokens / kRedSub;

__host__ __device__ constexpr int red_stage_bytes(int dki, int kes) { return kBlockTokens * dki * (8 + kes); }

template <typename TIn>
__global__ void __launch_bounds__(128, 2)
mobius_reduce_tma(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_qn,
                  const __grid_constant__ CUtensorMap tm_k, ScanArgs s, const float *__restrict__ beta,
                  float4 *__restrict__ agg, int nitems, int *status) {
    using namespace ptx;
    const int dki = min(s.dk, 64), nq = dki / 4, nhalf = s.dk / dki;
    const int stA = kBlockTokens * dki * 4, stK = kBlockTokens * dki * (int)sizeof(TIn);
    const int stB = 2 * stA + stK;
    extern __shared__ __align__(128) uint8_t smraw[];
    float4 *part = reinterpret_cast<float4 *>(smraw + kRedStages * stB);    // [kRedSub][64]
    uint64_t *full = reinterpret_cast<uint64_t *>(part + kRedSub * 64), *empty = full + kRedStages;
    const int quad = threadIdx.x % nq, sub = threadIdx.x / nq;
    // 32-bit index arithmetic (the host checks the item count and the token
    // axis fit): one unsigned division per decode
    const unsigned units = (unsigned)(s.N * s.H), H = (unsigned)s.H;
    const int step = gridDim.x;
    if (threadIdx.x == 0) {
        for (int j = 0; j < kRedStages; ++j) {
            mbar_init(&full[j], 1);
            mbar_init(&empty[j], blockDim.x);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_release();
    pdl_wait();
    struct Item { unsigned u, n, h; int blk, half; };
    auto decode = [&](int w) {
        Item it;
        const unsigned r = nhalf == 2 ? (unsigned)w >> 1 : (unsigned)w;   // nhalf is 1 or 2
        it.half = nhalf == 2 ? (w & 1) : 0;
        it.blk = (int)(r / units);
        it.u = r - (unsigned)it.blk * units;
        it.n = it.u / H;
        it.h = it.u - it.n * H;
        return it;
    };
    auto issue = [&](int w, int st) {
        const Item it = decode(w);
        const int blk = it.blk, half = it.half, h = (int)it.h;
        const int tok = (int)it.n * (int)s.T + blk * kBlockTokens;
        uint8_t *d = smraw + st * stB;
        mbar_expect_tx(&full[st], stB);
        tma_load_3d(d, &tm_a, &full[st], half * dki, h, tok);
        tma_load_3d(d + stA, &tm_qn, &full[st], half * dki, h, tok);
        tma_load_3d(d + 2 * stA, &tm_k, &full[st], half * dki, h, tok);
    };
    auto wait = [&](uint64_t *bar, uint32_t par) -> bool {
        if (mbar_try_wait(bar, par)) return true;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait_sleep(bar, par, 20000u))
            if (globaltimer() - t0 > 2000000000ull) { atomicOr(status, kStatusTimeout); return false; }
        return true;
    };
    int nmine = 0;
    if ((int)blockIdx.x < nitems) nmine = (nitems - 1 - (int)blockIdx.x) / step + 1;
    if (threadIdx.x == 0)
        for (int j = 0; j < kRedStages && j < nmine; ++j) issue((int)blockIdx.x + j * step, j);
    float bv[kRedLen];
    const int T = (int)s.T;
    auto load_beta = [&](const Item &it) {
        const int t0 = it.blk * kBlockTokens + sub * kRedLen;
        const float *bp = beta + ((long long)it.n * T + t0) * H + it.h;
#pragma unroll
        for (int r = 0; r < kRedLen; ++r) bv[r] = t0 + r < T ? __ldg(bp + r * H) : 0.f;
    };
    Item nxt = decode((int)blockIdx.x);
    if (nmine > 0) load_beta(nxt);
    bool ok = true;
    int issued = min(kRedStages, nmine), consumed = 0;
    for (int j = 0; j < nmine; ++j) {
        const int st = j % kRedStages;
        const int w = (int)blockIdx.x + j * step;
        const Item cur = nxt;
        const int blk = cur.blk, half = cur.half;
        const int t0 = blk * kBlockTokens + sub * kRedLen;
        const int len = max(0, min(kRedLen, T - t0));
        float cb[kRedLen];
#pragma unroll
        for (int r = 0; r < kRedLen; ++r) cb[r] = bv[r];
        if (j + 1 < nmine) {
            nxt = decode(w + step);
            load_beta(nxt);
        }
        // every thread waits; the CTA goes on only if all saw the copy land
        if (!__syncthreads_and(wait(&full[st], (uint32_t)((j / kRedStages) & 1)))) { ok = false; consumed = j; break; }
        const uint8_t *d = smraw + st * stB;
        const float *sa = reinterpret_cast<const float *>(d) + (sub * kRedLen) * dki + 4 * quad;
        const float *sq = reinterpret_cast<const float *>(d + stA) + (sub * kRedLen) * dki + 4 * quad;
        const TIn *sk = reinterpret_cast<const TIn *>(d + 2 * stA) + (sub * kRedLen) * dki + 4 * quad;
        float4 av[kRedLen], qv[kRedLen], kv[kRedLen];
#pragma unroll
        for (int r = 0; r < kRedLen; ++r) {
            av[r] = *reinterpret_cast<const float4 *>(sa + r * dki);
            qv[r] = *reinterpret_cast<const float4 *>(sq + r * dki);
            if constexpr (sizeof(TIn) == 2) {
                const uint2 x = *reinterpret_cast<const uint2 *>(sk + r * dki);
                kv[r] = make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u),
                                    __uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u));
            } else {
                kv[r] = *reinterpret_cast<const float4 *>(sk + r * dki);
            }
        }
        // stage read into registers: release it, and refill it with the item kRedStages ahead
        mbar_arrive(&empty[st]);
        if (threadIdx.x == 0 && issued < nmine) {
            if (!wait(&empty[st], (uint32_t)((j / kRedStages) & 1))) { ok = false; }
            else { issue(blockIdx.x + issued * step, st); ++issued; }
        }
        Mob m[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            // the two columns (n1, n2), (d1, d2) share a^2, qn and b: paired fp32
            float2 nn = make_float2(1.f, 0.f), dd = make_float2(0.f, 1.f);
#pragma unroll
            for (int r = 0; r < kRedLen; ++r) {
                if (r < len) {
                    const float ac = (&av[r].x)[c], qc = (&qv[r].x)[c], kc = (&kv[r].x)[c];
                    const float a2 = ac * ac, b = cb[r] * kc * kc;
                    dd = __ffma2_rn(make_float2(a2, a2), dd, __fmul2_rn(make_float2(qc, qc), nn));
                    nn = __ffma2_rn(make_float2(b, b), dd, nn);
                }
            }
            m[c] = mob_norm(Mob{nn.x, nn.y, dd.x, dd.y});
            part[sub * 64 + 4 * quad + c] = make_float4(m[c].m00, m[c].m01, m[c].m10, m[c].m11);
        }
#pragma unroll
        for (int wd = 1; wd < kRedSub; wd <<= 1) {
            __syncthreads();
            if ((sub & (2 * wd - 1)) == 0) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 x = part[(sub + wd) * 64 + 4 * quad + c];
                    m[c] = mob_norm(mob_mul(Mob{x.x, x.y, x.z, x.w}, m[c]));
                    if (2 * wd < kRedSub) part[sub * 64 + 4 * quad + c] = make_float4(m[c].m00, m[c].m01, m[c].m10, m[c].m11);
                }
            }
        }
        if (sub == 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                agg[((long long)cur.u * s.NB + blk) * s.dk + half * dki + 4 * quad + c] =
                    make_float4(m[c].m00, m[c].m01, m[c].m10, m[c].m11);
        }
        // part is rewritten by the next item; a failed refill stops every thread
        if (!__syncthreads_and(ok)) { ok = false; consumed = j + 1; break; }
    }
    // on a timeout, the copies issued but not consumed land before the CTA exits
    if (threadIdx.x == 0 && !ok)
        for (int j = consumed; j < issued; ++j) wait(&full[j % kRedStages], (uint32_t)((j / kRedStages) & 1));
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
    pdl_release();
    pdl_wait();
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
// One warp per (row, head, key), segments in order: the warp's lanes compose
// consecutive slices of the segment's blocks, a shuffle tree combines the
// slices in order into the segment's product, and lane 0 carries the prefix.
__device__ __forceinline__ Mob shfl_down_m(const Mob &m, int d) {
    return Mob{__shfl_down_sync(0xffffffffu, m.m00, d), __shfl_down_sync(0xffffffffu, m.m01, d),
               __shfl_down_sync(0xffffffffu, m.m10, d), __shfl_down_sync(0xffffffffu, m.m11, d)};
}

__global__ void __launch_bounds__(128)
mobius_carry(ScanArgs s, int nl, int P, int seg_blocks, const float4 *__restrict__ agg,
             const float *__restrict__ lambda0, float *__restrict__ lam_blk) {
    pdl_release();
    pdl_wait();
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (long long)s.N * s.H * nl) return;
    const long long u = gw / nl;
    const int i = (int)(gw % nl);
    const float l0 = lambda0 ? __ldg(lambda0 + gw) : 1.0f;
    const float4 *src = agg + u * s.NB * nl + i;
    Mob carry{1.f, 0.f, 0.f, 1.f};
    for (int p = 0; p < P; ++p) {
        if (lane == 0) lam_blk[(u * s.NB + (long long)p * seg_blocks) * nl + i] = mob_apply(carry, l0);
        if (p == P - 1) break;
        const int b0 = p * seg_blocks, b1 = min(b0 + seg_blocks, s.NB);
        const int per = (b1 - b0 + 31) / 32;
        // this lane's slice [b0 + lane * per, ...), composed in order
        Mob M{1.f, 0.f, 0.f, 1.f};
        for (int q0 = 0; q0 < per; q0 += 8) {
            float4 m[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int b = b0 + lane * per + q0 + r;
                if (q0 + r < per && b < b1) m[r] = __ldg(src + (long long)b * nl);
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int b = b0 + lane * per + q0 + r;
                if (q0 + r < per && b < b1) M = mob_norm(mob_mul(Mob{m[r].x, m[r].y, m[r].z, m[r].w}, M));
            }
        }
        // slices in order: lane l takes the product of lanes l .. l + 2d - 1
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const Mob o = shfl_down_m(M, d);
            if ((lane & (2 * d - 1)) == 0) M = mob_norm(mob_mul(o, M));
        }
        carry = mob_norm(mob_mul(M, carry));
    }
}

// Short segments (fewer than 32 blocks each, e.g. every block a segment):
// lane l composes the blocks of segments l, l+32, ..., a warp-shuffle scan of
// the 2x2 maps gives the exclusive prefixes, carried across groups of 32.
__device__ __forceinline__ Mob shfl_up_m(const Mob &m, int d) {
    return Mob{__shfl_up_sync(0xffffffffu, m.m00, d), __shfl_up_sync(0xffffffffu, m.m01, d),
               __shfl_up_sync(0xffffffffu, m.m10, d), __shfl_up_sync(0xffffffffu, m.m11, d)};
}
__device__ __forceinline__ Mob shfl_m(const Mob &m, int src) {
    return Mob{__shfl_sync(0xffffffffu, m.m00, src), __shfl_sync(0xffffffffu, m.m01, src),
               __shfl_sync(0xffffffffu, m.m10, src), __shfl_sync(0xffffffffu, m.m11, src)};
}

__global__ void __launch_bounds__(128)
mobius_carry_lanes(ScanArgs s, int nl, int P, int seg_blocks, const float4 *__restrict__ agg,
             const float *__restrict__ lambda0, float *__restrict__ lam_blk) {
    pdl_release();
    pdl_wait();
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
    pdl_release();
    pdl_wait();
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
    pdl_release();
    pdl_wait();
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

// ---- launch order of packed sequences -------------------------------------

// perm[r] = the packed sequence of rank r by length, longest first (ties by
// index). The walk kernels map their block index through it, so the longest
// walks start first and the short ones fill in behind (list scheduling).
__global__ void __launch_bounds__(256)
kla_seq_order(const int *__restrict__ cu, int N, int *__restrict__ perm) {
    pdl_release();
    pdl_wait();
    __shared__ int len[kMaxOrderSeqs];
    for (int i = threadIdx.x; i < N; i += blockDim.x) len[i] = cu[i + 1] - cu[i];
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int li = len[i];
        int r = 0;
        for (int j = 0; j < N; ++j) {
            const int lj = len[j];
            r += (lj > li) || (lj == li && j < i);
        }
        perm[r] = i;
    }
}

// ---- host launchers ------------------------------------------------------

static inline unsigned blocks_for(long long threads, int per) {
    return (unsigned)((threads + per - 1) / per);
}

template <typename TIn>
cudaError_t launch_mobius_reduce(const Plan &p, const void *k, const float *a, const float *qn,
                                 const float *beta, float4 *agg, int *status, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, nullptr};
    long long pairs = (long long)p.N * p.H * p.NB;
    if (p.iso) {
        return launch_pdl(mobius_reduce_iso<TIn>, blocks_for(pairs, 128), 128, 0, st, s, (const TIn *)k, a, qn,
                          beta, agg);
    }
    const int dki = p.dk < 64 ? p.dk : 64, nhalf = p.dk / dki;
    const int kes = (int)sizeof(TIn);
    const CUtensorMapDataType F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUtensorMapDataType KT = kes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : F32;
    CUtensorMap ma, mq, mk;
    if (!make_tma_map(&ma, a, F32, 4, p.dk, p.H, p.ntok, dki, kBlockTokens, false) ||
        !make_tma_map(&mq, qn, F32, 4, p.dk, p.H, p.ntok, dki, kBlockTokens, false) ||
        !make_tma_map(&mk, k, KT, kes, p.dk, p.H, p.ntok, dki, kBlockTokens, false))
        return cudaErrorInvalidValue;
    const int smem = kRedStages * red_stage_bytes(dki, kes) + kRedSub * 64 * 16 + 2 * kRedStages * 8;
    // the largest request (64-key items) once per device and input type
    static PerDevice<bool> attr;
    const int smax = kRedStages * red_stage_bytes(64, kes) + kRedSub * 64 * 16 + 2 * kRedStages * 8;
    const cudaError_t ea = ensure_smem_attr(attr, mobius_reduce_tma<TIn>, smax);
    if (ea != cudaSuccess) return ea;
    const long long nitems = pairs * nhalf;
    // the kernel indexes items and tokens in 32 bits (TMA coordinates are 32-bit too)
    if (nitems >= (1LL << 31) || p.ntok >= (1LL << 31)) return cudaErrorInvalidValue;
    const long long grid = std::min(nitems, 2LL * p.sms);
    return launch_pdl(mobius_reduce_tma<TIn>, (unsigned)grid, kRedSub * dki / 4, smem, st, ma, mq, mk, s, beta, agg,
                      (int)nitems, status);
}

cudaError_t launch_seq_order(const Plan &p, const int *cu, int *perm, cudaStream_t st) {
    if (p.N > kMaxOrderSeqs) return cudaErrorInvalidValue;
    return launch_pdl(kla_seq_order, 1, 256, 0, st, cu, p.N, perm);
}

cudaError_t launch_mobius_carry(const Plan &p, const float4 *agg, const float *lambda0,
                                float *lam_blk, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, nullptr};
    long long thr = (long long)p.N * p.H * p.nl * 32;
    return launch_pdl(p.seg_blocks >= 32 ? mobius_carry : mobius_carry_lanes, blocks_for(thr, 128), 128, 0, st,
                      s, p.nl, p.P, p.seg_blocks, agg, lambda0, lam_blk);
}

template <typename TIn>
cudaError_t launch_mobius_emit(const Plan &p, const int *cu, const void *k, const float *a,
                               const float *qn, const float *beta, const float *lam_blk,
                               const float *lambda0, float *lam_out, cudaStream_t st) {
    ScanArgs s{p.N, p.H, p.dk, p.T, p.NB, cu};
    long long pairs = cu ? (long long)p.N * p.H : (long long)p.N * p.H * p.NB;
    if (p.iso)
        return launch_pdl(mobius_emit_iso<TIn>, blocks_for(pairs, 128), 128, 0, st, s, (const TIn *)k, a, qn,
                          beta, lam_blk, lambda0, lam_out);
    return launch_pdl(mobius_emit_diag<TIn>, blocks_for(pairs * (p.dk / 4), 128), 128, 0, st, s,
                      (const TIn *)k, a, qn, beta, lam_blk, lambda0, lam_out);
}

template cudaError_t launch_mobius_reduce<float>(const Plan &, const void *, const float *,
                                                 const float *, const float *, float4 *, int *, cudaStream_t);
template cudaError_t launch_mobius_reduce<__nv_bfloat16>(const Plan &, const void *, const float *,
                                                         const float *, const float *, float4 *, int *,
                                                         cudaStream_t);
template cudaError_t launch_mobius_emit<float>(const Plan &, const int *, const void *, const float *,
                                               const float *, const float *, const float *,
                                               const float *, float *, cudaStream_t);
template cudaError_t launch_mobius_emit<__nv_bfloat16>(const Plan &, const int *, const void *,
                                                       const float *, const float *, const float *,
                                                       const float *, const float *, float *,
                                                       cudaStream_t);

}  // namespace kla
