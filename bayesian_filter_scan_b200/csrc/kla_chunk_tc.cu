// kla_chunk_tc.cu -- the chunked form of the filter's mean path on tcgen05
// tensor cores (sm_100a).
//
// Once the precision path is known, the information-vector update is affine in
// eta with a per-key, data-dependent gate (Kalman Linear Attention, technical
// summary sections 2-3: after the Moebius scan the mean recursion is a
// parallelisable affine map; the forget gate g = a/(a^2 + qn*lambda) comes from
// precision ratios). It is gated linear attention with
//     q~ = q / lambda,  k~ = beta * k,  gate g[t,i] = a/(a^2 + qn*lambda_{t-1}).
// Per chunk of C = 64 tokens with in-chunk cumulative log2-gate G[t,i] and a
// per-key reference R[i] (midpoint of the chunk's G range, so that neither
// factor leaves the fp32/bf16 exponent range):
//     Q'[t,i] = q~[t,i] 2^(G[t,i]-R[i]),   K'[s,i] = k~[s,i] 2^(R[i]-G[s,i])
//     U       = diag(2^R) eta_chunk_start                     (state, TMEM fp32)
//     out     = mask_causal(Q' K'^T) V + Q' U                  (tcgen05, TMEM fp32)
//     eta_chunk_end = diag(2^(G_last-R)) (U + K'^T V)          (tcgen05, TMEM fp32)
// The state never leaves the SM while a CTA walks its segment: it lives in
// TMEM as the accumulator of the K'^T V products (the pages' kernels likewise
// avoid expanding the state in HBM).
//
// CTA = one segment of one (row or packed sequence, head); 320 threads:
//   warps 0-3  gate: per key, the lambda recursion over the chunk (a, qn stream
//              through a TMA ring of three 16-token slots), log-gates, then Q'/K' written in
//              place over the TMA-loaded q/k tiles (bf16, 128B-swizzled), and
//              the bf16 remainder of K' for a two-term state update, slot by
//              slot (the gate warps fold every slot themselves);
//              isotropic mode runs a warp-level Moebius scan over the chunk;
//   warps 4-7  epilogue: rescale U in TMEM and snapshot it to bf16 shared
//              memory, mask the score tile into P, store the output rows;
//   warp 8     TMA producer (q, k, v tiles double-buffered; a, qn ring);
//   warp 9     TMEM owner and single-thread tcgen05.mma issuer.
// mode 0 walks whole rows or packed sequences (from lambda0, eta0); mode 2
// walks every segment of split rows from a zero state (segment 0 from eta0)
// and exports what the correction pass needs. The kernel is instantiated per
// (dk, dv, isotropic or diagonal precision), each variant with only its own
// gate code.
//
// Every wait is bounded: after kWaitLimitNs a waiter sets the abort flag and
// the library status bit, all roles fall through to the teardown, the
// producer waits (bounded) for its outstanding copies, the MMA thread for its
// outstanding MMAs, and the TMEM is released.
#include <cstdlib>

#include "kla_internal.cuh"
#include "kla_tc_ptx.cuh"

namespace kla {
using namespace ptx;

namespace {

constexpr int kC = 64;             // chunk tokens
constexpr int kSlotTok = 8;        // tokens per gate slot (one pass of the chain and fold)
constexpr int kSlotsPerChunk = kC / kSlotTok;
constexpr int kRingTok = 16;       // tokens per a/qn ring slot (two gate slots per wait)
constexpr int kRings = 3;          // ring depth (48 tokens of look-ahead)
constexpr int kRingsPerChunk = kC / kRingTok;
constexpr int kMaxOffset = 110;    // |G - R| (log2) kept inside the fp32/bf16 exponent range
constexpr int kRebase = 64;        // diagonal mode: predicted |G - rho| that moves the reference
// Warp roles. dk = 128: gate warps 0-3, epilogue 4-7, TMA producer 8, MMA 9.
// dk = 64: gate warps 0 and 2, producer 1, MMA 3, epilogue 4-7 (8 warps, so
// two CTAs fit on one SM when dv = 64 as well).
template <int DK, int DV>
struct Roles {
    static constexpr int NGW = (DK == 64) ? 2 : 4;
    static constexpr int THREADS = (NGW + 6) * 32;
    static constexpr int MIN_BLOCKS = (DK == 64 && DV == 64) ? 2 : 1;
    static constexpr int PRODW = (NGW == 2) ? 1 : 8;
    static constexpr int MMAW = (NGW == 2) ? 3 : 9;
};
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct TcArgs {
    int N, H, P, NB, seg_blocks, iso, mode;
    long long T, Lseg;
    const int *cu, *perm;
    const float *a, *qn, *beta;
    const float *lambda0, *eta0, *lam_blk;
    const float4 *agg;   // block aggregates when the segment-start precision is composed here
    float *S_io, *decay;
    __nv_bfloat16 *out;
    float *final_lambda, *final_eta;
    int *status;
    // mode 2 (segments from a zero state): per chunk and key, the log2 factor
    // that takes the folded q' of the chunk to the segment-start frame,
    // rlog[(u * NC + chunk of the row) * DK + key]; the folded q tiles go to
    // the tensor map of the q' buffer
    float *rlog;
    int NC;
};

template <int DK, int DV>
struct Layout {
    static constexpr int QK = kC * DK * 2;
    static constexpr int V = kC * DV * 2;
    static constexpr int PT = kC * kC * 2;
    static constexpr int UB = DK * DV * 2;
    static constexpr int RINGF = kRingTok * DK;   // floats of one of a / qn per ring slot
    static constexpr int q0 = 0;
    static constexpr int k0 = q0 + 2 * QK;
    static constexpr int v0 = k0 + 2 * QK;
    static constexpr int p0 = v0 + 2 * V;
    static constexpr int ub0 = p0 + PT;
    static constexpr int klo0 = ub0 + UB;          // low bf16 part of K' (state update), per stage
    static constexpr int ring0 = klo0 + 2 * QK;
    static constexpr int fac0 = ring0 + kRings * 2 * RINGF * 4;
    static constexpr int facf0 = fac0 + 2 * DK * 4;
    static constexpr int isof0 = facf0 + DK * 4;   // iso: per-token factors (q, beta k) of a chunk
    static constexpr int bar0 = ((isof0 + kC * 8) + 7) & ~7;
    static constexpr int NBAR = 6 + 2 * kRings + 9;
    static constexpr int hold0 = bar0 + NBAR * 8;
    static constexpr int bytes = hold0 + 16;
    static constexpr int alloc = bytes + 1024;
    static_assert(alloc <= 232448, "shared memory per CTA");
    static constexpr uint32_t NCOLS = (2 * DV + 64 <= 256) ? 256u : 512u;
    static constexpr uint32_t colU = 0, colO = DV, colS = 2 * DV;
};

// Byte offset of element (row, col) in a 128B-swizzled bf16 tile stored as
// 64-column atoms of `rows` rows of 128 bytes (rows 1024-byte aligned groups).
__device__ __forceinline__ int sw_off(int row, int col, int rows) {
    return (col >> 6) * (rows * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1);
}

__device__ __forceinline__ float bf_at(const uint8_t *base, int off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}
__device__ __forceinline__ void bf_put(uint8_t *base, int off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status,
                                       bool honour_abort) {
    const uint64_t t0 = globaltimer();
    for (;;) {
        // sleeps until the phase completes (or 0.1 ms), then re-checks the limits
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if (honour_abort && *abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ bool wait1(uint64_t *bar, uint32_t parity, volatile int *ab, int *st) {
    return mbar_try_wait(bar, parity) || wait_slow(bar, parity, ab, st, true);
}
// Warp-uniform wait: every lane waits, the warp proceeds only if all saw it.
__device__ __forceinline__ bool waitw(uint64_t *bar, uint32_t parity, volatile int *ab, int *st) {
    bool ok = wait1(bar, parity, ab, st);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ Mob shfl_up_mob(const Mob &m, int d) {
    return Mob{__shfl_up_sync(0xffffffffu, m.m00, d), __shfl_up_sync(0xffffffffu, m.m01, d),
               __shfl_up_sync(0xffffffffu, m.m10, d), __shfl_up_sync(0xffffffffu, m.m11, d)};
}

template <int DK>
__device__ __forceinline__ float row_sumsq(const uint8_t *ktile, int row) {
    float s = 0.f;
#pragma unroll
    for (int a = 0; a < DK / 64; ++a) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint4 x = *reinterpret_cast<const uint4 *>(ktile + a * kC * 128 + row * 128 + ch * 16);
            const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2 f = __bfloat1622float2(b[e]);
                s = fmaf(f.x, f.x, s);
                s = fmaf(f.y, f.y, s);
            }
        }
    }
    return s;
}

// One 8-token slot (rows 8j .. 8j+7 of the chunk) of the diagonal gate for the
// key i of this thread. The precision runs in projective form, lambda = n/d:
//   d <- a^2 d + qn n,   n <- n + b d   (b = beta k^2),   PA <- PA a,
// two FMAs per token on the serial chain; with G the cumulative log2 gate,
// 2^G = PA/d and 2^G / lambda = PA/n (n, d, PA carry exponents E, E, F). The
// slot's operands are then written over the q/k tiles:
//   K' = beta k 2^(R - G) = beta k (d/PA) mk   (bf16 hi + bf16 remainder)
//   Q' = q / lambda 2^(G - R) = q (PA/n) mq    (bf16)
// (mk = 2^(R - (F - E)), mq = 1/mk), packed to bf16 by integer rounding. The
// chain runs first, then every token's reciprocals and stores, which are
// independent of one another. Ends with the exact power-of-two rescale.
// a and qn come from the ring slot ra.
template <int DK>
__device__ __forceinline__ void gate_slot(int j, const float *ra, uint8_t *qt, uint8_t *kt, uint8_t *klo,
                                          const int (&offr)[kSlotTok], float bsrc, bool state_mode, int R,
                                          float &nn, float &dd, float &pa, int &E, int &F, float &mq, float &mk,
                                          float &rkmin, float &rkmax) {
    constexpr int RINGF = kRingTok * DK;    // qn follows a in the ring slot
    float xa[kSlotTok], xn[kSlotTok], xk[kSlotTok], xq[kSlotTok];
#pragma unroll
    for (int r = 0; r < kSlotTok; ++r) {
        xa[r] = ra[r * DK];
        xn[r] = ra[RINGF + r * DK];
        xk[r] = bf_at(kt, j * 1024 + offr[r]);
        xq[r] = state_mode ? 0.f : bf_at(qt, j * 1024 + offr[r]);
    }
    float bk[kSlotTok], nt[kSlotTok], pt[kSlotTok], dt[kSlotTok];
#pragma unroll
    for (int r = 0; r < kSlotTok; ++r) bk[r] = __shfl_sync(0xffffffffu, bsrc, (kSlotTok * j + r) & 31) * xk[r];
#pragma unroll
    for (int r = 0; r < kSlotTok; ++r) {
        const float at = xa[r];
        dd = fmaf(at * at, dd, xn[r] * nn);
        nn = fmaf(bk[r] * xk[r], dd, nn);
        pa *= at;
        nt[r] = nn;
        pt[r] = pa;
        dt[r] = dd;
    }
#pragma unroll
    for (int r = 0; r < kSlotTok; ++r) {
        const float rkm = (dt[r] * mk) * rcp_approx(pt[r]);      // 2^(R - G)
        rkmin = fminf(rkmin, rkm);
        rkmax = fmaxf(rkmax, rkm);
        const float ko = bk[r] * rkm;
        const uint32_t t = __float_as_uint(ko) + 0x8000u;         // K' hi, rounded
        const int off = j * 1024 + offr[r];
        *reinterpret_cast<uint16_t *>(kt + off) = (uint16_t)(t >> 16);
        *reinterpret_cast<uint16_t *>(klo + off) =
            (uint16_t)(__float_as_uint(ko - __uint_as_float(t & 0xffff0000u)) >> 16);
    }
    if (!state_mode) {
#pragma unroll
        for (int r = 0; r < kSlotTok; ++r) {
            const float qo = xq[r] * ((pt[r] * mq) * rcp_approx(nt[r]));
            *reinterpret_cast<uint16_t *>(qt + j * 1024 + offr[r]) = (uint16_t)((__float_as_uint(qo) + 0x8000u) >> 16);
        }
    }
    const int e = ((__float_as_int(dd) >> 23) & 0xff) - 127;
    const int f = ((__float_as_int(pa) >> 23) & 0xff) - 127;
    const float se = __int_as_float((127 - e) << 23);
    nn *= se;
    dd *= se;
    pa *= __int_as_float((127 - f) << 23);
    E += e;
    F += f;
    const int sh = max(-126, min(127, (F - E) - R));
    mq = __int_as_float((127 + sh) << 23);
    mk = __int_as_float((127 - sh) << 23);
}

}  // namespace

template <int DK, int DV, bool ISO, bool LOCAL>
__global__ void __launch_bounds__(Roles<DK, DV>::THREADS, Roles<DK, DV>::MIN_BLOCKS)
kla_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qs,
                    const TcArgs g) {
    using L = Layout<DK, DV>;
    using RL = Roles<DK, DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (128B-swizzle atoms), derived by pointer arithmetic
    // on the shared array so that every tile access stays a shared-space access
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar0);
    uint64_t *stage_full = bars + 0, *stage_empty = bars + 2, *qk_ready = bars + 4;
    uint64_t *ring_full = bars + 6, *ring_empty = bars + 6 + kRings;
    uint64_t *s_full = bars + 6 + 2 * kRings, *u_ready = s_full + 1, *u_done = s_full + 2, *p_full = s_full + 3;
    uint64_t *o_full = s_full + 4, *o_empty = s_full + 5, *td_bar = s_full + 6, *gate_sync = s_full + 7;
    uint64_t *gate_sync2 = s_full + 8;   // iso: the chunk's per-token factors are in shared memory
    uint32_t *tmem_hold = reinterpret_cast<uint32_t *>(sm + L::hold0);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::hold0 + 4);
    float *fac = reinterpret_cast<float *>(sm + L::fac0);
    float *fac_final = reinterpret_cast<float *>(sm + L::facf0);
    float2 *isof = reinterpret_cast<float2 *>(sm + L::isof0);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the transfer-only pass (mode 1) runs on the CUDA-core walk; this kernel
    // takes modes 0 and 2 and is instantiated per precision mode (ISO) and walk
    // mode (LOCAL), so that each variant holds only its own code
    constexpr bool state_mode = false;
    // mode 2: every segment walks from a zero state (segment 0 from eta0), writes
    // its transfer and decay, and segments p > 0 export their folded q tiles and
    // chunk references for the correction pass that adds the carried state
    constexpr bool local_mode = LOCAL;
    // one gate thread per key: each reads and rewrites only its own key column
    const int gate_threads = DK;
    const bool is_gate = (RL::NGW == 4) ? (warp < 4) : (warp == 0 || warp == 2);
    const int gt = (RL::NGW == 4) ? tid : ((warp >> 1) * 32 + lane);   // gate rank

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&stage_empty[s], 1);
            mbar_init(&qk_ready[s], gate_threads);
        }
        for (int j = 0; j < kRings; ++j) {
            mbar_init(&ring_full[j], 1);
            mbar_init(&ring_empty[j], gate_threads);
        }
        mbar_init(s_full, 1);
        mbar_init(u_ready, 128);
        mbar_init(u_done, 1);
        mbar_init(p_full, 128);
        mbar_init(o_full, 1);
        mbar_init(o_empty, 128);
        mbar_init(td_bar, 1);
        mbar_init(gate_sync, gate_threads);
        mbar_init(gate_sync2, gate_threads);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == RL::PRODW && lane == 0) {
        prefetch_map(&tm_q); prefetch_map(&tm_k); prefetch_map(&tm_v);
        if (!ISO) { prefetch_map(&tm_a); prefetch_map(&tm_qn); }
    }
    if (warp == RL::MMAW) tmem_alloc(tmem_hold, L::NCOLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_hold;
    pdl_release();
    pdl_wait();
    const int P_eff = state_mode ? g.P - 1 : g.P;
    // unit u = (row or packed sequence n, head h); packed sequences in the
    // longest-first order when one is given
    const long long ur = blockIdx.x / P_eff;
    const int p = (int)(blockIdx.x % P_eff);
    const int h = (int)(ur % g.H);
    const int n = g.perm ? g.perm[ur / g.H] : (int)(ur / g.H);
    const long long u = (long long)n * g.H + h;
    long long tb, te;
    if (g.cu) { tb = g.cu[n]; te = g.cu[n + 1]; }
    else {
        tb = (long long)n * g.T + (long long)p * g.Lseg;
        te = (long long)n * g.T + min((long long)(p + 1) * g.Lseg, g.T);
    }
    const int nchunks = te > tb ? (int)((te - tb + kC - 1) / kC) : 0;
    const bool last_seg = p == P_eff - 1;

    if (is_gate) {
      {
        // ================= gate warps: precision path and operand folding =====
        const int i = gt;                    // key owned by this thread
        const bool key = true;
        // byte offset of (row r of an 8-row group, key i) in a 64-row 128B-swizzled
        // tile; row 8j + r of the chunk is at j * 1024 + offr[r]
        int offr[kSlotTok];
#pragma unroll
        for (int r = 0; r < kSlotTok; ++r) offr[r] = sw_off(r, i, kC);
        float lam = 1.0f;
        {
            const int il = ISO ? 0 : i;
            if (key || ISO) {
                const int nl = ISO ? 1 : DK;
                lam = g.lambda0 ? g.lambda0[u * nl + il] : 1.0f;
                if (p > 0 && g.agg) {
                    // compose the Moebius aggregates of the blocks before this segment
                    // (in order) and apply them to lambda0
                    const float4 *src = g.agg + u * g.NB * nl + il;
                    const int nb = p * g.seg_blocks;
                    Mob M{1.f, 0.f, 0.f, 1.f};
                    for (int b0 = 0; b0 < nb; b0 += 16) {
                        float4 m[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r)
                            if (b0 + r < nb) m[r] = __ldg(src + (long long)(b0 + r) * nl);
#pragma unroll
                        for (int r = 0; r < 16; ++r)
                            if (b0 + r < nb) M = mob_norm(mob_mul(Mob{m[r].x, m[r].y, m[r].z, m[r].w}, M));
                    }
                    lam = mob_apply(M, lam);
                } else if (p > 0) {
                    lam = g.lam_blk[(u * g.NB + (long long)p * g.seg_blocks) * nl + il];
                }
            }
        }
        float e_prev = 1.f, log_decay = 0.f;   // e_prev = 2^(G_last - R) of the previous chunk
        bool ok = true;
        // Diagonal mode keeps the precision chain and the log-gate reference across
        // chunks: G is the cumulative log2 gate since the segment start, rho a
        // per-key integer reference that moves only when the next chunk's predicted
        // G range would leave [rho - kRebase, rho + kRebase]. The state in TMEM is
        // U = diag(2^(rho - G)) eta, so it needs no rescale while rho stays put.
        float nn = lam, dd = 1.0f, pa = 1.0f;
        int E = 0, F = 0, rho = 0, dpred = 0;
        float gprev = 0.f;
        // Per-token scalars of a chunk are loaded one chunk ahead into registers
        // and broadcast with shuffles (no global load sits on the recursion).
        // diag: beta of tokens (lane, lane+32); iso: a, qn, beta of (2 lane, 2 lane+1).
        float nb0 = 0.f, nb1 = 0.f, na0 = 1.f, na1 = 1.f, nq0 = 0.f, nq1 = 0.f;
        auto prefetch = [&](int c) {
            const long long t0 = tb + (long long)c * kC;
            const long long x0 = ISO ? t0 + 2 * lane : t0 + lane;
            const long long x1 = ISO ? x0 + 1 : t0 + 32 + lane;
            nb0 = x0 < te ? __ldg(g.beta + x0 * g.H + h) : 0.f;
            nb1 = x1 < te ? __ldg(g.beta + x1 * g.H + h) : 0.f;
            if (ISO) {
                na0 = x0 < te ? __ldg(g.a + x0 * g.H + h) : 1.f;
                na1 = x1 < te ? __ldg(g.a + x1 * g.H + h) : 1.f;
                nq0 = x0 < te ? __ldg(g.qn + x0 * g.H + h) : 0.f;
                nq1 = x1 < te ? __ldg(g.qn + x1 * g.H + h) : 0.f;
            }
        };
        if (nchunks > 0) prefetch(0);
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            const long long tok0 = tb + (long long)c * kC;
            uint8_t *qt = sm + L::q0 + s * L::QK;
            uint8_t *kt = sm + L::k0 + s * L::QK;
            const float cb0 = nb0, cb1 = nb1, ca0 = na0, ca1 = na1, cq0 = nq0, cq1 = nq1;
            if (c + 1 < nchunks) prefetch(c + 1);
            if (!waitw(&stage_full[s], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
            int R;                 // integer log2 reference of this chunk (per key)
            float fac_c = 1.f;     // diagonal mode: rescale of U at this chunk's start
            float e_cur;           // 2^(G_last - R)
            float glast_log2;      // G_last
            uint8_t *klo = sm + L::klo0 + s * L::QK;
            if (!ISO) {
                // One pass per chunk. Projective form of the precision: lambda = n/d with
                //   d <- a^2 d + qn n,  n <- n + b d   (b = beta k^2),
                // two FMAs per token on the serial chain. The gate is g = a d_prev / d,
                // so with PA = prod a the cumulative gate telescopes (d = 1 at the chunk
                // start): 2^G = PA/d and 2^G/lambda = PA/n. n, d and PA are floats times
                // 2^E (n, d) and 2^F (PA), rescaled by exact powers of two every 8 tokens.
                // The operands are written at once against the reference R predicted
                // from the previous chunk's decay; the chunk's actual G range is checked.
                const int nvalid = (int)min((long long)kC, te - tok0);
                float mq, mk;
                bool range_bad = false;
                {
                    // G at the chunk start is F - E to within one (n, d, PA are kept
                    // in [1, 2) by the per-slot rescale); dpred = the last chunk's drift
                    const int gs = F - E;
                    const int lo = gs + min(0, dpred) - 2, hi = gs + max(0, dpred) + 2;
                    int rnew = rho;
                    if (hi - rho > kRebase || rho - lo > kRebase) rnew = gs + dpred / 2;
                    fac_c = __int_as_float((127 + max(-126, min(127, rnew - rho))) << 23);
                    rho = rnew;
                    R = rho;
                    if (local_mode && p > 0)
                        g.rlog[(u * g.NC + (tok0 - tb) / kC + (long long)p * g.seg_blocks) * DK + i] = (float)R;
                    const int sh0 = max(-126, min(127, gs - R));
                    mq = __int_as_float((127 + sh0) << 23);
                    mk = __int_as_float((127 - sh0) << 23);
                }
                const int gs_chunk = F - E;
                if (nvalid == kC) {
                    // Full chunk: the chain and the operands of every slot.
                    float rkmin = 3.0e38f, rkmax = 0.f;
                    // not unrolled: one slot's code stays resident in the instruction cache
#pragma unroll 1
                    for (int j = 0; j < kSlotsPerChunk; ++j) {
                        const int n = c * kRingsPerChunk + (j >> 1), slot = n % kRings;
                        // one wait per ring slot of two gate slots
                        if (!(j & 1) && !waitw(&ring_full[slot], (n / kRings) & 1, abort_flag, g.status)) {
                            ok = false;
                            break;
                        }
                        const float *ra = reinterpret_cast<const float *>(sm + L::ring0) + slot * 2 * L::RINGF +
                                          (j & 1) * kSlotTok * DK + i;
                        const float bsrc = (j < 4) ? cb0 : cb1;
                        gate_slot<DK>(j, ra, qt, kt, klo, offr, bsrc, state_mode, R, nn, dd, pa, E, F, mq, mk, rkmin,
                                      rkmax);
                        if (j & 1) {
                            // ring slot read into registers: release it (generic reads
                            // ordered before the TMA refill)
                            fence_proxy_async();
                            mbar_arrive(&ring_empty[slot]);
                        }
                    }
                    if (!ok) break;
                    // rk = 2^(R - G): |G - R| beyond the kept range leaves the exponent window
                    range_bad = (((__float_as_int(rkmax) >> 23) & 0xff) - 127 >= kMaxOffset) ||
                                (((__float_as_int(rkmin) >> 23) & 0xff) - 127 < -kMaxOffset);
                } else {
                    // Partial chunk (end of a segment or sequence): same recursion, one
                    // slot at a time, with per-token validity.
                    int gmin = F - E, gmax = F - E;     // G at the chunk start (absolute)
#pragma unroll 1
                    for (int j = 0; j < kSlotsPerChunk; ++j) {
                        const int n = c * kRingsPerChunk + (j >> 1), slot = n % kRings;
                        if (!(j & 1) && !waitw(&ring_full[slot], (n / kRings) & 1, abort_flag, g.status)) {
                            ok = false;
                            break;
                        }
                        const float *ra = reinterpret_cast<const float *>(sm + L::ring0) + slot * 2 * L::RINGF +
                                          (j & 1) * kSlotTok * DK;
                        const float *rq = ra + L::RINGF;
                        const float bsrc = (j < 4) ? cb0 : cb1;
                        float kr[kSlotTok], qr[kSlotTok], ar[kSlotTok], qnr[kSlotTok], br[kSlotTok];
#pragma unroll
                        for (int r = 0; r < kSlotTok; ++r) {
                            const int off = j * 1024 + offr[r];
                            kr[r] = bf_at(kt, off);
                            qr[r] = state_mode ? 0.f : bf_at(qt, off);
                            ar[r] = ra[r * DK + i];
                            qnr[r] = rq[r * DK + i];
                            br[r] = __shfl_sync(0xffffffffu, bsrc, (kSlotTok * j + r) & 31);
                        }
                        if (j & 1) {
                            fence_proxy_async();
                            mbar_arrive(&ring_empty[slot]);
                        }
                        float qo[kSlotTok], ko[kSlotTok];
                        float rkmin = 3.0e38f, rkmax = 0.f;
#pragma unroll
                        for (int r = 0; r < kSlotTok; ++r) {
                            const bool valid = kSlotTok * j + r < nvalid;
                            const float at = valid ? ar[r] : 1.f;
                            const float bk = valid ? br[r] * kr[r] : 0.f;
                            dd = fmaf(at * at, dd, valid ? qnr[r] * nn : 0.f);
                            nn = fmaf(bk * kr[r], dd, nn);
                            pa *= at;
                            const float rk = __fdividef(dd, pa);
                            rkmin = fminf(rkmin, rk);
                            rkmax = fmaxf(rkmax, rk);
                            qo[r] = valid ? qr[r] * (__fdividef(pa, nn) * mq) : 0.f;
                            ko[r] = bk * (rk * mk);
                        }
                        // G = (F - E) - log2(rk); integer bounds of this slot's G range
                        gmin = min(gmin, (F - E) - (((__float_as_int(rkmax) >> 23) & 0xff) - 126));
                        gmax = max(gmax, (F - E) - (((__float_as_int(rkmin) >> 23) & 0xff) - 127));
#pragma unroll
                        for (int r = 0; r < kSlotTok; ++r) {
                            const int off = j * 1024 + offr[r];
                            if (!state_mode) bf_put(qt, off, qo[r]);
                            const __nv_bfloat16 khi = __float2bfloat16_rn(ko[r]);
                            *reinterpret_cast<__nv_bfloat16 *>(kt + off) = khi;
                            bf_put(klo, off, ko[r] - __bfloat162float(khi));
                        }
                        const int e = ((__float_as_int(dd) >> 23) & 0xff) - 127;
                        const int f = ((__float_as_int(pa) >> 23) & 0xff) - 127;
                        const float se = __int_as_float((127 - e) << 23);
                        nn *= se;
                        dd *= se;
                        pa *= __int_as_float((127 - f) << 23);
                        E += e;
                        F += f;
                        const int sh = max(-126, min(127, (F - E) - R));
                        mq = __int_as_float((127 + sh) << 23);
                        mk = __int_as_float((127 - sh) << 23);
                    }
                    if (!ok) break;
                    range_bad = gmax - R > kMaxOffset || R - gmin > kMaxOffset;
                }
                lam = nn / dd;
                const float gm = pa / dd;                 // 2^G = gm * 2^(F-E)
                const int sl = F - E;
                e_cur = gm * __int_as_float((127 + max(-126, min(127, sl - R))) << 23);   // 2^(G - rho)
                const float gnow = (float)sl + __log2f(gm);
                glast_log2 = gnow - gprev;                 // this chunk's log2 decay
                gprev = gnow;
                dpred = sl - gs_chunk;
                if (range_bad) atomicOr(g.status, kStatusRange);
            } else {
                // isotropic: one precision per head; warp-level Moebius scan over
                // the chunk (lane l owns tokens 2l, 2l+1), redundantly per warp.
                const int t0i = 2 * lane, t1i = 2 * lane + 1;
                const bool va = tok0 + t0i < te, vb = tok0 + t1i < te;
                const float inv_dk = 1.0f / (float)DK;
                const float a0 = ca0, q0 = cq0, a1 = ca1, q1 = cq1;
                const float b0 = va ? cb0 * row_sumsq<DK>(kt, t0i) * inv_dk : 0.f;
                const float b1 = vb ? cb1 * row_sumsq<DK>(kt, t1i) * inv_dk : 0.f;
                Mob Mp = mob_norm(mob_mul(mob_step(a1, q1, b1), mob_step(a0, q0, b0)));
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    Mob o = shfl_up_mob(Mp, d);
                    if (lane >= d) Mp = mob_norm(mob_mul(Mp, o));
                }
                Mob Ex = shfl_up_mob(Mp, 1);
                if (lane == 0) Ex = Mob{1.f, 0.f, 0.f, 1.f};
                const float lamA = mob_apply(Ex, lam);
                float g0 = 1.f, lamB = lamA, g1 = 1.f, lamC;
                if (va) { float rr = __frcp_rn(fmaf(a0, a0, q0 * lamA)); g0 = a0 * rr; lamB = fmaf(lamA, rr, b0); }
                lamC = lamB;
                if (vb) { float rr = __frcp_rn(fmaf(a1, a1, q1 * lamB)); g1 = a1 * rr; lamC = fmaf(lamB, rr, b1); }
                const float l0 = __log2f(g0), l1 = __log2f(g1);
                float sum = l0 + l1;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    float o = __shfl_up_sync(0xffffffffu, sum, d);
                    if (lane >= d) sum += o;
                }
                const float G1 = sum, G0 = sum - l1;
                float mn = fminf(0.f, fminf(G0, G1)), mx = fmaxf(0.f, fmaxf(G0, G1));
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, d));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
                }
                const int gmin = (int)floorf(mn), gmax = (int)ceilf(mx);
                R = (gmin + gmax) >> 1;
                const float Rf = (float)R;
                // G here runs from the chunk start: the segment-start frame adds the
                // log2 decay of the segment's earlier chunks
                if (local_mode && p > 0)
                    g.rlog[(u * g.NC + (tok0 - tb) / kC + (long long)p * g.seg_blocks) * DK + i] = Rf + log_decay;
                const float Glast = __shfl_sync(0xffffffffu, G1, 31);
                e_cur = exp2f(Glast - Rf);
                glast_log2 = Glast;
                lam = __shfl_sync(0xffffffffu, lamC, 31);
                // per-token factors, shared by all keys of the head
                if (gmax - gmin > 2 * kMaxOffset) atomicOr(g.status, kStatusRange);
                // every gate warp has read the raw k rows, and the previous chunk's
                // factors, before any of them is overwritten
                mbar_arrive(gate_sync);
                if (!waitw(gate_sync, c & 1, abort_flag, g.status)) { ok = false; break; }
                // per-token factors, shared by all keys of the head: q / lambda 2^(G-R)
                // and beta 2^(R-G), zero past the end of the sequence
                if (warp == 0) {
                    isof[t0i] = va ? make_float2(exp2f(G0 - Rf) / lamB, cb0 * exp2f(Rf - G0)) : make_float2(0.f, 0.f);
                    isof[t1i] = vb ? make_float2(exp2f(G1 - Rf) / lamC, cb1 * exp2f(Rf - G1)) : make_float2(0.f, 0.f);
                }
                mbar_arrive(gate_sync2);
                if (!waitw(gate_sync2, c & 1, abort_flag, g.status)) { ok = false; break; }
#pragma unroll 1
                for (int j = 0; j < kSlotsPerChunk; ++j) {
                    float qr[kSlotTok], kr[kSlotTok];
                    float2 fv[kSlotTok];
#pragma unroll
                    for (int r = 0; r < kSlotTok; ++r) {
                        const int off = j * 1024 + offr[r];
                        qr[r] = state_mode ? 0.f : bf_at(qt, off);
                        kr[r] = bf_at(kt, off);
                        fv[r] = isof[kSlotTok * j + r];
                    }
#pragma unroll
                    for (int r = 0; r < kSlotTok; ++r) {
                        const int off = j * 1024 + offr[r];
                        const float ko = kr[r] * fv[r].y;
                        const uint32_t t = __float_as_uint(ko) + 0x8000u;         // K' hi, rounded
                        *reinterpret_cast<uint16_t *>(kt + off) = (uint16_t)(t >> 16);
                        *reinterpret_cast<uint16_t *>(klo + off) =
                            (uint16_t)(__float_as_uint(ko - __uint_as_float(t & 0xffff0000u)) >> 16);
                        if (!state_mode)
                            *reinterpret_cast<uint16_t *>(qt + off) =
                                (uint16_t)((__float_as_uint(qr[r] * fv[r].x) + 0x8000u) >> 16);
                    }
                }
            }
            // state rescale factors: U_c = diag(2^R_c) S_c, S_{c+1} = diag(2^(G_last - R_c)) (U_c + K'^T V)
            fac[s * DK + i] = ISO ? e_prev * __int_as_float((127 + max(-126, min(127, R))) << 23) : fac_c;
            if (c == nchunks - 1) fac_final[i] = e_cur;
            e_prev = e_cur;
            log_decay += glast_log2;
            fence_proxy_async();
            mbar_arrive(&qk_ready[s]);
        }
        if (ok && !*abort_flag) {
            if (state_mode || local_mode) {
                if (ISO ? (gt == 0) : key) g.decay[(u * g.P + p) * (ISO ? 1 : DK) + (ISO ? 0 : i)] = exp2f(log_decay);
            }
            if (!state_mode && last_seg && g.final_lambda) {
                if (ISO ? (gt == 0) : key) g.final_lambda[u * (ISO ? 1 : DK) + (ISO ? 0 : i)] = lam;
            }
        }
      }
    } else if (warp >= 4 && warp < 8) {
        // ================= epilogue warps ====================================
        const int e = tid - 128, we = e >> 5, le = e & 31;
        const uint32_t lane_base = (uint32_t)(32 * we) << 16;
        const int row64 = 16 * we + le;
        const bool v64 = le < 16;
        const int rowU = (DK == 128) ? (32 * we + le) : row64;
        const bool vU = (DK == 128) || v64;
        uint8_t *ub = sm + L::ub0;
        uint8_t *pt = sm + L::p0;
        const float *eta0 = (!state_mode && (!local_mode || p == 0) && g.eta0) ? g.eta0 + u * DK * DV : nullptr;
        bool ok = true;
        // Belief at the segment start, written into the U columns of TMEM before
        // the first chunk (while the gate works on it): eta0 for whole rows and
        // first segments, zero for the later segments of split rows (their
        // carried state is added by the correction pass)
        if (!state_mode && nchunks > 0) {
#pragma unroll
            for (int cb = 0; cb < DV / 32; ++cb) {
                float acc[32];
#pragma unroll
                for (int x = 0; x < 32; x += 4) {
                    const float4 e4 = (vU && eta0) ? *reinterpret_cast<const float4 *>(eta0 + rowU * DV + cb * 32 + x)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                    acc[x] = e4.x; acc[x + 1] = e4.y; acc[x + 2] = e4.z; acc[x + 3] = e4.w;
                }
                uint32_t r[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(acc[x]);
                tmem_st32(tbase + lane_base + L::colU + cb * 32, r);
            }
            tmem_wait_st();
        }
        // output rows of chunk cc (TMEM O -> bf16 -> global)
        auto emit_out = [&](int cc) -> bool {
            if (!waitw(o_full, cc & 1, abort_flag, g.status)) return false;
            tc_fence_after();
            const long long tok0 = tb + (long long)cc * kC;
            const bool row_ok = v64 && (tok0 + row64 < te);
            __nv_bfloat16 *orow = g.out + ((tok0 + row64) * g.H + h) * DV;
#pragma unroll
            for (int cb = 0; cb < DV / 32; cb += 2) {
                uint32_t rr[2][32];
                tmem_ld32(tbase + lane_base + L::colO + cb * 32, rr[0]);
                tmem_ld32(tbase + lane_base + L::colO + cb * 32 + 32, rr[1]);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t *r = rr[hh];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 w;
                            w.x = pack_bf2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                            w.y = pack_bf2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                            w.z = pack_bf2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                            w.w = pack_bf2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                            *reinterpret_cast<uint4 *>(orow + (cb + hh) * 32 + q4 * 8) = w;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(o_empty);
            return true;
        };
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            // ---- output rows of the previous chunk (its MMAs finished meanwhile)
            if (!state_mode && c > 0 && !emit_out(c - 1)) { ok = false; break; }
            // ---- state U_c = diag(fac) * (eta_start or U_{c-1} + K'^T V)
            if (!waitw(&qk_ready[s], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
            if (c > 0 && !waitw(u_done, (c - 1) & 1, abort_flag, g.status)) { ok = false; break; }
            tc_fence_after();
            // diag: f = 1 unless the gate moved this key's reference; the warp then
            // only snapshots U (bf16, for the readout MMA) without rewriting TMEM
            const float f = vU ? fac[s * DK + rowU] : 1.f;
            const bool rmw = (c == 0) || __any_sync(0xffffffffu, f != 1.0f);
            auto snap = [&](const uint32_t (&r)[32], int cb) {
                if (!state_mode && vU) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 w;
                        w.x = pack_bf2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                        w.y = pack_bf2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                        w.z = pack_bf2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                        w.w = pack_bf2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                        *reinterpret_cast<uint4 *>(ub + sw_off(rowU, cb * 32 + q4 * 8, DK)) = w;
                    }
                }
            };
            if (c == 0 && state_mode) {
#pragma unroll
                for (int cb = 0; cb < DV / 32; ++cb) {
                    uint32_t r[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = 0u;
                    tmem_st32(tbase + lane_base + L::colU + cb * 32, r);
                }
            } else if (rmw || !state_mode) {
#pragma unroll
                for (int cb = 0; cb < DV / 32; cb += 2) {
                    uint32_t r0[32], r1[32];
                    const uint32_t ta = tbase + lane_base + L::colU + cb * 32;
                    tmem_ld32(ta, r0);
                    tmem_ld32(ta + 32, r1);
                    tmem_wait_ld();
                    if (rmw) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            r0[x] = __float_as_uint(__uint_as_float(r0[x]) * f);
                            r1[x] = __float_as_uint(__uint_as_float(r1[x]) * f);
                        }
                        tmem_st32(ta, r0);
                        tmem_st32(ta + 32, r1);
                    }
                    snap(r0, cb);
                    snap(r1, cb + 1);
                }
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(u_ready);
            if (state_mode) continue;
            // ---- P = causal mask of the score tile, bf16
            if (!waitw(s_full, c & 1, abort_flag, g.status)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(tbase + lane_base + L::colS, r0);
                tmem_ld32(tbase + lane_base + L::colS + 32, r1);
                tmem_wait_ld();
                if (v64) {
                    const int tau = row64;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float x[8];
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2) {
                            const int sg = ch * 8 + e2;
                            const float sv = __uint_as_float(sg < 32 ? r0[sg] : r1[sg - 32]);
                            x[e2] = sg <= tau ? sv : 0.f;
                        }
                        uint4 w;
                        w.x = pack_bf2(x[0], x[1]); w.y = pack_bf2(x[2], x[3]);
                        w.z = pack_bf2(x[4], x[5]); w.w = pack_bf2(x[6], x[7]);
                        *reinterpret_cast<uint4 *>(pt + tau * 128 + ((ch ^ (tau & 7)) << 4)) = w;
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && !state_mode && nchunks > 0 && !emit_out(nchunks - 1)) ok = false;
        // ---- final belief (last segment) or segment transfer (state mode)
        float *dst = nullptr;
        if (state_mode || local_mode) dst = g.S_io + (u * g.P + p) * DK * DV;
        else if (last_seg && g.final_eta) dst = g.final_eta + u * DK * DV;
        if (ok && dst && !*abort_flag) {
            if (nchunks > 0) {
                if (waitw(u_done, (nchunks - 1) & 1, abort_flag, g.status)) {
                    tc_fence_after();
                    const float ff = vU ? fac_final[rowU] : 0.f;
#pragma unroll
                    for (int cb = 0; cb < DV / 32; ++cb) {
                        uint32_t r[32];
                        tmem_ld32(tbase + lane_base + L::colU + cb * 32, r);
                        tmem_wait_ld();
                        if (vU) {
                            float4 *d4 = reinterpret_cast<float4 *>(dst + rowU * DV + cb * 32);
#pragma unroll
                            for (int x = 0; x < 8; ++x)
                                d4[x] = make_float4(__uint_as_float(r[4 * x]) * ff, __uint_as_float(r[4 * x + 1]) * ff,
                                                    __uint_as_float(r[4 * x + 2]) * ff, __uint_as_float(r[4 * x + 3]) * ff);
                        }
                    }
                }
            } else if (vU) {
                // no tokens (an empty packed sequence, a single segment): the belief is eta0
                for (int x = 0; x < DV; ++x) dst[rowU * DV + x] = eta0 ? eta0[rowU * DV + x] : 0.f;
            }
        }
    } else if (warp == RL::PRODW) {
        // ================= TMA producer =====================================
        if (lane == 0) {
            int last_ring[kRings], last_stage[2] = {-1, -1};
            for (int j = 0; j < kRings; ++j) last_ring[j] = -1;
            bool ok = true;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int tok0 = (int)(tb + (long long)c * kC);
                const int s = c & 1;
                if (c >= 2 && !wait1(&stage_empty[s], ((c >> 1) - 1) & 1, abort_flag, g.status)) { ok = false; break; }
                mbar_expect_tx(&stage_full[s], (state_mode ? 0 : L::QK) + L::QK + L::V);
#pragma unroll
                for (int a = 0; a < DK / 64; ++a) {
                    if (!state_mode)
                        tma_load_3d(sm + L::q0 + s * L::QK + a * kC * 128, &tm_q, &stage_full[s], 64 * a, h, tok0);
                    tma_load_3d(sm + L::k0 + s * L::QK + a * kC * 128, &tm_k, &stage_full[s], 64 * a, h, tok0);
                }
#pragma unroll
                for (int a = 0; a < DV / 64; ++a)
                    tma_load_3d(sm + L::v0 + s * L::V + a * kC * 128, &tm_v, &stage_full[s], 64 * a, h, tok0);
                last_stage[s] = c;
                // L2 prefetch of the chunk two ahead, so that the TMA copies above
                // and the ring refills below are served from L2
                if (c + 2 < nchunks) {
                    const int tp = tok0 + 2 * kC;
#pragma unroll
                    for (int a = 0; a < DK / 64; ++a) {
                        if (!state_mode) tma_prefetch_3d(&tm_q, 64 * a, h, tp);
                        tma_prefetch_3d(&tm_k, 64 * a, h, tp);
                    }
#pragma unroll
                    for (int a = 0; a < DV / 64; ++a) tma_prefetch_3d(&tm_v, 64 * a, h, tp);
                    if (!ISO)
                        for (int j = 0; j < kRingsPerChunk; ++j) {
                            tma_prefetch_3d(&tm_a, 0, h, tp + kRingTok * j);
                            tma_prefetch_3d(&tm_qn, 0, h, tp + kRingTok * j);
                        }
                }
                if (!ISO) {
                    for (int j = 0; j < kRingsPerChunk; ++j) {
                        const int n = c * kRingsPerChunk + j, slot = n % kRings;
                        if (n >= kRings && !wait1(&ring_empty[slot], ((n / kRings) - 1) & 1, abort_flag, g.status)) {
                            ok = false;
                            break;
                        }
                        float *ra = reinterpret_cast<float *>(sm + L::ring0) + slot * 2 * L::RINGF;
                        mbar_expect_tx(&ring_full[slot], 2 * L::RINGF * 4);
                        tma_load_3d(ra, &tm_a, &ring_full[slot], 0, h, tok0 + kRingTok * j);
                        tma_load_3d(ra + L::RINGF, &tm_qn, &ring_full[slot], 0, h, tok0 + kRingTok * j);
                        last_ring[slot] = n;
                    }
                }
            }
            if (!ok || *abort_flag) {
                // wait (bounded) until every copy this thread issued has landed
                for (int j = 0; j < kRings; ++j)
                    if (last_ring[j] >= 0)
                        wait_slow(&ring_full[j], (last_ring[j] / kRings) & 1, abort_flag, g.status, false);
                for (int s = 0; s < 2; ++s)
                    if (last_stage[s] >= 0)
                        wait_slow(&stage_full[s], (last_stage[s] >> 1) & 1, abort_flag, g.status, false);
            }
        }
    } else if (warp == RL::MMAW) {
        // ================= MMA issuer =======================================
        if (lane == 0) {
            constexpr uint32_t iS = idesc_bf16(64, 64, false, false);
            constexpr uint32_t iO = idesc_bf16(64, DV, false, true);
            constexpr uint32_t iU = idesc_bf16(DK, DV, true, true);
            const uint32_t tS = tbase + L::colS, tO = tbase + L::colO, tU = tbase + L::colU;
            const uint32_t pa = smem_u32(sm + L::p0), uba = smem_u32(sm + L::ub0);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (!wait1(&qk_ready[s], (c >> 1) & 1, abort_flag, g.status)) break;
                tc_fence_after();
                const uint32_t qa = smem_u32(sm + L::q0 + s * L::QK);
                const uint32_t ka = smem_u32(sm + L::k0 + s * L::QK);
                const uint32_t va = smem_u32(sm + L::v0 + s * L::V);
                const uint32_t kloa = smem_u32(sm + L::klo0 + s * L::QK);
                if (local_mode && p > 0) {
                    // export the folded q tile (the correction pass multiplies it by the
                    // carried segment-start state)
                    const int tok0 = (int)(tb + (long long)c * kC);
#pragma unroll
                    for (int a = 0; a < DK / 64; ++a)
                        tma_store_3d(&tm_qs, sm + L::q0 + s * L::QK + a * kC * 128, 64 * a, h, tok0);
                    tma_store_commit();
                }
                if (!state_mode) {
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * (kC * 128) + (kk & 3) * 32;
                        mma_bf16(tS, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), iS, kk > 0);
                    }
                    mma_commit(s_full);
                }
                if (!wait1(u_ready, c & 1, abort_flag, g.status)) break;
                tc_fence_after();
                if (!state_mode) {
                    // O of the previous chunk has been read out by the epilogue
                    if (c > 0 && !wait1(o_empty, (c - 1) & 1, abort_flag, g.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * (kC * 128) + (kk & 3) * 32;
                        mma_bf16(tO, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(uba + kk * 2048, DK * 128, 1024), iO,
                                 kk > 0);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk) {
                    const uint64_t bv = sdesc_sw128(va + kk * 2048, kC * 128, 1024);
                    mma_bf16(tU, sdesc_sw128(ka + kk * 2048, kC * 128, 1024), bv, iU, 1);
                    mma_bf16(tU, sdesc_sw128(kloa + kk * 2048, kC * 128, 1024), bv, iU, 1);
                }
                mma_commit(u_done);
                if (!state_mode) {
                    if (!wait1(p_full, c & 1, abort_flag, g.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kC / 16; ++kk)
                        mma_bf16(tO, sdesc_sw128(pa + kk * 32, 16, 1024), sdesc_sw128(va + kk * 2048, kC * 128, 1024),
                                 iO, 1);
                    mma_commit(o_full);
                }
                // the stage is refilled only after the q' export read it
                if (local_mode && p > 0) tma_store_wait_read();
                mma_commit(&stage_empty[s]);
            }
            if (local_mode && p > 0) tma_store_wait_all();
            // all MMAs this thread issued have completed before TMEM is released
            mma_commit(td_bar);
            wait_slow(td_bar, 0, abort_flag, g.status, false);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == RL::MMAW) tmem_dealloc(tbase, L::NCOLS);
}

// ---- host side ---------------------------------------------------------------

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

// 3-D map over [ntok][H][inner] (inner contiguous) with box (box_inner, 1, box_rows).
bool make_tma_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int inner, int H,
                  long long ntok, int box_inner, int box_rows, bool swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)box_rows};
    cuuint32_t es[3] = {1u, 1u, 1u};
    CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

template <int DK, int DV>
cudaError_t launch_t(const Plan &p, const int *cu, int mode, const void *q, const void *k, const void *v,
                     const float *a, const float *qn, const float *beta, const float *lambda0, const float *eta0,
                     const float *lam_blk, float *S_io, float *decay, void *out, float *final_lambda,
                     float *final_eta, int *status, cudaStream_t st) {
    using L = Layout<DK, DV>;
    CUtensorMap mq, mk, mv, ma, mqn, mqs;
    const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    bool ok = make_tma_map(&mq, q, BF, 2, DK, p.H, p.ntok, 64, kC, true) &&
              make_tma_map(&mk, k, BF, 2, DK, p.H, p.ntok, 64, kC, true) &&
              make_tma_map(&mv, v, BF, 2, DV, p.H, p.ntok, 64, kC, true);
    if (ok && !p.iso)
        ok = make_tma_map(&ma, a, F32, 4, DK, p.H, p.ntok, DK, kRingTok, false) &&
             make_tma_map(&mqn, qn, F32, 4, DK, p.H, p.ntok, DK, kRingTok, false);
    else { ma = mq; mqn = mq; }
    if (ok && mode == 2) ok = make_tma_map(&mqs, p.qbuf, BF, 2, DK, p.H, p.ntok, 64, kC, true);
    else mqs = mq;
    if (!ok) return cudaErrorInvalidValue;
    if (mode != 0 && mode != 2) return cudaErrorInvalidValue;
    static bool attr[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr[dev]) {
        void (*const kerns[4])(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                               TcArgs) = {kla_chunk_tc_kernel<DK, DV, false, false>,
                                          kla_chunk_tc_kernel<DK, DV, false, true>,
                                          kla_chunk_tc_kernel<DK, DV, true, false>,
                                          kla_chunk_tc_kernel<DK, DV, true, true>};
        for (auto kern : kerns) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::alloc);
            if (e != cudaSuccess) return e;
        }
        attr[dev] = true;
    }
    TcArgs g;
    g.N = p.N; g.H = p.H; g.P = p.P; g.NB = p.NB; g.seg_blocks = p.seg_blocks; g.iso = p.iso; g.mode = mode;
    g.T = p.T; g.Lseg = p.Lseg; g.cu = cu; g.perm = cu ? p.perm : nullptr;
    g.a = a; g.qn = qn; g.beta = beta; g.lambda0 = lambda0; g.eta0 = eta0; g.lam_blk = lam_blk;
    g.agg = p.inline_carry ? p.agg : nullptr;
    g.rlog = p.rlog; g.NC = p.NB;
    g.S_io = S_io; g.decay = decay; g.out = (__nv_bfloat16 *)out;
    g.final_lambda = final_lambda; g.final_eta = final_eta; g.status = status;
    const long long segs = p.P;
    const unsigned grid = (unsigned)((long long)p.N * p.H * segs);
    if (grid == 0) return cudaSuccess;
    auto kern = p.iso ? (mode == 2 ? kla_chunk_tc_kernel<DK, DV, true, true> : kla_chunk_tc_kernel<DK, DV, true, false>)
                      : (mode == 2 ? kla_chunk_tc_kernel<DK, DV, false, true>
                                   : kla_chunk_tc_kernel<DK, DV, false, false>);
    return launch_pdl(kern, grid, Roles<DK, DV>::THREADS, L::alloc, st, mq, mk, mv, ma, mqn,
                      mqs, g);
}

}  // namespace

bool chunk_tc_supported(const Plan &p) {
    const char *env = getenv("KLA_DISABLE_TC");
    if (env && *env && *env != '0') return false;
    return p.bf16 && (p.dk == 64 || p.dk == 128) && (p.dv == 64 || p.dv == 128) && p.ntok < (1LL << 31);
}

cudaError_t launch_chunk_tc(const Plan &p, const int *cu, int mode, const void *q, const void *k, const void *v,
                            const float *a, const float *qn, const float *beta, const float *lambda0,
                            const float *eta0, const float *lam_blk, float *S_io, float *decay, void *out,
                            float *final_lambda, float *final_eta, int *status, cudaStream_t st) {
#define KLA_TC_CASE(DK_, DV_)                                                                                  \
    if (p.dk == DK_ && p.dv == DV_)                                                                            \
        return launch_t<DK_, DV_>(p, cu, mode, q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay, out, \
                                  final_lambda, final_eta, status, st);
    KLA_TC_CASE(64, 64)
    KLA_TC_CASE(64, 128)
    KLA_TC_CASE(128, 64)
    KLA_TC_CASE(128, 128)
#undef KLA_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kla
