// kla_chunk_tc.cu -- the chunked form of the filter's mean path on tcgen05
// tensor cores (sm_100a).
//
// Once the precision path is known, the information-vector update is affine in
// eta with a per-key, data-dependent gate (Kalman Linear Attention, technical
// summary sections 2-3: after the Moebius scan the mean recursion is a
// parallelisable affine map; the forget gate g = a/(a^2 + qn*lambda) comes from
// precision ratios). It is gated linear attention with
//     q~ = q / lambda,  k~ = beta * k,  gate g[t,i] = a/(a^2 + qn*lambda_{t-1}).
// With G[t,i] the cumulative log2 gate since the segment start and a per-key
// integer reference rho[i] (the frame of the state):
//     Q'[t,i] = q~[t,i] 2^(G[t,i]-rho[i]),   K'[s,i] = k~[s,i] 2^(rho[i]-G[s,i])
//     U       = diag(2^(rho - G_chunk_start)) eta_chunk_start      (state, TMEM fp32)
//     out     = mask_causal(Q' K'^T) V + Q' U                       (tcgen05, TMEM fp32)
//     U      += K'^T V                                              (tcgen05, TMEM fp32)
// The state never leaves the SM while a CTA walks its segment: it lives in
// TMEM as the accumulator of the K'^T V products (the pages' kernels likewise
// avoid expanding the state in HBM).
//
// The reference: every factor 2^(+-(G - rho)) must stay inside the fp32/bf16
// exponent window. The gate warps compute the chunk's whole precision chain
// first, so the chunk's actual G range per key is known before any operand is
// folded. The reference stays where it is while that range fits within
// kStick of it (then the state needs no rescale); otherwise it moves to the
// range's midpoint. A chunk whose range spans more than 2 kLim for some key is
// processed as two passes of 32 tokens or four of 16, each with its own
// reference per key, the state rescaled between them (strong forgetting inside
// a chunk). A 16-token quarter spanning more than 2 kLim is outside what the
// factorised form represents: KLA_ERR_RANGE.
//
// CTA = one segment of one (row or packed sequence, head); 448 threads:
//   warps 0-7   gate. Diagonal precision: thread = (key pair, sub-block of 16
//               tokens at dk = 128, 8 at dk = 64). Each thread composes its
//               sub-block's Moebius matrices for its two keys, the matrices
//               are exchanged through shared memory, each thread walks its
//               sub-block from the exact start precision and forms the raw
//               operand factors, the per-key G ranges are exchanged, the
//               references chosen, and the thread writes Q', K' (bf16 hi) and
//               the bf16 remainder of K' over the TMA-loaded tiles.
//               Isotropic precision: warp 0 scans the chunk's 64 Moebius maps
//               with shuffles; all eight warps fold the rows.
//   warps 8-11  epilogue: rescale U in TMEM and snapshot it to bf16 shared
//               memory, mask the score tile into P, store the output rows;
//   warp 12     TMA producer (q, k, v tiles double-buffered; L2 prefetch of
//               later chunks, a and qn included);
//   warp 13     TMEM owner and single-thread tcgen05.mma issuer.
// mode 0 walks whole rows or packed sequences (from lambda0, eta0); mode 2
// walks every segment of split rows from a zero state (segment 0 from eta0)
// and exports what the correction pass needs. The kernel is instantiated per
// (dk, dv, isotropic or diagonal precision, walk mode).
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

constexpr int kC = 64;        // chunk tokens
constexpr int kQ = 16;        // tokens per pass quarter
constexpr int kLim = 80;      // |G - rho| (log2) a pass keeps inside the exponent window
constexpr int kStick = 48;    // the reference stays while the range fits [rho - kStick, rho + kStick]
constexpr int kLost = 100;    // the fold against the reference in force is exact while |G - rho| <= kLost
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kGateBar = 1;   // named barrier of the gate warps
constexpr int kEpiBar = 2;    // named barrier of the epilogue warps

template <int DK, int DV>
struct Roles {
    static constexpr int NGW = 8;                     // gate warps
    static constexpr int GT = NGW * 32;               // gate threads
    static constexpr int EPIW = 8;                    // first epilogue warp (TMEM lane quarter 0)
    static constexpr int THREADS = 12 * 32;           // 12 warps: up to 168 registers per thread
    static constexpr int MIN_BLOCKS = 1;
    // diagonal gate: sub-blocks per chunk and their length
    static constexpr int NSUB = (DK == 128) ? 4 : 8;
    static constexpr int SL = kC / NSUB;
};

struct TcArgs {
    int N, H, P, NB, seg_blocks, NC;
    long long T, Lseg;
    const int *cu, *perm;
    const float *a, *qn, *beta;
    const float *lambda0, *eta0, *lam_blk;
    const void *q, *k;   // inputs (the strong-forgetting re-walk reloads them)
    const float4 *agg;   // block aggregates when the segment-start precision is composed here
    float *S_io, *decay;
    __nv_bfloat16 *out;
    float *final_lambda, *final_eta;
    int *status;
    // mode 2: per chunk, pass quarter and key, the reference rho of the folded
    // q' (segment-start frame): rlog[((u * NC + chunk of the row) * 4 + quarter) * DK + key]
    float *rlog;
};

template <int DK, int DV>
struct Layout {
    static constexpr int QK = kC * DK * 2;
    static constexpr int V = kC * DV * 2;
    static constexpr int PT = kC * kC * 2;
    static constexpr int UB = DK * DV * 2;
    static constexpr int XN = 512;                   // sub-blocks x keys of the diagonal gate (NSUB * DK)
    static constexpr int q0 = 0;
    static constexpr int k0 = q0 + 2 * QK;
    static constexpr int v0 = k0 + 2 * QK;
    static constexpr int klo0 = v0 + 2 * V;          // low bf16 part of K' (state update), per stage
    static constexpr int p0 = klo0 + 2 * QK;
    static constexpr int ub0 = p0 + 2 * PT;         // (P double-buffered by pass)
    static constexpr int xch0 = ub0 + UB;            // [NSUB][DK] {float4 matrix, float4 {PA, EM, FM, -}}
    static constexpr int rng0 = xch0 + XN * 32;      // [NSUB][DK] int2 G range
    static constexpr int car0 = rng0 + XN * 8;       // [2][DK] chunk-start state {float4 n,d,pa; int4 E,F}
    static constexpr int fac0 = car0 + 2 * DK * 32;  // [2][4][DK] int: U rescale exponent at each pass quarter
    static constexpr int facf0 = fac0 + 2 * kQuarters * DK * 4;   // [DK] float: 2^(G_end - rho_end)
    static constexpr int isof0 = facf0 + DK * 4;     // [2][kC] float2: iso per-token factors
    static constexpr int lvl0 = isof0 + 2 * kC * 8;  // int[2]: pass level of the chunk, tagged with its index
    static constexpr int bar0 = lvl0 + 16;
    static constexpr int NBAR = 9;
    static constexpr int hold0 = bar0 + NBAR * 8;
    static constexpr int bytes = hold0 + 16;
    static constexpr int alloc = bytes + 1024;
    static_assert(alloc <= 232448, "shared memory per CTA");
    static_assert(Roles<DK, DV>::MIN_BLOCKS == 1 || 2 * (alloc + 1024) <= 233472, "two CTAs per SM");
    // TMEM columns: the state U, two output accumulators (by pass), the scores
    static constexpr uint32_t NCOLS = (3 * DV + 64 <= 256) ? 256u : 512u;
    static constexpr uint32_t colU = 0, colO = DV, colS = 3 * DV;
};

// Byte offset of element (row, col) in a 128B-swizzled bf16 tile stored as
// 64-column atoms of `rows` rows of 128 bytes (rows 1024-byte aligned groups).
__device__ __forceinline__ int sw_off(int row, int col, int rows) {
    return (col >> 6) * (rows * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1);
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ int expo(float x) { return ((__float_as_int(x) >> 23) & 0xff) - 127; }
// 2^e for e in [-126, 127]
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }
__device__ __forceinline__ int clampe(int e) { return max(-126, min(126, e)); }
// Multiplies the DV state columns of this thread's TMEM lane by 2^d (the
// reference of the lane's key moved). Warp-collective (every lane calls it, d
// = 0 where nothing moves). Out of line: it is rare, and keeping it out of
// the epilogue's loop body keeps the hot code small.
template <int DV>
__device__ __noinline__ void tmem_scale_lane(uint32_t taddr, int d) {
    const float f1 = pow2i(d / 2), f2 = pow2i(d - d / 2);
#pragma unroll 1
    for (int cb = 0; cb < DV / 32; ++cb) {
        uint32_t r[32];
        tmem_ld32(taddr + cb * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * f1 * f2);
        tmem_st32(taddr + cb * 32, r);
    }
    tmem_wait_st();
}

// R[q] for a runtime q without indexing the array (it stays in registers)
__device__ __forceinline__ int pick4(const int (&R)[4], int q) {
    return q == 0 ? R[0] : (q == 1 ? R[1] : (q == 2 ? R[2] : R[3]));
}
// x * 2^e for |e| <= 252, exact while the result is a normal float
__device__ __forceinline__ float scale2(float x, int e) {
    const int e1 = e / 2;
    return x * pow2i(e1) * pow2i(e - e1);
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
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = unpack_bf2(w[e]);
                s = fmaf(f.x, f.x, s);
                s = fmaf(f.y, f.y, s);
            }
        }
    }
    return s;
}

// ---- reference choice ------------------------------------------------------

__device__ __forceinline__ int2 runion(int2 a, int2 b) { return make_int2(min(a.x, b.x), max(a.y, b.y)); }
__device__ __forceinline__ int rspan(int2 a) { return a.y - a.x; }
__device__ __forceinline__ bool rfits(int2 a, int r) { return a.x >= r - kStick && a.y <= r + kStick; }
__device__ __forceinline__ int rmid(int2 a) { return (a.x + a.y) >> 1; }

// The references of one key for the four pass quarters of a chunk, from the
// integer bounds qr[q] of G over each quarter (including the value just before
// it) and the reference rho in force: level 0 = one pass (span <= 2 kLim),
// 1 = two passes of 32 tokens, 2 = four passes of 16. `bad` when a quarter's
// own span exceeds the window.
__device__ __forceinline__ int choose_refs(const int2 (&qr)[4], int rho, int (&R)[4], bool &bad) {
    const int2 h0 = runion(qr[0], qr[1]), h1 = runion(qr[2], qr[3]);
    const int2 all = runion(h0, h1);
    bad = false;
    if (rspan(all) <= 2 * kLim) {
        const int r = rfits(all, rho) ? rho : rmid(all);
        R[0] = R[1] = R[2] = R[3] = r;
        return 0;
    }
    if (rspan(h0) <= 2 * kLim && rspan(h1) <= 2 * kLim) {
        const int ra = rfits(h0, rho) ? rho : rmid(h0);
        const int rb = rfits(h1, ra) ? ra : rmid(h1);
        R[0] = R[1] = ra;
        R[2] = R[3] = rb;
        return 1;
    }
    int prev = rho;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        R[q] = rfits(qr[q], prev) ? prev : rmid(qr[q]);
        prev = R[q];
        bad |= rspan(qr[q]) > 2 * kLim;
    }
    return 2;
}

// Normalises a 2x2 map (two columns) of one key by the power of two of its
// largest entry; the exponent goes to `e`.
__device__ __forceinline__ void norm_cols(float &n1, float &n2, float &d1, float &d2, int &e) {
    const int x = clampe(expo(fmaxf(fmaxf(n1, n2), fmaxf(d1, d2))));
    const float s = pow2i(-x);
    n1 *= s; n2 *= s; d1 *= s; d2 *= s;
    e += x;
}
// Normalises the projective precision (n, d) by the power of two of d and the
// gate product pa by its own.
__device__ __forceinline__ void norm_state(float &n, float &d, float &pa, int &E, int &F) {
    const int e = clampe(expo(d)), f = clampe(expo(pa));
    const float se = pow2i(-e);
    n *= se;
    d *= se;
    pa *= pow2i(-f);
    E += e;
    F += f;
}

// The strong-forgetting path of the diagonal gate: walks a sub-block of SL
// tokens again from its start state and folds every token against the
// references R0, R1 of its two keys (a, qn, beta, q, k reloaded from global
// memory: the tile words were overwritten by the provisional fold). Out of line:
// it runs only when a provisional fold lost bits.
template <int DK, int SL>
__device__ __noinline__ void rewalk_fold(uint8_t *qt, uint8_t *kt, uint8_t *klo, int cbase, float2 n2s, float2 d2s,
                                         float2 p2s, int Ew0, int Ew1, int Fw0, int Fw1, int R0, int R1,
                                         const float *a, const float *qn, const float *beta, const __nv_bfloat16 *q,
                                         const __nv_bfloat16 *k, long long tok0, int nval, int H, int h, int i0) {
    int e0 = clampe(Fw0 - Ew0 - R0), e1 = clampe(Fw1 - Ew1 - R1);
    float2 mq = make_float2(pow2i(e0), pow2i(e1)), mk = make_float2(pow2i(-e0), pow2i(-e1));
#pragma unroll 1
    for (int r = 0; r < SL; ++r) {
        const long long tok = tok0 + r;
        const long long off = (tok * H + h) * DK + i0;
        float2 ar = make_float2(1.f, 1.f), qr = make_float2(0.f, 0.f), kf = qr, qf = qr;
        float be = 0.f;
        if (r < nval) {
            ar = __ldg(reinterpret_cast<const float2 *>(a + off));
            qr = __ldg(reinterpret_cast<const float2 *>(qn + off));
            kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(k + off));
            qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(q + off));
            be = __ldg(beta + tok * H + h);
        }
        const float2 bk = f2mul(make_float2(be, be), kf);
        d2s = f2fma(f2mul(ar, ar), d2s, f2mul(qr, n2s));
        n2s = f2fma(f2mul(bk, kf), d2s, n2s);
        p2s = f2mul(p2s, ar);
        const float2 pn = f2mul(p2s, n2s);
        const float2 rc = make_float2(__frcp_rn(pn.x), __frcp_rn(pn.y));
        const float2 qo = f2mul(f2mul(f2mul(qf, p2s), f2mul(p2s, rc)), mq);
        const float2 ko = f2mul(bk, f2mul(f2mul(d2s, f2mul(n2s, rc)), mk));
        const uint32_t kh = pack_bf2(ko.x, ko.y);
        const float2 khf = unpack_bf2(kh);
        const int o = (cbase + r * 128) ^ ((r & 7) << 4);
        *reinterpret_cast<uint32_t *>(qt + o) = pack_bf2(qo.x, qo.y);
        *reinterpret_cast<uint32_t *>(kt + o) = kh;
        *reinterpret_cast<uint32_t *>(klo + o) = pack_bf2(ko.x - khf.x, ko.y - khf.y);
        if ((r & 7) == 7) {
            norm_state(n2s.x, d2s.x, p2s.x, Ew0, Fw0);
            norm_state(n2s.y, d2s.y, p2s.y, Ew1, Fw1);
            e0 = clampe(Fw0 - Ew0 - R0);
            e1 = clampe(Fw1 - Ew1 - R1);
            mq = make_float2(pow2i(e0), pow2i(e1));
            mk = make_float2(pow2i(-e0), pow2i(-e1));
        }
    }
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
    uint64_t *stage_full = bars + 0, *qk_ready = bars + 2;
    // o_full[b]: the MMAs of the pass that used output accumulator b (one barrier
    // per accumulator, so that a pass's completion is waited for before the
    // barrier can complete again)
    uint64_t *s_full = bars + 4, *u_done = bars + 5, *td_bar = bars + 6, *o_full = bars + 7;
    uint32_t *tmem_hold = reinterpret_cast<uint32_t *>(sm + L::hold0);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::hold0 + 4);
    int *lvl = reinterpret_cast<int *>(sm + L::lvl0);
    int *facd = reinterpret_cast<int *>(sm + L::fac0);
    float *facf = reinterpret_cast<float *>(sm + L::facf0);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&qk_ready[s], RL::GT);
            lvl[s] = -1;
        }
        mbar_init(s_full, 1);
        mbar_init(u_done, 1);
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        mbar_init(td_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == RL::EPIW && lane == 0) {
        prefetch_map(&tm_q); prefetch_map(&tm_k); prefetch_map(&tm_v);
        if (!ISO) { prefetch_map(&tm_a); prefetch_map(&tm_qn); }
    }
    if (warp == RL::EPIW) tmem_alloc(tmem_hold, L::NCOLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_hold;
    pdl_release();
    pdl_wait();
    // unit u = (row or packed sequence n, head h); packed sequences in the
    // longest-first order when one is given
    const long long ur = blockIdx.x / g.P;
    const int p = (int)(blockIdx.x % g.P);
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
    const bool last_seg = p == g.P - 1;
    // chunk index of the row (for the exported references)
    const long long chunk_base = (long long)p * g.seg_blocks;

    // precision at the segment start, key i (iso: i = 0)
    auto seg_lambda = [&](int i) -> float {
        const int nl = ISO ? 1 : DK;
        float lam = g.lambda0 ? g.lambda0[u * nl + i] : 1.0f;
        if (p > 0 && g.agg) {
            // compose the Moebius aggregates of the blocks before this segment
            // (in order) and apply them to lambda0
            const float4 *src = g.agg + u * g.NB * nl + i;
            const int nb = p * g.seg_blocks;
            Mob M{1.f, 0.f, 0.f, 1.f};
            for (int b0 = 0; b0 < nb; b0 += 8) {
                float4 m[8];
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (b0 + r < nb) m[r] = __ldg(src + (long long)(b0 + r) * nl);
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (b0 + r < nb) M = mob_norm(mob_mul(Mob{m[r].x, m[r].y, m[r].z, m[r].w}, M));
            }
            lam = mob_apply(M, lam);
        } else if (p > 0) {
            lam = g.lam_blk[(u * g.NB + (long long)p * g.seg_blocks) * nl + i];
        }
        return lam;
    };

    if (warp < RL::NGW) {
        // ================= gate warps: precision path and operand folding =====
        bool ok = true;
        if constexpr (!ISO) {
            constexpr int NSUB = RL::NSUB, SL = RL::SL, NP = DK / 2;
            const int s = (DK == 128) ? (warp >> 1) : warp;           // sub-block
            const int pr = (DK == 128) ? ((warp & 1) * 32 + lane) : lane;   // key pair
            const int i0 = 2 * pr;
            const int quarter = (SL * s) / kQ;                        // pass quarter of this sub-block
            // exchange buffers, one float2 (the pair's two keys) per entry, so that a
            // warp's accesses are consecutive 8-byte words:
            //   sub-block maps  xch[(comp * NSUB + sub) * NP + pair], comp = n1 n2 d1 d2 PA EM FM
            //   chunk-start state car[(comp * 2 + parity) * NP + pair], comp = n d pa E F
            //   G ranges        rng[sub * NP + pair] = {lo, hi} of both keys, relative to rho
            float2 *xch = reinterpret_cast<float2 *>(sm + L::xch0);
            float2 *car = reinterpret_cast<float2 *>(sm + L::car0);
            int4 *rng = reinterpret_cast<int4 *>(sm + L::rng0);
            auto X = [&](int comp, int sj) -> float2 & { return xch[(comp * NSUB + sj) * NP + pr]; };
            auto CAR = [&](int comp, int par) -> float2 & { return car[(comp * 2 + par) * NP + pr]; };
            auto i2f = [](int x, int y) { return make_float2(__int_as_float(x), __int_as_float(y)); };
            // byte offset of (row SL*s + r, keys i0, i0+1) in a swizzled tile: the
            // sub-block starts on a multiple of 8 rows, so row & 7 = r & 7
            // (bits 4-6 of a row's base are zero, so the swizzled 16-byte chunk
            // index can be XORed into the sum)
            const int cbase = ((i0 >> 6) * (kC * 128) + (SL * s) * 128 + ((i0 & 7) << 1)) | (((i0 & 63) >> 3) << 4);
            auto offr = [&](int r) { return (cbase + r * 128) ^ ((r & 7) << 4); };
            if (s == 0) {
                // the belief at the segment start, as the first chunk's start state
                CAR(0, 0) = make_float2(seg_lambda(i0), seg_lambda(i0 + 1));
                CAR(1, 0) = make_float2(1.f, 1.f);
                CAR(2, 0) = make_float2(1.f, 1.f);
                CAR(3, 0) = i2f(0, 0);
                CAR(4, 0) = i2f(0, 0);
            }
            int rho0 = 0, rho1 = 0;          // references in force (segment-start frame)
            float2 av[SL], qv[SL];           // a, qn of the sub-block's tokens
            float bl = 0.f, bln = 0.f;       // beta of token SL*s + lane (lanes < SL): this chunk, next
            // a, qn of token r of this thread's sub-block in chunk c (identity step
            // past the segment end); the addresses step by H * DK floats per token
            const long long tstep = (long long)g.H * (DK / 2);   // in float2
            auto load_tok = [&](int c, int r, float2 &ra, float2 &rq) {
                const long long t0s = tb + (long long)c * kC + SL * s;
                const long long off = ((t0s * g.H + h) * DK + i0) / 2 + r * tstep;
                if (t0s + r < te) {
                    ra = __ldg(reinterpret_cast<const float2 *>(g.a) + off);
                    rq = __ldg(reinterpret_cast<const float2 *>(g.qn) + off);
                } else {
                    ra = make_float2(1.f, 1.f);
                    rq = make_float2(0.f, 0.f);
                }
            };
            auto load_beta = [&](int c) {
                const long long tok = tb + (long long)c * kC + SL * s + lane;
                return (lane < SL && tok < te) ? __ldg(g.beta + tok * g.H + h) : 0.f;
            };
            if (nchunks > 0) {
#pragma unroll
                for (int r = 0; r < SL; ++r) load_tok(0, r, av[r], qv[r]);
                bl = load_beta(0);
            }
            float lam_end0 = 0.f, lam_end1 = 0.f, gend0 = 1.f, gend1 = 1.f;
            int xend0 = 0, xend1 = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const long long tok0 = tb + (long long)c * kC;
                const int nval = (int)min((long long)SL, max(0LL, te - (tok0 + SL * s)));   // valid tokens of the sub-block
                uint8_t *qt = sm + L::q0 + st * L::QK;
                uint8_t *kt = sm + L::k0 + st * L::QK;
                uint8_t *klo = sm + L::klo0 + st * L::QK;
                const bool okw = waitw(&stage_full[st], (c >> 1) & 1, abort_flag, g.status);
                // ---- step 1: the sub-block's Moebius maps for both keys (columns
                // are the images of (1, 0) and (0, 1); chain d <- a^2 d + qn n,
                // n <- n + b d with b = beta k^2), and its product of a
                if (okw) {
                    float2 n1 = make_float2(1.f, 1.f), d1 = make_float2(0.f, 0.f);
                    float2 n2 = make_float2(0.f, 0.f), d2 = make_float2(1.f, 1.f), PA = make_float2(1.f, 1.f);
                    int em0 = 0, em1 = 0, fm0 = 0, fm1 = 0;
#pragma unroll
                    for (int b8 = 0; b8 < SL; b8 += 8) {
                        uint32_t kwb[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) kwb[x] = *reinterpret_cast<const uint32_t *>(kt + offr(b8 + x));
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const int r = b8 + x;
                            const float2 kf = unpack_bf2(kwb[x]);
                            const float be = __shfl_sync(0xffffffffu, bl, r);
                            const float2 a2 = f2mul(av[r], av[r]);
                            const float2 b = f2mul(f2mul(make_float2(be, be), kf), kf);
                            d1 = f2fma(a2, d1, f2mul(qv[r], n1));
                            n1 = f2fma(b, d1, n1);
                            d2 = f2fma(a2, d2, f2mul(qv[r], n2));
                            n2 = f2fma(b, d2, n2);
                            PA = f2mul(PA, av[r]);
                        }
                        norm_cols(n1.x, n2.x, d1.x, d2.x, em0);
                        norm_cols(n1.y, n2.y, d1.y, d2.y, em1);
                        const int f0 = clampe(expo(PA.x)), f1 = clampe(expo(PA.y));
                        PA.x *= pow2i(-f0); PA.y *= pow2i(-f1);
                        fm0 += f0; fm1 += f1;
                    }
                    X(0, s) = n1; X(1, s) = n2; X(2, s) = d1; X(3, s) = d2; X(4, s) = PA;
                    X(5, s) = i2f(em0, em1);
                    X(6, s) = i2f(fm0, fm1);
                }
                if (named_bar_or(kGateBar, RL::GT, !okw || *abort_flag)) { ok = false; break; }
                // ---- step 2: the state at this sub-block's start: the chunk-start
                // state with the maps of the sub-blocks before it applied
                float nn[2], dd[2], pa[2];
                int E[2], F[2];
                {
                    const float2 cn = CAR(0, st), cd = CAR(1, st), cp = CAR(2, st), cE = CAR(3, st), cF = CAR(4, st);
                    nn[0] = cn.x; nn[1] = cn.y; dd[0] = cd.x; dd[1] = cd.y; pa[0] = cp.x; pa[1] = cp.y;
                    E[0] = __float_as_int(cE.x); E[1] = __float_as_int(cE.y);
                    F[0] = __float_as_int(cF.x); F[1] = __float_as_int(cF.y);
                }
                for (int sj = 0; sj < s; ++sj) {
                    const float2 m00 = X(0, sj), m01 = X(1, sj), m10 = X(2, sj), m11 = X(3, sj), mp = X(4, sj);
                    const float2 me = X(5, sj), mf = X(6, sj);
                    const float n0v = fmaf(m00.x, nn[0], m01.x * dd[0]), d0v = fmaf(m10.x, nn[0], m11.x * dd[0]);
                    const float n1v = fmaf(m00.y, nn[1], m01.y * dd[1]), d1v = fmaf(m10.y, nn[1], m11.y * dd[1]);
                    nn[0] = n0v; dd[0] = d0v; nn[1] = n1v; dd[1] = d1v;
                    pa[0] *= mp.x; pa[1] *= mp.y;
                    E[0] += __float_as_int(me.x); E[1] += __float_as_int(me.y);
                    F[0] += __float_as_int(mf.x); F[1] += __float_as_int(mf.y);
                    norm_state(nn[0], dd[0], pa[0], E[0], F[0]);
                    norm_state(nn[1], dd[1], pa[1], E[1], F[1]);
                }
                // the sub-block's start state, kept for a re-walk
                const float2 n2s0 = make_float2(nn[0], nn[1]), d2s0 = make_float2(dd[0], dd[1]);
                const float2 p2s0 = make_float2(pa[0], pa[1]);
                const int E00 = E[0], E01 = E[1], F00 = F[0], F01 = F[1];
                bln = (c + 1 < nchunks) ? load_beta(c + 1) : 0.f;
                // ---- step 3: walk the sub-block and fold every token against the
                // reference in force (exact while |G - rho| stays within kLost):
                //   Q' = q/lambda 2^(G - rho) = q pa/n 2^((F-E) - rho)
                //   K' = beta k 2^(rho - G)   = beta k d/pa 2^(rho - (F-E))
                // tracking fk = 2^(rho - G) for the chunk's G range; the next chunk's
                // a, qn go into the freed registers
                int2 glo, ghi;
                bool clamped = false;
                {
                    float2 n2s = n2s0, d2s = d2s0, p2s = p2s0;
                    int Ew0 = E00, Ew1 = E01, Fw0 = F00, Fw1 = F01;
                    // x = (F - E) - rho of the current 8-token group (unclamped): with
                    // rk = d/pa, G - rho lies in (x - expo(rk) - 1, x - expo(rk)]
                    int x0 = Fw0 - Ew0 - rho0, x1 = Fw1 - Ew1 - rho1;
                    clamped = x0 != clampe(x0) || x1 != clampe(x1);
                    float2 mq = make_float2(pow2i(clampe(x0)), pow2i(clampe(x1)));
                    float2 mk = make_float2(pow2i(-clampe(x0)), pow2i(-clampe(x1)));
                    // G just before the sub-block
                    float2 rkmin = make_float2(__fdividef(d2s.x, p2s.x), __fdividef(d2s.y, p2s.y));
                    float2 rkmax = rkmin;
                    // four tokens at a time: their chain steps (the serial part), then
                    // their folds, which are independent of one another; each token's
                    // a, qn registers take the next chunk's once it is folded
                    constexpr int TG = 4;
#pragma unroll
                    for (int r0 = 0; r0 < SL; r0 += TG) {
                        uint32_t kwb[TG], qwb[TG];
#pragma unroll
                        for (int x = 0; x < TG; ++x) {
                            kwb[x] = *reinterpret_cast<const uint32_t *>(kt + offr(r0 + x));
                            qwb[x] = *reinterpret_cast<const uint32_t *>(qt + offr(r0 + x));
                        }
                        float2 nt[TG], dt[TG], pt2[TG], bkt[TG];
#pragma unroll
                        for (int x = 0; x < TG; ++x) {
                            const int r = r0 + x;
                            const float2 kf = unpack_bf2(kwb[x]);
                            const float be = __shfl_sync(0xffffffffu, bl, r);
                            bkt[x] = f2mul(make_float2(be, be), kf);
                            d2s = f2fma(f2mul(av[r], av[r]), d2s, f2mul(qv[r], n2s));
                            n2s = f2fma(f2mul(bkt[x], kf), d2s, n2s);
                            p2s = f2mul(p2s, av[r]);
                            nt[x] = n2s; dt[x] = d2s; pt2[x] = p2s;
                        }
#pragma unroll
                        for (int x = 0; x < TG; ++x) {
                            const int r = r0 + x;
                            // (rows past the segment end are never stored and their K' is
                            // zero, so their Q' needs no masking)
                            const float2 qf = unpack_bf2(qwb[x]);
                            const float2 pn = f2mul(pt2[x], nt[x]);
                            const float2 rc = make_float2(rcp_approx(pn.x), rcp_approx(pn.y));
                            const float2 qo = f2mul(f2mul(qf, f2mul(pt2[x], mq)), f2mul(pt2[x], rc));   // q pa/n 2^x
                            const float2 rk = f2mul(dt[x], f2mul(nt[x], rc));                         // d/pa
                            const float2 ko = f2mul(bkt[x], f2mul(rk, mk));                            // beta k d/pa 2^-x
                            rkmin = make_float2(fminf(rkmin.x, rk.x), fminf(rkmin.y, rk.y));
                            rkmax = make_float2(fmaxf(rkmax.x, rk.x), fmaxf(rkmax.y, rk.y));
                            const uint32_t kh = pack_bf2(ko.x, ko.y);
                            const float2 khf = unpack_bf2(kh);
                            *reinterpret_cast<uint32_t *>(qt + offr(r)) = pack_bf2(qo.x, qo.y);
                            *reinterpret_cast<uint32_t *>(kt + offr(r)) = kh;
                            *reinterpret_cast<uint32_t *>(klo + offr(r)) = pack_bf2(ko.x - khf.x, ko.y - khf.y);
                            if (c + 1 < nchunks) load_tok(c + 1, r, av[r], qv[r]);
                        }
                        if (((r0 + TG) & 7) == 0) {
                            // the 8-token group's G range, renormalisation, next factors
                            const int r = r0 + TG - 1;
                            const int lo0 = x0 - expo(rkmax.x) - 1, lo1 = x1 - expo(rkmax.y) - 1;
                            const int hi0 = x0 - expo(rkmin.x), hi1 = x1 - expo(rkmin.y);
                            glo = (r == 7) ? make_int2(lo0, lo1) : make_int2(min(glo.x, lo0), min(glo.y, lo1));
                            ghi = (r == 7) ? make_int2(hi0, hi1) : make_int2(max(ghi.x, hi0), max(ghi.y, hi1));
                            norm_state(n2s.x, d2s.x, p2s.x, Ew0, Fw0);
                            norm_state(n2s.y, d2s.y, p2s.y, Ew1, Fw1);
                            rkmin = make_float2(3.0e38f, 3.0e38f);
                            rkmax = make_float2(0.f, 0.f);
                            if (r + 1 < SL) {
                                x0 = Fw0 - Ew0 - rho0;
                                x1 = Fw1 - Ew1 - rho1;
                                clamped |= x0 != clampe(x0) || x1 != clampe(x1);
                                mq = make_float2(pow2i(clampe(x0)), pow2i(clampe(x1)));
                                mk = make_float2(pow2i(-clampe(x0)), pow2i(-clampe(x1)));
                            }
                        }
                    }
                    if (s == NSUB - 1) {
                        // the chunk-end state starts the next chunk
                        const int nst = (c + 1) & 1;
                        CAR(0, nst) = n2s; CAR(1, nst) = d2s; CAR(2, nst) = p2s;
                        CAR(3, nst) = i2f(Ew0, Ew1);
                        CAR(4, nst) = i2f(Fw0, Fw1);
                        if (c == nchunks - 1) {
                            lam_end0 = n2s.x / d2s.x;
                            lam_end1 = n2s.y / d2s.y;
                            gend0 = p2s.x / d2s.x;
                            gend1 = p2s.y / d2s.y;
                            xend0 = Fw0 - Ew0;
                            xend1 = Fw1 - Ew1;
                        }
                    }
                }
                rng[s * NP + pr] = make_int4(glo.x, ghi.x, glo.y, ghi.y);
                if (named_bar_or(kGateBar, RL::GT, *abort_flag != 0)) { ok = false; break; }
                // ---- step 4: references of the pass quarters from the G ranges of
                // every sub-block (relative to rho): R = 0 keeps the reference
                int R0[4], R1[4];
                int lv;
                bool bad0, bad1;
                {
                    int2 qa[4], qb[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        constexpr int per = NSUB / 4;
                        int4 x = rng[(q * per) * NP + pr];
                        int2 ra = make_int2(x.x, x.y), rb = make_int2(x.z, x.w);
#pragma unroll
                        for (int y = 1; y < per; ++y) {
                            x = rng[(q * per + y) * NP + pr];
                            ra = runion(ra, make_int2(x.x, x.y));
                            rb = runion(rb, make_int2(x.z, x.w));
                        }
                        qa[q] = ra;
                        qb[q] = rb;
                    }
                    const int l0 = choose_refs(qa, 0, R0, bad0);
                    const int l1 = choose_refs(qb, 0, R1, bad1);
                    lv = max(l0, l1);
                }
                const int ra = pick4(R0, quarter), rb = pick4(R1, quarter);
                // the provisional fold of this sub-block is exact while its |G - rho|
                // stays within kLost and no exponent was clamped; a rescale by more
                // than 2^100 is not taken in one step either: re-walk instead
                const bool lost = clamped || glo.x < -kLost || ghi.x > kLost || glo.y < -kLost || ghi.y > kLost ||
                                  abs(ra) > kLost || abs(rb) > kLost;
                if (s == 0) {
                    atomicMax(&lvl[st], (c << 2) | lv);
                    if (bad0 || bad1) atomicOr(g.status, kStatusRange);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        facd[(st * 4 + q) * DK + i0] = R0[q] - (q ? R0[q - 1] : 0);
                        facd[(st * 4 + q) * DK + i0 + 1] = R1[q] - (q ? R1[q - 1] : 0);
                    }
                    if (LOCAL && p > 0) {
                        float *rl = g.rlog + ((u * g.NC + chunk_base + c) * 4) * DK + i0;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<float2 *>(rl + q * DK) =
                                make_float2((float)(rho0 + R0[q]), (float)(rho1 + R1[q]));
                    }
                }
                if (lost) {
                    // ---- step 5a (strong forgetting): walk the sub-block again from its
                    // start and fold against the pass reference (a, qn reloaded)
                    rewalk_fold<DK, SL>(qt, kt, klo, cbase, n2s0, d2s0, p2s0, E00, E01, F00, F01, rho0 + ra, rho1 + rb,
                                        g.a, g.qn, g.beta, reinterpret_cast<const __nv_bfloat16 *>(g.q),
                                        reinterpret_cast<const __nv_bfloat16 *>(g.k), tok0 + SL * s, nval, g.H, h, i0);
                } else if (ra != 0 || rb != 0) {
                    // ---- step 5b: the reference moved: rescale the folded bf16 words
                    // exactly by powers of two (Q' by 2^-R, K' by 2^R)
                    const __nv_bfloat162 sq = __floats2bfloat162_rn(pow2i(-ra), pow2i(-rb));
                    const __nv_bfloat162 sk = __floats2bfloat162_rn(pow2i(ra), pow2i(rb));
#pragma unroll 1
                    for (int r = 0; r < SL; ++r) {
                        __nv_bfloat162 *wq = reinterpret_cast<__nv_bfloat162 *>(qt + offr(r));
                        __nv_bfloat162 *wk = reinterpret_cast<__nv_bfloat162 *>(kt + offr(r));
                        __nv_bfloat162 *wl = reinterpret_cast<__nv_bfloat162 *>(klo + offr(r));
                        *wq = __hmul2(*wq, sq);
                        *wk = __hmul2(*wk, sk);
                        *wl = __hmul2(*wl, sk);
                    }
                }
                rho0 += R0[3];
                rho1 += R1[3];
                if (c == nchunks - 1 && s == NSUB - 1) {
                    // final outputs of the segment: 2^(G_end - rho) for the state
                    // export, the precision, and the segment's gate product
                    facf[i0] = scale2(gend0, xend0 - rho0);
                    facf[i0 + 1] = scale2(gend1, xend1 - rho1);
                    if (LOCAL) {
                        auto prod = [](float gm, int x) {
                            return x < -250 ? 0.f : (x > 250 ? __int_as_float(0x7f800000) : scale2(gm, x));
                        };
                        g.decay[(u * g.P + p) * DK + i0] = prod(gend0, xend0);
                        g.decay[(u * g.P + p) * DK + i0 + 1] = prod(gend1, xend1);
                    }
                    if (last_seg && g.final_lambda) {
                        g.final_lambda[u * DK + i0] = lam_end0;
                        g.final_lambda[u * DK + i0 + 1] = lam_end1;
                    }
                }
                bl = bln;
                fence_proxy_async();
                mbar_arrive(&qk_ready[st]);
            }
            if (nchunks == 0 && s == 0 && last_seg && g.final_lambda) {
                const float2 l0 = CAR(0, 0);
                g.final_lambda[u * DK + i0] = l0.x;
                g.final_lambda[u * DK + i0 + 1] = l0.y;
            }
        } else {
            // ---- isotropic: one precision per head ---------------------------
            float2 *isof = reinterpret_cast<float2 *>(sm + L::isof0);
            float lam = 0.f, D = 0.f, Gc = 0.f;   // warp 0: precision, G - rho and G at the chunk start
            // per-token scalars of a chunk, loaded one chunk ahead (lane: tokens 2 lane, 2 lane + 1)
            float nb0 = 0.f, nb1 = 0.f, na0 = 1.f, na1 = 1.f, nq0 = 0.f, nq1 = 0.f;
            auto prefetch = [&](int c) {
                const long long x0 = tb + (long long)c * kC + 2 * lane, x1 = x0 + 1;
                nb0 = x0 < te ? __ldg(g.beta + x0 * g.H + h) : 0.f;
                nb1 = x1 < te ? __ldg(g.beta + x1 * g.H + h) : 0.f;
                na0 = x0 < te ? __ldg(g.a + x0 * g.H + h) : 1.f;
                na1 = x1 < te ? __ldg(g.a + x1 * g.H + h) : 1.f;
                nq0 = x0 < te ? __ldg(g.qn + x0 * g.H + h) : 0.f;
                nq1 = x1 < te ? __ldg(g.qn + x1 * g.H + h) : 0.f;
            };
            if (warp == 0) {
                lam = seg_lambda(0);
                if (nchunks > 0) prefetch(0);
            }
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const long long tok0 = tb + (long long)c * kC;
                uint8_t *qt = sm + L::q0 + st * L::QK;
                uint8_t *kt = sm + L::k0 + st * L::QK;
                uint8_t *klo = sm + L::klo0 + st * L::QK;
                bool okw = true;
                if (warp == 0) {
                    const float cb0 = nb0, cb1 = nb1, a0 = na0, a1 = na1, q0 = nq0, q1 = nq1;
                    if (c + 1 < nchunks) prefetch(c + 1);
                    okw = waitw(&stage_full[st], (c >> 1) & 1, abort_flag, g.status);
                    if (okw) {
                        // warp-level Moebius scan of the chunk (lane: tokens 2l, 2l+1)
                        const int t0i = 2 * lane, t1i = t0i + 1;
                        const bool va = tok0 + t0i < te, vb = tok0 + t1i < te;
                        const float inv_dk = 1.0f / (float)DK;
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
                        // G (relative to the chunk start) after tokens 2l and 2l+1, and
                        // just before 2l; in the frame x = G_abs - rho: D + G
                        const float G1 = sum, G0 = sum - l1, Gp = G0 - l0;
                        float mn = fminf(Gp, fminf(G0, G1)), mx = fmaxf(Gp, fmaxf(G0, G1));
                        // quarter q = lanes 8q .. 8q+7
#pragma unroll
                        for (int d = 1; d < 8; d <<= 1) {
                            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, d));
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
                        }
                        int2 qr[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float lo = __shfl_sync(0xffffffffu, mn, 8 * q);
                            const float hi = __shfl_sync(0xffffffffu, mx, 8 * q);
                            qr[q] = make_int2((int)floorf(D + lo), (int)ceilf(D + hi));
                        }
                        int R[4];
                        bool bad;
                        const int lv = choose_refs(qr, 0, R, bad);
                        const int myq = lane >> 3;
                        const float Rq = (float)pick4(R, myq);
                        // per-token factors: q / lambda 2^(G - rho_q), beta 2^(rho_q - G)
                        const float e0 = D + G0 - Rq, e1 = D + G1 - Rq;
                        isof[st * kC + t0i] = va ? make_float2(exp2f(e0) / lamB, cb0 * exp2f(-e0)) : make_float2(0.f, 0.f);
                        isof[st * kC + t1i] = vb ? make_float2(exp2f(e1) / lamC, cb1 * exp2f(-e1)) : make_float2(0.f, 0.f);
                        for (int i = lane; i < DK; i += 32) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) facd[(st * 4 + q) * DK + i] = R[q] - (q ? R[q - 1] : 0);
                        }
                        if (lane == 0) {
                            lvl[st] = (c << 2) | lv;
                            if (bad) atomicOr(g.status, kStatusRange);
                        }
                        if (LOCAL && p > 0) {
                            // segment-start frame: rho_q = G_chunk_start - D + R_q
                            float *rl = g.rlog + ((u * g.NC + chunk_base + c) * 4) * DK;
                            for (int i = lane; i < DK; i += 32) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) rl[q * DK + i] = Gc - D + (float)R[q];
                            }
                        }
                        const float Gend = __shfl_sync(0xffffffffu, G1, 31);
                        lam = __shfl_sync(0xffffffffu, lamC, 31);
                        D = D + Gend - (float)R[3];
                        Gc += Gend;
                        if (c == nchunks - 1) {
                            for (int i = lane; i < DK; i += 32) facf[i] = exp2f(D);
                            if (lane == 0) {
                                if (LOCAL) g.decay[u * g.P + p] = exp2f(Gc);
                                if (last_seg && g.final_lambda) g.final_lambda[u] = lam;
                            }
                        }
                    }
                }
                if (named_bar_or(kGateBar, RL::GT, !okw || *abort_flag)) { ok = false; break; }
                // fold the rows: Q' = q fq, K' = k fk (hi + remainder); thread = (row, key pair)
                constexpr int NP = DK / 2;
#pragma unroll 4
                for (int it = tid; it < kC * NP; it += RL::GT) {
                    const int row = it / NP, i0 = 2 * (it % NP);
                    const int off = sw_off(row, i0, kC);
                    const float2 f = isof[st * kC + row];
                    const float2 qf = unpack_bf2(*reinterpret_cast<const uint32_t *>(qt + off));
                    const float2 kf = unpack_bf2(*reinterpret_cast<const uint32_t *>(kt + off));
                    const float2 ko = make_float2(kf.x * f.y, kf.y * f.y);
                    const uint32_t kh = pack_bf2(ko.x, ko.y);
                    const float2 khf = unpack_bf2(kh);
                    *reinterpret_cast<uint32_t *>(qt + off) = pack_bf2(qf.x * f.x, qf.y * f.x);
                    *reinterpret_cast<uint32_t *>(kt + off) = kh;
                    *reinterpret_cast<uint32_t *>(klo + off) = pack_bf2(ko.x - khf.x, ko.y - khf.y);
                }
                fence_proxy_async();
                mbar_arrive(&qk_ready[st]);
            }
            if (warp == 0 && lane == 0 && nchunks == 0 && last_seg && g.final_lambda) g.final_lambda[u] = lam;
        }
        (void)ok;
    } else {
        // ================= epilogue warps; thread 0 also issues the TMA loads and
        // the tcgen05 MMAs at the points where the epilogue synchronises ========
        const int we = warp - RL::EPIW;        // TMEM lane quarter (warp % 4)
        const bool issuer = we == 0 && lane == 0;
        const uint32_t lane_base = (uint32_t)(32 * we) << 16;
        const int row64 = 16 * we + lane;
        const bool v64 = lane < 16;
        const int rowU = (DK == 128) ? (32 * we + lane) : row64;
        const bool vU = (DK == 128) || v64;
        uint8_t *ub = sm + L::ub0;
        uint8_t *pt = sm + L::p0;
        const float *eta0 = ((!LOCAL || p == 0) && g.eta0) ? g.eta0 + u * DK * DV : nullptr;
        bool ok = true;
        // q, k, v tiles of chunk c into stage c & 1, and an L2 prefetch of the
        // chunk two ahead (its tiles, a and qn: the gate loads those itself)
        auto load_chunk = [&](int c) {
            const int tok0 = (int)(tb + (long long)c * kC);
            const int s = c & 1;
            mbar_expect_tx(&stage_full[s], 2 * L::QK + L::V);
#pragma unroll
            for (int a = 0; a < DK / 64; ++a) {
                tma_load_3d(sm + L::q0 + s * L::QK + a * kC * 128, &tm_q, &stage_full[s], 64 * a, h, tok0);
                tma_load_3d(sm + L::k0 + s * L::QK + a * kC * 128, &tm_k, &stage_full[s], 64 * a, h, tok0);
            }
#pragma unroll
            for (int a = 0; a < DV / 64; ++a)
                tma_load_3d(sm + L::v0 + s * L::V + a * kC * 128, &tm_v, &stage_full[s], 64 * a, h, tok0);
            if (c + 2 < nchunks) {
                const int tp = tok0 + 2 * kC;
#pragma unroll
                for (int a = 0; a < DK / 64; ++a) {
                    tma_prefetch_3d(&tm_q, 64 * a, h, tp);
                    tma_prefetch_3d(&tm_k, 64 * a, h, tp);
                }
#pragma unroll
                for (int a = 0; a < DV / 64; ++a) tma_prefetch_3d(&tm_v, 64 * a, h, tp);
                if (!ISO) {
                    tma_prefetch_3d(&tm_a, 0, h, tp);
                    tma_prefetch_3d(&tm_qn, 0, h, tp);
                }
            }
        };
        int loaded = 0;                                 // chunks whose loads were issued
        if (issuer) {
            // a and qn of chunk 1 (chunk 0 is read at once)
            if (!ISO && nchunks > 1) {
                tma_prefetch_3d(&tm_a, 0, h, (int)(tb + kC));
                tma_prefetch_3d(&tm_qn, 0, h, (int)(tb + kC));
            }
            for (; loaded < 2 && loaded < nchunks; ++loaded) load_chunk(loaded);
        }
        // Belief at the segment start, written into the U columns of TMEM before
        // the first chunk (while the gate works on it): eta0 for whole rows and
        // first segments, zero for the later segments of split rows (their
        // carried state is added by the correction pass)
        if (nchunks > 0) {
#pragma unroll
            for (int cb = 0; cb < DV / 32; ++cb) {
                uint32_t r[32];
#pragma unroll
                for (int x = 0; x < 32; x += 4) {
                    const float4 e4 = (vU && eta0) ? *reinterpret_cast<const float4 *>(eta0 + rowU * DV + cb * 32 + x)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                    r[x] = __float_as_uint(e4.x); r[x + 1] = __float_as_uint(e4.y);
                    r[x + 2] = __float_as_uint(e4.z); r[x + 3] = __float_as_uint(e4.w);
                }
                tmem_st32(tbase + lane_base + L::colU + cb * 32, r);
            }
            tmem_wait_st();
        }
        constexpr uint32_t iS = idesc_bf16(64, 64, false, false);
        constexpr uint32_t iO = idesc_bf16(64, DV, false, true);
        constexpr uint32_t iU = idesc_bf16(DK, DV, true, true);
        const uint32_t tS = tbase + L::colS, tO = tbase + L::colO, tU = tbase + L::colU;
        const uint32_t uba = smem_u32(sm + L::ub0);
        int pc = 0;                                   // passes so far (barrier phases)
        // The output rows of a pass are read out during the next pass (after its
        // P mask), from the other of two output accumulators, so the epilogue
        // does not wait for the pass's last MMAs; P is double-buffered likewise.
        int pend_c = -1, pend_m0 = 0, pend_m1 = 0;    // the pass whose rows are pending
        auto emit = [&](int pcx, int cc, int m0, int m1) {
            if (!waitw(&o_full[pcx & 1], (pcx >> 1) & 1, abort_flag, g.status)) { ok = false; return; }
            tc_fence_after();
            const long long tok0 = tb + (long long)cc * kC;
            const bool row_ok = v64 && row64 >= m0 && row64 < m1 && (tok0 + row64 < te);
            __nv_bfloat16 *orow = g.out + ((tok0 + row64) * g.H + h) * DV;
            const uint32_t to = tbase + lane_base + L::colO + (pcx & 1) * DV;
            uint32_t r2[DV / 32][32];
#pragma unroll
            for (int cb = 0; cb < DV / 32; ++cb) tmem_ld32(to + cb * 32, r2[cb]);
            tmem_wait_ld();
            if (row_ok) {
#pragma unroll
                for (int hh = 0; hh < DV / 32; ++hh) {
                    const uint32_t *r = r2[hh];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 w;
                        w.x = pack_bf2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                        w.y = pack_bf2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                        w.z = pack_bf2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                        w.w = pack_bf2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                        *reinterpret_cast<uint4 *>(orow + hh * 32 + q4 * 8) = w;
                    }
                }
            }
            tc_fence_before();
        };
        // every exit from this loop goes through a reducing barrier, so that the
        // four warps leave it together
        for (int c = 0; c < nchunks; ++c) {
            const int st = c & 1;
            if (!waitw(&qk_ready[st], (c >> 1) & 1, abort_flag, g.status)) { ok = false; }
            if (named_bar_or(kEpiBar, 128, !ok || *abort_flag)) { ok = false; break; }
            tc_fence_after();
            const int lv = lvl[st] & 3;
            const int np = 1 << lv, qper = 4 >> lv;
            const uint32_t qa = smem_u32(sm + L::q0 + st * L::QK);
            const uint32_t ka = smem_u32(sm + L::k0 + st * L::QK);
            const uint32_t va = smem_u32(sm + L::v0 + st * L::V);
            const uint32_t kloa = smem_u32(sm + L::klo0 + st * L::QK);
            if (issuer) {
                if (LOCAL && p > 0) {
                    // export the folded q tile (the correction pass multiplies it by
                    // the carried segment-start state)
                    const int tok0 = (int)(tb + (long long)c * kC);
#pragma unroll
                    for (int a = 0; a < DK / 64; ++a)
                        tma_store_3d(&tm_qs, sm + L::q0 + st * L::QK + a * kC * 128, 64 * a, h, tok0);
                    tma_store_commit();
                }
                // scores of the whole chunk (each pass masks its own block); the
                // K step moves a descriptor's start address by (bytes >> 4)
                const uint64_t dq = sdesc_sw128(qa, 16, 1024), dk = sdesc_sw128(ka, 16, 1024);
#pragma unroll 1
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * (kC * 128) + (kk & 3) * 32) >> 4;
                    mma_bf16(tS, dq + off, dk + off, iS, kk > 0);
                }
                mma_commit(s_full);
            }
            for (int k = 0; k < np; ++k) {
                const int m0 = kQ * qper * k, m1 = m0 + kQ * qper;
                const int s0 = k * qper, s1 = s0 + qper;      // 16-token slices of this pass
                const uint32_t tOp = tO + (pc & 1) * DV;      // this pass's output accumulator
                uint8_t *ptp = pt + (pc & 1) * L::PT;         // and its P buffer
                // ---- state: U <- 2^d U for this pass's reference, snapshot to bf16
                if (pc > 0 && !waitw(u_done, (pc - 1) & 1, abort_flag, g.status)) ok = false;
                tc_fence_after();
                const int d = vU ? facd[(st * 4 + k * qper) * DK + rowU] : 0;
                const bool rmw = __any_sync(0xffffffffu, d != 0);
                if (ok) {
                    if (rmw) tmem_scale_lane<DV>(tbase + lane_base + L::colU, d);
                    uint32_t r2[DV / 32][32];
#pragma unroll
                    for (int cb = 0; cb < DV / 32; ++cb) tmem_ld32(tbase + lane_base + L::colU + cb * 32, r2[cb]);
                    tmem_wait_ld();
                    if (vU) {
#pragma unroll
                        for (int hh = 0; hh < DV / 32; ++hh) {
                            const uint32_t *r = r2[hh];
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                uint4 w;
                                w.x = pack_bf2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                                w.y = pack_bf2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                                w.z = pack_bf2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                                w.w = pack_bf2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                                *reinterpret_cast<uint4 *>(ub + sw_off(rowU, hh * 32 + q4 * 8, DK)) = w;
                            }
                        }
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                if (named_bar_or(kEpiBar, 128, !ok || *abort_flag)) { ok = false; break; }
                if (issuer) {
                    tc_fence_after();
                    // O = Q' U into this pass's accumulator (its previous contents, two
                    // passes back, were read out before the barrier)
                    const uint64_t dq = sdesc_sw128(qa, 16, 1024), du = sdesc_sw128(uba, DK * 128, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * (kC * 128) + (kk & 3) * 32) >> 4;
                        mma_bf16(tOp, dq + off, du + kk * (2048 >> 4), iO, kk > 0);
                    }
                }
                // ---- P = the pass's block of the causal score tile, bf16
                if (k == 0 && !waitw(s_full, c & 1, abort_flag, g.status)) ok = false;
                tc_fence_after();
                if (ok) {
                    uint32_t r2[2][32];
                    tmem_ld32(tbase + lane_base + L::colS, r2[0]);
                    tmem_ld32(tbase + lane_base + L::colS + 32, r2[1]);
                    tmem_wait_ld();
                    if (v64) {
                        const int tau = row64;
                        const bool in_row = tau >= m0 && tau < m1;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            float x[8];
#pragma unroll
                            for (int e2 = 0; e2 < 8; ++e2) {
                                const int sg = ch * 8 + e2;
                                const float sv = __uint_as_float(r2[sg >> 5][sg & 31]);
                                x[e2] = (in_row && sg >= m0 && sg <= tau) ? sv : 0.f;
                            }
                            uint4 w;
                            w.x = pack_bf2(x[0], x[1]); w.y = pack_bf2(x[2], x[3]);
                            w.z = pack_bf2(x[4], x[5]); w.w = pack_bf2(x[6], x[7]);
                            *reinterpret_cast<uint4 *>(ptp + tau * 128 + ((ch ^ (tau & 7)) << 4)) = w;
                        }
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                if (named_bar_or(kEpiBar, 128, !ok || *abort_flag)) { ok = false; break; }
                if (issuer) {
                    tc_fence_after();
                    // O += P V over this pass's tokens; then the state update, whose
                    // completion (u_done) the next pass's snapshot waits for
                    const uint64_t dp = sdesc_sw128(smem_u32(ptp), 16, 1024), dv = sdesc_sw128(va, kC * 128, 1024);
                    const uint64_t dk = sdesc_sw128(ka, kC * 128, 1024), dl = sdesc_sw128(kloa, kC * 128, 1024);
#pragma unroll 1
                    for (int kk = s0; kk < s1; ++kk) mma_bf16(tOp, dp + kk * (32 >> 4), dv + kk * (2048 >> 4), iO, 1);
                    mma_commit(&o_full[pc & 1]);
                    // U += K'^T V over this pass's tokens (hi and remainder of K')
#pragma unroll 1
                    for (int kk = s0; kk < s1; ++kk) {
                        mma_bf16(tU, dk + kk * (2048 >> 4), dv + kk * (2048 >> 4), iU, 1);
                        mma_bf16(tU, dl + kk * (2048 >> 4), dv + kk * (2048 >> 4), iU, 1);
                    }
                    mma_commit(u_done);
                }
                // ---- output rows of the previous pass (its MMAs have finished
                // while this pass was prepared)
                if (ok && pend_c >= 0) emit(pc - 1, pend_c, pend_m0, pend_m1);
                pend_c = c; pend_m0 = m0; pend_m1 = m1;
                ++pc;
            }
            if (named_bar_or(kEpiBar, 128, !ok || *abort_flag)) { ok = false; break; }
            // every MMA of this chunk has completed once its last u_done has (the
            // state update is the last reader of K' and V): the stage takes the
            // chunk two ahead once the q' export has read it. Only the issuing
            // thread waits; the other warps go on to the next chunk.
            if (issuer) {
                ok = wait_slow(u_done, (pc - 1) & 1, abort_flag, g.status, true) && ok;
                if (LOCAL && p > 0) tma_store_wait_read();
                if (ok && loaded < nchunks) { load_chunk(loaded); ++loaded; }
            }
        }
        if (ok && pend_c >= 0) emit(pc - 1, pend_c, pend_m0, pend_m1);
        // ---- final belief (last segment) or segment transfer (mode 2)
        float *dst = nullptr;
        if (LOCAL) dst = g.S_io + (u * g.P + p) * DK * DV;
        else if (last_seg && g.final_eta) dst = g.final_eta + u * DK * DV;
        if (ok && dst && !*abort_flag) {
            if (nchunks > 0) {
                if (waitw(u_done, (pc - 1) & 1, abort_flag, g.status)) {
                    tc_fence_after();
                    const float ff = vU ? facf[rowU] : 0.f;
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
                // no tokens (an empty packed sequence): the belief is eta0
                for (int x = 0; x < DV; ++x) dst[rowU * DV + x] = eta0 ? eta0[rowU * DV + x] : 0.f;
            }
        }
        if (issuer) {
            if (LOCAL && p > 0) tma_store_wait_all();
            if (!ok || *abort_flag) {
                // wait (bounded) until every tile load issued has landed
                for (int c = max(0, loaded - 2); c < loaded; ++c)
                    wait_slow(&stage_full[c & 1], (c >> 1) & 1, abort_flag, g.status, false);
            }
            // all MMAs issued have completed before TMEM is released
            mma_commit(td_bar);
            wait_slow(td_bar, 0, abort_flag, g.status, false);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == RL::EPIW) tmem_dealloc(tbase, L::NCOLS);
}

// ---- host side ---------------------------------------------------------------

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(ptr);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
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
    // a and qn: L2 prefetch boxes of a whole chunk (the gate loads them itself)
    if (ok && !p.iso)
        ok = make_tma_map(&ma, a, F32, 4, DK, p.H, p.ntok, DK, kC, false) &&
             make_tma_map(&mqn, qn, F32, 4, DK, p.H, p.ntok, DK, kC, false);
    else { ma = mq; mqn = mq; }
    if (ok && mode == 2) ok = make_tma_map(&mqs, p.qbuf, BF, 2, DK, p.H, p.ntok, 64, kC, true);
    else mqs = mq;
    if (!ok) return cudaErrorInvalidValue;
    if (mode != 0 && mode != 2) return cudaErrorInvalidValue;
    static PerDevice<bool> attr[4];
    void (*const kerns[4])(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                           TcArgs) = {kla_chunk_tc_kernel<DK, DV, false, false>,
                                      kla_chunk_tc_kernel<DK, DV, false, true>,
                                      kla_chunk_tc_kernel<DK, DV, true, false>,
                                      kla_chunk_tc_kernel<DK, DV, true, true>};
    const int which = (p.iso ? 2 : 0) + (mode == 2 ? 1 : 0);
    const cudaError_t e = ensure_smem_attr(attr[which], kerns[which], L::alloc);
    if (e != cudaSuccess) return e;
    TcArgs g;
    g.N = p.N; g.H = p.H; g.P = p.P; g.NB = p.NB; g.seg_blocks = p.seg_blocks; g.NC = p.NB;
    g.T = p.T; g.Lseg = p.Lseg; g.cu = cu; g.perm = cu ? p.perm : nullptr;
    g.a = a; g.qn = qn; g.beta = beta; g.lambda0 = lambda0; g.eta0 = eta0; g.lam_blk = lam_blk;
    g.q = q; g.k = k;
    g.agg = p.inline_carry ? p.agg : nullptr;
    g.rlog = p.rlog;
    g.S_io = S_io; g.decay = decay; g.out = (__nv_bfloat16 *)out;
    g.final_lambda = final_lambda; g.final_eta = final_eta; g.status = status;
    const unsigned grid = (unsigned)((long long)p.N * p.H * p.P);
    if (grid == 0) return cudaSuccess;
    return launch_pdl(kerns[which], grid, Roles<DK, DV>::THREADS, L::alloc, st, mq, mk, mv, ma, mqn, mqs, g);
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
