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
// CTA = one segment of one (row or packed sequence, head), warp-specialised:
//   gate        Diagonal precision: dk / 32 warps, thread = key. Each thread
//               walks its key through every token of the segment (precision
//               chain and exponents in registers), folding each token's Q',
//               K' (bf16 hi) and the bf16 remainder of K' over the TMA-loaded
//               tiles against the reference in force; then the chunk's G
//               ranges per pass quarter fix the references, and rows whose
//               reference moved are rescaled exactly (or re-walked where the
//               provisional fold lost bits).
//               Isotropic precision: three warps; warp 0 scans the chunk's 64
//               Moebius maps with shuffles, all three fold the rows.
//   epilogue    four warps (TMEM lane quarter = warp % 4): rescale U in TMEM
//               and snapshot it to bf16 shared memory, mask the score tile into
//               P, store the output rows;
//   producer    (diagonal) streams a and qn into the gate's ring of 16-token
//               slots, with an L2 prefetch two chunks ahead;
//   MMA warp    TMEM owner; lane 0 loads the q, k, v tiles (double-buffered,
//               L2 prefetch of later chunks), exports q' of split rows, and
//               issues every tcgen05.mma, synchronised with the gate and the
//               epilogue through mbarriers only.
// mode 0 walks whole rows or packed sequences (from lambda0, eta0); mode 2
// walks every segment of split rows from a zero state (segment 0 from eta0)
// and exports what the correction pass needs. The kernel is instantiated per
// (dk, dv, isotropic or diagonal precision, walk mode).
//
// Every wait is bounded: after kWaitLimitNs a waiter sets the abort flag and
// the library status bit, all roles fall through to the teardown, the
// producer and the MMA thread wait (bounded) for their outstanding copies, the
// MMA thread for its outstanding MMAs, and the TMEM is released.
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
constexpr int kMove = 32;     // the reference moves to a chunk's start once G has drifted beyond kMove from it
constexpr int kSl = 8;        // tokens per slice of the diagonal gate's walk
constexpr int kRt = 16;       // tokens per a / qn ring slot of the diagonal gate (two slices)
constexpr int kRpc = kC / kRt;             // ring slots per chunk
constexpr int kRs = 2;                     // ring slots
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Gate warps first, then the four epilogue warps (TMEM lane quarter = warp % 4),
// the warp that streams a and qn into the diagonal gate's ring (diagonal only),
// and the MMA warp. Diagonal precision: one gate thread per key (dk / 32
// warps); isotropic: three gate warps (warp 0 scans, all three fold), so that
// no scheduler holds more than two warps' registers.
template <int DK, int DV, bool ISO>
struct Roles {
    static constexpr int NGW = ISO ? 3 : DK / 32;     // gate warps
    static constexpr int GT = NGW * 32;               // gate threads
    // threads that arrive on qk_ready: every diagonal gate thread; the isotropic
    // gate's folding warps (warp 0 scans ahead of them)
    static constexpr int QKA = ISO ? (NGW - 1) * 32 : GT;
    static constexpr int EPIW = NGW;                  // first epilogue warp
    static constexpr int MMAW = NGW + (ISO ? 4 : 5);  // TMEM owner, tile loads, MMA issue
    static constexpr int THREADS = (MMAW + 1) * 32;
    // two CTAs per SM at dk = dv = 64 (the planner counts on it): 128 registers
    // per thread, half the shared memory and TMEM each
    static constexpr int MIN_BLOCKS = (DK == 64 && DV == 64) ? 2 : 1;
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
    // test switch (KLA_TEST_WITHHOLD_TILES): the MMA warp issues no tile loads,
    // so the first wait on them runs out and the bounded-wait path is exercised
    int withhold_tiles;
};

template <int DK, int DV>
struct Layout {
    static constexpr int QK = kC * DK * 2;
    static constexpr int V = kC * DV * 2;
    static constexpr int PT = kC * kC * 2;
    static constexpr int UB = DK * DV * 2;
    static constexpr int RSLOT = 2 * kRt * DK * 4;   // a / qn ring slot: [a: kRt x DK][qn: kRt x DK] floats
    static constexpr int q0 = 0;
    static constexpr int k0 = q0 + 2 * QK;
    static constexpr int v0 = k0 + 2 * QK;
    static constexpr int klo0 = v0 + 2 * V;          // low bf16 part of K' (state update), per stage
    static constexpr int p0 = klo0 + 2 * QK;
    static constexpr int ub0 = p0 + 2 * PT;         // (P double-buffered by pass)
    static constexpr int ring0 = ub0 + UB;           // [kRs] a / qn ring slots of the diagonal gate
    static constexpr int fac0 = ring0 + kRs * RSLOT; // [2][4][DK] int: U rescale exponent at each pass quarter
    static constexpr int facf0 = fac0 + 2 * kQuarters * DK * 4;   // [DK] float: 2^(G_end - rho_end)
    static constexpr int isof0 = facf0 + DK * 4;     // [2][kC] float2: iso per-token factors
    static constexpr int lvl0 = isof0 + 2 * kC * 8;  // int[2]: pass level of the chunk, tagged with its index
    static constexpr int bar0 = lvl0 + 16;
    static constexpr int NBAR = 14 + 2 * kRs;
    static constexpr int hold0 = bar0 + NBAR * 8;
    static constexpr int bytes = hold0 + 16;
    static constexpr int alloc = bytes + 1024;
    static_assert(alloc <= 232448, "shared memory per CTA");
    static_assert(!(DK == 64 && DV == 64) || 2 * (alloc + 1024) <= 233472, "two CTAs per SM at dk = dv = 64");
    // TMEM columns: the state U, two output accumulators (by pass), the scores
    static constexpr uint32_t NCOLS = (3 * DV + 64 <= 256) ? 256u : 512u;
    static constexpr uint32_t colU = 0, colO = DV, colS = 3 * DV;
    static_assert(!(DK == 64 && DV == 64) || NCOLS <= 256, "two CTAs' TMEM at dk = dv = 64");
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

// Sum of squares of row `row` of a 128B-swizzled bf16 tile (the order of its
// 16-byte chunks does not matter). Lane l starts at chunk l, so that a warp
// reading different rows spreads over the banks (a 4-way conflict, not 32).
template <int DK>
__device__ __forceinline__ float row_sumsq(const uint8_t *ktile, int row, int lane) {
    float s = 0.f;
#pragma unroll
    for (int a = 0; a < DK / 64; ++a) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            const int ch = (c8 + lane) & 7;
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

__device__ __forceinline__ uint16_t bf16_bits(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
__device__ __forceinline__ float bf16_val(uint32_t bits) { return __uint_as_float(bits << 16); }

// One key's walk in the diagonal gate. The projective precision lambda = n/d
// and the gate product p are renormalised at every slice end, their exponents
// kept in E and F, so that G = log2(p/d) + F - E.
struct KeyWalk {
    float n, d, p;
    int E, F;
    int x;                  // F - E - rho at the slice start (unclamped)
    float mq, mk;           // 2^clamp(x), 2^-clamp(x)
    float rkmin, rkmax;     // range of d/p over the slice
    bool clamped;           // some slice's x left the exponent window
    int2 cl, q0, q1, q2, q3;   // integer bounds of G - rho: this quarter, the completed ones
};

// Walks the kSl tokens of slice s8 for one key (a, qn at ra[x * DK], rq[x * DK]
// for token x of the slice): per token the precision step
// (the serial part) and the provisional fold against the reference rho, exact
// while |G - rho| stays within kLost and no exponent clamps:
//   Q' = q/lambda 2^(G - rho) = q p/n 2^x,   K' = beta k 2^(rho - G) = beta k d/p 2^-x
// written over the q and k tiles (bf16; the K' remainder into the klo tile).
// The slice's G range is folded into the quarter's (the first slice of a
// quarter also counts G just before it); then the state is renormalised.
template <bool SECOND, int DK>
__device__ __forceinline__ void walk_slice(KeyWalk &w, uint8_t *qt, uint8_t *kt, uint8_t *klo, const int (&sw)[8],
                                           int s8, float bsrc, const float *ra, const float *rq, int rho) {
    const int rb = s8 * kSl * 128, bl0 = (s8 * kSl) & 31;
    if (!SECOND) {
        w.rkmin = __fdividef(w.d, w.p);
        w.rkmax = w.rkmin;
    }
    uint32_t kw[kSl], qw[kSl];
    float be[kSl], A[kSl], Q[kSl];
#pragma unroll
    for (int x = 0; x < kSl; ++x) {
        A[x] = ra[x * DK];
        Q[x] = rq[x * DK];
        kw[x] = *reinterpret_cast<const uint16_t *>(kt + sw[x] + rb + x * 128);
        qw[x] = *reinterpret_cast<const uint16_t *>(qt + sw[x] + rb + x * 128);
        be[x] = __shfl_sync(0xffffffffu, bsrc, bl0 + x);
    }
#pragma unroll
    for (int x = 0; x < kSl; ++x) {
        const int o = sw[x] + rb + x * 128;
        const float kf = bf16_val(kw[x]);
        const float bk = be[x] * kf;
        w.d = fmaf(A[x] * A[x], w.d, Q[x] * w.n);
        w.n = fmaf(bk * kf, w.d, w.n);
        w.p *= A[x];
        const float rc = rcp_approx(w.p * w.n);
        const float qo = (bf16_val(qw[x]) * (w.p * w.mq)) * (w.p * rc);
        const float rk = w.d * (w.n * rc);
        const float ko = bk * (rk * w.mk);
        w.rkmin = fminf(w.rkmin, rk);
        w.rkmax = fmaxf(w.rkmax, rk);
        const uint16_t kh = bf16_bits(ko);
        *reinterpret_cast<uint16_t *>(qt + o) = bf16_bits(qo);
        *reinterpret_cast<uint16_t *>(kt + o) = kh;
        *reinterpret_cast<uint16_t *>(klo + o) = bf16_bits(ko - bf16_val(kh));
    }
    // with d/p in [2^e, 2^(e+1)), G - rho lies in (x - e - 1, x - e]
    const int2 gr = make_int2(w.x - expo(w.rkmax) - 1, w.x - expo(w.rkmin));
    if (!SECOND) {
        w.cl = gr;
    } else {
        w.cl = runion(w.cl, gr);
        w.q0 = w.q1; w.q1 = w.q2; w.q2 = w.q3; w.q3 = w.cl;
    }
    norm_state(w.n, w.d, w.p, w.E, w.F);
    w.x = w.F - w.E - rho;
    w.clamped |= w.x != clampe(w.x);
    w.mq = pow2i(clampe(w.x));
    w.mk = pow2i(-clampe(w.x));
}

// The strong-forgetting path of the diagonal gate: walks one key through the
// chunk again from its start state and folds every token of quarter q against
// the reference ref[q] (a, qn, beta, q, k reloaded from global memory: the tile
// words were overwritten by the provisional fold). Out of line: it runs only
// when a provisional fold lost bits.
template <int DK>
__device__ __noinline__ void rewalk_key(uint8_t *qt, uint8_t *kt, uint8_t *klo, int cb, float n, float d, float p,
                                        int E, int F, int4 ref, const float *a, const float *qn, const float *beta,
                                        const __nv_bfloat16 *q, const __nv_bfloat16 *k, long long tok0, int nval,
                                        int H, int h, int i) {
    float mq = 1.f, mk = 1.f;
#pragma unroll 1
    for (int r = 0; r < kC; ++r) {
        if ((r & 7) == 0) {
            const int qq = r >> 4;
            const int rr = qq == 0 ? ref.x : qq == 1 ? ref.y : qq == 2 ? ref.z : ref.w;
            const int e = clampe(F - E - rr);
            mq = pow2i(e);
            mk = pow2i(-e);
        }
        const long long tok = tok0 + r;
        const long long off = (tok * H + h) * DK + i;
        float ar = 1.f, qr = 0.f, kf = 0.f, qf = 0.f, be = 0.f;
        if (r < nval) {
            ar = __ldg(a + off);
            qr = __ldg(qn + off);
            kf = __bfloat162float(k[off]);
            qf = __bfloat162float(q[off]);
            be = __ldg(beta + tok * H + h);
        }
        const float bk = be * kf;
        d = fmaf(ar * ar, d, qr * n);
        n = fmaf(bk * kf, d, n);
        p *= ar;
        const float rc = __frcp_rn(p * n);
        const float qo = ((qf * p) * (p * rc)) * mq;
        const float ko = bk * ((d * (n * rc)) * mk);
        const uint16_t kh = bf16_bits(ko);
        const int o = (cb + r * 128) ^ ((r & 7) << 4);
        *reinterpret_cast<uint16_t *>(qt + o) = bf16_bits(qo);
        *reinterpret_cast<uint16_t *>(kt + o) = kh;
        *reinterpret_cast<uint16_t *>(klo + o) = bf16_bits(ko - bf16_val(kh));
        if ((r & 7) == 7) norm_state(n, d, p, E, F);
    }
}

}  // namespace

template <int DK, int DV, bool ISO, bool LOCAL>
__global__ void __launch_bounds__(Roles<DK, DV, ISO>::THREADS, Roles<DK, DV, ISO>::MIN_BLOCKS)
kla_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qs,
                    const TcArgs g) {
    using L = Layout<DK, DV>;
    using RL = Roles<DK, DV, ISO>;
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
    // the epilogue's hand-offs to the MMA warp: the pass's state snapshot is in
    // shared memory; its P tile is (one barrier per P buffer, so that a phase is
    // seen before the barrier can complete again)
    uint64_t *snap_ready = bars + 9, *p_ready = bars + 10;
    // isotropic gate: the chunk's per-token factors are in shared memory (per stage)
    uint64_t *scan_done = bars + 12;
    // a / qn ring of the diagonal gate: slot landed, slot read by every gate warp
    uint64_t *ring_full = bars + 14, *ring_empty = bars + 14 + kRs;
    uint32_t *tmem_hold = reinterpret_cast<uint32_t *>(sm + L::hold0);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::hold0 + 4);
    int *lvl = reinterpret_cast<int *>(sm + L::lvl0);
    int *facd = reinterpret_cast<int *>(sm + L::fac0);
    float *facf = reinterpret_cast<float *>(sm + L::facf0);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&qk_ready[s], RL::QKA);
            lvl[s] = -1;
        }
        mbar_init(s_full, 1);
        mbar_init(u_done, 1);
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        mbar_init(td_bar, 1);
        mbar_init(snap_ready, 128);
        mbar_init(&scan_done[0], 32);
        mbar_init(&scan_done[1], 32);
        mbar_init(&p_ready[0], 128);
        mbar_init(&p_ready[1], 128);
        if (!ISO)
            for (int r = 0; r < kRs; ++r) {
                mbar_init(&ring_full[r], 1);
                mbar_init(&ring_empty[r], RL::NGW);
            }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == RL::MMAW && lane == 0) {
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
            // ---- diagonal: thread = key i; it walks every token of the segment, so
            // the precision chain and its exponents stay in registers
            const int i = warp * 32 + lane;
            // byte offset of (row r, key i) in a 128B-swizzled tile: sw[r & 7] + 128 r
            // (the 16-byte chunk index, bits 4-6 of cb, is XORed with r & 7; the row
            // term leaves those bits alone)
            const int cb = ((i >> 6) * (kC * 128) + ((i & 7) << 1)) | (((i & 63) >> 3) << 4);
            int sw[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) sw[x] = cb ^ (x << 4);
            // beta of tokens lane and 32 + lane of chunk c
            auto load_beta = [&](int c, int half) {
                const long long tok = tb + (long long)c * kC + 32 * half + lane;
                return tok < te ? __ldg(g.beta + tok * g.H + h) : 0.f;
            };
            KeyWalk w;
            w.n = seg_lambda(i);
            w.d = 1.f;
            w.p = 1.f;
            w.E = w.F = 0;
            w.cl = w.q0 = w.q1 = w.q2 = w.q3 = make_int2(0, 0);
            int rho = 0;   // reference in force (segment-start frame)
            float bA = 0.f, bB = 0.f;
            if (nchunks > 0) {
                bA = load_beta(0, 0);
                bB = load_beta(0, 1);
            }
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const long long tok0 = tb + (long long)c * kC;
                uint8_t *qt = sm + L::q0 + st * L::QK;
                uint8_t *kt = sm + L::k0 + st * L::QK;
                uint8_t *klo = sm + L::klo0 + st * L::QK;
                const float cA = bA, cB = bB;
                if (c + 1 < nchunks) {
                    bA = load_beta(c + 1, 0);
                    bB = load_beta(c + 1, 1);
                }
                if (!waitw(&stage_full[st], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
                // the chunk-start state, for a re-walk
                const float nc = w.n, dc = w.d, pc0 = w.p;
                const int Ec = w.E, Fc = w.F;
                // d and p are normalised at a slice end, so G - rho lies within 1 of
                // x = (F - E) - rho; the reference moves to the chunk start once x
                // has drifted beyond kMove (then the provisional fold needs no rescale
                // unless G moves by more than kStick - kMove inside the chunk)
                int x = w.F - w.E - rho;
                const int pre = abs(x) > kMove ? x : 0;
                rho += pre;
                x -= pre;
                w.x = x;
                w.clamped = false;
                w.mq = pow2i(clampe(x));
                w.mk = pow2i(-clampe(x));
                // the chunk's ring slots (two slices each), released once read
#pragma unroll 1
                for (int s16 = 0; s16 < kRpc; ++s16) {
                    const int j = c * kRpc + s16, slot = j % kRs;
                    if (!waitw(&ring_full[slot], (j / kRs) & 1, abort_flag, g.status)) { ok = false; break; }
                    float *ra = reinterpret_cast<float *>(sm + L::ring0 + slot * L::RSLOT) + i;
                    float *rq = ra + kRt * DK;
                    const long long ts = tok0 + s16 * kRt;
                    if (ts + kRt > te) {
                        // past the segment end: identity steps (beta is 0 there); each
                        // thread rewrites its own key's column only
                        for (int x = 0; x < kRt; ++x)
                            if (ts + x >= te) {
                                ra[x * DK] = 1.f;
                                rq[x * DK] = 0.f;
                            }
                        fence_proxy_async();
                    }
                    const float bs = s16 < kRpc / 2 ? cA : cB;
                    walk_slice<false, DK>(w, qt, kt, klo, sw, 2 * s16, bs, ra, rq, rho);
                    walk_slice<true, DK>(w, qt, kt, klo, sw, 2 * s16 + 1, bs, ra + kSl * DK, rq + kSl * DK, rho);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ring_empty[slot]);
                }
                if (!ok) break;
                // ---- references of the pass quarters (relative to rho; R = 0 keeps it)
                int R[4];
                bool bad;
                {
                    const int2 qr[4] = {w.q0, w.q1, w.q2, w.q3};
                    const int lv = choose_refs(qr, 0, R, bad);
                    const int lvw = __reduce_max_sync(0xffffffffu, lv);
                    if (lane == 0) atomicMax(&lvl[st], (c << 2) | lvw);
                }
                if (bad) atomicOr(g.status, kStatusRange);
#pragma unroll
                for (int q = 0; q < 4; ++q) facd[(st * 4 + q) * DK + i] = q ? R[q] - R[q - 1] : pre + R[0];
                if (LOCAL && p > 0) {
                    float *rl = g.rlog + ((u * g.NC + chunk_base + c) * 4) * DK + i;
#pragma unroll
                    for (int q = 0; q < 4; ++q) rl[q * DK] = (float)(rho + R[q]);
                }
                const int2 wr = runion(runion(w.q0, w.q1), runion(w.q2, w.q3));
                bool far = false, moved = false;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    far |= abs(R[q]) > kLost;
                    moved |= R[q] != 0;
                }
                // the provisional fold is exact while |G - rho| stayed within kLost and
                // no exponent clamped; a rescale by more than 2^kLost is not taken in
                // one step either: re-walk instead
                if (w.clamped || far || wr.x < -kLost || wr.y > kLost) {
                    rewalk_key<DK>(qt, kt, klo, cb, nc, dc, pc0, Ec, Fc,
                                   make_int4(rho + R[0], rho + R[1], rho + R[2], rho + R[3]), g.a, g.qn, g.beta,
                                   reinterpret_cast<const __nv_bfloat16 *>(g.q),
                                   reinterpret_cast<const __nv_bfloat16 *>(g.k), tok0,
                                   (int)min((long long)kC, te - tok0), g.H, h, i);
                } else if (moved) {
                    // a quarter's reference moved: rescale its folded bf16 values
                    // exactly by powers of two (Q' by 2^-R, K' by 2^R)
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        const int r = pick4(R, q);
                        if (r == 0) continue;
                        const float fq = pow2i(-r), fk = pow2i(r);
#pragma unroll 1
                        for (int row = kQ * q; row < kQ * (q + 1); ++row) {
                            const int o = sw[row & 7] + row * 128;
                            uint16_t *wq = reinterpret_cast<uint16_t *>(qt + o);
                            uint16_t *wk = reinterpret_cast<uint16_t *>(kt + o);
                            uint16_t *wl = reinterpret_cast<uint16_t *>(klo + o);
                            *wq = bf16_bits(bf16_val(*wq) * fq);
                            *wk = bf16_bits(bf16_val(*wk) * fk);
                            *wl = bf16_bits(bf16_val(*wl) * fk);
                        }
                    }
                }
                rho += R[3];
                if (c == nchunks - 1) {
                    // final outputs of the segment: 2^(G_end - rho) for the state
                    // export, the precision, and the segment's gate product
                    const float ge = w.p / w.d;
                    const int xe = w.F - w.E;
                    facf[i] = scale2(ge, xe - rho);
                    if (LOCAL)
                        g.decay[(u * g.P + p) * DK + i] =
                            xe < -250 ? 0.f : (xe > 250 ? __int_as_float(0x7f800000) : scale2(ge, xe));
                    if (last_seg && g.final_lambda) g.final_lambda[u * DK + i] = w.n / w.d;
                }
                fence_proxy_async();
                mbar_arrive(&qk_ready[st]);
            }
            if (nchunks == 0 && last_seg && g.final_lambda) g.final_lambda[u * DK + i] = w.n;
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
            // warp 0 scans each chunk's precision path and writes its per-token
            // factors (up to two chunks ahead of the folding); the other gate warps
            // fold the rows once a chunk's factors are in (scan_done)
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
                        const float b0 = va ? cb0 * row_sumsq<DK>(kt, t0i, lane) * inv_dk : 0.f;
                        const float b1 = vb ? cb1 * row_sumsq<DK>(kt, t1i, lane) * inv_dk : 0.f;
                        Mob Mp = mob_norm(mob_mul(mob_step(a1, q1, b1), mob_step(a0, q0, b0)));
#pragma unroll
                        for (int d = 1; d < 32; d <<= 1) {
                            Mob o = shfl_up_mob(Mp, d);
                            if (lane >= d) Mp = mob_norm(mob_mul(Mp, o));
                        }
                        Mob Ex = shfl_up_mob(Mp, 1);
                        if (lane == 0) Ex = Mob{1.f, 0.f, 0.f, 1.f};
                        const float lamA = fmaf(Ex.m00, lam, Ex.m01) * rcp_approx(fmaf(Ex.m10, lam, Ex.m11));
                        float g0 = 1.f, lamB = lamA, g1 = 1.f, lamC;
                        if (va) { float rr = rcp_approx(fmaf(a0, a0, q0 * lamA)); g0 = a0 * rr; lamB = fmaf(lamA, rr, b0); }
                        lamC = lamB;
                        if (vb) { float rr = rcp_approx(fmaf(a1, a1, q1 * lamB)); g1 = a1 * rr; lamC = fmaf(lamB, rr, b1); }
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
                        isof[st * kC + t0i] =
                            va ? make_float2(ex2_approx(e0) * rcp_approx(lamB), cb0 * ex2_approx(-e0)) : make_float2(0.f, 0.f);
                        isof[st * kC + t1i] =
                            vb ? make_float2(ex2_approx(e1) * rcp_approx(lamC), cb1 * ex2_approx(-e1)) : make_float2(0.f, 0.f);
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
                if (warp == 0) {
                    if (!okw) { ok = false; break; }
                    mbar_arrive(&scan_done[st]);
                    continue;
                }
                if (!waitw(&scan_done[st], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
                // fold the rows: Q' = q fq, K' = k fk (hi + remainder). A folding thread
                // keeps one key pair and a fixed set of rows within every 8-row group
                // (so that its swizzled offsets are fixed); a warp shares the rows, so
                // the row factors are broadcast reads
                {
                    constexpr int NP = DK / 2, FT = RL::GT - 32;
                    constexpr int RS = FT / NP, XR = 8 / RS;      // threads per pair, rows per group
                    const int ft = tid - 32, i0 = 2 * (ft % NP), s = ft / NP;
                    const int cbp = ((i0 >> 6) * (kC * 128) + ((i0 & 7) << 1)) | (((i0 & 63) >> 3) << 4);
                    const int x0 = s * XR;
#pragma unroll 2
                    for (int r8 = 0; r8 < kC; r8 += 8) {
#pragma unroll
                        for (int x = 0; x < XR; ++x) {
                            const int row = r8 + x0 + x;
                            const int off = (cbp ^ ((x0 + x) << 4)) + row * 128;
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
                    }
                }
                fence_proxy_async();
                mbar_arrive(&qk_ready[st]);
            }
            if (warp == 0 && lane == 0 && nchunks == 0 && last_seg && g.final_lambda) g.final_lambda[u] = lam;
        }
        (void)ok;
    } else if (!ISO && warp == RL::EPIW + 4) {
        // ================= a / qn producer (diagonal precision): the gate's ring
        // slots of kRt tokens, and an L2 prefetch of the slot two chunks ahead
        if (!ISO && lane == 0) {
            uint8_t *ring = sm + L::ring0;
            const int nrs = nchunks * kRpc;
            auto prefetch = [&](int j) {
                const int tok = (int)(tb + (long long)j * kRt);
                tma_prefetch_3d(&tm_a, 0, h, tok);
                tma_prefetch_3d(&tm_qn, 0, h, tok);
            };
            for (int j = kRs; j < min(nrs, 2 * kRpc); ++j) prefetch(j);
            int j = 0;
            for (; j < nrs; ++j) {
                const int slot = j % kRs;
                if (j >= kRs && !wait1(&ring_empty[slot], ((j / kRs) - 1) & 1, abort_flag, g.status)) break;
                float *dst = reinterpret_cast<float *>(ring + slot * L::RSLOT);
                const int tok = (int)(tb + (long long)j * kRt);
                mbar_expect_tx(&ring_full[slot], L::RSLOT);
                tma_load_3d(dst, &tm_a, &ring_full[slot], 0, h, tok);
                tma_load_3d(dst + kRt * DK, &tm_qn, &ring_full[slot], 0, h, tok);
                if (j + 2 * kRpc < nrs) prefetch(j + 2 * kRpc);
            }
            // the copies issued land before the CTA exits
            for (int r = max(0, j - kRs); r < j; ++r)
                wait_slow(&ring_full[r % kRs], (r / kRs) & 1, abort_flag, g.status, false);
        }
    } else if (warp < RL::EPIW + 4) {
        // ================= epilogue warps: rescale U in TMEM and snapshot it to
        // bf16 shared memory, mask the score tile into P, store the output rows;
        // each pass is handed to the MMA warp through mbarriers ==============
        const int we = warp & 3;               // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(32 * we) << 16;
        const int row64 = 16 * we + lane;
        const bool v64 = lane < 16;
        const int rowU = (DK == 128) ? (32 * we + lane) : row64;
        const bool vU = (DK == 128) || v64;
        uint8_t *ub = sm + L::ub0;
        uint8_t *pt = sm + L::p0;
        const float *eta0 = ((!LOCAL || p == 0) && g.eta0) ? g.eta0 + u * DK * DV : nullptr;
        bool ok = true;
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
        for (int c = 0; c < nchunks && ok; ++c) {
            const int st = c & 1;
            if (!waitw(&qk_ready[st], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
            const int lv = lvl[st] & 3;
            const int np = 1 << lv, qper = 4 >> lv;
            for (int k = 0; k < np; ++k) {
                const int m0 = kQ * qper * k, m1 = m0 + kQ * qper;
                uint8_t *ptp = pt + (pc & 1) * L::PT;         // this pass's P buffer
                // ---- state: U <- 2^d U for this pass's reference, snapshot to bf16
                // (the previous pass's state update, and its Q' U reading the old
                // snapshot, have completed)
                if (pc > 0 && !waitw(u_done, (pc - 1) & 1, abort_flag, g.status)) { ok = false; break; }
                tc_fence_after();
                const int d = vU ? facd[(st * 4 + k * qper) * DK + rowU] : 0;
                const bool rmw = __any_sync(0xffffffffu, d != 0);
                {
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
                mbar_arrive(snap_ready);
                // ---- P = the pass's block of the causal score tile, bf16
                if (k == 0 && !waitw(s_full, c & 1, abort_flag, g.status)) { ok = false; break; }
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
                mbar_arrive(&p_ready[pc & 1]);
                // ---- output rows of the previous pass (its MMAs have finished
                // while this pass was prepared)
                if (pend_c >= 0) emit(pc - 1, pend_c, pend_m0, pend_m1);
                pend_c = c; pend_m0 = m0; pend_m1 = m1;
                ++pc;
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
    } else if (warp == RL::MMAW) {
        // ================= MMA warp: the q, k, v tile loads, the q' export of
        // split rows (lane 0), and the tcgen05 MMAs (the converged warp, one
        // elected lane issuing: see mma_bf16_warp) ===========================
        bool ok = true;
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
            }
        };
        int loaded = 0;                                 // chunks whose loads were issued
        const int nload = g.withhold_tiles ? 0 : nchunks;
        if (lane == 0)
            for (; loaded < 2 && loaded < nload; ++loaded) load_chunk(loaded);
        loaded = min(2, nload);
        constexpr uint32_t iS = idesc_bf16(64, 64, false, false);
        constexpr uint32_t iO = idesc_bf16(64, DV, false, true);
        constexpr uint32_t iU = idesc_bf16(DK, DV, true, true);
        const uint32_t tS = tbase + L::colS, tO = tbase + L::colO, tU = tbase + L::colU;
        const uint64_t du = sdesc_sw128(smem_u32(sm + L::ub0), DK * 128, 1024);
        int pc = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int st = c & 1;
            if (!waitw(&qk_ready[st], (c >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
            const int lv = lvl[st] & 3;
            const int np = 1 << lv, qper = 4 >> lv;
            if (LOCAL && p > 0 && lane == 0) {
                // export the folded q tile (the correction pass multiplies it by
                // the carried segment-start state)
                const int tok0 = (int)(tb + (long long)c * kC);
#pragma unroll
                for (int a = 0; a < DK / 64; ++a)
                    tma_store_3d(&tm_qs, sm + L::q0 + st * L::QK + a * kC * 128, 64 * a, h, tok0);
                tma_store_commit();
            }
            __syncwarp();
            tc_fence_after();
            // scores of the whole chunk (each pass masks its own block); a K step
            // moves a descriptor's start address by (bytes >> 4)
            const uint32_t qa = smem_u32(sm + L::q0 + st * L::QK), ka = smem_u32(sm + L::k0 + st * L::QK);
            const uint64_t dq = sdesc_sw128(qa, 16, 1024), dk = sdesc_sw128(ka, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * (kC * 128) + (kk & 3) * 32) >> 4;
                mma_bf16_warp(tS, dq + off, dk + off, iS, kk > 0);
            }
            mma_commit_warp(s_full);
            const uint64_t dv = sdesc_sw128(smem_u32(sm + L::v0 + st * L::V), kC * 128, 1024);
            const uint64_t dkm = sdesc_sw128(ka, kC * 128, 1024);
            const uint64_t dl = sdesc_sw128(smem_u32(sm + L::klo0 + st * L::QK), kC * 128, 1024);
            for (int k = 0; k < np; ++k) {
                const int s0 = k * qper;                      // first 16-token slice of this pass
                const uint32_t tOp = tO + (pc & 1) * DV;      // this pass's output accumulator
                const uint64_t dp = sdesc_sw128(smem_u32(sm + L::p0 + (pc & 1) * L::PT), 16, 1024);
                // O = Q' U (the snapshot) into this pass's accumulator (its contents
                // two passes back were read out before the snapshot), then the state
                // update over the pass's tokens (hi and remainder of K'): it reads
                // only K' and V, so it runs while P is masked
                if (!waitw(snap_ready, pc & 1, abort_flag, g.status)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * (kC * 128) + (kk & 3) * 32) >> 4;
                    mma_bf16_warp(tOp, dq + off, du + kk * (2048 >> 4), iO, kk > 0);
                }
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    if (x < qper) {
                        const uint32_t ko = (s0 + x) * (2048 >> 4);
                        mma_bf16_warp(tU, dkm + ko, dv + ko, iU, 1);
                        mma_bf16_warp(tU, dl + ko, dv + ko, iU, 1);
                    }
                mma_commit_warp(u_done);
                // O += P V over the pass's tokens: its last MMA
                if (!waitw(&p_ready[pc & 1], (pc >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    if (x < qper) mma_bf16_warp(tOp, dp + (s0 + x) * (32 >> 4), dv + (s0 + x) * (2048 >> 4), iO, 1);
                mma_commit_warp(&o_full[pc & 1]);
                ++pc;
            }
            if (!ok) break;
            // every MMA of the chunk has completed once its last P V has: the
            // stage takes the chunk two ahead once the q' export has read it
            if (!waitw(&o_full[(pc - 1) & 1], ((pc - 1) >> 1) & 1, abort_flag, g.status)) { ok = false; break; }
            if (lane == 0) {
                if (LOCAL && p > 0) tma_store_wait_read();
                if (loaded < nload) load_chunk(loaded);
            }
            if (loaded < nload) ++loaded;
        }
        if (lane == 0) {
            if (LOCAL && p > 0) tma_store_wait_all();
            if (!ok || *abort_flag) {
                // wait (bounded) until every tile load issued has landed
                for (int c = max(0, loaded - 2); c < loaded; ++c)
                    wait_slow(&stage_full[c & 1], (c >> 1) & 1, abort_flag, g.status, false);
            }
        }
        __syncwarp();
        // all MMAs issued have completed before TMEM is released
        mma_commit_warp(td_bar);
        if (lane == 0) wait_slow(td_bar, 0, abort_flag, g.status, false);
        __syncwarp();
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
    // a and qn: ring slots of kRt tokens (their L2 prefetch uses the same boxes)
    if (ok && !p.iso)
        ok = make_tma_map(&ma, a, F32, 4, DK, p.H, p.ntok, DK, kRt, false) &&
             make_tma_map(&mqn, qn, F32, 4, DK, p.H, p.ntok, DK, kRt, false);
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
    const char *wt = getenv("KLA_TEST_WITHHOLD_TILES");
    g.withhold_tiles = (wt && *wt && *wt != '0') ? 1 : 0;
    const unsigned grid = (unsigned)((long long)p.N * p.H * p.P);
    if (grid == 0) return cudaSuccess;
    const int threads = p.iso ? Roles<DK, DV, true>::THREADS : Roles<DK, DV, false>::THREADS;
    return launch_pdl(kerns[which], grid, threads, L::alloc, st, mq, mk, mv, ma, mqn, mqs, g);
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
