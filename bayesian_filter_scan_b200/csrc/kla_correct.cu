// kla_correct.cu -- the carried state of rows split into segments.
//
// The mean recursion is affine in eta (Kalman Linear Attention, technical
// summary section 2), so the output of a segment that starts from the belief
// eta_start is the output it gives from a zero start plus the readout of
// eta_start carried through the segment's gates:
//     out_t = out_t|0 + sum_i q[t,i] / lambda[t,i] 2^(G[t,i]) eta_start[i,:],
// G the cumulative log2 gate from the segment start. The chunk kernel (mode 2)
// walks every segment from a zero start, writes the segment's transfer and gate
// product, and exports its folded q tiles Q' = q/lambda 2^(G - rho) with the
// log2 factor rlog = rho (per chunk, 16-token pass quarter and key) that takes
// them to the segment start. Here: first the segment-start beliefs of every row,
//     eta_start(1) = T_0, eta_start(q+1) = D_q eta_start(q) + T_q,
// and the final belief D_{P-1} eta_start(P-1) + T_{P-1} (T_0 is segment 0's
// end state from eta0; T_q, D_q the transfers and gate products); then, per
// chunk of every segment p >= 1, on the tensor cores,
//     out[chunk rows] += Q' (64 x dk) . diag(2^rlog) eta_start(p) (dk x dv),
// one product per chunk when its four quarters share their references (a
// chunk the walk took in one pass), else one per quarter, each adding only its
// quarter's rows.
//
// Correction CTA = a range of chunks of one (row, head, segment p >= 1), 128
// threads, two per SM. Chunks whose operand diag(2^rlog) eta_start rounds to
// zero for every key (the carried state has decayed below bf16 range there) add
// exactly zero and are skipped. The Q' and output tiles of the others stream
// through a 2-stage TMA ring; thread 0 issues the copies and the tcgen05 MMAs
// into a TMEM accumulator; the operand is rebuilt in shared memory (bf16),
// the rows of the keys whose factor changed; all threads add the TMEM result to
// the output tile in shared memory, which a TMA store writes back.
// Every wait is bounded: on a timeout the status bit is set and the CTA stops
// after its copies in flight have landed.
#include <algorithm>

#include "kla_internal.cuh"
#include "kla_tc_ptx.cuh"

namespace kla {
using namespace ptx;

namespace {

constexpr int kCC = 64;   // chunk tokens (the chunk kernel's)
constexpr int kQ = 16;    // tokens per pass quarter (the chunk kernel's)
constexpr uint64_t kCorrWaitNs = 2000000000ull;
constexpr int kMaxRange = 256;   // chunks per correction CTA at most
// log2 of a size below which bf16(2^rlog eta) rounds to zero, with margin
constexpr float kZeroLog2 = -140.f;

struct CorrArgs {
    int H, P, NB, seg_blocks, iso, cpr;
    long long T, Lseg;
    const float *S_io, *rlog;
    __nv_bfloat16 *out;
    int *status;
};

template <int DK, int DV>
struct CLayout {
    static constexpr int QT = kCC * DK * 2;        // one folded q tile (128B-swizzled 64-column atoms)
    static constexpr int OT = kCC * DV * 2;        // one output tile (same layout)
    static constexpr int ST = QT + OT;             // one stage
    static constexpr int st0 = 0;                  // two stages
    static constexpr int b0 = 2 * ST;              // diag(2^rlog) eta_start, bf16 [DK][DV] swizzled
    static constexpr int r0 = b0 + DK * DV * 2;    // rlog the operand was built with, [DK]
    static constexpr int m0 = r0 + DK * 4;         // log2 max |eta_start| per key, [DK]
    static constexpr int l0 = m0 + DK * 4;         // chunks of the range that can contribute, [kMaxRange + 1]
    static constexpr int bar0 = (l0 + (kMaxRange + 1) * 4 + 7) & ~7;
    static constexpr int bytes = bar0 + 8 * 8;
    static constexpr int alloc = bytes + 1024;
    static_assert(2 * (alloc + 1024) <= 233472, "two CTAs per SM");
    static constexpr uint32_t NCOLS = (DV <= 32) ? 32u : (uint32_t)DV;   // one fp32 accumulator
};

__device__ __forceinline__ int csw_off(int row, int col, int rows) {
    return (col >> 6) * (rows * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1);
}

__device__ __forceinline__ uint32_t cpack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __noinline__ bool cwait(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait_sleep(bar, parity, 20000u))
        if (globaltimer() - t0 > kCorrWaitNs) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    return true;
}

// Segment-start beliefs of a row's segments from their transfers, in place:
// S_io[q-1] <- eta_start(q) = D_{q-1} eta_start(q-1) + T_{q-1} (eta_start(0) = 0
// here: T_0 already starts from eta0), and the final belief
// D_{P-1} eta_start(P-1) + T_{P-1}. One thread per state element.
__global__ void __launch_bounds__(256)
kla_segment_starts(long long units, int DKV, int dv, int nl, int P, const float *__restrict__ decay,
                   float *__restrict__ S_io, float *__restrict__ final_eta) {
    pdl_release();
    pdl_wait();
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= units * DKV) return;
    const long long u = gid / DKV;
    const int e = (int)(gid % DKV);
    const int il = nl == 1 ? 0 : e / dv;
    float x[8], dc[8];
    float S = 0.f;
    for (int q0 = 0; q0 < P; q0 += 8) {
#pragma unroll
        for (int r = 0; r < 8; ++r)
            if (q0 + r < P) {
                x[r] = S_io[(u * P + q0 + r) * DKV + e];
                dc[r] = decay[(u * P + q0 + r) * nl + il];
            }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int q = q0 + r;
            if (q < P) {
                S = fmaf(dc[r], S, x[r]);          // the belief at the end of segment q
                if (q < P - 1) S_io[(u * P + q) * DKV + e] = S;
                else if (final_eta) final_eta[u * DKV + e] = S;
            }
        }
    }
}

}  // namespace

template <int DK, int DV>
__global__ void __launch_bounds__(128, 2)
kla_correct_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_o,
                   const CorrArgs g) {
    using L = CLayout<DK, DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar0);
    uint64_t *full = bars, *mma_done = bars + 2;          // [2] each
    uint32_t *tmem_hold = reinterpret_cast<uint32_t *>(bars + 4);
    uint8_t *Bt = sm + L::b0;
    float *rcur = reinterpret_cast<float *>(sm + L::r0);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA = (row x head u, segment p >= 1, range r of cpr chunks)
    const int ranges = (g.seg_blocks + g.cpr - 1) / g.cpr;
    const long long ur = blockIdx.x / ranges;
    const int r = (int)(blockIdx.x % ranges);
    const int ps = g.P - 1;
    const long long u = ur / ps;
    const int p = 1 + (int)(ur % ps);
    const int n = (int)(u / g.H), h = (int)(u % g.H);
    const long long tb = (long long)n * g.T + (long long)p * g.Lseg;
    const long long te = (long long)n * g.T + min((long long)(p + 1) * g.Lseg, g.T);
    const int seg_chunks = te > tb ? (int)((te - tb + kCC - 1) / kCC) : 0;
    const int c0 = r * g.cpr, c1 = min(seg_chunks, c0 + g.cpr);
    const int nch = max(0, c1 - c0);
    const float *Sst = g.S_io + (u * g.P + p - 1) * DK * DV;   // eta_start(p)

    if (tid == 0) {
        for (int j = 0; j < 2; ++j) {
            mbar_init(&full[j], 1);
            mbar_init(&mma_done[j], 1);
        }
        fence_mbar_init();
        prefetch_map(&tm_qs);
        prefetch_map(&tm_o);
    }
    if (warp == 0) tmem_alloc(tmem_hold, L::NCOLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_hold;
    pdl_release();
    pdl_wait();

    float *lmax = reinterpret_cast<float *>(sm + L::m0);
    int *list = reinterpret_cast<int *>(sm + L::l0);
    // references of this range's chunks: rl[(chunk * kQuarters + quarter) * DK + key]
    const float *rl = g.rlog + ((u * g.NB + (long long)p * g.seg_blocks + c0) * kQuarters) * DK;
    // short ranges take every chunk (the zero test would cost more than it saves)
    const bool test = nch > 2;
    // log2 max |eta_start| per key
    if (test && tid < DK) {
        float mx = 0.f;
        const float4 *src = reinterpret_cast<const float4 *>(Sst + tid * DV);
        for (int jj = 0; jj < DV / 4; ++jj) {
            const float4 x = __ldg(src + jj);
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
        }
        lmax[tid] = __log2f(mx);   // -inf for a zero row
    }
    __syncthreads();
    // The chunks whose operand diag(2^rlog) eta_start is not zero in bf16 for
    // some key and quarter; the others add exactly zero and are skipped.
    // list[0] = count.
    if (!test) {
        if (tid == 0) list[0] = nch;
        if (tid < nch) list[1 + tid] = tid;
    } else if (warp == 0) {
        int cnt = 0;
        for (int j0 = 0; j0 < nch; j0 += 32) {
            const int jj = j0 + lane;
            bool need = false;
            if (jj < nch)
                for (int x = 0; x < kQuarters * DK; ++x)
                    need |= __ldg(rl + (long long)jj * kQuarters * DK + x) + lmax[x % DK] >= kZeroLog2;
            const unsigned m = __ballot_sync(0xffffffffu, need);
            if (need) list[1 + cnt + __popc(m & ((1u << lane) - 1u))] = jj;
            cnt += __popc(m);
        }
        if (lane == 0) list[0] = cnt;
    }
    __syncthreads();
    const int nl2 = list[0];
    auto issue = [&](int k) {   // k-th listed chunk into stage k & 1
        const int s = k & 1;
        const int tok = (int)(tb + (long long)(c0 + list[1 + k]) * kCC);
        uint8_t *d = sm + L::st0 + s * L::ST;
        mbar_expect_tx(&full[s], L::ST);
#pragma unroll
        for (int a = 0; a < DK / 64; ++a) tma_load_3d(d + a * kCC * 128, &tm_qs, &full[s], 64 * a, h, tok);
#pragma unroll
        for (int a = 0; a < DV / 64; ++a) tma_load_3d(d + L::QT + a * kCC * 128, &tm_o, &full[s], 64 * a, h, tok);
    };
    int issued = 0;
    if (tid == 0) {
        for (int k = 0; k < 2 && k < nl2; ++k) issue(k);
        issued = min(2, nl2);
    }
    if (tid < DK) rcur[tid] = __int_as_float(0x7fc00000);   // NaN: the first chunk builds the operand
    __syncthreads();

    const uint32_t idesc = idesc_bf16(64, DV, false, true);
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int row64 = 16 * warp + lane;
    const bool v64 = lane < 16;
    bool ok = true;
    int nmma = 0;   // MMAs committed so far (phases of mma_done[0])
    for (int k = 0; k < nl2; ++k) {
        const int s = k & 1, c = c0 + list[1 + k];
        const float *rc = rl + (long long)list[1 + k] * kQuarters * DK;
        // one group when the four quarters share their references, else one per quarter
        bool same = true;
        if (tid < DK)
            for (int q = 1; q < kQuarters; ++q) same &= rc[q * DK + tid] == rc[tid];
        const int ngr = __syncthreads_and(same) ? 1 : kQuarters;
        if (!__syncthreads_and(cwait(&full[s], (k >> 1) & 1, g.status))) { ok = false; break; }
        uint8_t *ot = sm + L::st0 + s * L::ST + L::QT;
        for (int gi = 0; gi < ngr; ++gi) {
            const int q0 = ngr == 1 ? 0 : gi, q1 = ngr == 1 ? kQuarters : gi + 1;
            // rebuild the operand rows of the keys whose reference moved (thread =
            // key); the previous MMA, the last reader, has completed
            const float rnew = tid < DK ? rc[q0 * DK + tid] : 0.f;
            const bool changed = tid < DK && !(rnew == rcur[tid]);
            if (__syncthreads_or(changed)) {
                if (changed) {
                    rcur[tid] = rnew;
                    const float f = exp2f(rnew);
                    const float4 *src = reinterpret_cast<const float4 *>(Sst + tid * DV);
#pragma unroll 4
                    for (int jj = 0; jj < DV; jj += 8) {
                        const float4 a = __ldg(src + jj / 4), b = __ldg(src + jj / 4 + 1);
                        uint4 w;
                        w.x = cpack_bf2(f * a.x, f * a.y); w.y = cpack_bf2(f * a.z, f * a.w);
                        w.z = cpack_bf2(f * b.x, f * b.y); w.w = cpack_bf2(f * b.z, f * b.w);
                        *reinterpret_cast<uint4 *>(Bt + csw_off(tid, jj, DK)) = w;
                    }
                }
                fence_proxy_async();
                __syncthreads();
            }
            // D[64 x DV] = Q'[64 x DK] . B[DK x DV]
            if (tid == 0) {
                tc_fence_after();
                const uint32_t qa = smem_u32(sm + L::st0 + s * L::ST), ba = smem_u32(Bt);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (kCC * 128) + (kk & 3) * 32;
                    mma_bf16(tbase, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ba + kk * 2048, DK * 128, 1024),
                             idesc, kk > 0);
                }
                mma_commit(&mma_done[0]);
            }
            if (!__syncthreads_and(cwait(&mma_done[0], nmma & 1, g.status))) { ok = false; break; }
            ++nmma;
            tc_fence_after();
            // add the carried-state readout of this group's rows to the output tile
            const bool row_ok = v64 && row64 >= kQ * q0 && row64 < kQ * q1 && tb + (long long)c * kCC + row64 < te;
#pragma unroll
            for (int cb = 0; cb < DV / 32; cb += 2) {
                uint32_t rr[2][32];
                tmem_ld32(tbase + lane_base + cb * 32, rr[0]);
                tmem_ld32(tbase + lane_base + cb * 32 + 32, rr[1]);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 *dst = reinterpret_cast<uint4 *>(ot + csw_off(row64, (cb + hh) * 32 + q4 * 8, kCC));
                            const uint4 o = *dst;
                            const uint32_t ow[4] = {o.x, o.y, o.z, o.w};
                            uint32_t nw[4];
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float lo = __uint_as_float(ow[x] << 16) + __uint_as_float(rr[hh][q4 * 8 + 2 * x]);
                                const float hi =
                                    __uint_as_float(ow[x] & 0xffff0000u) + __uint_as_float(rr[hh][q4 * 8 + 2 * x + 1]);
                                nw[x] = cpack_bf2(lo, hi);
                            }
                            *dst = make_uint4(nw[0], nw[1], nw[2], nw[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
        }
        if (!ok) break;
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            // Write the tile back; its stage is reloaded once the store has read it.
            // The tile's rows past the segment end (a last partial chunk) were
            // loaded and are stored back unchanged: they are the first tokens of
            // the next row, which only segment 0 of that row writes, in the walk
            // launch that finished before this one.
            const int tok = (int)(tb + (long long)c * kCC);
#pragma unroll
            for (int a = 0; a < DV / 64; ++a) tma_store_3d(&tm_o, ot + a * kCC * 128, 64 * a, h, tok);
            tma_store_commit();
            if (issued < nl2) {
                tma_store_wait_read();
                issue(issued);
                ++issued;
            }
        }
    }
    if (tid == 0) {
        tma_store_wait_all();
        // on a timeout, the tiles issued but not consumed land before the CTA exits
        if (!ok)
            for (int k = 0; k < issued; ++k) mbar_try_wait_sleep(&full[k & 1], (k >> 1) & 1, 1000000u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, L::NCOLS);
}

namespace {

template <int DK, int DV>
cudaError_t launch_correct_t(const Plan &p, const float *S_io, void *out, int *status, cudaStream_t st) {
    using L = CLayout<DK, DV>;
    CUtensorMap mqs, mo;
    if (!make_tma_map(&mqs, p.qbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, p.H, p.ntok, 64, kCC, true) ||
        !make_tma_map(&mo, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, p.H, p.ntok, 64, kCC, true))
        return cudaErrorInvalidValue;
    static PerDevice<bool> attr;
    const cudaError_t ea = ensure_smem_attr(attr, kla_correct_kernel<DK, DV>, L::alloc);
    if (ea != cudaSuccess) return ea;
    CorrArgs g;
    g.H = p.H; g.P = p.P; g.NB = p.NB; g.seg_blocks = p.seg_blocks; g.iso = p.iso;
    g.T = p.T; g.Lseg = p.Lseg;
    g.S_io = S_io; g.rlog = p.rlog; g.status = status;
    g.out = (__nv_bfloat16 *)out;
    // chunks per CTA: enough ranges per segment for about four CTAs per SM (a
    // CTA's cost is mostly latency: its first tiles, then the chunks that
    // survive the zero test, which for decaying gates are the first few)
    const long long segs = (long long)p.N * p.H * (p.P - 1);
    if (segs <= 0) return cudaSuccess;
    int ranges = (int)std::max(1LL, (4LL * p.sms + segs - 1) / segs);
    ranges = std::min(ranges, p.seg_blocks);
    ranges = std::max(ranges, (p.seg_blocks + kMaxRange - 1) / kMaxRange);
    g.cpr = (p.seg_blocks + ranges - 1) / ranges;
    ranges = (p.seg_blocks + g.cpr - 1) / g.cpr;
    return launch_pdl(kla_correct_kernel<DK, DV>, (unsigned)(segs * ranges), 128, L::alloc, st, mqs, mo, g);
}

}  // namespace

cudaError_t launch_correct(const Plan &p, const float *S_io, const float *decay, void *out, float *final_eta,
                           int *status, cudaStream_t st) {
    // segment-start beliefs (and the final belief) first
    const long long units = (long long)p.N * p.H;
    const long long thr = units * p.dk * p.dv;
    cudaError_t e = launch_pdl(kla_segment_starts, (unsigned)((thr + 255) / 256), 256, 0, st, units, p.dk * p.dv,
                               p.dv, p.nl, p.P, decay, (float *)S_io, final_eta);
    if (e != cudaSuccess) return e;
#define KLA_CORR_CASE(DK_, DV_) \
    if (p.dk == DK_ && p.dv == DV_) return launch_correct_t<DK_, DV_>(p, S_io, out, status, st);
    KLA_CORR_CASE(64, 64)
    KLA_CORR_CASE(64, 128)
    KLA_CORR_CASE(128, 64)
    KLA_CORR_CASE(128, 128)
#undef KLA_CORR_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kla
