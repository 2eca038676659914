// kla_recurrent.cu -- token-by-token walk of the information-form filter on
// CUDA cores (fp32 throughout).
//
// Serves the fp32-input build (its tolerance needs fp32 products, which bf16
// or tf32 tensor-core operands cannot give), head dims the tensor-core chunk
// kernel does not take, and the one-token decode step. Per token it applies
// the filter exactly as stated (Kalman Linear Attention, technical summary
// section 1): OU predict of lambda and eta (gate g = a/(a^2+qn*lambda)),
// observation update (+beta*k^2, +beta*k*v), posterior-mean readout through q.
//
// One CTA walks one segment of one (row or packed sequence, head):
//   mode kOutput : starts from (lambda, eta) at the segment start, writes out
//                  (and the final belief on the last segment);
//   mode kState  : starts from eta = 0 and records the segment's transfer,
//                  eta_end = diag(prod g) eta_start + dS, for the carry kernel.
// 256 threads; thread (kg, j) holds eta[i, j] for KPG consecutive keys i of
// key group kg in registers. Tokens are processed in tiles of TT: the gate
// threads advance lambda and publish g, q/lambda, beta*k per (token, key) in
// shared memory, then every thread updates its slice of eta and its partial
// readout, then the partials are summed per value column.
#include "kla_internal.cuh"

namespace kla {

enum WalkMode : int { kOutput = 0, kState = 1 };

struct WalkArgs {
    int N, H, dk, dv, nl;
    long long T, Lseg;
    int P, NB, seg_blocks;
    const int *cu;             // packed sequence offsets or nullptr
    bool iso;
    int mode;
    const void *q, *k, *v;
    const float *a, *qn, *beta;
    const float *lambda0, *eta0;
    const float *lam_blk;      // lambda at block starts (segments p > 0)
    float *S_io;               // [u][P][dk][dv] transfer / segment-start eta
    float *decay;              // [u][P][nl] product of gates over a segment
    void *out;
    float *final_lambda, *final_eta;
    const int *perm;           // longest-first order of packed sequences or nullptr
};

constexpr int kWalkThreads = 256;
constexpr int kTT = 16;

__host__ __device__ inline size_t walk_smem_bytes(int dk, int dv) {
    int nkg = kWalkThreads / dv;
    return sizeof(float) * ((size_t)kTT * dk * 3 + (size_t)kTT * dv + (size_t)kTT * nkg * dv + 2 * kTT);
}

template <typename TIn, int KPG>
__global__ void __launch_bounds__(kWalkThreads)
kla_walk_simt(WalkArgs w) {
    pdl_release();
    pdl_wait();
    extern __shared__ float sm[];
    const int dk = w.dk, dv = w.dv;
    const int nkg = kWalkThreads / dv;
    float *gs = sm;                         // [kTT][dk]
    float *qts = gs + kTT * dk;             // [kTT][dk]
    float *kts = qts + kTT * dk;            // [kTT][dk]
    float *vs = kts + kTT * dk;             // [kTT][dv]
    float *part = vs + kTT * dv;            // [kTT][nkg][dv]
    float *lam_s = part + kTT * nkg * dv;   // [kTT] (iso)
    float *g1_s = lam_s + kTT;              // [kTT] (iso)

    const int tid = threadIdx.x;
    const int j = tid % dv, kg = tid / dv;
    const int P_eff = (w.mode == kState) ? (w.P - 1) : w.P;
    const long long ur = blockIdx.x / P_eff;
    const int p = (int)(blockIdx.x % P_eff);
    const int h = (int)(ur % w.H);
    const int n = w.perm ? w.perm[ur / w.H] : (int)(ur / w.H);
    const long long u = (long long)n * w.H + h;
    long long tb, te;
    if (w.cu) { tb = w.cu[n]; te = w.cu[n + 1]; }
    else {
        tb = (long long)n * w.T + (long long)p * w.Lseg;
        te = (long long)n * w.T + min((long long)(p + 1) * w.Lseg, w.T);
    }
    const TIn *q = (const TIn *)w.q, *k = (const TIn *)w.k, *v = (const TIn *)w.v;

    // belief at the segment start
    float lam = 1.0f, gprod = 1.0f;
    const bool gate_thread = w.iso ? (tid < 32) : (tid < dk);
    if (gate_thread) {
        int il = w.iso ? 0 : tid;
        if (p == 0) lam = w.lambda0 ? w.lambda0[u * w.nl + il] : 1.0f;
        else lam = w.lam_blk[(u * w.NB + (long long)p * w.seg_blocks) * w.nl + il];
    }
    float S[KPG];
#pragma unroll
    for (int r = 0; r < KPG; ++r) {
        int i = kg * KPG + r;
        float s0 = 0.0f;
        if (w.mode == kOutput) {
            if (p == 0) { if (w.eta0) s0 = w.eta0[(u * dk + i) * dv + j]; }
            else s0 = w.S_io[((u * w.P + p - 1) * dk + i) * dv + j];
        }
        S[r] = s0;
    }
    const float inv_dk = 1.0f / (float)dk;

    for (long long t0 = tb; t0 < te; t0 += kTT) {
        // ---- phase A: advance the precision, publish per-(token, key) factors
        if (!w.iso) {
            if (tid < dk) {
                const int i = tid;
#pragma unroll 4
                for (int tau = 0; tau < kTT; ++tau) {
                    long long tok = t0 + tau;
                    float g = 1.0f, qt = 0.0f, kt = 0.0f;
                    if (tok < te) {
                        long long th = tok * w.H + h;
                        float at = w.a[th * dk + i], qnt = w.qn[th * dk + i];
                        float kk = ld_in(k + th * dk + i), bt = w.beta[th];
                        float den = fmaf(at, at, qnt * lam);
                        g = at / den;
                        lam = fmaf(bt * kk, kk, lam / den);
                        kt = bt * kk;
                        if (w.mode == kOutput) qt = ld_in(q + th * dk + i) / lam;
                        gprod *= g;
                    }
                    gs[tau * dk + i] = g; qts[tau * dk + i] = qt; kts[tau * dk + i] = kt;
                }
            }
        } else {
            if (tid < 32) {
                for (int tau = 0; tau < kTT; ++tau) {
                    long long tok = t0 + tau;
                    float g = 1.0f;
                    if (tok < te) {
                        long long th = tok * w.H + h;
                        float ks = 0.0f;
                        for (int i = tid; i < dk; i += 32) { float x = ld_in(k + th * dk + i); ks = fmaf(x, x, ks); }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) ks += __shfl_xor_sync(0xffffffffu, ks, o);
                        float at = w.a[th], den = fmaf(at, at, w.qn[th] * lam);
                        g = at / den;
                        lam = fmaf(w.beta[th] * ks, inv_dk, lam / den);
                        gprod *= g;
                    }
                    if (tid == 0) { g1_s[tau] = g; lam_s[tau] = lam; }
                }
            }
            __syncthreads();
            for (int idx = tid; idx < kTT * dk; idx += kWalkThreads) {
                int tau = idx / dk, i = idx % dk;
                long long tok = t0 + tau;
                float qt = 0.0f, kt = 0.0f;
                if (tok < te) {
                    long long th = tok * w.H + h;
                    kt = w.beta[th] * ld_in(k + th * dk + i);
                    if (w.mode == kOutput) qt = ld_in(q + th * dk + i) / lam_s[tau];
                }
                gs[idx] = g1_s[tau]; qts[idx] = qt; kts[idx] = kt;
            }
        }
        for (int idx = tid; idx < kTT * dv; idx += kWalkThreads) {
            int tau = idx / dv, jj = idx % dv;
            long long tok = t0 + tau;
            vs[idx] = (tok < te) ? ld_in(v + (tok * w.H + h) * dv + jj) : 0.0f;
        }
        __syncthreads();
        // ---- phase B: eta update and partial readout
#pragma unroll 2
        for (int tau = 0; tau < kTT; ++tau) {
            float vj = vs[tau * dv + j], acc = 0.0f;
#pragma unroll
            for (int r = 0; r < KPG; ++r) {
                int i = kg * KPG + r;
                S[r] = fmaf(gs[tau * dk + i], S[r], kts[tau * dk + i] * vj);
                acc = fmaf(qts[tau * dk + i], S[r], acc);
            }
            if (w.mode == kOutput) part[(tau * nkg + kg) * dv + j] = acc;
        }
        __syncthreads();
        // ---- phase C: sum the partial readouts per value column
        if (w.mode == kOutput) {
            TIn *out = (TIn *)w.out;
            for (int idx = tid; idx < kTT * dv; idx += kWalkThreads) {
                int tau = idx / dv, jj = idx % dv;
                long long tok = t0 + tau;
                if (tok < te) {
                    float o = 0.0f;
                    for (int g2 = 0; g2 < nkg; ++g2) o += part[(tau * nkg + g2) * dv + jj];
                    st_out(out + (tok * w.H + h) * dv + jj, o);
                }
            }
        }
    }

    // ---- end of segment
    if (w.mode == kState) {
#pragma unroll
        for (int r = 0; r < KPG; ++r)
            w.S_io[((u * w.P + p) * dk + kg * KPG + r) * dv + j] = S[r];
        if (gate_thread && (!w.iso || tid == 0))
            w.decay[(u * w.P + p) * w.nl + (w.iso ? 0 : tid)] = gprod;
    } else if (p == P_eff - 1) {
        if (w.final_eta) {
#pragma unroll
            for (int r = 0; r < KPG; ++r)
                w.final_eta[(u * dk + kg * KPG + r) * dv + j] = S[r];
        }
        if (w.final_lambda && gate_thread && (!w.iso || tid == 0))
            w.final_lambda[u * w.nl + (w.iso ? 0 : tid)] = lam;
    }
}

template <typename TIn, int KPG>
static cudaError_t launch_walk_t(const WalkArgs &w, unsigned grid, cudaStream_t st) {
    size_t smem = walk_smem_bytes(w.dk, w.dv);
    static PerDevice<bool> attr;
    const cudaError_t e = ensure_smem_attr(attr, kla_walk_simt<TIn, KPG>, 64 * 1024);
    if (e != cudaSuccess) return e;
    return launch_pdl(kla_walk_simt<TIn, KPG>, grid, kWalkThreads, smem, st, w);
}

template <typename TIn>
static cudaError_t launch_walk_kpg(const WalkArgs &w, unsigned grid, cudaStream_t st) {
    switch (w.dk * w.dv / kWalkThreads) {
        case 1: return launch_walk_t<TIn, 1>(w, grid, st);
        case 2: return launch_walk_t<TIn, 2>(w, grid, st);
        case 4: return launch_walk_t<TIn, 4>(w, grid, st);
        case 8: return launch_walk_t<TIn, 8>(w, grid, st);
        case 16: return launch_walk_t<TIn, 16>(w, grid, st);
        case 32: return launch_walk_t<TIn, 32>(w, grid, st);
        case 64: return launch_walk_t<TIn, 64>(w, grid, st);
        case 128: return launch_walk_t<TIn, 128>(w, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

// mode kState launches segments 0..P-2 of every unit; kOutput all of them.
cudaError_t launch_walk(const Plan &p, const int *cu, int mode, const void *q, const void *k,
                        const void *v, const float *a, const float *qn, const float *beta,
                        const float *lambda0, const float *eta0, const float *lam_blk, float *S_io,
                        float *decay, void *out, float *final_lambda, float *final_eta,
                        cudaStream_t st) {
    WalkArgs w{p.N, p.H, p.dk, p.dv, p.nl, p.T, p.Lseg, p.P, p.NB, p.seg_blocks, cu, p.iso, mode,
               q, k, v, a, qn, beta, lambda0, eta0, lam_blk, S_io, decay, out, final_lambda, final_eta,
               cu ? p.perm : nullptr};
    long long segs = (mode == kState) ? (p.P - 1) : p.P;
    unsigned grid = (unsigned)((long long)p.N * p.H * segs);
    if (grid == 0) return cudaSuccess;
    return p.bf16 ? launch_walk_kpg<__nv_bfloat16>(w, grid, st) : launch_walk_kpg<float>(w, grid, st);
}

// ---- inter-segment carry of eta ------------------------------------------
// eta_start[p] = diag(decay[p-1]) eta_start[p-1] + dS[p-1], eta_start[0] = eta0.
// In place: eta_start[p] overwrites the dS slot p-1 it was made from.
__global__ void __launch_bounds__(256)
kla_state_carry(int N, int H, int dk, int dv, int nl, int P, const float *__restrict__ eta0,
                const float *__restrict__ decay, float *__restrict__ S_io) {
    pdl_release();
    pdl_wait();
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long per = (long long)dk * dv;
    if (gid >= (long long)N * H * per) return;
    long long u = gid / per, e = gid % per;
    int il = (nl == 1) ? 0 : (int)(e / dv);
    float S = eta0 ? eta0[gid] : 0.0f;
    // segments in batches of 8: every transfer of a batch is read before any
    // carried state is written back, so the loads overlap
    for (int p0 = 1; p0 < P; p0 += 8) {
        float x[8], dc[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int p = p0 + r;
            if (p < P) {
                x[r] = S_io[(u * P + p - 1) * per + e];
                dc[r] = decay[(u * P + p - 1) * nl + il];
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int p = p0 + r;
            if (p < P) {
                S = fmaf(dc[r], S, x[r]);
                S_io[(u * P + p - 1) * per + e] = S;
            }
        }
    }
}

cudaError_t launch_state_carry(const Plan &p, const float *eta0, const float *decay, float *S_io,
                               cudaStream_t st) {
    long long thr = (long long)p.N * p.H * p.dk * p.dv;
    return launch_pdl(kla_state_carry, (unsigned)((thr + 255) / 256), 256, 0, st, p.N, p.H, p.dk, p.dv, p.nl,
                      p.P, eta0, decay, S_io);
}

}  // namespace kla
