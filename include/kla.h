/*
 * kla.h -- C ABI of libkla, the B200 (sm_100a) forward pass of a Kalman
 * linear-attention (KLA) sequence-mixing layer.
 *
 * The operation (Kalman Linear Attention, technical summary section 1,
 * "probabilistic formulation"; Kalman Delta Networks abstract for the
 * isotropic variant). Per sequence n and head h an information-form Kalman
 * filter keeps a precision lambda and an information matrix eta[dk][dv].
 * For every token t, first a predict with an exactly discretised
 * Ornstein-Uhlenbeck prior (decay a, process noise qn), then an update that
 * treats the token as a noisy observation through the key k with value
 * precision beta, then a readout of the posterior mean through the query q:
 *
 *   den = a^2 + qn*lambda ;  g = a/den                (forget gate)
 *   lambda <- lambda/den + beta*k^2                   (a Moebius map of lambda,
 *                                                      technical summary sec. 2)
 *   eta[i,:] <- g*eta[i,:] + beta*k[i]*v              (affine once g is known)
 *   out[t,:] = sum_i q[i]*eta[i,:]/lambda[i]
 *
 * KLA_DIAG: lambda, a, qn per key dimension i.  KLA_ISO: one lambda per head,
 * a and qn per (token, head), increment beta*|k|^2/dk, shared gate.
 * Every token predicts and then updates (the first one included), so
 * lambda0/eta0 is the belief before the first token and the final state of one
 * call is a valid lambda0/eta0 for the next: two calls over a split sequence
 * equal one call over the whole.
 *
 * Layouts (row-major, tokens flattened over the batch, Ntok = B*T):
 *   q, k        [Ntok, H, dk]        bf16 (KLA_BF16) or fp32 (KLA_FP32)
 *   v, out      [Ntok, H, dv]        same dtype as q
 *   a, qn       [Ntok, H, dk] fp32   (KLA_ISO: [Ntok, H])
 *   beta        [Ntok, H]     fp32
 *   lambda0, final_lambda  [N, H, dk] fp32 (KLA_ISO: [N, H])
 *   eta0, final_eta        [N, H, dk, dv] fp32
 * N = B, or num_seqs with packed variable-length sequences (cu_seqlens).
 *
 * Ownership: the caller owns every buffer, including the workspace; all device
 * pointers must stay valid until the stream work completes. Calls enqueue work
 * on `stream` and return without synchronising (except kla_check and
 * kla_forward_host, which say so). The library never allocates device memory.
 *
 * Preconditions not checked on the device: a > 0, qn >= 0, beta >= 0,
 * lambda0 > 0, finite inputs. Identical inputs give bitwise identical outputs
 * on the same device and configuration (no atomics in any reduction).
 */
#ifndef KLA_H_
#define KLA_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KLA_OK = 0,
    KLA_ERR_INVALID_ARG = 1,  /* bad shape, null required pointer, misaligned
                                 pointer, workspace too small; nothing launched */
    KLA_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement */
    KLA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    KLA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (kla_check);
                                 the kernel left through its teardown and the
                                 context stays usable */
    KLA_ERR_RANGE = 5         /* a 16-token stretch of one key (or of the head, in
                                 isotropic mode) has a cumulative gate below 2^-160
                                 (log2 span above 160), beyond what the factorised
                                 chunk form represents (kla_check); outputs of that
                                 call are unreliable. Faster forgetting spread over
                                 longer stretches is computed exactly. */
} kla_status;

typedef enum { KLA_BF16 = 0, KLA_FP32 = 1 } kla_dtype;   /* dtype of q, k, v, out */
typedef enum { KLA_DIAG = 0, KLA_ISO = 1 } kla_mode;      /* lambda per key / per head */

typedef struct {
    int B, T, H;          /* batch, tokens per batch row, heads (B*T = Ntok) */
    int dk, dv;           /* key and value head dims: dk, dv in {16,32,64,128}, dv also 256 */
    kla_dtype dtype;
    kla_mode mode;
    const int *cu_seqlens;  /* device int32 [num_seqs+1]: packed sequence offsets
                               into the Ntok axis (0 = first, Ntok = last), or NULL
                               for B independent rows of T tokens */
    int num_seqs;           /* number of packed sequences when cu_seqlens != NULL */
} kla_desc;

/* Bytes of device workspace kla_forward needs for this descriptor on the
 * current device (0 means the workspace pointer may be NULL): when rows are
 * split into segments, the Moebius block aggregates and the segment states,
 * and on the tensor-core path also the segments' folded queries (2*dk bytes
 * per token and head) and per-chunk factors for the correction pass; one int
 * per packed sequence (up to 1024 sequences) for the longest-first launch
 * order. Pure host computation. Returns 0 for an invalid descriptor as well. */
size_t kla_workspace_bytes(const kla_desc *desc);

/* Bytes of device workspace kla_precision needs (0: the pointer may be NULL). */
size_t kla_precision_workspace_bytes(const kla_desc *desc);

/* The forward pass (the whole hot path: precision scan, state passing, chunked
 * gated linear attention). q, k, v, a, qn, out: device pointers in the
 * layouts above, 16-byte aligned; beta 4-byte aligned. lambda0 (4-byte aligned) / eta0 (16-byte
 * aligned): device pointers, or NULL for lambda0 = 1 and eta0 = 0. final_lambda/final_eta: device pointers or NULL to
 * skip. workspace: device, 256-byte aligned, >= kla_workspace_bytes(desc).
 * Ntok == 0 is a no-op. Errors: KLA_ERR_INVALID_ARG / KLA_ERR_UNSUPPORTED
 * before any launch; KLA_ERR_CUDA if a launch fails. Stream order holds as
 * for any launch: the library's kernels use programmatic dependent launch
 * among themselves, and each waits for the work before it in the stream to
 * complete before it touches global memory. */
kla_status kla_forward(const kla_desc *desc,
                       const void *q, const void *k, const void *v,
                       const float *a, const float *qn, const float *beta,
                       const float *lambda0, const float *eta0,
                       void *out, float *final_lambda, float *final_eta,
                       void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* kla_forward that also records seven caller-created CUDA events on `stream`:
 * events[0] before the first launch (the length ranking of packed sequences
 * falls between events[0] and events[1]) and events[1..6] after the stages
 * 1 Moebius block reduction, 2 Moebius carry, 3 segment state pass and
 * 4 segment state carry (CUDA-core walk only), 5 the walk (whole rows, or
 * every segment of split rows), 6 segment-start beliefs and correction pass
 * (split rows on the tensor-core path: the carried segment-start states added
 * to the outputs of segments walked from a zero state). Stages that do not run
 * for this descriptor record at the same point as the previous one. For
 * measuring the stages; otherwise identical to kla_forward. */
kla_status kla_forward_profiled(const kla_desc *desc,
                                const void *q, const void *k, const void *v,
                                const float *a, const float *qn, const float *beta,
                                const float *lambda0, const float *eta0,
                                void *out, float *final_lambda, float *final_eta,
                                void *workspace, size_t workspace_bytes,
                                cudaStream_t stream, cudaEvent_t *events);

/* The work plan kla_forward uses for this descriptor on the current device:
 * segments each row is split into (1: one CTA walks a whole row or packed
 * sequence), kernel launches per call (1 unsplit; split rows on the
 * tensor-core path: Moebius reduce, Moebius carry unless the chunk kernel
 * composes the short segments' aggregates itself, chunk kernel, segment starts
 * and correction, so 4 or 5; 5 on the CUDA-core walk; plus 1 for the launch
 * order of packed sequences), and
 * whether the chunk stages
 * run on the tcgen05 tensor-core kernel (1) or the CUDA-core walk (0).
 * Any output pointer may be NULL. Pure host computation. */
kla_status kla_plan(const kla_desc *desc, int *segments_per_row, int *launches,
                    int *tensor_core);

/* The precision path alone: lambda_out[Ntok, H, dk] (KLA_ISO: [Ntok, H]) fp32
 * receives the posterior precision after every token -- the filter's explicit
 * uncertainty (Kalman Linear Attention, technical summary section 2: the
 * Moebius recursion computed by a parallel prefix scan). Same argument rules
 * as kla_forward, with a workspace of kla_precision_workspace_bytes(desc). */
kla_status kla_precision(const kla_desc *desc, const void *k,
                         const float *a, const float *qn, const float *beta,
                         const float *lambda0, float *lambda_out,
                         void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/* One recurrent decode step per sequence (T = 1 per sequence, B = N rows):
 * reads the belief lambda/eta in place, applies predict + update for token
 * q,k,v,a,qn,beta ([N,H,...] with Ntok = N) and writes out[N,H,dv]; lambda and
 * eta are overwritten with the new belief (constant-memory decoding, Kalman
 * Delta Networks abstract). desc->T must be 1 and cu_seqlens NULL. */
kla_status kla_decode_step(const kla_desc *desc,
                           const void *q, const void *k, const void *v,
                           const float *a, const float *qn, const float *beta,
                           float *lambda, float *eta, void *out,
                           cudaStream_t stream);

/* Bytes of one device buffer kla_forward_host needs (inputs, outputs and
 * workspace, each 256-byte aligned). */
size_t kla_host_device_bytes(const kla_desc *desc);

/* kla_forward on HOST buffers (pinned host memory gives asynchronous copies):
 * copies the inputs into device_buffer (>= kla_host_device_bytes), runs the
 * forward pass, copies out (and final states when the pointers are non-NULL)
 * back, and synchronises the stream before returning. cu_seqlens in desc is a
 * HOST pointer for this call. */
kla_status kla_forward_host(const kla_desc *desc,
                            const void *q, const void *k, const void *v,
                            const float *a, const float *qn, const float *beta,
                            const float *lambda0, const float *eta0,
                            void *out, float *final_lambda, float *final_eta,
                            void *device_buffer, size_t device_bytes,
                            cudaStream_t stream);

/* Size of the fixed device scratch area kla_forward_noalloc uses, per GPU. */
#define KLA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* kla_forward for callers that cannot allocate device memory: code that runs
 * inside an allocator or memory-pool callback, plug-ins whose host framework
 * owns every device allocation, or processes that must keep a fixed device
 * footprint after start-up. The pages have no counterpart of this call; it is
 * plumbing around the same forward pass. Instead of a caller-provided
 * workspace it uses a file-scope device array of KLA_NOALLOC_SCRATCH_BYTES,
 * which every GPU that loads the library holds until the process exits.
 * Arguments, layouts and errors as kla_forward. A descriptor whose
 * kla_workspace_bytes exceeds KLA_NOALLOC_SCRATCH_BYTES (long rows with few
 * heads, e.g. 16 heads x 128k tokens at dk = dv = 128) returns
 * KLA_ERR_UNSUPPORTED before any launch. The first call on each device looks
 * up the array's device address (cudaGetSymbolAddress), so make that first
 * call before any stream capture. All calls share the one array: nothing in
 * it needs to start at zero (each call writes every scratch value before
 * reading it), but calls whose GPU work overlaps -- on different streams or
 * from different host threads -- race on it and must be serialised by the
 * caller. Never allocates, never synchronises. */
kla_status kla_forward_noalloc(const kla_desc *desc,
                               const void *q, const void *k, const void *v,
                               const float *a, const float *qn, const float *beta,
                               const float *lambda0, const float *eta0,
                               void *out, float *final_lambda, float *final_eta,
                               cudaStream_t stream);

/* Kalman Delta Network forward with the Kalman-gain residual (delta-style)
 * write (Kalman Delta Networks abstract: the memory is the state of a
 * linear-Gaussian model, the Kalman gain weights each residual write, the
 * one-step posterior is projected onto diagonal Gaussians (diagonal mode) or
 * kept isotropic with one uncertainty per head). The state is the posterior
 * mean M [N,H,dk,dv] and the precision lambda; per token t:
 *   lambda~ = lambda / (a^2 + qn lambda),  w = k / lambda~,
 *   gamma = beta / (1 + beta k.w),  r = v - (a M)^T k,
 *   M = a M + gamma w r^T,  lambda = lambda~ + beta k^2 (iso: + beta |k|^2 / dk),
 *   o = M^T q.
 * Arguments as kla_forward, with M0 (prior mean before the first token, or
 * NULL for 0; 16-byte aligned) and final_M (or NULL) in place of eta0 /
 * final_eta; no workspace. dk and dv in {16, 32, 64, 128}, else
 * KLA_ERR_UNSUPPORTED. One CTA per (row or packed sequence, head, block of 32
 * value columns) walks its tokens with its columns of the mean in registers
 * (CUDA cores). Errors as kla_forward. */
kla_status kla_kdn_forward(const kla_desc *desc,
                           const void *q, const void *k, const void *v,
                           const float *a, const float *qn, const float *beta,
                           const float *lambda0, const float *M0,
                           void *out, float *final_lambda, float *final_M,
                           cudaStream_t stream);

/* The mixer's input prologue in one pass (Kalman Linear Attention, technical
 * summary section 4: a Mamba-like block with a 1-D causal convolution and SiLU
 * before the mixer): from the pre-activations it writes the forward pass's
 * inputs,
 *   q = l2norm(silu(conv(xq))), k = l2norm(silu(conv(xk))), v = silu(conv(xv)),
 *   a = sigmoid(xa), qn = softplus(xqn), beta = sigmoid(xbeta),
 * conv: depthwise and causal, y[t,c] = b[c] + sum_{w<W} wgt[c,w] x[t-(W-1)+w,c]
 * with x = 0 before the start of t's row or packed sequence; l2norm over dk:
 * y / sqrt(sum y^2 + 1e-6). xq, xk, q, k [Ntok,H,dk] and xv, v [Ntok,H,dv] in
 * desc->dtype; xa, xqn, a, qn [Ntok,H,dk] (iso [Ntok,H]) and xbeta, beta
 * [Ntok,H] fp32; weights wq, wk [H,dk,W], wv [H,dv,W] fp32; biases bq, bk
 * [H,dk], bv [H,dv] fp32 or NULL for none. W = conv_width in 1..4. Device
 * pointers: the token tensors 16-byte aligned (rows move as vectors), xbeta,
 * beta, weights and biases 4-byte aligned. Errors as kla_forward. */
kla_status kla_prologue(const kla_desc *desc, int conv_width,
                        const void *xq, const void *xk, const void *xv,
                        const float *xa, const float *xqn, const float *xbeta,
                        const float *wq, const float *wk, const float *wv,
                        const float *bq, const float *bk, const float *bv,
                        void *q, void *k, void *v, float *a, float *qn, float *beta,
                        cudaStream_t stream);

/* Gradients of kla_forward (Kalman Linear Attention abstract: the layer is
 * meant for efficient parallel training): given the inputs of a forward call
 * and dout = dL/dout, plus optionally dL/dfinal_lambda and dL/dfinal_eta (NULL
 * for zero), writes dL/d of every input in fp32, in the layout of that input:
 * dq, dk [Ntok,H,dk]; dv [Ntok,H,dv]; da, dqn [Ntok,H,dk] (iso [Ntok,H]);
 * dbeta [Ntok,H]; dlambda0 [N,H,dk] (iso [N,H]) and deta0 [N,H,dk,dv] (either
 * may be NULL when not wanted). q, k, v, dout in desc->dtype, 16-byte aligned;
 * the rest fp32, 4-byte aligned. With q^ = q/lambda, k^ = beta k and the gate
 * g, the mean recursion is the gated linear one eta_t = g_t eta_{t-1} +
 * k^_t v_t^T, out_t = eta_t^T q^_t; the library runs a forward sweep (the
 * mean in registers, dq^ = eta do), two reverse sweeps of the adjoint
 * d_t = g_{t+1} d_{t+1} + q^_t do_t^T (one over key rows for dk^ and the gate
 * term g dL/dg = sum over later tokens of q^ dq^ - k^ dk^, one over value
 * columns for dv), and the scalar precision chain in reverse; no per-token
 * state is stored (CUDA cores, fp32; one CTA per (row or packed sequence,
 * head) for each sweep). The workspace (kla_backward_workspace_bytes, caller
 * owned, 16-byte aligned) holds per-token precisions, gates and partial
 * gradients. dk and dv in {16, 32, 64, 128}, else KLA_ERR_UNSUPPORTED.
 * Preconditions as kla_forward (a > 0 in particular: dL/dg is recovered as
 * (g dL/dg) / g). Errors as kla_forward. */
size_t kla_backward_workspace_bytes(const kla_desc *desc);
kla_status kla_backward(const kla_desc *desc,
                        const void *q, const void *k, const void *v,
                        const float *a, const float *qn, const float *beta,
                        const float *lambda0, const float *eta0, const void *dout,
                        const float *dfinal_lambda, const float *dfinal_eta,
                        float *dq, float *dk, float *dv, float *da, float *dqn, float *dbeta,
                        float *dlambda0, float *deta0,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the library's device status
 * word on the current device: KLA_OK, KLA_ERR_RANGE or KLA_ERR_TIMEOUT from any
 * kernel that ran since the last check, or KLA_ERR_CUDA if the stream failed.
 * (The environment variable KLA_TEST_WITHHOLD_TILES=1, read at each launch of the
 * tensor-core walk, withholds its tile loads so that its first bounded wait runs
 * out: a test switch for this status path, off unless set.) */
kla_status kla_check(cudaStream_t stream);

/* Static description of an error code. */
const char *kla_status_string(kla_status status);

/* Library version, major*10000 + minor*100 + patch. */
int kla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KLA_H_ */
