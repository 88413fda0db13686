/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) operator.
 *
 * The operator (Kimi Linear: An Expressive, Efficient Attention Architecture,
 * summary, §3 "Kimi Delta Attention"):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t
 *
 * with the lower-bounded channel-wise gate (Kimi K3 architecture summary,
 * hybrid KDA / Gated MLA section)
 *
 *   g_t = -5 * sigmoid(exp(A_h) * z_t),   alpha_t = exp(g_t)   (per channel)
 *
 * and q, k normalised to unit length inside the operator as
 * x / sqrt(sum x^2 + 1e-6) (Kimi Linear summary, §4).  No 1/sqrt(d) scale is
 * applied to q.  The memory is decayed before the delta correction, and o_t
 * reads the state after token t's update.
 *
 * Prefill uses the chunkwise form (Kimi Linear summary, §3.1 "Hardware-
 * Efficient Chunkwise Algorithm"; §6.3 for the chunk size): per-chunk
 * cumulative log-decay, a WY / UT-transform of the rank-1 updates whose
 * lower-triangular inverse is formed by forward substitution on 16-token
 * sub-tiles, a sequential inter-chunk state carry, and the intra-chunk causal
 * output plus the incoming-state term.  Decode is the recurrent form, one
 * token per sequence (§6.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor pointer is a DEVICE pointer, 16-byte aligned, contiguous,
 *   row-major.  T = total tokens, N = sequences, H = heads.
 *     q, k, z : [T, H, dk]      v, o : [T, H, dv]      beta : [T, H]
 *     A       : [H]    float32
 *     states  : [N, H, dk, dv]  float32, S[key][value]
 *   q, k, v, z, beta and o share the element type `dt`.
 * - Supported sizes: dk, dv in {32, 64, 128}; chunk in {16, 64}; H >= 1.
 * - The caller owns every buffer, including the workspace.  The library never
 *   allocates on the call path and keeps no global state between calls; calls
 *   on different workspaces are independent.
 * - All calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL
 *   is the legacy default stream).  Nothing is copied device-to-host.
 * - Errors that the host can see return synchronously and enqueue nothing:
 *   KDA_ERR_INVALID_ARG (null pointer, misalignment, inconsistent sizes,
 *   workspace too small), KDA_ERR_UNSUPPORTED (dims, chunk or dtype outside
 *   the supported set).  A failed launch returns KDA_ERR_CUDA.  Errors only
 *   the device can see (a cu_seqlens that is not non-decreasing from 0 to
 *   total_tokens, or has a length above max_seqlen) are recorded in the
 *   workspace's error word; the kernels then skip all work (o and S_final
 *   are left unwritten) and kda_check_device_error() reports
 *   KDA_ERR_INVALID_ARG.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = -1,
  KDA_ERR_UNSUPPORTED = -2,
  KDA_ERR_CUDA = -3,
  KDA_ERR_TIMEOUT = -4
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Opaque stream handle; pass a cudaStream_t (or NULL). */
typedef void* kda_stream_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char* kda_status_string(kda_status s);

/* Library version as an integer (major*10000 + minor*100 + patch). */
int32_t kda_version(void);

/*
 * Bytes of device workspace kda_forward / kda_forward_g need for this
 * problem.  Returns 0 when the arguments are invalid or unsupported.
 * max_seqlen bounds every sequence's length; with cu_seqlens == NULL the
 * batch is num_seqs sequences of max_seqlen tokens each.
 */
size_t kda_forward_workspace_size(int32_t num_seqs, int32_t total_tokens,
                                  int32_t max_seqlen, int32_t H, int32_t dk,
                                  int32_t dv, kda_dtype dt, int32_t chunk);

/*
 * Number of kernel launches one kda_forward / kda_forward_g call with these
 * arguments enqueues (0 when the arguments are invalid or unsupported).  The
 * same count holds for kda_forward_scalar_gate, kda_forward_checkpoints and,
 * on the tensor-core path, kda_forward_norm_gate and kda_forward_conv; on the
 * CUDA-core path kda_forward_norm_gate and kda_forward_conv enqueue one
 * launch more.
 */
int32_t kda_forward_launches(int32_t num_seqs, int32_t total_tokens,
                             int32_t max_seqlen, int32_t H, int32_t dk,
                             int32_t dv, kda_dtype dt, int32_t chunk);

/*
 * Chunkwise KDA prefill over packed sequences.
 *
 *  q, k, v, z, beta : inputs in `dt`, layouts above.
 *  A          : [H] float32, per-head gate scale (the gate uses exp(A_h)).
 *  S0         : [N, H, dk, dv] float32 initial states; NULL means zeros.
 *  cu_seqlens : device int32 [N+1] token offsets (0 = cu[0] <= cu[1] <= ...
 *               <= cu[N] = total_tokens, every length <= max_seqlen), or NULL
 *               for N equal sequences of max_seqlen tokens
 *               (total_tokens must then equal num_seqs * max_seqlen).
 *               The chunk grid restarts at every sequence; the last chunk of a
 *               sequence may be partial; an empty sequence passes S0 through.
 *  o          : [T, H, dv] in `dt`, output; must not overlap any input.
 *  S_final    : [N, H, dk, dv] float32 final states, or NULL to skip.  It may
 *               equal S0 (in-place state passing); any other overlap with an
 *               input is undefined.
 *  chunk      : 16 or 64 tokens (the result does not depend on it beyond
 *               rounding).
 *  workspace  : device buffer of at least kda_forward_workspace_size() bytes,
 *               16-byte aligned; its contents need no initialisation and are
 *               overwritten.  Do not share one workspace between calls that
 *               may run concurrently.
 */
kda_status kda_forward(const void* q, const void* k, const void* v,
                       const void* z, const float* A, const void* beta,
                       const float* S0, const int32_t* cu_seqlens,
                       int32_t num_seqs, int32_t total_tokens,
                       int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                       kda_dtype dt, int32_t chunk, void* o, float* S_final,
                       void* workspace, size_t workspace_bytes,
                       kda_stream_t stream);

/*
 * Same operator with the log-decay given directly instead of (z, A):
 *  g : [T, H, dk] float32 log-decay, alpha = exp(g).
 * Precondition g in [-5, 0] (the range the gate produces); outside it the
 * 16-token sub-tile rescaling loses its overflow guarantee and results are
 * undefined (not checked).  g = 0 gives DeltaNet (Kimi Linear summary §2.2);
 * g equal across a head's channels gives Gated DeltaNet's scalar gate.
 */
kda_status kda_forward_g(const void* q, const void* k, const void* v,
                         const float* g, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, int32_t num_seqs,
                         int32_t total_tokens, int32_t max_seqlen, int32_t H,
                         int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk,
                         void* o, float* S_final, void* workspace,
                         size_t workspace_bytes, kda_stream_t stream);

/*
 * The Gated DeltaNet special case (Kimi Linear summary, §2.2 "Linear Attention
 * and the Gated Delta Rule": one scalar forget gate per head): the decay of
 * token t in head h is one value shared by all dk channels,
 * alpha_t = exp(g_head[t, h]).  Same algorithm and kernels as kda_forward with
 * the gate broadcast over the channels; z is not read, so the call moves
 * 2·dk bytes (bf16) less per token and head.
 *
 *  g_head : [T, H] float32 log-decay, in [-5, 0] (the range the lower-bounded
 *           KDA gate guarantees and the 16-token sub-tile bound relies on;
 *           values outside it give undefined results: not checked).
 * Everything else, including the workspace size, is kda_forward's.
 */
kda_status kda_forward_scalar_gate(const void* q, const void* k, const void* v,
                                   const float* g_head, const void* beta, const float* S0,
                                   const int32_t* cu_seqlens, int32_t num_seqs,
                                   int32_t total_tokens, int32_t max_seqlen, int32_t H,
                                   int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk,
                                   void* o, float* S_final, void* workspace,
                                   size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_forward that also writes sparse state checkpoints: the state after
 * every `interval` tokens of each sequence.  This is the operator's side of a
 * prefix cache that keeps KDA states at fixed token boundaries inside a paged
 * pool (Kimi K3 review, romaanj.github.io, Significance: a KDA-aware prefix cache
 * that keeps MLA blocks and sparse KDA checkpoint boundaries in one paged
 * pool; Kimi K3 architecture summary, serving engine);
 * the pages describe the cache, not a kernel for it.
 *
 *  interval : tokens between checkpoints, a positive multiple of `chunk`
 *             (else KDA_ERR_INVALID_ARG).
 *  S_ckpt   : [N, H, J, dk, dv] float32 with J = max_seqlen / interval
 *             (rounded down).  Entry (n, h, j) receives the state after the
 *             first (j+1)·interval tokens of sequence n when (j+1)·interval
 *             is at most its length; the other entries are not written.
 *             16-byte aligned; may be NULL only when J = 0; must not overlap
 *             any other argument.
 * Everything else, including the workspace size, is kda_forward's.
 */
kda_status kda_forward_checkpoints(const void* q, const void* k, const void* v,
                                   const void* z, const float* A, const void* beta,
                                   const float* S0, const int32_t* cu_seqlens,
                                   int32_t num_seqs, int32_t total_tokens,
                                   int32_t max_seqlen, int32_t H, int32_t dk,
                                   int32_t dv, kda_dtype dt, int32_t chunk, void* o,
                                   float* S_final, float* S_ckpt, int32_t interval,
                                   void* workspace, size_t workspace_bytes,
                                   kda_stream_t stream);

/*
 * kda_forward followed by the layer's output epilogue, fused into the kernels
 * that write o (Kimi Linear summary, §4 "The Kimi Linear Model Architecture":
 * head-wise RMSNorm of the output, then a data-dependent sigmoid gate; §5.2:
 * the gate is a sigmoid, not Swish).  For every token t and head h, over the
 * head's dv features j:
 *
 *   o[t,h,j] = a[t,h,j] / sqrt(mean_j' a[t,h,j']^2 + eps) * w[j] * sigmoid(r[t,h,j])
 *
 * where a is the attention output kda_forward would write.  The output
 * projection that follows in the layer is not part of this call.
 *
 *  out_gate    : r, [T, H, dv] in `dt`, the gate input (the layer's low-rank
 *                projection of its input, computed by the caller).  Required
 *                when total_tokens > 0; must not overlap o.
 *  norm_weight : w, [dv] float32, the RMSNorm gain shared by the heads, or
 *                NULL for ones.  The pages name no gain; this one is optional.
 *  eps         : added to the mean square, finite and >= 0 (else
 *                KDA_ERR_INVALID_ARG); the pages give no value.
 * On the tensor-core path the epilogue runs in the full chain pass, which
 * writes o, from the fp32 attention output in Tensor Memory; on the
 * CUDA-core path it is one extra launch after the state pass
 * (kda_forward_launches + 1), since that pass splits a head's dv features
 * over several blocks.  Everything else is kda_forward's.
 */
kda_status kda_forward_norm_gate(const void* q, const void* k, const void* v,
                                 const void* z, const float* A, const void* beta,
                                 const float* S0, const int32_t* cu_seqlens,
                                 int32_t num_seqs, int32_t total_tokens,
                                 int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                                 kda_dtype dt, int32_t chunk, const void* out_gate,
                                 const float* norm_weight, float eps, void* o,
                                 float* S_final, void* workspace, size_t workspace_bytes,
                                 kda_stream_t stream);

/*
 * One recurrent KDA step for B independent sequences (one token each),
 * updating the float32 states in place (Kimi Linear summary §6.3: token
 * generation uses the recurrent update).
 *
 *  q, k, z : [B, H, dk] in `dt`;  v : [B, H, dv];  beta : [B, H];
 *  A       : [H] float32;
 *  S_inout : [B, H, dk, dv] float32, read and overwritten with the new state;
 *  o       : [B, H, dv] in `dt`, must not overlap any input.
 * No workspace is needed; the call has no device-side error paths.
 */
kda_status kda_decode_step(const void* q, const void* k, const void* v,
                           const void* z, const float* A, const void* beta,
                           float* S_inout, int32_t B, int32_t H, int32_t dk,
                           int32_t dv, kda_dtype dt, void* o,
                           kda_stream_t stream);

/*
 * kda_decode_step with the output epilogue of kda_forward_norm_gate fused
 * into the step: o[b,h,:] is the RMS-normalised attention output times the
 * gain times sigmoid(out_gate[b,h,:]).
 *
 *  out_gate    : [B, H, dv] in `dt`; required when B > 0.
 *  norm_weight : [dv] float32 or NULL (ones).   eps : finite, >= 0.
 * Everything else is kda_decode_step's.
 */
kda_status kda_decode_step_norm_gate(const void* q, const void* k, const void* v,
                                     const void* z, const float* A, const void* beta,
                                     float* S_inout, int32_t B, int32_t H, int32_t dk,
                                     int32_t dv, kda_dtype dt, const void* out_gate,
                                     const float* norm_weight, float eps, void* o,
                                     kda_stream_t stream);

/*
 * kda_forward without a caller-provided workspace, for callers that cannot
 * allocate device memory.  No passage of the pages corresponds to this entry
 * point; it exists for integration only.
 *
 * Who needs it: a host whose device memory is owned by another allocator (a
 * framework pool that reserved the GPU's memory up front, so a new cudaMalloc
 * fails or fragments it), and code that must not call the CUDA allocator at
 * all, since cudaMalloc/cudaFree can synchronise the whole device.
 *
 * Arguments and results are those of kda_forward, minus the workspace.  The
 * scratch comes from one fixed array of KDA_NOALLOC_SCRATCH_BYTES in device
 * memory that the library defines at file scope.  The array is reserved on a
 * GPU when the library's device code is loaded there -- with CUDA's default
 * lazy module loading at the first kernel of this library launched on that
 * GPU (any entry point, decode included), with CUDA_MODULE_LOADING=EAGER when
 * the context is created -- and stays reserved until the process exits.  The
 * call itself allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).
 *  - Problems needing more scratch than KDA_NOALLOC_SCRATCH_BYTES (see
 *    kda_forward_workspace_size) are rejected with KDA_ERR_UNSUPPORTED before
 *    anything is enqueued; use kda_forward with your own workspace instead.
 *  - The first call on a device, made with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it; make that
 *    first call before any stream capture begins on that device.  The cached
 *    address belongs to that device's primary context: do not use this entry
 *    point after cudaDeviceReset (or any teardown of the primary context) in
 *    the same process, since the array may then live at another address.
 *  - Every call on a device shares the one array, and it keeps the previous
 *    call's contents (nothing in it needs to start at zero).  Calls whose GPU
 *    work may overlap -- different streams, or different host threads without
 *    ordering -- race on it: order them on one stream.
 *  - A bad cu_seqlens seen on the device is recorded in the shared array,
 *    where it cannot be queried: validate cu_seqlens beforehand.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

kda_status kda_forward_noalloc(const void* q, const void* k, const void* v,
                               const void* z, const float* A, const void* beta,
                               const float* S0, const int32_t* cu_seqlens,
                               int32_t num_seqs, int32_t total_tokens,
                               int32_t max_seqlen, int32_t H, int32_t dk,
                               int32_t dv, kda_dtype dt, int32_t chunk,
                               void* o, float* S_final, kda_stream_t stream);

/*
 * kda_decode_step with the input prologue (Kimi Linear summary, §4: short
 * convolution and Swish on q, k, v, as in kda_short_conv_swish) carried
 * across steps: each sequence keeps a rolling window of its last
 * conv_width - 1 inputs per channel, so that a run of steps equals
 * kda_forward_conv over the same tokens.
 *
 *  x_q, x_k : [B, H, dk]; x_v : [B, H, dv]: this token's convolution inputs.
 *  w_q, w_k : [H*dk, conv_width]; w_v : [H*dv, conv_width] float32
 *             (4-byte aligned); conv_width : 1..4 (else KDA_ERR_UNSUPPORTED).
 *  conv_state : [B, H*(2*dk + dv), conv_width - 1] in `dt`, channels in the
 *             order q (h*dk + i), k (H*dk + h*dk + i), v (2*H*dk + h*dv + j);
 *             element m holds the input of the token conv_width - 1 - m
 *             steps back (m = 0 the oldest).  Read, then overwritten with the
 *             window of the next step (zeros before a sequence's first token).
 *             May be NULL when conv_width = 1.  Must not overlap any other
 *             argument.
 * Everything else is kda_decode_step's; the step is one launch.
 */
kda_status kda_decode_step_conv(const void* x_q, const void* x_k, const void* x_v,
                                const float* w_q, const float* w_k, const float* w_v,
                                int32_t conv_width, void* conv_state, const void* z,
                                const float* A, const void* beta, float* S_inout, int32_t B,
                                int32_t H, int32_t dk, int32_t dv, kda_dtype dt, void* o,
                                kda_stream_t stream);

/*
 * The layer's input prologue on one tensor (Kimi Linear summary, §4 "The Kimi
 * Linear Model Architecture": a short convolution captures dependencies
 * between neighbouring tokens, and a Swish nonlinearity is applied to the
 * queries, keys and values).  The pages give neither the width nor the form
 * of the convolution; this is a causal depthwise convolution along the tokens
 * of each sequence, no bias, never reaching across a sequence boundary:
 *
 *   u[t,c] = sum_{i<width} w[c,i] * x[t-(width-1)+i, c]   (x = 0 before the
 *            first token of t's sequence)
 *   y[t,c] = u[t,c] * sigmoid(u[t,c])
 *
 *  x, y      : [T, channels] in `dt` (channels = H * d for a [T, H, d]
 *              tensor), 16-byte aligned; y must not overlap x.
 *  w         : [channels, width] float32 (4-byte aligned); w[c, width-1]
 *              weighs the current token.
 *  cu_seqlens, num_seqs, total_tokens, max_seqlen : as in kda_forward
 *              (cu_seqlens is not validated here: a malformed one gives
 *              undefined values, never an out-of-range access).
 *  channels  : a positive multiple of 8;  width : 1..4 (else
 *              KDA_ERR_UNSUPPORTED).
 * One launch; no workspace.
 */
kda_status kda_short_conv_swish(const void* x, const float* w, const int32_t* cu_seqlens,
                                int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen,
                                int32_t channels, int32_t width, kda_dtype dt, void* y,
                                kda_stream_t stream);

/* Workspace bytes for kda_forward_conv: kda_forward's on the tensor-core
 * path (bf16, dk = dv = 128, chunk 64), where the prologue runs inside the
 * chunk preparation; elsewhere kda_forward's plus room for the prologue's q,
 * k and v (0 for unsupported arguments). */
size_t kda_forward_conv_workspace_size(int32_t num_seqs, int32_t total_tokens,
                                       int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                                       kda_dtype dt, int32_t chunk);

/*
 * kda_forward on the prologue's outputs: q = Swish(conv(x_q)), k = Swish(
 * conv(x_k)), v = Swish(conv(x_v)) as in kda_short_conv_swish, then the
 * operator, which normalises q and k to unit length itself.  z (the
 * forget-gate input) and beta are used as given.
 *
 *  x_q, x_k : [T, H, dk]; x_v : [T, H, dv], in `dt`.
 *  w_q, w_k : [H*dk, conv_width]; w_v : [H*dv, conv_width] float32.
 *  conv_width : 1..4.
 *  workspace_bytes >= kda_forward_conv_workspace_size(...).
 * Everything else is kda_forward's.  On the tensor-core path the prologue is
 * fused into the chunk preparation: it stages each chunk's x rows with the
 * three tokens before them, convolves and applies Swish in registers (q and
 * k stay fp32 up to their norms; v is rounded to bf16 for the WY product), so
 * the call reads x_q, x_k, x_v once and launches what kda_forward launches.
 * On the CUDA-core path the prologue is one extra launch that writes q, k, v
 * into the workspace.
 */
kda_status kda_forward_conv(const void* x_q, const void* x_k, const void* x_v,
                            const float* w_q, const float* w_k, const float* w_v,
                            int32_t conv_width, const void* z, const float* A, const void* beta,
                            const float* S0, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk,
                            int32_t dv, kda_dtype dt, int32_t chunk, void* o, float* S_final,
                            void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Context parallelism: one long sequence split over ranks (Kimi K3
 * architecture summary, infrastructure section: KDA context parallelism
 * computes the local state updates on each rank and merges them with a prefix
 * scan over a fixed-size all-gather).  The recurrence is affine in the state,
 * so a shard of tokens acts on the state entering it as
 *
 *   S_after = M S_before + N     (M: dk x dk, N: dk x dv, per sequence and head)
 *
 * with M the product of the shard's per-token transitions
 * (I - beta k k^T) Diag(alpha) and N the state the shard leaves from S = 0.
 * Protocol, for the shards 0 .. R-1 of a sequence in token order, shard r on
 * rank r:
 *   1. kda_cp_local(shard r) -> (M_r, N_r); the workspace keeps the shard's
 *      chunk preparation and segment transitions for step 4;
 *   2. the caller all-gathers (M_j, N_j) of every rank (a fixed size: 2 x 64 KB
 *      per head at d = 128), e.g. with one NCCL all-gather;
 *   3. S_in(r) = fold of kda_state_compose over j = 0 .. r-1, starting from
 *      the sequence's initial state: S_in(j+1) = M_j S_in(j) + N_j;
 *   4. kda_cp_finish(S_in(r)) on the same workspace -> o of shard r and the
 *      state after it (on the last rank, the sequence's final state).
 * Several sequences may be processed together (num_seqs > 1 with their own
 * cu_seqlens); each (sequence, head) has its own M and N.  The tensor-core
 * configuration only (bf16, dk = dv = 128, chunk 64); others return
 * KDA_ERR_UNSUPPORTED.  Step 1 is kda_forward's preparation and transition
 * passes plus the last segment's transition and a fold; step 4 is its
 * composition and full passes: the two together cost one kda_forward call plus
 * one segment transition, with no preparation redone.
 */
size_t kda_cp_workspace_size(int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen,
                             int32_t H, int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk);

/*  q, k, v, z, A, beta, cu_seqlens, sizes: the shard, as in kda_forward.
 *  M_out : [N, H, dk, dk] float32;  N_out : [N, H, dk, dv] float32.
 *  workspace : kda_cp_workspace_size bytes, kept unchanged until the matching
 *  kda_cp_finish.  Three launches. */
kda_status kda_cp_local(const void* q, const void* k, const void* v, const void* z,
                        const float* A, const void* beta, const int32_t* cu_seqlens,
                        int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen, int32_t H,
                        int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk, float* M_out,
                        float* N_out, void* workspace, size_t workspace_bytes,
                        kda_stream_t stream);

/*  S_in : [N, H, dk, dv] float32, the state entering the shard (NULL: zeros).
 *  o : [T, H, dv] bf16;  S_final : [N, H, dk, dv] float32 or NULL.
 *  The sizes and cu_seqlens must be those of the kda_cp_local call that
 *  filled the workspace.  One or two launches. */
kda_status kda_cp_finish(const float* S_in, const int32_t* cu_seqlens, int32_t num_seqs,
                         int32_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk,
                         int32_t dv, kda_dtype dt, int32_t chunk, void* o, float* S_final,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*  S_out[i] = M[i] S_in[i] + N[i] for i < count (fp32; M [count, dk, dk],
 *  N, S_in, S_out [count, dk, dv]; S_in NULL reads as zeros; S_out may be
 *  S_in but not M or N).  dk, dv in {32, 64, 128}.  One launch. */
kda_status kda_state_compose(const float* M, const float* N, const float* S_in, float* S_out,
                             int32_t count, int32_t dk, int32_t dv, kda_stream_t stream);

/*
 * Test hook for the failure path; no passage of the pages corresponds to it.
 * Every device-side wait of the tensor-core prefill kernels (on a TMA or bulk
 * copy, or on the completion of tensor-core products) is bounded: by default
 * a wait that has not finished after about 2 s of SM clock gives up, records
 * KDA_ERR_TIMEOUT in the workspace's error word, lets the copies and products
 * it already issued land (each again bounded by about 2 s), frees its Tensor
 * Memory and leaves; the kernels after it in the same call give up the same
 * way.  This call sets the limit of the first, giving-up waits to `cycles` SM
 * cycles for later calls in this process (cycles <= 0 restores the default),
 * so that a test can make a wait run out without any fault.  Not for
 * production use: a small limit fails every call.  Returns KDA_OK.
 */
kda_status kda_debug_set_wait_limit(int64_t cycles);

/*
 * Reads the workspace's error word of the most recent kda_forward /
 * kda_forward_g call on that workspace (synchronises `stream`).  Each call
 * clears the word (a 4-byte cudaMemsetAsync ordered before its first kernel)
 * and its kernels only OR errors into it.  Returns
 * KDA_OK, KDA_ERR_INVALID_ARG (bad cu_seqlens seen on the device),
 * KDA_ERR_TIMEOUT (a bounded device wait gave up) or KDA_ERR_CUDA.
 */
kda_status kda_check_device_error(const void* workspace, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
