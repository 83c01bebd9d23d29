/*
 * gdn.h -- C ABI of libgdn.so: the gated delta rule (Gated DeltaNet sequence
 * mixer) on NVIDIA B200 (sm_100a).
 *
 * The operation.  For every sequence and every value head, a d_v x d_k
 * matrix state S evolves token by token as
 *
 *     S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,                     alpha_t = exp(g_t),
 *
 * the gated delta rule of "Architecture Thread I: Gated Attention, DeltaNet,
 * and Hybrid Models" (section "Gated DeltaNet") and of "Gated Attention
 * Architectures" (section 3, Gated DeltaNet, "Mathematical Formulation"),
 * with the read-out o_t = S_t q_t of the same page's section 1.  The state
 * does not grow with the sequence ("The Transformer Isn't Alone Anymore",
 * the long-context section), so prefill returns it and decode updates it.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, row-major and token-major; every pointer is device
 *     memory owned by the caller.  The library allocates nothing, keeps no
 *     state between calls, never synchronises, and is stream-ordered: work
 *     is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and runs asynchronously.
 *   - q, k: [tokens, Hk, d_k]; v, o: [tokens, Hv, d_v], all of `dtype`.
 *     g, beta: [tokens, Hv] fp32.  States: [N, Hv, d_v, d_k] fp32, row =
 *     value index, key index fastest.
 *   - Value head h reads query/key head h / (Hv / Hk) (grouped heads share
 *     their q/k head in contiguous groups); Hv % Hk must be 0.
 *   - Unchecked preconditions (documented, not verified): q and k are
 *     L2-normalised by the caller, beta in (0, 1) and g <= 0 -- unless the
 *     flags below hand those steps to the library.  The kernels
 *     read g as max(g, -20): exp(-20) is about 2e-9, below fp32 resolution
 *     relative to the state, and the floor keeps the chunk-local prefix
 *     sums of g finite and accurate (g = -inf would make them undefined).
 *   - The output reads the state after the update at the same token.
 *   - Base pointers must be 16-byte aligned (tensor-memory-accelerator
 *     loads); violations return GDN_ERR_MISALIGNED before any launch.
 *   - Errors are returned as a status; nothing aborts or prints.  A status
 *     other than GDN_OK means nothing was enqueued, except GDN_ERR_CUDA
 *     raised by a launch, which reports the CUDA error of that launch.
 *   - The last error's detail text is kept per host thread
 *     (gdn_last_error_message).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad shape, Hv % Hk != 0 */
    GDN_ERR_UNSUPPORTED = 2,        /* valid but not implemented (sizes)     */
    GDN_ERR_MISALIGNED = 3,         /* a base pointer not 16-byte aligned    */
    GDN_ERR_WORKSPACE_TOO_SMALL = 4,
    GDN_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed  */
    GDN_ERR_DEVICE_CHECK = 6        /* a kernel rejected its inputs (see
                                       gdn_read_device_status)               */
} gdn_status_t;

typedef enum { GDN_DTYPE_F32 = 0, GDN_DTYPE_BF16 = 1 } gdn_dtype_t;

/* Flags for gdn_shape_t.flags (and the flags argument of gdn_decode_step_ex). */
#define GDN_FLAG_FORCE_SIMT 1u  /* run the fp32 CUDA-core kernel even where the
                                   tensor-core kernel applies (cross-checks) */
/* The mixer's input side, done inside the kernels so that no separate pass
 * over q, k, g and beta is needed ("Gated Attention Architectures", the
 * Gated DeltaNet code listing: q and k L2-normalised per head, decay and
 * write gates as sigmoids of per-head logits; "Architecture Thread I",
 * "Modern Architecture Improvements": L2 normalisation keeps the
 * transition's eigenvalue along k in (0, 1)).                              */
#define GDN_FLAG_QK_L2NORM 2u    /* q and k are raw: each (token, head) row is
                                    used as x / max(||x||_2, 1e-12)          */
#define GDN_FLAG_GATE_LOGITS 4u  /* g holds the decay logit a and beta the
                                    write logit b: alpha = sigmoid(a), i.e.
                                    the log-decay is log sigmoid(a), and the
                                    write strength is sigmoid(b)            */
/* The bf16 tensor-core prefill (d_k = d_v = 128, C = 64) has two forms.  The
 * single kernel inverts each chunk's triangular WY factor T = (I + A)^-1 in
 * place, one chunk ahead of the state; its workspace holds only the schedule
 * tables (a few bytes per sequence), and it needs the value heads in
 * multiples of 4.  The two-kernel form computes the factors of all chunks at
 * once (they do not depend on the state) into the workspace, 16,640 bytes
 * per (chunk, value head), then runs the state-carrying chunk loop that
 * reads them; it takes any head count.  By default the single kernel runs where it
 * applies and the two-kernel form where it does not (value heads not a
 * multiple of 4).  GDN_FLAG_SPLIT asks for the two-kernel form wherever it
 * applies; GDN_FLAG_ONE_KERNEL never runs it (shapes the single kernel does
 * not take then run the fp32 CUDA-core kernel).  Setting both is an invalid
 * argument.  The results agree within rounding.                            */
#define GDN_FLAG_ONE_KERNEL 8u
#define GDN_FLAG_SPLIT 16u

/* Shape of a prefill problem.
 *   batch, seq_len  without cu_seqlens: B sequences of T tokens each
 *                   (tokens = B * T).  With cu_seqlens: batch must be 1 and
 *                   seq_len is the total packed token count.
 *   num_seqs        N = batch, or the number of packed sequences.
 *   chunk_size      C, the chunk length of the chunkwise algorithm: 16, 32
 *                   or 64.  It changes rounding only, never the result.
 *   dtype           gdn_dtype_t of q, k, v, o.                             */
typedef struct {
    int32_t batch;
    int32_t seq_len;
    int32_t num_seqs;
    int32_t num_qk_heads;
    int32_t num_v_heads;
    int32_t head_dim_k;
    int32_t head_dim_v;
    int32_t chunk_size;
    int32_t dtype;
    uint32_t flags;
} gdn_shape_t;

/* Bytes of device workspace gdn_chunk_forward needs for `shape` (a pure
 * function of the shape, flags included; the caller allocates it, 256-byte
 * aligned).  Where the two-kernel tensor-core form runs, this includes
 * 16,640 bytes per (chunk, value head) for the chunk factors (T', T'' and
 * the decay prefix sums): at most
 * ((tokens + 63 N) / 64) Hv of them.  With a workspace below that size (but
 * at least the size queried with GDN_FLAG_ONE_KERNEL set) the call runs as
 * if GDN_FLAG_ONE_KERNEL were set. */
GDN_API gdn_status_t gdn_chunk_forward_workspace_size(const gdn_shape_t *shape, size_t *bytes);

/* Kernel paths of gdn_chunk_forward. */
#define GDN_PATH_SIMT 0          /* fp32 CUDA-core kernel                      */
#define GDN_PATH_TC_ONE_KERNEL 1 /* single tensor-core kernel                  */
#define GDN_PATH_TC_SPLIT 2      /* two-kernel tensor-core form (chunk factors
                                    for all chunks, then the chunk loop)      */

/* Which path gdn_chunk_forward takes for `shape` with a workspace of
 * `workspace_bytes` on the current device, written to *path (a GDN_PATH_*
 * value).  The page has no counterpart for this query: it lets a caller see
 * that a shape runs on the CUDA cores (an fp32 or non-128 head size, or the
 * flags), or that a workspace below the two-kernel size kept a shape of
 * value heads not a multiple of 4 off the tensor cores.  Errors: those of
 * gdn_chunk_forward_workspace_size, GDN_ERR_WORKSPACE_TOO_SMALL below the
 * minimum workspace, GDN_ERR_CUDA without a usable device.  Launches
 * nothing. */
GDN_API gdn_status_t gdn_chunk_forward_path(const gdn_shape_t *shape, size_t workspace_bytes, int32_t *path);

/* Chunkwise prefill ("Gated Attention Architectures", sections 2 and 3: the
 * WY representation of the generalised Householder transitions, extended
 * with per-chunk cumulative decay products, and the decay-masked chunk
 * output of section 1).  Computes o for every token and, if final_state is
 * not NULL, the state after each sequence's last token.
 *   q, k            [tokens, Hk, d_k] dtype
 *   v               [tokens, Hv, d_v] dtype
 *   g, beta         [tokens, Hv] fp32 (log-decay, write strength)
 *   initial_state   [N, Hv, d_v, d_k] fp32, or NULL for zeros
 *   cu_seqlens      [N + 1] int32 device array of sequence starts
 *                   (cu[0] = 0, non-decreasing, cu[N] = tokens), or NULL
 *                   for the batched layout.  Chunks never cross a sequence
 *                   boundary; empty sequences are allowed (final = initial).
 *                   Its contents are checked on the device: a violation
 *                   makes every kernel skip its work and records
 *                   GDN_ERR_DEVICE_CHECK in the workspace status word.
 *   o               [tokens, Hv, d_v] dtype (written)
 *   final_state     [N, Hv, d_v, d_k] fp32 or NULL; may alias initial_state.
 *   workspace       device scratch of at least the queried size.
 * Paths: bf16 with d_k = d_v = 128 and C = 64 runs the tensor-core
 * (tcgen05/TMEM, TMA-fed) kernel; every other supported shape (d_k, d_v <=
 * 128, C in {16, 32, 64}) runs the fp32 CUDA-core kernel. */
GDN_API gdn_status_t gdn_chunk_forward(const gdn_shape_t *shape,
                               const void *q, const void *k, const void *v,
                               const float *g, const float *beta,
                               const float *initial_state,
                               const int32_t *cu_seqlens,
                               void *o, float *final_state,
                               void *workspace, size_t workspace_bytes,
                               void *stream);

/* gdn_chunk_forward without a caller-provided workspace.  The source pages
 * have no counterpart for this entry point: it exists for callers that
 * cannot allocate device memory, such as a plugin that a host runtime hands
 * only tensor pointers and no allocator, or a serving loop that must not
 * call cudaMalloc on the request path (cudaMalloc may synchronise the whole
 * device).  The scratch the prefill needs (schedule tables and status word)
 * lives instead in a device array built into the library: 196,864 bytes on
 * every GPU that loads the library, held until the process exits, enough
 * for at most 16,384 sequences per call (more returns GDN_ERR_UNSUPPORTED
 * with a message; nothing is launched).  Arguments and results are those of
 * gdn_chunk_forward with GDN_FLAG_ONE_KERNEL set (the scratch holds no chunk
 * factors).  Every call looks up the array's device address in the
 * current device's context (cudaGetSymbolAddress, a host-side query); the
 * first lookup in a context may load the library's device code, so make the
 * first call on a device before any stream capture.  No call allocates or frees memory.
 * All calls on a device share the one array: calls that overlap on the GPU
 * (two streams, or two host threads) race on it and give wrong results, so
 * serialise them.  Each call re-initialises the scratch before use, so what
 * an earlier call left there is harmless.  gdn_noalloc_read_device_status
 * reads back the device status word the last call on the current device
 * left in the array. */
GDN_API gdn_status_t gdn_chunk_forward_noalloc(const gdn_shape_t *shape,
                                       const void *q, const void *k, const void *v,
                                       const float *g, const float *beta,
                                       const float *initial_state,
                                       const int32_t *cu_seqlens,
                                       void *o, float *final_state,
                                       void *stream);

/* Reads the device status word that gdn_chunk_forward, gdn_kda_forward or
 * gdn_chunk_backward left in `workspace` into *device_status: GDN_OK, or
 * GDN_ERR_DEVICE_CHECK when the schedule rejected cu_seqlens or a
 * tensor-core kernel's bounded wait timed out (the outputs are then not, or
 * not all, written).  Synchronises `stream`.  This and
 * gdn_noalloc_read_device_status are the only entry points that wait for
 * the GPU. */
GDN_API gdn_status_t gdn_read_device_status(const void *workspace, int32_t *device_status, void *stream);

/* The same for gdn_chunk_forward_noalloc: reads the device status word that
 * the last such call on the current device left in the library's built-in
 * scratch array (a cu_seqlens rejected on the device, or a tensor-core wait
 * that timed out, reads GDN_ERR_DEVICE_CHECK; o and final_state are then
 * not written).  Synchronises `stream`.  Like the scratch array itself it
 * has no counterpart in the source pages.  Errors: GDN_ERR_INVALID_ARGUMENT
 * for a NULL device_status, GDN_ERR_CUDA when the array's address cannot be
 * resolved or the read fails. */
GDN_API gdn_status_t gdn_noalloc_read_device_status(int32_t *device_status, void *stream);

/* One decode token for each of N sequences, state updated in place
 * ("The Transformer Isn't Alone Anymore": the recurrent state is read and
 * updated every step, which makes decoding memory-bound).  Per value head
 * and per state row i: p_i = s_i . k, r_i = s_i . q,
 * u_i = beta (v_i - alpha p_i), s_i <- alpha s_i + u_i k^T,
 * o_i = alpha r_i + u_i (k . q)  (= s_i,new . q): one read and one write
 * of S.
 *   q, k   [N, Hk, d_k] dtype;  v, o [N, Hv, d_v] dtype
 *   g, beta [N, Hv] fp32
 *   state  [N, Hv, d_v, d_k] fp32, read and written in place.
 * d_k = 128 takes the vectorised kernel; other d_k <= 256 a generic one. */
GDN_API gdn_status_t gdn_decode_step(int32_t num_seqs, int32_t num_qk_heads, int32_t num_v_heads,
                             int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                             const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             float *state, void *o, void *stream);

/* gdn_decode_step with flags: GDN_FLAG_QK_L2NORM and GDN_FLAG_GATE_LOGITS
 * (as for prefill: raw q and k normalised per head inside the kernel; g and
 * beta given as logits).  flags = 0 is gdn_decode_step.  Other bits return
 * GDN_ERR_INVALID_ARGUMENT. */
GDN_API gdn_status_t gdn_decode_step_ex(int32_t num_seqs, int32_t num_qk_heads, int32_t num_v_heads,
                                int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                const void *q, const void *k, const void *v,
                                const float *g, const float *beta,
                                float *state, void *o, uint32_t flags, void *stream);

/* The mixer's output side, applied to every (token, value head) output row
 * o of d_v values before it is stored:
 *
 *     y_i = o_i / sqrt(mean_j(o_j^2) + eps) * s_i * act(z_i)
 *
 * RMS normalisation of the mixer output ahead of the output projection
 * ("Architecture Thread I", "Modern Architecture Improvements"), with the
 * gate of the gated RMSNorm ("The Transformer Isn't Alone Anymore", the
 * model-reconstruction section; "Gated Attention Architectures", the
 * Gated DeltaNet code listing, whose gate is SiLU of a projection; the
 * same page's Gated Attention section for the sigmoid form) and the
 * zero-centred scale 1 + delta of the Qwen3-Next passage of "Architecture
 * Thread I".  The normalisation runs in fp32 on the unrounded output. */
#define GDN_OUT_GATE_SILU 1u        /* act(z) = z * sigmoid(z)                 */
#define GDN_OUT_GATE_SIGMOID 2u     /* act(z) = sigmoid(z)                     */
#define GDN_OUT_ZERO_CENTRED 4u     /* s_i = 1 + w_i (else s_i = w_i)          */
#define GDN_OUT_WEIGHT_PER_HEAD 8u  /* w is [Hv, d_v] (else [d_v], shared by
                                       all value heads)                       */
typedef struct {
    const float *weight;  /* fp32 scale w, [d_v] or [Hv, d_v], 16-byte aligned;
                             NULL reads as w = 1 (plain) or w = 0 (zero-
                             centred), i.e. a unit scale either way          */
    const void *gate;     /* z, [tokens, Hv, d_v] of the problem's dtype,
                             16-byte aligned; NULL = no gate (then neither
                             gate flag may be set; with a gate exactly one
                             must be)                                        */
    float eps;            /* added to the mean square; finite and > 0        */
    uint32_t flags;       /* GDN_OUT_* bits; others are invalid              */
} gdn_output_side_t;

/* gdn_chunk_forward with the output side applied: `o` receives y instead of
 * the raw read-out.  out_side = NULL is gdn_chunk_forward.  The tensor-core
 * kernel applies it in its output epilogue (the gate tile arrives by TMA
 * beside the chunk); the fp32 CUDA-core kernel, whose blocks each own a
 * slice of d_v, stores o and then runs one more kernel over o in place.
 * Invalid output-side arguments return GDN_ERR_INVALID_ARGUMENT or
 * GDN_ERR_MISALIGNED before any launch. */
GDN_API gdn_status_t gdn_chunk_forward_out(const gdn_shape_t *shape,
                                   const void *q, const void *k, const void *v,
                                   const float *g, const float *beta,
                                   const float *initial_state,
                                   const int32_t *cu_seqlens,
                                   const gdn_output_side_t *out_side,
                                   void *o, float *final_state,
                                   void *workspace, size_t workspace_bytes,
                                   void *stream);

/* gdn_decode_step_ex with the output side applied inside the decode kernel
 * (gate z: [N, Hv, d_v]).  out_side = NULL is gdn_decode_step_ex.  With an
 * output side, d_v must be at most 256 (GDN_ERR_UNSUPPORTED otherwise). */
GDN_API gdn_status_t gdn_decode_step_out(int32_t num_seqs, int32_t num_qk_heads, int32_t num_v_heads,
                                 int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                 const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 float *state, const gdn_output_side_t *out_side,
                                 void *o, uint32_t flags, void *stream);

/* Kimi Delta Attention: the delta rule with one decay per key channel
 * ("Gated Attention Architectures", section 8, "Mathematical Formulation":
 * S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t,
 * D_t = diag(alpha_t)).  With this library's d_v x d_k state the update is
 *     S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,   alpha_t[c] = exp(g[t, h, c]),
 * which is the gated delta rule when every alpha_t[c] is the same.
 * Arguments are those of gdn_chunk_forward_out except
 *   g     [tokens, Hv, d_k] fp32: one log-decay per key channel (with
 *         GDN_FLAG_GATE_LOGITS: one decay logit per key channel, alpha =
 *         sigmoid(logit)); read as max(g, -20) like the scalar gate.
 * Two paths.  bf16 with d_k = d_v = 128 and C = 64 runs the chunkwise WY
 * form on the tensor cores: a first kernel forms every chunk's decay-masked
 * products, its triangular factor and the decay-scaled keys and queries at
 * once, then the chunk loop carries the state through tcgen05 products.  It
 * needs the workspace gdn_kda_forward_workspace_size returns (66,048 bytes
 * per (chunk, value head) on top of the schedule tables).  Every other shape,
 * GDN_FLAG_FORCE_SIMT, or a smaller workspace walks the tokens of each
 * sequence in order on CUDA cores (state in registers, a block per sequence,
 * value head and 32 rows of d_v; shape->chunk_size is checked but not used),
 * with the workspace of gdn_chunk_forward.  Supports d_k <= 128 and
 * d_v <= 128, fp32 or bf16; the input flags; an output side (applied as a
 * second pass over o). */
GDN_API gdn_status_t gdn_kda_forward(const gdn_shape_t *shape,
                             const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             const float *initial_state,
                             const int32_t *cu_seqlens,
                             const gdn_output_side_t *out_side,
                             void *o, float *final_state,
                             void *workspace, size_t workspace_bytes,
                             void *stream);

/* Bytes of workspace gdn_kda_forward needs for `shape` (the tensor-core path's
 * chunk operands where it applies, else the schedule tables alone). */
GDN_API gdn_status_t gdn_kda_forward_workspace_size(const gdn_shape_t *shape, size_t *bytes);

/* One Kimi Delta Attention token per sequence, state updated in place: per
 * state row s_i, s' = alpha .* s_i, u_i = beta (v_i - s' . k),
 * s_i <- s' + u_i k^T, o_i = s' . q + u_i (k . q); one read and one write of
 * S.  g is [N, Hv, d_k] fp32; the other arguments are those of
 * gdn_decode_step_out (out_side may be NULL). */
GDN_API gdn_status_t gdn_kda_decode_step(int32_t num_seqs, int32_t num_qk_heads, int32_t num_v_heads,
                                 int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                 const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 float *state, const gdn_output_side_t *out_side,
                                 void *o, uint32_t flags, void *stream);

/* Several decode tokens per sequence in one pass, for verifying draft
 * tokens: multi-token prediction drafts a few tokens ahead and the model
 * confirms several at once ("Architecture Thread I", the Qwen3-Next
 * passage).  For each sequence the K = num_tokens tokens are applied in
 * order from `state` with the decode step's update; o receives every
 * token's output and `snapshots` the state after every token.  `state` is
 * only read: after checking the drafts, gdn_decode_commit moves the state
 * of the accepted prefix into it.  One read of S and K snapshot writes,
 * instead of K reads and K writes for K decode steps.
 *   q, k       [N, K, Hk, d_k] dtype;  v, o [N, K, Hv, d_v] dtype
 *   g, beta    [N, K, Hv] fp32
 *   state      [N, Hv, d_v, d_k] fp32 (read only)
 *   snapshots  [N, K, Hv, d_v, d_k] fp32 (written; must not overlap state)
 *   flags      GDN_FLAG_QK_L2NORM, GDN_FLAG_GATE_LOGITS
 * Supports d_k = 128 and 1 <= K <= 16 (GDN_ERR_UNSUPPORTED otherwise). */
GDN_API gdn_status_t gdn_decode_multi(int32_t num_seqs, int32_t num_tokens, int32_t num_qk_heads,
                              int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                              const void *q, const void *k, const void *v,
                              const float *g, const float *beta, const float *state,
                              float *snapshots, void *o, uint32_t flags, void *stream);

/* Keeps the accepted prefix of a gdn_decode_multi call: for each sequence
 * n, accepted[n] (device int32 [N]) in 1..K copies snapshot accepted[n] - 1
 * into state[n]; 0 keeps state[n].  Values outside 0..K leave state[n]
 * alone and, if bad_count (device int32) is not NULL, add one to it.
 * Shapes as for gdn_decode_multi. */
GDN_API gdn_status_t gdn_decode_commit(int32_t num_seqs, int32_t num_tokens, int32_t num_v_heads,
                               int32_t head_dim_k, int32_t head_dim_v, const float *snapshots,
                               const int32_t *accepted, float *state, int32_t *bad_count, void *stream);

/* Gradients for training ("Architecture Thread I", the Gated DeltaNet
 * section, and "Gated Attention Architectures", sections 2 and 3: the
 * chunked form is how the layer is trained).  For the upstream gradients
 * d_o (of o) and d_final_state (of the final states; NULL = zero), writes
 * the gradients of L = sum d_o . o + sum d_final_state . S_final:
 *   dq, dk             [tokens, Hk, d_k] fp32 (summed over the value heads
 *                      of each q/k group)
 *   dv                 [tokens, Hv, d_v] fp32
 *   dg, dbeta          [tokens, Hv] fp32 (dg is zero where g < -20, the
 *                      kernels' floor on g)
 *   d_initial_state    [N, Hv, d_v, d_k] fp32, or NULL
 * Inputs are those of gdn_chunk_forward (the plain path: no input-side
 * flags, GDN_ERR_UNSUPPORTED otherwise, and neither GDN_FLAG_ONE_KERNEL nor
 * GDN_FLAG_SPLIT); d_o has the dtype of v.  d_k, d_v <= 128.  Two forms:
 *   - bf16 with d_k = d_v = 128 on sm_100 (unless GDN_FLAG_FORCE_SIMT):
 *     tcgen05 tensor-core kernels over chunks of 64 tokens -- the chunk
 *     factors of every (chunk, value head), the state and state-gradient
 *     recurrences (one product per chunk each, every chunk's boundary state
 *     kept), then the gradients of every (chunk, value head, half of d_v).
 *     Workspace: the schedule plus 344,064 bytes per (chunk, value head)
 *     (gdn_chunk_backward_workspace_size).
 *   - otherwise one kernel per (sequence, value head, 32 rows of d_v) that
 *     walks 32-token chunks forward, keeping each chunk's start state and
 *     intra-chunk products (about 3 d_v d_k fp32 values per chunk and value
 *     head), then backward.
 * fp32 results: products of fp32 operands split each operand into a bf16
 * value and a bf16 residual (tensor cores, fp32 accumulation) for bf16
 * inputs, fp32 CUDA-core tiles for fp32 inputs.  dg and dbeta (both forms)
 * and dq, dk (the single-kernel form) are accumulated with atomic adds
 * (their summation order, and so their last bits, can vary between runs). */
GDN_API gdn_status_t gdn_chunk_backward_workspace_size(const gdn_shape_t *shape, size_t *bytes);
GDN_API gdn_status_t gdn_chunk_backward(const gdn_shape_t *shape,
                                const void *q, const void *k, const void *v,
                                const float *g, const float *beta,
                                const float *initial_state,
                                const int32_t *cu_seqlens,
                                const void *d_o, const float *d_final_state,
                                float *dq, float *dk, float *dv, float *dg, float *dbeta,
                                float *d_initial_state,
                                void *workspace, size_t workspace_bytes,
                                void *stream);

/* The input side's short causal convolution, with an optional SiLU after it
 * ("Architecture Thread I", "Modern Architecture Improvements": after the
 * projections, q and k pass through a short convolution, SiLU and L2
 * normalisation -- the last step is GDN_FLAG_QK_L2NORM of the mixer calls --
 * and v through a short convolution and SiLU).  Causal and depthwise, one
 * filter of W taps per channel:
 *     y[t, c] = act( sum_{j<W} weight[c, j] x[t - (W-1) + j, c] ),
 * the last tap on the current token; act = SiLU with GDN_CONV_SILU, else the
 * identity.  Inputs before a sequence's first token come from the
 * sequence's conv state, its W-1 preceding inputs oldest first (zeros when
 * state_in is NULL); a sequence never reads another's tokens.
 *   num_seqs, seq_len, cu_seqlens
 *                   N sequences: without cu_seqlens, of seq_len tokens each
 *                   (tokens = N * seq_len); with cu_seqlens ([N + 1] int32
 *                   device array of sequence starts, as for
 *                   gdn_chunk_forward; seq_len ignored), packed.  Its
 *                   contents are not checked: contents that break its
 *                   contract give unspecified values, never an access out
 *                   of bounds.
 *   x, y            [tokens, channels] of `dtype` (q, k or v as [tokens,
 *                   H, d] with channels = H * d); y must not overlap x.
 *   weight          [channels, W] fp32.
 *   state_in        [N, channels, W-1] fp32, or NULL for zeros.
 *   state_out       [N, channels, W-1] fp32, or NULL: each sequence's last
 *                   W-1 inputs (reaching into state_in when the sequence is
 *                   shorter), for decode to continue from; must not overlap
 *                   state_in.
 * 1 <= W <= 8; channels a multiple of 4.  HBM-bound: one read of x and one
 * write of y. */
#define GDN_CONV_SILU 1u
GDN_API gdn_status_t gdn_short_conv(int32_t num_seqs, int32_t seq_len, const int32_t *cu_seqlens, int64_t tokens,
                                    int32_t channels, int32_t width, int32_t dtype, const void *x,
                                    const float *weight, const float *state_in, float *state_out, void *y,
                                    uint32_t flags, void *stream);

/* Static text for a status code. */
GDN_API const char *gdn_status_string(gdn_status_t status);

/* Detail of the last error returned on the calling host thread ("" if none). */
GDN_API const char *gdn_last_error_message(void);

/* Number of kernels this library has launched in this process (all host
 * threads), for accounting of launches inside a timed region. */
GDN_API uint64_t gdn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
