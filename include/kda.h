/*
 * kda.h -- C ABI of libkda: the Kimi Delta Attention (KDA) recurrence on B200 (sm_100a).
 *
 * The operation (per sequence n and head h; state S is d_k x d_v fp32, row c =
 * key channel, column j = value channel), for each token t in order:
 *
 *     S   <- Diag(alpha_t) S,            alpha_t = exp(log_alpha_t), one gate per key channel
 *     S   <- S + beta_t k_t (v_t - S^T k_t)^T                   (delta rule: write only the error)
 *     o_t  = S^T q_t                                             (read after the write)
 *
 * Sources: "Kimi K3 -- the architecture and infrastructure, explained"
 * (shivam2003.com), sections "How the delta rule actually works" (the update
 * S <- S - beta (S k - v) k^T, written there for the transposed d_v x d_k
 * state) and "Kimi Delta Attention: the load-bearing choice" (channel-wise
 * gating; blockwise computation that maps onto matrix units; constant per-token
 * decode cost); aitrending.vip "Inside Kimi K3", section "Technical Details"
 * (beta = writing strength, alpha = forgetting factor, 128 dials per head);
 * same shivam2003.com article, section "Serving infrastructure: supernodes and
 * the prefill cache" (a cached prefill state is restored so a returning request
 * only pays for the new suffix: initial/final state I/O).
 *
 * Conventions shared by every entry point
 *   - Device pointers unless a name ends in _host. All tensors are dense and
 *     row-major with the last dimension contiguous, 16-byte aligned base.
 *   - q, k: [T, H, d_k]; v, out: [T, H, d_v] in the input dtype (fp32 or bf16).
 *     log_alpha: [T, H, d_k] fp32 (must be <= 0); beta: [T, H] fp32 (in [0, 1]);
 *     states: [N, H, d_k, d_v] fp32. q and k are used as given (the caller
 *     normalises them; no 1/sqrt(d_k) scale is applied).
 *   - Ownership: the caller allocates and frees every buffer, including the
 *     workspace. The library does not allocate, free or synchronise inside
 *     kda_prefill / kda_decode_step: both only enqueue work on `stream` and
 *     return. Buffers must stay valid until the stream has run the work. The
 *     prefill, decode and speculative-decode calls can therefore be captured
 *     into a CUDA graph (after one call outside the capture, which sets each
 *     kernel's shared-memory limit) and replayed on the same buffers; the decode
 *     step's kernel is launched with programmatic stream serialization, so
 *     consecutive steps overlap their launch, in a stream or in a graph.
 *   - Aliasing: final_state may alias initial_state (in-place resume); the
 *     decode state is updated in place; out must not alias any input.
 *   - Errors: arguments are checked on the host before anything is enqueued;
 *     a non-OK status means nothing was enqueued (except KDA_ERR_CUDA, which
 *     reports a failed launch). kda_last_error() returns a message for the
 *     calling thread's last non-OK status. No C++ exception crosses this ABI.
 *   - Values are not checked on the device: inputs must be finite, log_alpha <= 0
 *     and beta in [0, 1]; otherwise results are unspecified (but memory-safe).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size, shape, or cu_seqlens            */
    KDA_ERR_UNSUPPORTED = 2,      /* a dtype / head-size combination with no kernel       */
    KDA_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed                 */
    KDA_ERR_TIMEOUT = 4,          /* a bounded on-device wait gave up (device status word) */
    KDA_ERR_INTERNAL = 5          /* a debug build (-DKDA_DEBUG) caught an access outside its
                                     buffer (device status word); never set by release builds */
} kda_status_t;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* Supported head sizes: d_k, d_v in {32, 64, 128}. */

/*
 * Bytes of device workspace that let kda_prefill take its fastest path for this
 * problem (a multiple of 256). Problems with few (sequence, head) pairs get room
 * for the split-role kernel's ring of chunk images (704 KiB per pair); any
 * workspace of at least 256 + 4 * num_seqs bytes (rounded up to 256) is accepted,
 * and a smaller one than returned here selects the single-role kernel. Host
 * function: queries the current device's SM count; returns 0 only for
 * arguments kda_prefill would reject.
 */
KDA_API size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H,
                                  int32_t d_k, int32_t d_v, kda_dtype_t dtype);

/*
 * Chunked prefill over packed variable-length sequences.
 *
 * Defined by: the recurrence of "How the delta rule actually works" with the
 * per-key-channel forgetting of "Kimi Delta Attention: the load-bearing choice"
 * (shivam2003.com Kimi K3 article; that section also says the update is computed
 * blockwise so it maps onto matrix units: the 64-token chunks here), and the
 * state save/restore of "Serving infrastructure: supernodes and the prefill
 * cache" (same article: a cached state lets a returning request pay only for
 * its new suffix), which initial_state / final_state carry.
 *
 *   q, k        [total_tokens, H, d_k]  dtype
 *   v           [total_tokens, H, d_v]  dtype
 *   log_alpha   [total_tokens, H, d_k]  fp32
 *   beta        [total_tokens, H]       fp32
 *   initial_state [num_seqs, H, d_k, d_v] fp32, or NULL for a zero start
 *   cu_seqlens_dev  [num_seqs + 1] int32 device copy of the token offsets
 *   cu_seqlens_host [num_seqs + 1] int32 host copy of the same offsets (read
 *                   during the call only; used to validate and plan)
 *   out         [total_tokens, H, d_v]  dtype  (written)
 *   final_state [num_seqs, H, d_k, d_v] fp32, or NULL if not wanted (written;
 *               may alias initial_state)
 *   workspace   device memory, 256-byte aligned, contents on entry ignored: at
 *               least 256 + 4 * num_seqs bytes rounded up to 256, and
 *               kda_prefill_workspace_size(...) bytes for the fastest path.
 *
 * cu_seqlens must start at 0, be non-decreasing and end at total_tokens.
 * Zero-length sequences are allowed (their final state is their initial state).
 * A dense [B, T] batch is cu_seqlens = {0, T, 2T, ..., B*T}.
 *
 * Tokens are processed in chunks of 64 per sequence: bf16 inputs with
 * d_k = d_v = 128 run on the tensor-core chunk kernels (with few (sequence,
 * head) pairs and a full-size workspace, a split-role kernel in which some
 * thread blocks run the per-head state chains and the others prepare the
 * state-independent half of upcoming chunks); every other supported
 * combination runs the token-serial fp32 kernel (see kda_prefill_recurrent).
 * The result does not depend on that choice beyond rounding.
 *
 * Status: KDA_ERR_INVALID_ARGUMENT for a NULL required pointer, H <= 0,
 * num_seqs < 0, an unsupported d_k/d_v, bad cu_seqlens_host, or a workspace
 * smaller than the minimum; KDA_ERR_CUDA if a launch fails.
 */
KDA_API kda_status_t kda_prefill(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         const float *initial_state,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int32_t num_seqs, int64_t total_tokens, int32_t H,
                         int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                         void *out, float *final_state,
                         void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_prefill with context parallelism inside the GPU: each sequence is cut
 * into up to `segments` segments of whole 64-token chunks (fewer if it has
 * fewer chunks), and their state chains run side by side instead of one after
 * another.
 *
 * Defined by: the blockwise, context-parallel computation of the KDA update in
 * "Kimi Delta Attention: the load-bearing choice" (shivam2003.com Kimi K3
 * article). The state map of a segment is affine, S_end = F S_start + S0_end
 * (F: the product of the segment's per-chunk transitions, S0: the segment run
 * from a zero state), so segments after the first run from zero alongside the
 * product F and a per-chunk correction term; a scan then finds each segment's
 * true start state (and the final state) and a fix-up pass adds the start
 * state's contribution to the outputs. The result is kda_prefill's up to
 * rounding.
 *
 * Applies to bf16 inputs with d_k = d_v = 128; with segments = 1, other
 * dtypes / head sizes, sequences too short to split, or more chains than the
 * GPU can hold at once (2 * segments * H thread blocks resident), it runs
 * kda_prefill's own path. The workspace must hold
 * kda_prefill_cp_workspace_size(...) bytes (about 16 KiB per chunk and head of
 * every segment after a sequence's first, plus the split kernel's ring).
 * Arguments, layouts and status as kda_prefill; segments in [1, 64].
 */
KDA_API kda_status_t kda_prefill_cp(const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta,
                            const float *initial_state,
                            const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                            int32_t num_seqs, int64_t total_tokens, int32_t H,
                            int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                            void *out, float *final_state, int32_t segments,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Workspace bytes kda_prefill_cp needs for these sequences (it reads
 * cu_seqlens_host[0..num_seqs]) and `segments`; at least
 * kda_prefill_workspace_size. 0 for arguments kda_prefill_cp rejects.
 */
KDA_API size_t kda_prefill_cp_workspace_size(int32_t num_seqs, const int32_t *cu_seqlens_host,
                                             int32_t H, int32_t d_k, int32_t d_v,
                                             kda_dtype_t dtype, int32_t segments);

/*
 * The same operation as kda_prefill, always on the token-serial kernel: one
 * thread block per (sequence, head, 32-wide slice of d_v) walks the tokens in
 * order with the state slice in registers and fp32 arithmetic throughout. It
 * needs no workspace. Arguments and status as kda_prefill.
 */
KDA_API kda_status_t kda_prefill_recurrent(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   const float *initial_state,
                                   const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                   int32_t num_seqs, int64_t total_tokens, int32_t H,
                                   int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                                   void *out, float *final_state, kda_stream_t stream);

/*
 * One decode step: one new token for each of num_seqs sequences, state updated
 * in place (constant cost per token: the state of each head is read once and
 * written once).
 *
 * Defined by: the same per-token recurrence ("How the delta rule actually
 * works", "Kimi Delta Attention: the load-bearing choice", shivam2003.com Kimi
 * K3 article); the second section also gives the property this kernel is built
 * around, a decode cost per token that stays the same however long the context.
 *
 *   q, k        [num_seqs, H, d_k]  dtype
 *   v           [num_seqs, H, d_v]  dtype
 *   log_alpha   [num_seqs, H, d_k]  fp32
 *   beta        [num_seqs, H]       fp32
 *   state       [num_seqs, H, d_k, d_v] fp32, read and written in place
 *   out         [num_seqs, H, d_v]  dtype (written)
 *   workspace   may be NULL with workspace_bytes == 0 (the decode kernel has no
 *               on-device waits and needs no scratch); reserved for future use.
 *
 * Status: KDA_ERR_INVALID_ARGUMENT for a NULL required pointer, num_seqs < 0,
 * H <= 0 or unsupported head sizes; KDA_ERR_CUDA if the launch fails.
 * num_seqs == 0 is a no-op.
 */
KDA_API kda_status_t kda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             float *state, int32_t num_seqs, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                             void *out, void *workspace, size_t workspace_bytes,
                             kda_stream_t stream);

/* Prologue flags for kda_prefill_prologue: which inputs hold the layer's raw projections. */
#define KDA_PROLOGUE_QK_L2NORM 1u     /* q and k: each (token, head) row x becomes x / sqrt(x.x + 1e-6) */
#define KDA_PROLOGUE_GATE_SOFTPLUS 2u /* log_alpha holds gates g: log alpha = -gate_scale * softplus(g) */
#define KDA_PROLOGUE_BETA_SIGMOID 4u  /* beta holds logits b: beta = 1 / (1 + e^-b) */

/*
 * kda_prefill with the KDA layer's elementwise prologue fused into the
 * kernels' input staging: with the flags above, q and k are L2-normalised per
 * (token, head) row, the forgetting gate is log alpha = -gate_scale *
 * softplus(g) per key channel and beta = sigmoid(b), each applied as the chunk
 * kernels (and the token-serial kernel) load their inputs, so the activated
 * tensors are never written to HBM. ("Kimi Delta Attention: the load-bearing
 * choice" in the shivam2003.com Kimi K3 article: per-channel forgetting gates
 * and a writing strength; the L2 normalisation of q and k keeps the delta
 * rule's step within its stable range.) prologue_flags is any combination of
 * KDA_PROLOGUE_* (0: exactly kda_prefill); gate_scale must be finite and > 0
 * when KDA_PROLOGUE_GATE_SOFTPLUS is set. Tokens past a sequence's end are
 * never read. Arguments, workspace, results and status otherwise as
 * kda_prefill; the results equal kda_prefill's on the activated inputs up to
 * rounding (the activated q and k are rounded to bf16 once more for bf16
 * inputs).
 */
KDA_API kda_status_t kda_prefill_prologue(const void *q, const void *k, const void *v,
                                          const float *log_alpha, const float *beta,
                                          const float *initial_state,
                                          const int32_t *cu_seqlens_dev,
                                          const int32_t *cu_seqlens_host, int32_t num_seqs,
                                          int64_t total_tokens, int32_t H, int32_t d_k,
                                          int32_t d_v, kda_dtype_t dtype, void *out,
                                          float *final_state, void *workspace,
                                          size_t workspace_bytes, uint32_t prologue_flags,
                                          float gate_scale, kda_stream_t stream);

/*
 * kda_prefill with the states held in a pool of slots instead of one state per
 * sequence: the prefill cache of "Kimi K3 -- the architecture and
 * infrastructure, explained" (shivam2003.com), section "Serving
 * infrastructure: supernodes and the prefill cache" keeps computed states and
 * restores them so that a returning request pays only for its new suffix; a
 * pool addressed by slot lets one call resume many requests from cached states
 * (several may start from the same slot) and store their new states, without
 * gathering them into a dense array first.
 *
 *   state_pool      [pool_slots, H, d_k, d_v] fp32: read and written
 *   init_slot_dev   [num_seqs] int32 (device): sequence n starts from slot
 *                   init_slot_dev[n], or from zeros if it is -1
 *   final_slot_dev  [num_seqs] int32 (device): sequence n's final state goes to
 *                   slot final_slot_dev[n], or nowhere if it is -1
 *
 * A slot may be both read and written by the same sequence (in-place resume).
 * A slot written by one sequence must not be read or written by another
 * sequence of the same call (the result would be unspecified). Slot values
 * outside [-1, pool_slots) are treated as -1 and recorded in the device status
 * word, for which kda_read_device_status then returns KDA_ERR_INVALID_ARGUMENT.
 * state_pool may be NULL only if pool_slots == 0 (then every slot must be -1).
 * Everything else (workspace, kernels, status) is as kda_prefill; the results
 * equal kda_prefill's with the states gathered and scattered by slot.
 */
KDA_API kda_status_t kda_prefill_slots(const void *q, const void *k, const void *v,
                                       const float *log_alpha, const float *beta,
                                       float *state_pool, int64_t pool_slots,
                                       const int32_t *init_slot_dev, const int32_t *final_slot_dev,
                                       const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                       int32_t num_seqs, int64_t total_tokens, int32_t H,
                                       int32_t d_k, int32_t d_v, kda_dtype_t dtype, void *out,
                                       void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_decode_step on states held in a pool of slots (the same prefill cache):
 * sequence n's state is slot slot_dev[n] of state_pool ([pool_slots, H, d_k,
 * d_v] fp32), read and written in place; slot -1 means a zero state that is
 * not stored. Two sequences must not name the same slot. Out-of-range slots
 * are treated as -1 and recorded in the device status word at the start of
 * `workspace` (required here: at least 256 bytes, 256-byte aligned), which
 * kda_read_device_status reports as KDA_ERR_INVALID_ARGUMENT. Other arguments
 * and status as kda_decode_step.
 */
KDA_API kda_status_t kda_decode_step_slots(const void *q, const void *k, const void *v,
                                           const float *log_alpha, const float *beta,
                                           float *state_pool, int64_t pool_slots,
                                           const int32_t *slot_dev, int32_t num_seqs, int32_t H,
                                           int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                                           void *out, void *workspace, size_t workspace_bytes,
                                           kda_stream_t stream);

/* Most draft tokens per sequence that kda_decode_verify / kda_decode_commit take. */
#define KDA_MAX_DRAFT_TOKENS 16

/*
 * Speculative (multi-token) decode, verify half. The draft model proposes T
 * tokens per sequence and the main model checks them all in one pass
 * ("Optimization for Inference: 4-Bit and Speculative Decoding" in the Kimi K3
 * article, EAGLE-3 with a multi-token-prediction draft layer). For each
 * (sequence, head) this reads the state once, runs the T tokens through the
 * recurrence, and leaves the state UNCHANGED; kda_decode_commit then advances
 * it by however many tokens were accepted. Row n*T + t holds draft token t of
 * sequence n:
 *
 *   q, k        [num_seqs*T, H, d_k]  dtype
 *   v           [num_seqs*T, H, d_v]  dtype
 *   log_alpha   [num_seqs*T, H, d_k]  fp32
 *   beta        [num_seqs*T, H]       fp32
 *   state       slot_dev == NULL: [num_seqs, H, d_k, d_v] fp32, sequence n's
 *               state is entry n; otherwise a pool [pool_slots, H, d_k, d_v]
 *               and sequence n's state is slot slot_dev[n] (-1: zeros). Only read.
 *   out         [num_seqs*T, H, d_v]  dtype (written): token t's output, as if
 *               tokens 0..t had been decoded one by one
 *   u_cache     [num_seqs*T, H, d_v]  fp32 (written): token t's correction
 *               u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t), the value
 *               written into the memory, so that
 *               S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T
 *               ("How the delta rule actually works" in the same article)
 *   workspace   required: >= 256 bytes, 256-byte aligned; its first word is
 *               the device status word (out-of-range slots, as
 *               kda_decode_step_slots)
 *
 * 1 <= T <= KDA_MAX_DRAFT_TOKENS. The outputs equal those of T calls of
 * kda_decode_step on a copy of the states, bit for bit. Status as
 * kda_decode_step_slots.
 */
KDA_API kda_status_t kda_decode_verify(const void *q, const void *k, const void *v,
                                       const float *log_alpha, const float *beta,
                                       const float *state, int64_t pool_slots,
                                       const int32_t *slot_dev, int32_t num_seqs, int32_t T,
                                       int32_t H, int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                                       void *out, float *u_cache, void *workspace,
                                       size_t workspace_bytes, kda_stream_t stream);

/*
 * Speculative decode, commit half: advances sequence n's state in place by its
 * first accepted_dev[n] draft tokens (0 <= accepted <= T; 0 leaves it as it
 * is), using the k, log_alpha and u_cache of the kda_decode_verify call that
 * checked them (same T, layouts, state / pool and slot_dev). Each state that
 * moves is read once and written once; the result equals accepted_dev[n] calls
 * of kda_decode_step, bit for bit. An accepted count outside [0, T] leaves the
 * sequence untouched and is recorded in the device status word, which
 * kda_read_device_status reports as KDA_ERR_INVALID_ARGUMENT; slot -1 stores
 * nothing; two sequences must not name the same slot. Workspace and status as
 * kda_decode_verify.
 */
KDA_API kda_status_t kda_decode_commit(const void *k, const float *log_alpha,
                                       const float *u_cache, float *state, int64_t pool_slots,
                                       const int32_t *slot_dev, const int32_t *accepted_dev,
                                       int32_t num_seqs, int32_t T, int32_t H, int32_t d_k,
                                       int32_t d_v, kda_dtype_t dtype, void *workspace,
                                       size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_decode_commit of the previous draft followed by kda_decode_verify of the
 * next one, in one pass over the states: each state is read once, advanced by
 * accepted_dev[n] tokens of the previous draft (prev_k, prev_log_alpha,
 * prev_u: rows n*T_prev + t, as that draft's verify call took and returned
 * them), stored if it moved, and the T new draft tokens are run from it. A
 * speculative decode loop thus moves each state through HBM once per step,
 * like a single kda_decode_step, however many tokens the step accepts. Results
 * (out, u_cache, states) equal those of the two calls bit for bit; u_cache and
 * out must not alias prev_k, prev_log_alpha or prev_u (use two buffers in turn).
 * 1 <= T_prev <= KDA_MAX_DRAFT_TOKENS; two sequences must not name the same
 * slot. Other arguments, workspace and status as the two calls.
 */
KDA_API kda_status_t kda_decode_commit_verify(const void *prev_k, const float *prev_log_alpha,
                                              const float *prev_u, const int32_t *accepted_dev,
                                              int32_t T_prev, const void *q, const void *k,
                                              const void *v, const float *log_alpha,
                                              const float *beta, float *state, int64_t pool_slots,
                                              const int32_t *slot_dev, int32_t num_seqs, int32_t T,
                                              int32_t H, int32_t d_k, int32_t d_v,
                                              kda_dtype_t dtype, void *out, float *u_cache,
                                              void *workspace, size_t workspace_bytes,
                                              kda_stream_t stream);

/*
 * Number of this library's kernels that the calling thread's last successful
 * prefill, decode or speculative-decode call enqueued (memsets and copies are
 * not counted): 2 for the chunked prefill (a planning or initialisation kernel
 * and the chunk kernel), 1 for the token-serial prefill, the decode step and
 * each speculative-decode call. 0 before any such call. Diagnostic only.
 */
KDA_API int32_t kda_last_launch_count(void);

/* Static string naming a status code. Never NULL. */
KDA_API const char *kda_status_string(kda_status_t status);

/* Message for the calling thread's last non-OK status ("" if none). The
 * pointer stays valid until the thread's next call into the library. */
KDA_API const char *kda_last_error(void);

/*
 * Reads the device status word that kda_prefill keeps at the start of its
 * workspace: KDA_OK; KDA_ERR_TIMEOUT if a bounded on-device wait of the last
 * prefill that used this workspace gave up (its outputs are then invalid); or
 * KDA_ERR_INVALID_ARGUMENT if the last kda_prefill_slots /
 * kda_decode_step_slots / kda_decode_verify / kda_decode_commit /
 * kda_decode_commit_verify that used it
 * met a slot outside [-1, pool_slots) or an accepted count outside [0, T].
 * Synchronises `stream` (this is the only call that does).
 */
KDA_API kda_status_t kda_read_device_status(const void *workspace, kda_stream_t stream);

/*
 * Diagnostic: launches a one-block kernel that waits on an on-device barrier
 * nothing will ever release, using the same bounded wait as the prefill
 * kernels, so callers can check that a stuck wait ends by itself: after
 * timeout_ns (in (0, 1e10]) the kernel records KDA_ERR_TIMEOUT in the status
 * word at the start of `workspace` (>= 256 bytes) and exits, leaving the
 * context usable; kda_read_device_status then reports KDA_ERR_TIMEOUT.
 */
KDA_API kda_status_t kda_selftest_bounded_wait(void *workspace, size_t workspace_bytes,
                                               uint64_t timeout_ns, kda_stream_t stream);

/*
 * Diagnostic: the same check for the other kind of wait in the prefill
 * kernels, a spin on a flag in global memory that another thread block
 * releases (the split-role kernel's hand-off between its thread blocks). One
 * thread waits, with that kernel's bounded flag wait, for a word at byte 128 of
 * `workspace` that this call zeroes and nothing then writes; after timeout_ns
 * (in (0, 1e10]) it records KDA_ERR_TIMEOUT in the status word at the start of
 * `workspace` (>= 256 bytes) and exits, leaving the context usable.
 */
KDA_API kda_status_t kda_selftest_flag_wait(void *workspace, size_t workspace_bytes,
                                            uint64_t timeout_ns, kda_stream_t stream);

/*
 * kda_prefill without a workspace argument, for callers that cannot allocate
 * device memory when they run a prefill (code inside an allocator or pool
 * callback, a serving loop whose memory is fixed at start-up). The pages
 * describe no counterpart; this is a library convenience.
 *
 * The scratch kda_prefill keeps in its workspace lives instead in a fixed
 * 64 KiB array in the library's device memory, held on every GPU that loads
 * the library until the process exits. That caps num_seqs at 16320; larger
 * values return KDA_ERR_INVALID_ARGUMENT. No device memory is allocated or
 * freed. The first call on a device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every call shares the one array and rewrites all of it that it uses, so
 * calls that overlap on the GPU (different streams, or different host threads)
 * race and must be serialised by the caller. The device status word is kept in
 * that array; kda_prefill_noalloc_status reads it. The looked-up address is
 * kept until the process exits: after cudaDeviceReset on a device, do not call
 * this entry point on that device again in the same process. Other arguments,
 * results and status codes are those of kda_prefill.
 */
KDA_API kda_status_t kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                         const float *log_alpha, const float *beta,
                                         const float *initial_state,
                                         const int32_t *cu_seqlens_dev,
                                         const int32_t *cu_seqlens_host,
                                         int32_t num_seqs, int64_t total_tokens, int32_t H,
                                         int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                                         void *out, float *final_state, kda_stream_t stream);

/*
 * Status word of the last kda_prefill_noalloc on the current device (the
 * device-side report that kda_read_device_status gives for a caller's
 * workspace): KDA_OK, KDA_ERR_TIMEOUT if a bounded on-device wait of that call
 * gave up (its outputs are then invalid), or KDA_ERR_CUDA if the scratch
 * array's address cannot be looked up. Synchronises `stream`; call it on the
 * stream of the kda_prefill_noalloc it checks. No counterpart in the pages.
 */
KDA_API kda_status_t kda_prefill_noalloc_status(kda_stream_t stream);

/* Library version: major * 10000 + minor * 100 + patch. */
KDA_API int32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
