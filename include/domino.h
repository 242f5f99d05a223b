/*
 * domino.h - C ABI of the Domino draft-block hot path for NVIDIA B200 (sm_100a).
 *
 * The library computes one speculative-decoding draft block per request, as the
 * Domino pages describe it:
 *   1. base logits   L_i^base = W_lm h_i for every block position i, once per block
 *      (Domino study notes, gsyq.cn, §二.1(1) 并行草稿主干; yhxrc.cn article, §三);
 *   2. a sequential correction over the block: a GRU causal encoder reads the
 *      embedding of each token already fixed, a rank-r head computes
 *      dL_i = W2 SiLU(W1 [h_i ; S_{i-1}]), L_i = L_i^base + dL_i, and a token is
 *      picked and fed back (study notes §二.1(2); yhxrc.cn §四);
 *   3. greedy verification against target tokens, giving the acceptance length
 *      tau (study notes §一.1; digest page "大三本科生一作…" §4).
 * Beside the block: the teacher-forced training forward with its base-anchored
 * curriculum loss (study notes §二.2), stochastic verification at T > 0, and a
 * precomputed token->gate table for the GRU's input side (see below).
 *
 * Conventions shared by every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller, except where an
 *     entry point says "host".  Row-major, dense, no padding.  Every tensor
 *     pointer must be 16-byte aligned.
 *   - bf16 tensors hold IEEE bfloat16 values; f32 tensors hold IEEE binary32.
 *     Base logits, final logits and GRU biases are always f32.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  All device
 *     work is enqueued on it asynchronously; no entry point synchronises except
 *     domino_poll, domino_draft_block_host and domino_selftest_wait_timeout.
 *   - The library never allocates device memory.  Scratch lives in a
 *     caller-provided workspace of at least domino_workspace_bytes() bytes that
 *     must be initialised once with domino_workspace_init().  One workspace may
 *     serve one call at a time; calls on distinct workspaces may overlap.
 *   - Argument errors are detected on the host before any launch and returned
 *     synchronously (nothing is enqueued).  Errors found on the device (a token
 *     outside [0, V), a wait that ran out of time) set bits in an error word in
 *     the workspace; domino_poll reports and clears them.  No C++ exception
 *     crosses this boundary.
 *   - Sizes: B >= 1, 1 <= K <= 32, every model dimension a positive multiple of
 *     8, rank <= 256 (bf16) or <= 128 (f32).
 */
#ifndef DOMINO_H_
#define DOMINO_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DOMINO_API __attribute__((visibility("default")))
#else
#define DOMINO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DOMINO_OK = 0,
  DOMINO_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment, mode or temperature      */
  DOMINO_ERR_UNSUPPORTED = 2,  /* valid request outside what this build implements      */
  DOMINO_ERR_LAUNCH = 3,       /* a kernel could not be launched (e.g. too few free SMs  */
                               /* for the co-resident correction grid)                   */
  DOMINO_ERR_CUDA = 4,         /* a CUDA runtime call failed                             */
  DOMINO_ERR_TIMEOUT = 5,      /* a bounded device wait ran out of time (device-side)    */
  DOMINO_ERR_BAD_TOKEN = 6,    /* an anchor, forced, label or drafted token was outside  */
                               /* [0, V); it was clamped and the work still ran          */
                               /* (device-side)                                          */
  DOMINO_ERR_WORKSPACE = 7     /* workspace missing, too small or misaligned             */
} domino_status;

typedef enum { DOMINO_BF16 = 0, DOMINO_F32 = 1 } domino_dtype;

/* Token pick.  GREEDY: t_i = argmax_j L_i[j], ties to the lowest index (the
 * pages' T=0 runs).  GUMBEL: t_i = argmax_j (L_i[j] / T + g_j) with
 * g_j = -log(-log u_j), u_j from Philox4x32-10 keyed by the 64-bit seed, counter
 * (j >> 2, i - 1, b, 0), word j & 3, u = (2 (w >> 9) + 1) 2^-24 - a draw from
 * softmax(L_i / T) (the pages report T=1 runs but state no mechanism). */
typedef enum { DOMINO_GREEDY = 0, DOMINO_GUMBEL = 1 } domino_mode;

/* Domino-head weights plus the frozen LM head and the embedding table.
 * All pointers are device pointers; the caller keeps them alive for the call. */
typedef struct {
  int32_t vocab;       /* V                                                        */
  int32_t d_model;     /* d: width of the backbone hidden states                   */
  int32_t embed_dim;   /* E: width of the token embedding fed to the GRU           */
  int32_t gru_hidden;  /* H: GRU state width (1024 in the pages)                   */
  int32_t rank;        /* r: correction bottleneck width (256 in the pages)        */
  int32_t dtype;       /* domino_dtype of every matrix below and of the hidden     */
                       /* states                                                   */
  const void* w_lm;    /* [V, d]   frozen target LM head                           */
  const void* embed;   /* [V, E]   token embedding table; may equal w_lm (tied)    */
  const void* w_ih;    /* [3H, E]  GRU input weights, gate blocks r, z, n          */
  const void* w_hh;    /* [3H, H]  GRU recurrent weights, gate blocks r, z, n      */
  const float* b_ih;   /* [3H] f32 GRU input bias, or NULL for zero                */
  const float* b_hh;   /* [3H] f32 GRU recurrent bias (b_hn sits inside r*(.)),    */
                       /* or NULL for zero                                         */
  const void* w1;      /* [r, d + H] bottleneck; columns [0, d) act on h_i,        */
                       /* columns [d, d + H) on the GRU state S_{i-1}               */
  const void* w2;      /* [V, r]   vocabulary projection of the correction         */
  const float* gate_table; /* [V, 3H] f32 token -> gate table G[t] = W_ih E[t] + b_ih  */
                       /* (domino_build_gate_table), or NULL.  When set, the       */
                       /* correction loop reads the fed token's row instead of     */
                       /* multiplying W_ih (domino_correct_loop_noalloc ignores    */
                       /* it).  Not from the pages: an inference-time              */
                       /* restructuring of the GRU's input side.                   */
} domino_weights;

/* Workspace bytes needed by domino_draft_block / domino_lm_head /
 * domino_correct_loop for batch B and block K (base logits included), or 0 if
 * the arguments are invalid. */
DOMINO_API size_t domino_workspace_bytes(const domino_weights* w, int32_t B, int32_t K);

/* Number of kernels one domino_draft_block call launches for batch B and block
 * K (the LM head, the correction loop's kernels with verification fused into
 * them; asynchronous memsets not counted), or -1 if the arguments are invalid.
 * Host-only: no CUDA call.  Batches of bf16 weights from 4 requests (and
 * 16-byte aligned E, H, d, r) take the per-step tensor-core loop; the rest take
 * the persistent loop, one launch per group of up to 8 requests. */
DOMINO_API int32_t domino_launches_per_block(const domino_weights* w, int32_t B, int32_t K);

/* Zero the workspace control block (error word, barrier and flag counters).
 * Call once after allocating a workspace; domino_poll re-initialises it after
 * reporting a device error. */
DOMINO_API domino_status domino_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* One draft block for B requests (stage 1 + stage 2 + stage 3).
 *   hidden      [B, K, d]  backbone hidden states h_i (dtype of w)
 *   anchor      [B] int32  last confirmed token x_t: the GRU's first input
 *   mode, temperature, seed: token pick (temperature > 0 needed for GUMBEL,
 *               ignored for GREEDY)
 *   forced      [B, K] int32 or NULL: teacher-forced GRU inputs; forced[b, i] is
 *               fed after position i instead of the pick (study notes §二.2(1));
 *               the last column is never fed.  draft_out still gets the picks.
 *   target      [B, K] int32 or NULL: target tokens for verification
 *   draft_out   [B, K] int32: picked tokens t_1..t_K
 *   logits_out  [B, K, V] f32 or NULL: final logits L_i (before T and noise)
 *   tau_out     [B] int32: acceptance length; required iff target != NULL
 * Launches: see domino_launches_per_block. */
DOMINO_API domino_status domino_draft_block(const domino_weights* w, const void* hidden, const int32_t* anchor,
                                 int32_t B, int32_t K, int32_t mode, float temperature, uint64_t seed,
                                 const int32_t* forced, const int32_t* target, int32_t* draft_out,
                                 float* logits_out, int32_t* tau_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* domino_draft_block that also records CUDA events on `stream` around its
 * stages: events[0] before stage 1, events[1] between stage 1 and stage 2,
 * events[2] after stage 2 (each a cudaEvent_t created by the caller; NULL
 * entries are skipped).  For timing the stages of one draft block in place. */
DOMINO_API domino_status domino_draft_block_events(const domino_weights* w, const void* hidden, const int32_t* anchor,
                                        int32_t B, int32_t K, int32_t mode, float temperature, uint64_t seed,
                                        const int32_t* forced, const int32_t* target, int32_t* draft_out,
                                        float* logits_out, int32_t* tau_out, void* workspace,
                                        size_t workspace_bytes, void* stream, void* const* events);

/* Stage 1 only: base_out[b, i, v] = sum_k W_lm[v, k] hidden[b, i, k]  ([B, K, V] f32).
 * bf16 runs on the tcgen05 tensor cores, f32 on CUDA cores (no tf32). */
DOMINO_API domino_status domino_lm_head(const domino_weights* w, const void* hidden, int32_t B, int32_t K,
                             float* base_out, void* workspace, size_t workspace_bytes, void* stream);

/* Stage 2 only, given base logits base[B, K, V] f32 (e.g. from domino_lm_head).
 * Arguments as for domino_draft_block; target / tau_out as there (may be NULL). */
DOMINO_API domino_status domino_correct_loop(const domino_weights* w, const void* hidden, const float* base,
                                  const int32_t* anchor, int32_t B, int32_t K, int32_t mode,
                                  float temperature, uint64_t seed, const int32_t* forced,
                                  const int32_t* target, int32_t* draft_out, float* logits_out,
                                  int32_t* tau_out, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Allocation-free variant of domino_correct_loop.  The pages have no
 * counterpart: this exists for callers that cannot provide device memory —
 * engines that reserve all device memory in their own arena and forbid other
 * allocations, plugins running inside them, and deployments that must not
 * allocate after start-up (cudaMalloc may synchronise the device and has no
 * latency bound).  It takes no workspace and allocates nothing: its scratch is
 * one fixed device array of 657,664 bytes inside the library, which every GPU
 * that loads the library keeps until the process exits.  Arguments are those
 * of domino_correct_loop without the workspace.
 *   - Limits of that array: B <= 8, K <= 32, rank <= 256, gru_hidden <= 4096;
 *     larger requests return DOMINO_ERR_UNSUPPORTED before any work.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - The call waits for its own work and returns what the device flagged
 *     (DOMINO_OK, DOMINO_ERR_TIMEOUT or DOMINO_ERR_BAD_TOKEN).
 *   - All calls share the array: calls whose work overlaps on one GPU (other
 *     streams or host threads) race; run them one after another. */
DOMINO_API domino_status domino_correct_loop_noalloc(const domino_weights* w, const void* hidden, const float* base,
                                          const int32_t* anchor, int32_t B, int32_t K, int32_t mode,
                                          float temperature, uint64_t seed, const int32_t* forced,
                                          const int32_t* target, int32_t* draft_out, float* logits_out,
                                          int32_t* tau_out, void* stream);

/* ---- Token -> gate table ----
 * G[t, :] = W_ih E[t, :] + b_ih for every token t (fp32, [V, 3H] row-major,
 * domino_gate_table_bytes(w) bytes), computed once per weight set: the GRU's
 * input-side pre-activation depends on the fed token only, so a loop given the
 * table (domino_weights.gate_table) gathers one 3H row per request per position
 * instead of streaming W_ih.  bf16 weights: one tcgen05 GEMM launch (fp32
 * accumulation, as in the loop) plus a bias launch; fp32: SIMT.  workspace:
 * at least 1024 bytes, 256-byte aligned, zeroed once (error word).  Asynchronous. */
DOMINO_API size_t domino_gate_table_bytes(const domino_weights* w);
DOMINO_API domino_status domino_build_gate_table(const domino_weights* w, float* table_out, void* workspace,
                                                 size_t workspace_bytes, void* stream);

/* ---- Training forward (Domino study notes, gsyq.cn, §二.2 配套专属训练方案) ----
 *
 * Base-anchored curriculum loss (§二.2(2)) on given logits:
 *   loss = (1 - lambda) L_final + lambda L_base,
 *   L_x  = sum_{b,i} gamma^i CE(x[b,i,:], labels[b,i]) / (B sum_i gamma^i),
 *   CE(l, y) = logsumexp(l) - l[y]   (no temperature),
 * i = 0..K-1 the block position minus one (exponentially decaying position
 * weights; the notes give no decay constant, gamma is the caller's).
 *   final_logits, base_logits [B, K, V] fp32 device, 16-byte aligned
 *   labels      [B, K] int32 ground-truth tokens; out-of-range values are
 *               clamped and flagged (DOMINO_ERR_BAD_TOKEN via domino_poll)
 *   lambda      in [0, 1] (the notes anneal it linearly from 1 to 0 over training)
 *   gamma       > 0 (1 = uniform weights)
 *   ce_out      [B, K, 2] fp32 or NULL: per-position (final, base) cross-entropy
 *   loss_out    [1] fp32 device
 *   workspace   domino_curriculum_loss_workspace_bytes(B, K, V) bytes, 256-byte
 *               aligned, zeroed once with domino_workspace_init.
 * Two launches (one CTA per row chunk, then one combining CTA); deterministic.
 * Argument errors (NULL, misaligned, lambda or gamma out of range, B K > 32767)
 * return synchronously. */
DOMINO_API size_t domino_curriculum_loss_workspace_bytes(int32_t B, int32_t K, int32_t V);
DOMINO_API domino_status domino_curriculum_loss(const float* final_logits, const float* base_logits,
                                                const int32_t* labels, int32_t B, int32_t K, int32_t V, float lambda,
                                                float gamma, float* ce_out, float* loss_out, void* workspace,
                                                size_t workspace_bytes, void* stream);

/* Teacher-forced training forward (§二.2(1) Teacher-Forced, §二.2(2)): one draft
 * block per request whose GRU reads the ground truth (labels[b, i] is the
 * target of position i+1 and the GRU input after it, i.e. domino_draft_block
 * with forced = labels), then the curriculum loss of its final and base logits
 * against the labels.  Arguments as for domino_draft_block and
 * domino_curriculum_loss; the final logits are written to the workspace, whose
 * size is domino_draft_loss_workspace_bytes(w, B, K). */
DOMINO_API size_t domino_draft_loss_workspace_bytes(const domino_weights* w, int32_t B, int32_t K);
DOMINO_API domino_status domino_draft_loss(const domino_weights* w, const void* hidden, const int32_t* anchor,
                                           const int32_t* labels, int32_t B, int32_t K, float lambda, float gamma,
                                           float* ce_out, float* loss_out, void* workspace,
                                           size_t workspace_bytes, void* stream);

/* ---- Stochastic verification at T > 0 ----
 * The pages report acceptance at T = 1 (study notes §三.2(1)) but give no
 * mechanism; this is standard lossless speculative sampling.  With
 * p_i = softmax(draft_logits[b, i, :] / T) (the final logits L_i the drafted
 * tokens were sampled from, e.g. domino_draft_block's logits_out in GUMBEL mode)
 * and q_i = softmax(target_logits[b, i, :] / T):
 *   for i = 1..K: accept draft[b, i-1] with probability min(1, q_i(t) / p_i(t));
 *   at the first rejection emit a token drawn from norm(max(0, q_i - p_i));
 *   after K acceptances emit a bonus token drawn from q_{K+1}.
 * A rejection whose residual max(0, q_i - p_i) has no positive fp32 entry
 * (p_i and q_i agree to working precision except at the drafted token, whose
 * probability lies below it) emits a token drawn from q_i instead.
 *   draft_logits  [B, K, V] fp32 device; target_logits [B, K+1, V] fp32 device
 *   draft         [B, K] int32: the drafted tokens (out of range: clamped, flagged)
 *   temperature   > 0; seed: Philox4x32-10 key (seed low, seed high); acceptance
 *                 uniforms use counter (0, i-1, b, 2) word 0, the resampling
 *                 Gumbel noise counter (j >> 2, i-1, b, 1) word j & 3 (streams
 *                 the draft's Gumbel picks never use)
 *   tau_out       [B] int32: accepted draft tokens (0..K)
 *   token_out     [B] int32: the emitted residual or bonus token
 *   workspace     domino_verify_sample_workspace_bytes(B, K, V) bytes, 256-byte
 *                 aligned, zeroed once with domino_workspace_init.
 * Four launches and one memset; asynchronous.  Argument errors (NULL,
 * misaligned, T <= 0, K outside 1..32, B (2K+1) > 65535) return synchronously. */
DOMINO_API size_t domino_verify_sample_workspace_bytes(int32_t B, int32_t K, int32_t V);
DOMINO_API domino_status domino_verify_sample(const float* draft_logits, const float* target_logits,
                                              const int32_t* draft, int32_t B, int32_t K, int32_t V,
                                              float temperature, uint64_t seed, int32_t* tau_out, int32_t* token_out,
                                              void* workspace, size_t workspace_bytes, void* stream);

/* Stage 3 only: tau_out[b] = number of leading i with draft[b, i] == target[b, i]. */
DOMINO_API domino_status domino_verify(const int32_t* draft, const int32_t* target, int32_t B, int32_t K,
                            int32_t* tau_out, void* stream);

/* End-to-end variant with HOST buffers: copies hidden / anchor / forced / target
 * from host memory (pinned memory makes the copies asynchronous), runs the
 * block, copies draft_out / tau_out back to host memory, and synchronises the
 * stream before returning.  Weights and workspace stay device pointers; device
 * staging for the copied tensors comes from the workspace, which must hold
 * domino_workspace_bytes_host() bytes.  logits are not returned. */
DOMINO_API size_t domino_workspace_bytes_host(const domino_weights* w, int32_t B, int32_t K);
DOMINO_API domino_status domino_draft_block_host(const domino_weights* w, const void* hidden_host,
                                      const int32_t* anchor_host, int32_t B, int32_t K, int32_t mode,
                                      float temperature, uint64_t seed, const int32_t* forced_host,
                                      const int32_t* target_host, int32_t* draft_out_host,
                                      int32_t* tau_out_host, void* workspace, size_t workspace_bytes,
                                      void* stream);

/* Synchronise `stream`, read and clear the workspace error word.  Returns
 * DOMINO_OK, DOMINO_ERR_TIMEOUT or DOMINO_ERR_BAD_TOKEN (timeout wins), or
 * DOMINO_ERR_CUDA if the stream itself failed. */
DOMINO_API domino_status domino_poll(void* workspace, void* stream);

/* Budget of every bounded device wait (grid barriers, pipeline waits), in
 * nanoseconds; process-wide, default 2e9.  A wait that exceeds it sets
 * DOMINO_ERR_TIMEOUT and the kernel returns early. */
DOMINO_API void domino_set_wait_budget_ns(uint64_t ns);

/* Self-test of the bounded grid barrier: launches the correction grid with one
 * barrier whose arrival count can never be reached, using `budget_ns` as the
 * wait budget; synchronises and returns what domino_poll returns (expected:
 * DOMINO_ERR_TIMEOUT).  The GPU stays usable afterwards. */
DOMINO_API domino_status domino_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t budget_ns,
                                           void* stream);

/* Human-readable name of a status code (static storage). */
DOMINO_API const char* domino_status_str(domino_status s);

#ifdef __cplusplus
}
#endif
#endif /* DOMINO_H_ */
