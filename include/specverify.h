/* libspecverify — draft-token verification for speculative decoding on B200 (sm_100a).
 *
 * The library verifies the drafts of one speculative-decoding round on the GPU:
 *   - chain speculative sampling (temperature / top-k / top-p, ratio test,
 *     residual resample, bonus token) and its temperature-0 greedy form;
 *   - MEDUSA typical acceptance over a candidate tree;
 *   - the probability transform and the residual draw as separate calls.
 *
 * Sources, by page and section (the pages carry prose; their formulas were lost
 * in extraction and are restated here in the standard form that prose describes):
 *   [SD] taking-lying-flat.github.io/blog/posts/spec-decoding-i/ —
 *        "Speculative Decoding" (accept, resample at the first rejection, bonus
 *        token), "Speculative Sampling" (acceptance probability min(1, p/q), residual
 *        norm(max(0, p - q)), transforms applied before the rejection scheme),
 *        "Key Components" (MEDUSA tree, typical acceptance).
 *   [SV] blog.csdn.net/yorkhunter/article/details/139214590 — "推测解码"
 *        (blockwise parallel decoding: greedy longest-prefix verification; MEDUSA
 *        typical acceptance, first token greedy, longest accepted prefix).
 *
 * Conventions for every call
 *   - Pointers named *_logits, *_tokens, uniforms, parent_idx, workspace and all
 *     outputs are DEVICE pointers, allocated and owned by the caller. The library
 *     allocates nothing and keeps no pointer after a call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *     default stream). Calls are asynchronous: they return before the GPU runs, and
 *     no call synchronises the host (except spec_get_device_status).
 *   - Logit tensors are row-major with the vocabulary contiguous, element type
 *     SPEC_F32 (float) or SPEC_BF16 (bfloat16 bit patterns). 1 <= V <= SPEC_MAX_VOCAB.
 *   - The return value reports argument and launch errors only, before or at launch;
 *     on error nothing has been enqueued (SPEC_ERR_CUDA: a launch may have failed
 *     part-way).
 *   - Data errors are reported in-band per batch row: accepted_len[b] = -1 and every
 *     other output of that row = -1. A row is in error when the verification reaches
 *     a logit row that holds NaN or +inf or is entirely -inf, or a token outside
 *     [0, V). Rows the rule never reaches (positions after the first rejection, tree
 *     nodes under a rejected parent) are not inspected.
 *   - accepted_len[b] = -2 marks a row whose device-side copy wait exceeded its time
 *     limit (about 2 s); spec_get_device_status then returns SPEC_ERR_DEVICE_TIMEOUT.
 *   - Results are deterministic: the same inputs give the same outputs, bit for bit.
 *   - Temperature: temp == 0 selects the greedy limit; temp must be finite and >= 0.
 *     top_k <= 0 or top_k >= V disables top-k; top_p >= 1 disables top-p; top_p must
 *     be > 0. Transforms are applied in the order temperature -> top-k -> softmax ->
 *     top-p -> renormalise, ties broken by the lower token id, the token whose mass
 *     crosses top_p kept.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPEC_OK = 0,
  SPEC_ERR_INVALID_ARG = -1,    /* NULL where required, bad size, bad dtype, bad knob */
  SPEC_ERR_UNSUPPORTED = -2,    /* valid but beyond this build's limits */
  SPEC_ERR_CUDA = -3,           /* a CUDA runtime call or launch failed */
  SPEC_ERR_WORKSPACE = -4,      /* workspace NULL, misaligned or too small */
  SPEC_ERR_DEVICE_TIMEOUT = -5  /* reported by spec_get_device_status only */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

#define SPEC_MAX_VOCAB (1 << 20)
#define SPEC_MAX_TREE_NODES 4096

/* Human-readable name of a status code (static string). */
const char* spec_status_string(int status);

/* Bytes of workspace that spec_verify_chain(B, K, V), spec_verify_tree_typical(B,
 * N = K_or_N, V), spec_verify_tree_greedy(B, N, V) and spec_verify_tree_sampling(B, N, V)
 * need; each call accepts any workspace at least this large. The
 * workspace must be 16-byte aligned. Returns 0 for invalid sizes. */
size_t spec_workspace_size(int B, int K_or_N, int V);

/* Chain verification of one round — [SD] "Speculative Decoding", "Speculative
 * Sampling"; greedy form [SV] "推测解码".
 *   target_logits [B][K+1][V]: target scores for draft positions 1..K and the bonus
 *                  position K+1 (row i = distribution p_i of token i given the prefix).
 *   draft_logits  [B][K][V]:   draft scores q_i (may be NULL iff temp == 0).
 *   draft_tokens  [B][K] int32: the drafted tokens x_i.
 *   uniforms      [B][K+1] float in [0,1): u[0..K-1] for the accept tests,
 *                  u[K] for the single resample-or-bonus draw.
 *   accepted_len  [B] int32 out: a in [0, K]; a + 1 tokens are emitted.
 *   out_tokens    [B][K+1] int32 out: x_0..x_{a-1}, then the drawn token, then -1.
 * With temp > 0: x_i is accepted iff u_i < min(1, p_i(x_i) / q_i(x_i)) (r = +inf when
 * q_i(x_i) = 0 < p_i(x_i), r = 0 when both are 0), scanning i = 0.. and stopping at
 * the first rejection, whose token is redrawn from norm(max(0, p_a - q_a)) (p_a when
 * that is empty); if all K are accepted the bonus token is drawn from p_K. A draw
 * returns the smallest token id v (ascending) with mass > 0 whose cumulative mass
 * exceeds u[K] times the total. With temp == 0: a is the length of the longest
 * prefix with x_i == argmax p_i (lowest id on ties) and the emitted token is
 * argmax p_a. K >= 1, B >= 1. */
spec_status spec_verify_chain(const void* target_logits, const void* draft_logits,
                              spec_dtype dtype, int B, int K, int V,
                              const int32_t* draft_tokens, const float* uniforms, float temp,
                              int top_k, float top_p, int32_t* accepted_len,
                              int32_t* out_tokens, void* workspace, size_t workspace_bytes,
                              void* stream);

/* MEDUSA typical acceptance over a candidate tree — [SD] "Key Components";
 * [SV] "推测解码".
 *   target_logits [B][N][V]: row n = the target's next-token scores after node n.
 *   node_tokens   [B][N] int32: token of each node; node 0 is the root (the greedy
 *                  first token, accepted unconditionally; its token is not read).
 *   parent_idx    [N] int32, shared by the batch: parent_idx[0] = -1 and
 *                  0 <= parent_idx[c] < c (parents precede children). A violation
 *                  puts every batch row in error.
 *   best_path     [B][path_cap] int32 out: node indices of the chosen path, root
 *                  first, -1 padded. A path longer than path_cap is a row error.
 *   accepted_len  [B] int32 out: nodes on the path, root included (>= 1).
 * Node c >= 1 is accepted iff its parent is and p(tok_c) > min(eps, delta *
 * exp(-H(p))), with p = softmax of the parent's row (temperature 1) and H its entropy
 * in nats; the deepest accepted node wins, the lowest node index on ties. Only the rows
 * of nodes that have a child are read (a leaf's row is never inspected).
 * 1 <= N <= SPEC_MAX_TREE_NODES, eps and delta finite. */
spec_status spec_verify_tree_typical(const void* target_logits, spec_dtype dtype, int B, int N,
                                     int V, const int32_t* node_tokens,
                                     const int32_t* parent_idx, float eps, float delta,
                                     int32_t* best_path, int path_cap, int32_t* accepted_len,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Greedy verification over a candidate tree: several candidate continuations checked
 * against the target at once, the longest correct one kept — [SV] "推测解码" (blockwise
 * parallel decoding accepts a draft token while it equals the target's argmax; Lookahead
 * decoding verifies candidate branches in parallel and keeps the longest correct prefix).
 * Branches that share a prefix share their nodes; independent branches all hang off node
 * 0. Layout, conventions and outputs as spec_verify_tree_typical, plus
 *   next_token    [B] int32 out or NULL: the argmax of the deepest accepted node's row,
 *                  the token the round emits after the path (-1 on an error row).
 * Node c >= 1 is accepted iff its parent is and node_tokens[b][c] is the argmax of the
 * parent's row (lowest id on ties); the deepest accepted node wins, the lowest node
 * index on ties. Only argmaxes are computed: the row stage reads each row once and does
 * no exp. The deepest accepted node's own row must be valid (it gives next_token).
 * 1 <= N <= SPEC_MAX_TREE_NODES. */
spec_status spec_verify_tree_greedy(const void* target_logits, spec_dtype dtype, int B, int N,
                                    int V, const int32_t* node_tokens, const int32_t* parent_idx,
                                    int32_t* best_path, int path_cap, int32_t* accepted_len,
                                    int32_t* next_token, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Rejection sampling over a candidate tree — [SD] "Key Components" (MEDUSA's step (3)
 * may reuse the rejection rule of speculative sampling, which keeps the target's output
 * distribution), with the rule of "Speculative Decoding" / "Speculative Sampling".
 *   target_logits [B][N][V]: row n = the target's scores after node n (p_n).
 *   draft_logits  [B][N][V]: row n = the drafter's scores after node n (q_n); the
 *                  children of n carry tokens drawn independently from q_n. NULL allowed
 *                  iff temp == 0.
 *   node_tokens, parent_idx, best_path, path_cap, accepted_len: as
 *                  spec_verify_tree_typical; next_token [B] out or NULL: the token emitted
 *                  after the path.
 *   uniforms      [B][N+1] float in [0,1): u[c] tests child c (u[0] unused), u[N] is the
 *                  final draw.
 * From the root, at the current node n the children are tried in index order: child c
 * is accepted iff u[c] < min(1, r(x_c)/q_n(x_c)), r the current residual (p_n at first);
 * a rejection replaces r by norm(max(0, r - q_n)) (unchanged if that is empty). An
 * accepted child becomes the current node; when none is accepted the emitted token is
 * drawn from r with u[N] (the inverse CDF of spec_verify_chain). temp, top_k, top_p
 * transform p and q as in spec_verify_chain; temp == 0 accepts the first child whose
 * token is the argmax of p_n and emits that argmax. The draws and tests read only the
 * rows on the walked path. 1 <= N <= SPEC_MAX_TREE_NODES. */
spec_status spec_verify_tree_sampling(const void* target_logits, const void* draft_logits,
                                      spec_dtype dtype, int B, int N, int V,
                                      const int32_t* node_tokens, const int32_t* parent_idx,
                                      const float* uniforms, float temp, int top_k, float top_p,
                                      int32_t* best_path, int path_cap, int32_t* accepted_len,
                                      int32_t* next_token, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* The sampling transform alone — [SD] "Speculative Sampling" (last bullet).
 *   logits [rows][V]; probs [rows][V] float out: the transformed distribution
 *   (temp == 0: one-hot at the argmax); entropy [rows] float out or NULL: its
 *   entropy in nats. Rows that hold NaN or +inf, or are entirely -inf, get NaN
 *   probabilities and entropy. rows >= 1. probs must not overlap logits or entropy: the
 *   call also uses the probs buffer as its scratch space (bfloat16 rows keep their row
 *   statistics there until the probabilities overwrite them), so its contents are defined
 *   only once the call's work on the stream has finished. */
spec_status spec_logits_to_probs(const void* logits, spec_dtype dtype, int rows, int V,
                                 float temp, int top_k, float top_p, float* probs,
                                 float* entropy, void* stream);

/* Residual draw alone — [SD] "Speculative Sampling".
 *   p, q [rows][V] float probability rows (q may be NULL: draw from p);
 *   uniforms [rows] float; tokens [rows] int32 out.
 * Draws from norm(max(0, p - q)) (from p when that is empty) with the same
 * inverse-CDF rule as spec_verify_chain. A row holding an entry that is NaN or
 * outside [0, 1], or whose p has no positive entry, gets token -1. rows >= 1. */
spec_status spec_residual_sample(const float* p, const float* q, int rows, int V,
                                 const float* uniforms, int32_t* tokens, void* stream);

/* Chain verification straight from the scoring forward's hidden states — [SD]
 * "Speculative Sampling" (the K drafts are scored in one forward whose cost lies in its
 * linear layers) and the chain rule of spec_verify_chain. The LM-head product
 * logits = hidden . weight^T runs on the tensor cores (bf16 x bf16, fp32 accumulation) and
 * its epilogue keeps only what the rule needs of each logit row, the top-k entries (the
 * argmax at temperature 0), so no logit row is written to memory.
 *   target_hidden [B][K+1][d], draft_hidden [B][K][d] (NULL iff temp == 0): bf16, row-major.
 *   target_weight, draft_weight [V][d] bf16 (row v = token v's output embedding; the draft
 *                  weight may be NULL iff temp == 0).
 *   draft_tokens, uniforms, accepted_len, out_tokens: as spec_verify_chain.
 *   temp == 0: greedy (draft rows unused); temp > 0 needs 1 <= top_k <= 64, top_k < V
 *   (top-k sampling; other transforms return SPEC_ERR_UNSUPPORTED). The decisions are those of
 *   spec_verify_chain applied to the fp32 logits this product computes.
 *   logits_out: NULL, or float [B*(K+1) + B*K][V] (target rows, then draft rows) that also
 *   receives those logits, for checking.
 *   d a multiple of 64; hidden, weight and workspace 16-byte aligned; workspace at least
 *   spec_lmhead_workspace_size(B, K, V, d, top_k) bytes (top_k = 0 for greedy). */
size_t spec_lmhead_workspace_size(int B, int K, int V, int d, int top_k);
spec_status spec_verify_chain_lmhead(const void* target_hidden, const void* draft_hidden,
                                     const void* target_weight, const void* draft_weight, int B,
                                     int K, int V, int d, const int32_t* draft_tokens,
                                     const float* uniforms, float temp, int top_k,
                                     int32_t* accepted_len, int32_t* out_tokens,
                                     float* logits_out, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Linear-attention state commit after verification — [SpecLA] gist.science summary of
 * "SpecLA: Efficient Speculative Decoding for Linear-Attention Models" (a linear-attention
 * target keeps one dense state per head; after the verdict the state is brought to the
 * accepted prefix from compact per-step factors saved during verification, with no replay).
 * The state of sequence b, head h is S in R^{dk x dv} (row-major, float32) and follows the
 * gated delta rule S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T over the
 * S steps of one round (e.g. the previous round's emitted token, whose update was
 * deferred, then the K drafts).
 *
 * spec_linear_state_factors: the factors of every prefix, from the round's per-step data.
 *   alpha, beta [B][H][S], keys [B][H][S][dk], values [B][H][S][dv] (float32, device);
 *   w [B][H][S][dk], u [B][H][S][dv], gamma [B][H][S] out (device, caller-allocated):
 *   gamma_t = alpha_1 .. alpha_t, w_t = beta_t (k_t - sum_{s<t} (k_t . k_s) w_s),
 *   u_t = beta_t (v_t / gamma_t - sum_{s<t} (k_t . k_s) u_s). 1 <= S <= 32, dk <= 256. The
 *   values are divided by the cumulative gate, so gates far below 1 over many steps lose
 *   float32 precision.
 * spec_commit_linear_state: state [B][H][dk][dv] (device; it, keys, w and u 16-byte aligned,
 *   else SPEC_ERR_UNSUPPORTED) is replaced, in
 *   place, by the state after steps[b] steps (int32 [B], device):
 *   S_a = gamma_a (S_0 + sum_{t<=a} k_t (u_t - S_0^T w_t)^T). A sequence with steps[b] = 0,
 *   or outside [0, S], is left untouched (not read or written). dk in {32, 64, 128, 256},
 *   dv a multiple of 4, S <= 32. One read and one write of each committed state. */
spec_status spec_linear_state_factors(const float* alpha, const float* beta, const float* keys,
                                      const float* values, int B, int H, int S, int dk, int dv,
                                      float* w, float* u, float* gamma, void* stream);
spec_status spec_commit_linear_state(float* state, int B, int H, int dk, int dv, int S,
                                     const float* keys, const float* w, const float* u,
                                     const float* gamma, const int32_t* steps, void* stream);

/* spec_verify_chain without a caller workspace. The pages have no counterpart: they
 * state the verification rule, not an interface; this call is the library's own.
 *
 * For callers that cannot allocate device memory around the call: code recording a
 * stream capture it does not own, plain C hosts with no device allocator, decode loops
 * whose memory pool is fixed at start-up. Arguments, semantics and outputs are those of
 * spec_verify_chain minus workspace / workspace_bytes. The scratch is one device array of
 * SPEC_STATIC_SCRATCH_BYTES inside the library, one per device; the call allocates
 * nothing and looks the array's address up once per device (with that device current).
 *   - A call whose spec_workspace_size(B, K, V) exceeds SPEC_STATIC_SCRATCH_BYTES returns
 *     SPEC_ERR_WORKSPACE before any CUDA call (32 MiB holds about 4,000 logit rows,
 *     B * (2K + 1)).
 *   - Every call on a device uses the same scratch: calls that overlap in time (on
 *     different streams, or from host threads without ordering) race on it and give
 *     undefined results. Order them (one stream, or events).
 *   - Make the first call on each device outside any stream capture: it resolves the
 *     array's address, which may load the library's device code.
 *   - The scratch is the current device's: make the device that holds the tensors current
 *     before the call. target_logits that is not device (or managed) memory of the current
 *     device gets SPEC_ERR_INVALID_ARG before any launch.
 *   - spec_get_device_status cannot see this scratch: a row whose copy wait timed out
 *     shows as accepted_len[b] = -2. */
#define SPEC_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
spec_status spec_verify_chain_noalloc(const void* target_logits, const void* draft_logits,
                                      spec_dtype dtype, int B, int K, int V,
                                      const int32_t* draft_tokens, const float* uniforms,
                                      float temp, int top_k, float top_p,
                                      int32_t* accepted_len, int32_t* out_tokens,
                                      void* stream);

/* Copies the device status word of `workspace` to the host (synchronises `stream`):
 * SPEC_OK, or SPEC_ERR_DEVICE_TIMEOUT if a kernel of an earlier call on this
 * workspace gave up waiting for a copy (or, for spec_verify_chain_lmhead, for a tensor-core
 * stage). The word is cleared by every verify call. It works on the workspaces of
 * spec_verify_chain, spec_verify_tree_typical, spec_verify_tree_sampling and
 * spec_verify_chain_lmhead alike (the word is the first 4 bytes of each). */
spec_status spec_get_device_status(const void* workspace, int32_t* status_out, void* stream);

/* Timing hook for measurement tools: while set, every spec_verify_chain and
 * spec_verify_tree_typical call records `before` (a cudaEvent_t) on its stream just
 * before its row-statistics kernel and `after` just after it. NULL, NULL clears. */
void spec_set_row_kernel_events(void* before, void* after);

/* Largest number of kernels one call enqueues (for launch accounting): the row
 * statistics kernel, the exact finisher for rows it lists (chain calls with top-k or
 * top-p only), the double-precision placement of top-p boundaries (top-p without top-k),
 * the per-batch-row kernel, and for typical acceptance the kernel that lists the rows of
 * nodes with a child. -1 for an unknown name. */
int spec_kernels_per_call(const char* entry_point);

#ifdef __cplusplus
}
#endif

#endif /* SPECVERIFY_H */
