/*
 * s3r.h - C ABI of libs3r: one S3R decode step on NVIDIA B200 (sm_100a).
 *
 * S3R ("S3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative
 * Decoding", weekinpapers.com, Abstract) drafts tokens with sparse attention
 * over the KV cache, then verifies them with full attention over the complete
 * history and commits them by exact speculative sampling, with drafter and
 * verifier sharing the same parameters and the same KV cache. This library
 * implements the attention and sampling steps of one such round over a paged
 * GQA KV cache:
 *
 *   s3r_page_summaries     per-page key min/max (Quest page metadata)
 *   s3r_sparse_draft_attn  score pages, keep the top-B per KV head, attend
 *   s3r_verify_attn        dense causal attention of the gamma+1 verify rows
 *   s3r_spec_sample        accept/reject, residual or bonus draw
 *   s3r_sample_tokens      the drafter's own draw x ~ softmax(logits / T)
 *   s3r_kv_append          a round's keys and values into the paged cache
 *   s3r_kv_rollback        back to the committed prefix after sampling
 *   s3r_verify_attn_tree   verification of a token tree (ancestor masks)
 *   s3r_tree_spec_sample   exact speculative sampling walked over the tree
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument is a caller-owned DEVICE pointer unless stated
 *   otherwise. The library allocates and frees nothing and keeps no data
 *   between calls; scratch space comes from the caller's workspace (the one
 *   exception, s3r_spec_sample_noalloc, uses a static array of its own). Host
 *   side it remembers only launch choices: the TMA driver entry point, and
 *   the cluster size s3r_tree_spec_sample picked per device and problem size.
 * - A workspace must be zero-filled before its first use. Calls leave it
 *   ready for the next call (its counters return to zero as each call ends),
 *   so no call clears it and consecutive kernels of the library overlap
 *   their launch with the previous kernel's tail (programmatic dependent
 *   launch). After a call that reported S3R_DEV_WAIT_TIMEOUT, zero the
 *   workspace again before reusing it.
 * - A call may read its inputs (queries, KV cache, page summaries, block
 *   table, context lengths, logits) while the previous kernel on the stream
 *   is still finishing, when that kernel is one of this library's attention
 *   or sampling kernels (none of them writes another call's inputs;
 *   s3r_page_summaries, s3r_kv_append and s3r_kv_rollback, which do, let the
 *   next kernel start only when they are done). A kernel of the caller's
 *   that writes an input must not signal programmatic launch completion
 *   before that write.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream). Work is enqueued asynchronously on it; outputs are ready when the
 *   stream reaches that point.
 * - Argument errors are detected on the host and returned synchronously
 *   before anything is enqueued. A failed launch returns S3R_ERR_CUDA.
 * - Data the host cannot see (context lengths, page ids, draft token ids) is
 *   checked on the device: a bad value is skipped, never dereferenced, and
 *   recorded in the workspace's status word; s3r_device_status() reports it.
 *   A kernel wait that exceeds its time limit (about one second) is recorded
 *   the same way and the kernel returns instead of hanging.
 * - Shapes: S sequences, Hq query heads, Hkv KV heads, G = Hq / Hkv, head dim
 *   D, page size P, context length L_b of sequence b, n_b = ceil(L_b / P)
 *   pages, R = gamma + 1 verify rows.
 * - Supported: D in {64, 128}; P in {16, 64}; dtype f32 or bf16 (KV cache,
 *   queries and attention outputs share it); G <= 8; G * rows <= 128;
 *   1 <= gamma <= 16; max_pages_per_seq <= 8192.
 * - No exception crosses this ABI.
 */
#ifndef S3R_H_
#define S3R_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S3R_OK = 0,
  S3R_ERR_INVALID_ARG = 1,   /* null pointer, bad size or inconsistent shape   */
  S3R_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes/dtypes  */
  S3R_ERR_WORKSPACE = 3,     /* workspace null or smaller than required        */
  S3R_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
  S3R_ERR_DEVICE_CHECK = 5   /* a device-side check failed (s3r_device_status) */
} s3r_status;

typedef enum { S3R_F32 = 0, S3R_BF16 = 1 } s3r_dtype;

/* Bits of the device status word (s3r_device_status). */
#define S3R_DEV_BAD_CONTEXT_LEN  0x1u  /* L_b < 1, L_b > max_pages*P, or L_b < rows (verify) */
#define S3R_DEV_BAD_PAGE_ID      0x2u  /* block-table entry outside [0, num_pages_total)    */
#define S3R_DEV_BAD_TOKEN_ID     0x4u  /* draft token outside [0, vocab)                    */
#define S3R_DEV_WAIT_TIMEOUT     0x8u  /* an in-kernel wait ran past its limit              */
#define S3R_DEV_BAD_TREE         0x10u /* a tree parent entry outside [0, node) (root: -1)  */

/*
 * A paged KV cache (PagedAttention's block tables, cited on the mlsanity.com
 * page's reference list).
 * k_cache, v_cache: [num_pages_total, Hkv, P, D] row-major in `dtype`; the
 *   (page, head) tile of P*D values is contiguous. Base addresses must be
 *   16-byte aligned.
 * block_table: int32 [num_seqs, max_pages_per_seq]; entry i of row b is the
 *   physical page holding tokens i*P .. i*P+P-1 of sequence b. Entries past
 *   n_b are never read.
 * context_lens: int32 [num_seqs], L_b >= 1. Cache slots of positions >= L_b
 *   in a sequence's last page may hold anything (they are never used).
 */
typedef struct {
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t max_pages_per_seq;
  int32_t num_pages_total;
  s3r_dtype dtype;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* context_lens;
} s3r_paged_kv;

/*
 * Per-page key summaries (Quest: query-aware page sparsity, cited on the
 * mlsanity.com page's reference list; S3R page, Abstract, "uses sparse
 * attention to propose tokens").
 *   kmin[p, h, d] = min over the valid tokens t of page p of K[p, h, t, d];
 *   kmax likewise. Valid tokens of page i of sequence b: t < L_b - i*P.
 * kmin, kmax: [num_pages_total, Hkv, D] in kv->dtype (min and max are exact).
 * tail_only = 0 recomputes every page used by a sequence; tail_only = 1
 * recomputes only each sequence's last page (the one a decode step appends
 * to) and leaves every other entry untouched. Pages no sequence uses are never
 * written.
 */
s3r_status s3r_page_summaries(const s3r_paged_kv* kv, int32_t tail_only,
                              void* kmin, void* kmax, void* stream);

/*
 * Sparse draft attention (S3R page, Abstract: "uses sparse attention to
 * propose tokens"; page choice after Quest).
 * For each sequence b and KV head h:
 *   score(p) = sum over the G query heads g of group h, sum over d, of
 *              max(q[b,g,d] * kmin[p,h,d], q[b,g,d] * kmax[p,h,d])
 *   (accumulated in float64, unscaled) for every page p < n_b; keep the
 *   budget_pages highest scores, ties to the lower page index (all pages if
 *   n_b <= budget_pages); then for every query head of the group
 *   out = softmax(q k^T * scale) v over the valid tokens of the kept pages,
 *   the query sitting at position L_b - 1.
 * q: [S, Hq, D] in kv->dtype. out: [S, Hq, D] in kv->dtype.
 * lse: float32 [S, Hq] natural-log log-sum-exp of the scaled scores, or NULL.
 * selected: int32 [S, Hkv, budget_pages], the kept logical page indices in
 *   ascending order, -1 after the first min(n_b, budget_pages) entries.
 * kmin, kmax: as written by s3r_page_summaries, for pages p < n_b - 1. The
 *   tail page n_b - 1 is the only one whose keys change as a sequence
 *   decodes; the call summarises it from k_cache itself (min / max over its
 *   valid tokens), so no summary refresh is needed between draft steps and
 *   kmin/kmax are only read. kmin, kmax, q and out must be 16-byte aligned
 *   (S3R_ERR_INVALID_ARG otherwise): the summary rows are bulk-copied.
 * workspace: at least s3r_attn_workspace_bytes(kv, 1, budget_pages) bytes;
 * it also carries the physical ids of the selected pages from the selection
 * kernel to the attention kernel.
 */
s3r_status s3r_sparse_draft_attn(const s3r_paged_kv* kv, const void* kmin, const void* kmax,
                                 const void* q, int32_t budget_pages, float scale,
                                 int32_t* selected, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dense verification attention (S3R page, Abstract: "full-attention
 * verification"; "dense verification still requires the complete historical
 * KV cache").
 * Row r (0 <= r < rows) of sequence b sits at position L_b - rows + r and
 * attends causally to every key at position <= its own:
 *   out[b,r,hq] = softmax(q[b,r,hq] k^T * scale) v, keys of KV head hq / G.
 * q, out: [S, rows, Hq, D] in kv->dtype; lse: float32 [S, rows, Hq] or NULL.
 * Requires L_b >= rows (checked on the device).
 * workspace: at least s3r_attn_workspace_bytes(kv, rows, 0) bytes.
 */
s3r_status s3r_verify_attn(const s3r_paged_kv* kv, const void* q, int32_t rows, float scale,
                           void* out, float* lse,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Tree verification attention (the ai.info SpecRoll page: sparse-tree
 * verification of candidate continuations, exact target verification at every
 * visited node). The round's R = `nodes` tree nodes of sequence b occupy
 * positions L_b - R .. L_b - 1 in node order; node i sees every key before
 * L_b - R and the slots of its ancestors and itself:
 *   visible(i, L_b - R + j) = j is i or an ancestor of i.
 * A chain (parents[b, i] = i - 1) gives s3r_verify_attn with rows = R.
 * parents: int32 [S, R], parents[b, 0] = -1, 0 <= parents[b, i] < i; an
 *   entry breaking that rule is flagged (S3R_DEV_BAD_TREE) and the node's
 *   ancestor walk ends there.
 * q, out: [S, R, Hq, D] in kv->dtype; lse: float32 [S, R, Hq] or NULL.
 * Supported: R <= 64, G * R <= 64 (bf16) or <= 128 (f32).
 * workspace: at least s3r_attn_workspace_bytes(kv, R, 0) bytes.
 */
s3r_status s3r_verify_attn_tree(const s3r_paged_kv* kv, const void* q, int32_t nodes,
                                const int32_t* parents, float scale, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Exact speculative sampling over a token tree (the ai.info SpecRoll page:
 * exact rejection sampling and the target-residual fallback at every visited
 * node keep the committed tokens on the target distribution).
 *   p_v = softmax(target_logits[b,v] / T); q_v = softmax(draft_logits[b,v] / T),
 *   the distribution the children of node v were drawn from.
 *   From the root v = 0: the children c of v (ascending index) are tested in
 *   turn, accept c iff u_accept[b,c] < p'(x_c) / q_v(x_c) (q_v(x_c) = 0
 *   rejects), x_c = tokens[b,c]; p' = p_v at first and after each rejection
 *   p' <- max(p' - q_v, 0) normalised (p' renormalised where that is zero
 *   everywhere). An accepted child commits its token and becomes v. When no
 *   child is accepted, or v is a leaf, the token drawn from p' with
 *   u_sample[b,v] (the inverse-CDF rule of s3r_spec_sample) is committed.
 * target_logits, draft_logits: [S, R, V] in logit_dtype (draft rows of leaves
 *   are not read). tokens, parents: int32 [S, R] (tokens[b,0] unused; parents
 *   as for s3r_verify_attn_tree; a tree breaking the rule is flagged and the
 *   walk draws at the root). u_accept, u_sample: float32 [S, R] in [0, 1).
 * out_tokens: int32 [S, R], the n_acc accepted tokens, the drawn token, then
 *   -1. num_accepted: int32 [S]. path: int32 [S, R] or NULL, the accepted
 *   nodes in order, then -1 (which cache rows to keep).
 * Sums and decisions in float64. Supported: R <= 64.
 * workspace: at least s3r_tree_sample_workspace_bytes(S, R, V) bytes (the
 *   status word).
 */
size_t s3r_tree_sample_workspace_bytes(int32_t num_seqs, int32_t nodes, int32_t vocab);
s3r_status s3r_tree_spec_sample(const void* target_logits, const void* draft_logits,
                                s3r_dtype logit_dtype, const int32_t* tokens, const int32_t* parents,
                                const float* u_accept, const float* u_sample,
                                int32_t num_seqs, int32_t nodes, int32_t vocab, float temperature,
                                int32_t* out_tokens, int32_t* num_accepted, int32_t* path,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Concurrency-aware node budget of the ai.info SpecRoll page (host):
 *   N_t = clip(floor(capacity / active), n_min, n_max)
 * with `active` the unfinished responses B_t and `capacity` the profiled
 * verification capacity C_hw in tree nodes. Returns -1 for active < 1,
 * n_min < 1, n_max < n_min or capacity < 0.
 */
int32_t s3r_tree_node_budget(int64_t capacity, int32_t active, int32_t n_min, int32_t n_max);

/*
 * Exact speculative sampling of one round (S3R page, Abstract: "exact
 * speculative sampling", the committed responses "follow the dense-policy
 * distribution"; rule of the speculative-sampling papers on the mlsanity.com
 * reference list, restated on the ai.info SpecRoll page).
 *   p_i = softmax(target_logits[b,i] / T), i = 0..gamma
 *   q_i = softmax(draft_logits[b,i] / T),  i = 0..gamma-1
 *   for i = 0..gamma-1: accept x_i = draft_tokens[b,i] iff
 *       u_accept[b,i] < p_i(x_i) / q_i(x_i)          (q_i(x_i) = 0 rejects)
 *   at the first rejection j: draw from max(p_j - q_j, 0) normalised (from
 *   p_j if that is all zero); if all gamma are accepted: draw from p_gamma.
 *   A draw from weights w with uniform u is the smallest k whose running sum
 *   C(k) exceeds u * C(V-1) (the last positive-weight index if rounding
 *   leaves none); it uses u_sample[b, j].
 * target_logits: [S, gamma+1, V]; draft_logits: [S, gamma, V]; both in
 *   logit_dtype. draft_tokens: int32 [S, gamma]. u_accept: float32 [S, gamma];
 *   u_sample: float32 [S, gamma+1]; uniforms in [0, 1).
 * out_tokens: int32 [S, gamma+1], the n_acc accepted drafts, the drawn token,
 *   then -1. num_accepted: int32 [S] = n_acc.
 * Row statistics accumulate in float64; decisions are taken in float64.
 * workspace: at least s3r_sample_workspace_bytes(S, gamma, V) bytes.
 */
s3r_status s3r_spec_sample(const void* target_logits, const void* draft_logits,
                           s3r_dtype logit_dtype, const int32_t* draft_tokens,
                           const float* u_accept, const float* u_sample,
                           int32_t num_seqs, int32_t gamma, int32_t vocab, float temperature,
                           int32_t* out_tokens, int32_t* num_accepted,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * The drafter's own sampling step: tokens[r] = inverse-CDF draw from
 * softmax(logits[r] / T) with uniform u[r] (same draw rule as above). In a
 * round it draws each x_i ~ q_i from the draft logits.
 * logits: [num_rows, V] in logit_dtype; u: float32 [num_rows];
 * tokens: int32 [num_rows].
 * workspace: at least s3r_sample_workspace_bytes(num_rows, 0, V) bytes.
 */
s3r_status s3r_sample_tokens(const void* logits, s3r_dtype logit_dtype, int32_t num_rows,
                             int32_t vocab, float temperature, const float* u,
                             int32_t* tokens, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * As s3r_sample_tokens, also writing each row's statistics at temperature T:
 *   row_stats[r] = { M_r, Z_r },  float64 [num_rows, 2],
 *   M_r = the row's largest logit (-inf for a row of -inf only),
 *   Z_r = sum over k of exp((logits[r, k] - M_r) / T), accumulated in float64
 *         from float64 exponentials (the normaliser of q_r = softmax(logits / T)).
 * row_stats may be NULL (then this is s3r_sample_tokens). It must be 8-byte
 * aligned. The draw of the round's draft tokens visits every draft logit
 * once; handing these statistics to s3r_spec_sample_ex spares it a second
 * pass over the draft rows.
 */
s3r_status s3r_sample_tokens_ex(const void* logits, s3r_dtype logit_dtype, int32_t num_rows,
                                int32_t vocab, float temperature, const float* u,
                                int32_t* tokens, double* row_stats, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * As s3r_spec_sample, with the draft rows' statistics given: draft_stats,
 * float64 [S, gamma, 2], row (b, i) = { M, Z } of draft_logits[b, i] at the
 * same temperature, as s3r_sample_tokens_ex writes them (NULL: computed here,
 * which is s3r_spec_sample). With them the call reads the gamma + 1 target
 * rows for their statistics and, after a rejection at j, only target row j
 * for its exact normaliser; the draft rows are read at the drafted token and,
 * after a rejection, draft row j for the residual draw. Results are those of
 * s3r_spec_sample up to the float64 rounding of the normalisers.
 */
s3r_status s3r_spec_sample_ex(const void* target_logits, const void* draft_logits,
                              s3r_dtype logit_dtype, const int32_t* draft_tokens,
                              const float* u_accept, const float* u_sample,
                              const double* draft_stats, int32_t num_seqs, int32_t gamma,
                              int32_t vocab, float temperature, int32_t* out_tokens,
                              int32_t* num_accepted, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * s3r_spec_sample without a workspace argument, for callers that cannot
 * allocate device memory themselves (a plug-in inside a host framework whose
 * device memory belongs to the framework's pooling allocator, code that must
 * not allocate while a stream is being captured, and the like). This entry
 * point has no counterpart on the S3R pages: it only changes where the
 * scratch memory comes from. Same arguments and results as s3r_spec_sample.
 * - Scratch: a 4 MiB device array owned by the library (a file-scope
 *   __device__ variable), held on every GPU that loads the library until the
 *   process exits. Shapes whose scratch need exceeds it
 *   (s3r_sample_workspace_bytes(num_seqs, gamma, vocab) > 4 MiB) return
 *   S3R_ERR_UNSUPPORTED before anything is enqueued.
 * - The first call on a device looks up the array's device address for that
 *   device (with the device current) and keeps it for the device's current
 *   CUDA context; make that first call before any stream capture. A call made
 *   in another context (after cudaDeviceReset, say) looks the address up
 *   again, so make its first call before any capture as well.
 * - The function allocates nothing (no cudaMalloc, cudaFree or allocating
 *   library routine); it clears the part of the array that must start at
 *   zero with cudaMemsetAsync on `stream`.
 * - Every call shares the one array and leaves its contents behind: calls
 *   that can overlap on the GPU (other streams, other host threads) race and
 *   must be serialised by the caller. Device-check results land in the
 *   shared array and cannot be read back; use s3r_spec_sample to get them.
 */
s3r_status s3r_spec_sample_noalloc(const void* target_logits, const void* draft_logits,
                                   s3r_dtype logit_dtype, const int32_t* draft_tokens,
                                   const float* u_accept, const float* u_sample,
                                   int32_t num_seqs, int32_t gamma, int32_t vocab, float temperature,
                                   int32_t* out_tokens, int32_t* num_accepted, void* stream);

/*
 * KV-cache upkeep of a round (S3R page, Abstract: the drafter and the
 * verifier share the policy's parameters and its KV cache; speculative
 * sampling commits the accepted drafts and one drawn token, so the later
 * positions leave the cache). A round over a cache of committed length C:
 *   draft step i (i < gamma): s3r_kv_append(n = 1, overwrite = 0) writes the
 *     step's key and value at position C + i, then s3r_sparse_draft_attn
 *     attends from that position;
 *   verification: s3r_kv_append(n = gamma + 1, overwrite = gamma) writes the
 *     verifier's keys and values over positions C .. C + gamma (the drafter's
 *     rows and one more), then s3r_verify_attn (rows = gamma + 1);
 *   commit: s3r_spec_sample, then s3r_kv_rollback(rows = gamma + 1) keeps
 *     positions up to C + n_acc.
 * Both calls write the KV cache and the summaries (kv->k_cache, kv->v_cache
 * are written although the struct holds them as const) and update the
 * lengths in place: context_lens must be kv->context_lens (else
 * S3R_ERR_INVALID_ARG). They order themselves after the previous kernel on
 * the stream and let the next one start only when they are done, so the next
 * call reads what they wrote.
 *
 * s3r_kv_append: for each sequence b with length L_b, the n rows
 * k_new[b, t], v_new[b, t] go to positions L_b - overwrite + t (t < n), the
 * length becomes L_b - overwrite + n, and kmin / kmax of every page holding a
 * written position are recomputed over that page's valid tokens under the new
 * length (the definition of s3r_page_summaries). k_new, v_new: [S, n, Hkv, D]
 * in kv->dtype, 16-byte aligned. 0 <= n, overwrite <= 1024; n = 0 with
 * overwrite = 0 does nothing. Device checks: a sequence with
 * overwrite > L_b or a new length outside [1, max_pages_per_seq * P] is left
 * unchanged (S3R_DEV_BAD_CONTEXT_LEN); a row whose page id is out of range is
 * not written (S3R_DEV_BAD_PAGE_ID). The block-table entries of the new
 * positions must be set by the caller beforehand (the library allocates no
 * pages).
 *
 * s3r_kv_rollback: after a round of R = rows positions ending the cache,
 * with num_accepted[b] = n_acc from s3r_spec_sample: L_b becomes
 * L_b - rows + n_acc + 1, and the summary of the page holding the new last
 * position is recomputed over its valid tokens. n_acc outside [0, rows - 1],
 * or a length that would drop below 1, leaves the sequence unchanged
 * (S3R_DEV_BAD_CONTEXT_LEN). Positions past the new length keep their old
 * rows (never read again); their pages stay in the block table.
 *
 * workspace: at least s3r_kv_workspace_bytes(num_seqs) bytes, zero-filled
 * before first use (status word and per-sequence counters, which every call
 * leaves at zero); s3r_device_status() reads its status word.
 */
s3r_status s3r_kv_append(const s3r_paged_kv* kv, int32_t* context_lens, const void* k_new,
                         const void* v_new, int32_t n, int32_t overwrite, void* kmin, void* kmax,
                         void* workspace, size_t workspace_bytes, void* stream);
s3r_status s3r_kv_rollback(const s3r_paged_kv* kv, int32_t* context_lens,
                           const int32_t* num_accepted, int32_t rows, void* kmin, void* kmax,
                           void* workspace, size_t workspace_bytes, void* stream);
size_t s3r_kv_workspace_bytes(int32_t num_seqs);

/*
 * Draft-length policy (host only; every pointer here is a host pointer): the
 * acceptance-aware draft length with a regime toggle that the researchpod.app
 * page describes for EfficientRollout (drafting only when it speeds the step
 * up, which depends on whether the step is compute- or memory-bound; a draft
 * length that follows how often drafts are accepted).
 *   alpha    = accepted / tested draft positions (a round tests the accepted
 *              drafts and the first rejected one), each round's counts
 *              weighted by decay^age, started from prior_accept with weight
 *              prior_weight;
 *   E(g)     = sum_{i=0}^{g} alpha^i committed tokens per sequence and round
 *              (the speculative-decoding papers on the mlsanity.com list);
 *   rate(g)  = E(g) / cost_us[g] for g >= 1, rate(0) = 1 / cost_us[0] (a
 *              plain decode step commits one token);
 *   choose   = the g in 0..gamma_max with the largest rate (the smaller g on
 *              ties); 0 switches drafting off.
 * cost_us[g]: the time of a round with g drafts, measured by the caller or
 * from s3r_round_cost_us. The struct is plain data owned by the caller.
 */
typedef struct {
  int32_t gamma_max;
  double decay;
  double accepted;
  double tested;
  double cost_us[17];
} s3r_gamma_policy;

s3r_status s3r_gamma_policy_init(s3r_gamma_policy* policy, int32_t gamma_max, double decay,
                                 double prior_accept, double prior_weight, const double* cost_us);
/* One round's acceptance counts (num_accepted: host int32 [num_seqs], each in
 * [0, gamma_used]). */
s3r_status s3r_gamma_policy_update(s3r_gamma_policy* policy, const int32_t* num_accepted,
                                   int32_t num_seqs, int32_t gamma_used);
/* The next draft length (0: drafting off) and, if not NULL, the acceptance
 * estimate and the chosen rate (committed tokens per microsecond). */
s3r_status s3r_gamma_policy_choose(const s3r_gamma_policy* policy, int32_t* gamma, double* alpha,
                                   double* rate);
/*
 * Roofline times in microseconds (NaN for invalid arguments). Dense attention
 * of `rows` query rows per sequence over the whole cache: max(bytes of every
 * key and value / hbm_gbs, 4 Hq rows L D flops / tensor_tflops), so it is
 * memory-bound at small batch x rows and compute-bound beyond. A round with
 * gamma >= 1 drafts: gamma sparse draft calls (every page's summary and the
 * kept pages' keys and values), verification of gamma + 1 rows, the drafter's
 * draws (gamma rows) and speculative sampling (2 gamma + 1 rows and two
 * re-read); gamma = 0: one dense decode row and one draw.
 */
double s3r_attend_cost_us(int32_t num_seqs, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                          int32_t kv_bytes, double mean_context, int32_t rows, double hbm_gbs,
                          double tensor_tflops);
double s3r_round_cost_us(int32_t num_seqs, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                         int32_t page_size, int32_t kv_bytes, double mean_context, int32_t budget_pages,
                         int32_t vocab, int32_t logit_bytes, int32_t gamma, double hbm_gbs,
                         double tensor_tflops);

/* Workspace sizes. Return 0 for an invalid or unsupported request.
 * Attention: rows = 1 and budget_pages > 0 for s3r_sparse_draft_attn;
 * rows = gamma + 1 and budget_pages = 0 for s3r_verify_attn; rows = nodes
 * (up to 64) and budget_pages = 0 for s3r_verify_attn_tree.
 * Sampling: (num_seqs, gamma, vocab) for s3r_spec_sample;
 * (num_rows, 0, vocab) for s3r_sample_tokens. */
size_t s3r_attn_workspace_bytes(const s3r_paged_kv* kv, int32_t rows, int32_t budget_pages);
size_t s3r_sample_workspace_bytes(int32_t num_seqs, int32_t gamma, int32_t vocab);

/*
 * Number of kernels one s3r_sparse_draft_attn call with these arguments
 * launches: 1 when page scoring, top-B and attention run as one kernel (bf16
 * cache, at most one (sequence, KV head) unit per SM, G <= 8, budget <= 128,
 * max_pages_per_seq <= 1024), 2 when a selection kernel precedes the
 * attention kernel; 0 for an invalid or unsupported request. Host-only query
 * (it reads the current device's SM count).
 */
int32_t s3r_sparse_draft_kernels(const s3r_paged_kv* kv, int32_t budget_pages);

/*
 * Synchronises `stream`, then reads the status word of `workspace`: S3R_OK,
 * or S3R_ERR_DEVICE_CHECK with the S3R_DEV_* bits in *bits (bits may be
 * NULL). The bits accumulate over the calls made with the workspace since the
 * word was last read; reading it clears it. s3r_page_summaries has no
 * workspace; its device checks use the status word at `status_word` if given
 * via s3r_page_summaries_checked.
 */
s3r_status s3r_device_status(const void* workspace, uint32_t* bits, void* stream);

/* As s3r_page_summaries, also recording device-check failures in the 4-byte
 * device word status_word (which it clears first). */
s3r_status s3r_page_summaries_checked(const s3r_paged_kv* kv, int32_t tail_only,
                                      void* kmin, void* kmax, uint32_t* status_word,
                                      void* stream);

/*
 * Diagnostic: the float64 exponential the sampling kernels use for their
 * draw weights (a table-driven method after P. T. P. Tang, ACM TOMS 15(2),
 * 1989, with its range fix-up), y_tbl[i] = exp(x[i]), beside CUDA's own
 * exp(x[i]) in y_ref[i] evaluated on the same device. x, y_tbl, y_ref:
 * float64 device arrays of n elements. For tests of the sampler's arithmetic;
 * no part of the decode step calls it.
 */
s3r_status s3r_debug_exp64(const double* x, double* y_tbl, double* y_ref, int32_t n, void* stream);

/* Human-readable name of a status code (static storage). */
const char* s3r_status_str(s3r_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t s3r_version(void);

#ifdef __cplusplus
}
#endif

#endif /* S3R_H_ */
