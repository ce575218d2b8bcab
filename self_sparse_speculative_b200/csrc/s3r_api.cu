// C ABI of libs3r: argument validation, workspace planning and launches.
// Every argument error is returned before anything is enqueued; launches are
// asynchronous on the caller's stream. No allocation, no global state beyond
// the cached driver entry point used to encode TMA descriptors.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "s3r_internal.h"

#define S3R_EXPORT extern "C" __attribute__((visibility("default")))

using namespace s3r;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

s3r_status check_kv(const s3r_paged_kv* kv) {
  if (!kv) return S3R_ERR_INVALID_ARG;
  if (kv->num_seqs < 1 || kv->num_q_heads < 1 || kv->num_kv_heads < 1 || kv->max_pages_per_seq < 1 ||
      kv->num_pages_total < 1)
    return S3R_ERR_INVALID_ARG;
  if (kv->num_q_heads % kv->num_kv_heads != 0) return S3R_ERR_INVALID_ARG;
  if (kv->dtype != S3R_F32 && kv->dtype != S3R_BF16) return S3R_ERR_INVALID_ARG;
  if (!kv->k_cache || !kv->v_cache || !kv->block_table || !kv->context_lens) return S3R_ERR_INVALID_ARG;
  if (!aligned16(kv->k_cache) || !aligned16(kv->v_cache)) return S3R_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return S3R_ERR_UNSUPPORTED;
  if (kv->page_size != 16 && kv->page_size != 64) return S3R_ERR_UNSUPPORTED;
  if (kv->num_q_heads / kv->num_kv_heads > 8) return S3R_ERR_UNSUPPORTED;
  if (kv->max_pages_per_seq > kMaxPagesPerSeq) return S3R_ERR_UNSUPPORTED;
  if ((uint64_t)kv->num_pages_total * (uint64_t)kv->num_kv_heads >= (1ull << 31)) return S3R_ERR_UNSUPPORTED;
  return S3R_OK;
}

// max_dense_rows: rows of a dense call (gamma + 1 for s3r_verify_attn; the
// workspace query also serves s3r_verify_attn_tree's up to 64 nodes)
s3r_status check_attn(const s3r_paged_kv* kv, int32_t rows, int32_t budget, bool sparse,
                      int32_t max_dense_rows = kMaxGamma + 1) {
  s3r_status s = check_kv(kv);
  if (s != S3R_OK) return s;
  if (rows < 1) return S3R_ERR_INVALID_ARG;
  if (sparse && budget < 1) return S3R_ERR_INVALID_ARG;
  const int G = kv->num_q_heads / kv->num_kv_heads;
  if ((int64_t)G * rows > 128) return S3R_ERR_UNSUPPORTED;
  if (!sparse && rows > max_dense_rows) return S3R_ERR_UNSUPPORTED;
  if (kv->num_seqs > kMaxSeqs) return S3R_ERR_UNSUPPORTED;
  return S3R_OK;
}

s3r_status from_cuda(cudaError_t e) { return e == cudaSuccess ? S3R_OK : S3R_ERR_CUDA; }

AttnParams make_attn_params(const s3r_paged_kv* kv, const AttnPlan& pl, const void* q, void* out, float* lse,
                            int32_t R, int32_t budget, const int32_t* page_list, float scale, void* ws) {
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.block_table = kv->block_table;
  p.context_lens = kv->context_lens;
  p.page_list = page_list;
  p.page_phys = nullptr;
  p.k_cache = kv->k_cache;
  p.v_cache = kv->v_cache;
  p.S = kv->num_seqs;
  p.Hq = kv->num_q_heads;
  p.Hkv = kv->num_kv_heads;
  p.G = kv->num_q_heads / kv->num_kv_heads;
  p.D = kv->head_dim;
  p.P = kv->page_size;
  p.R = R;
  p.rows = p.G * R;
  p.max_pages = kv->max_pages_per_seq;
  p.num_pages_total = kv->num_pages_total;
  p.budget = budget;
  p.nsplit = pl.nsplit;
  p.chunk_pages = pl.chunk_pages;
  p.scale_log2 = scale * 1.4426950408889634f;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.status = reinterpret_cast<uint32_t*>(w);
  p.tickets = reinterpret_cast<uint32_t*>(w + pl.off_tickets);
  p.part_ml = reinterpret_cast<float*>(w + pl.off_ml);
  p.part_o = reinterpret_cast<float*>(w + pl.off_o);
  return p;
}

}  // namespace

S3R_EXPORT const char* s3r_status_str(s3r_status s) {
  switch (s) {
    case S3R_OK: return "S3R_OK";
    case S3R_ERR_INVALID_ARG: return "S3R_ERR_INVALID_ARG";
    case S3R_ERR_UNSUPPORTED: return "S3R_ERR_UNSUPPORTED";
    case S3R_ERR_WORKSPACE: return "S3R_ERR_WORKSPACE";
    case S3R_ERR_CUDA: return "S3R_ERR_CUDA";
    case S3R_ERR_DEVICE_CHECK: return "S3R_ERR_DEVICE_CHECK";
  }
  return "S3R_UNKNOWN_STATUS";
}

S3R_EXPORT int32_t s3r_version(void) { return 100; }

S3R_EXPORT size_t s3r_attn_workspace_bytes(const s3r_paged_kv* kv, int32_t rows, int32_t budget_pages) {
  if (check_attn(kv, rows, budget_pages, budget_pages > 0, kMaxTreeNodes) != S3R_OK || budget_pages < 0) return 0;
  return plan_attention(*kv, rows, budget_pages).ws_bytes;
}

S3R_EXPORT size_t s3r_sample_workspace_bytes(int32_t num_seqs, int32_t gamma, int32_t vocab) {
  if (num_seqs < 1 || vocab < 1 || gamma < 0 || gamma > kMaxGamma) return 0;
  // enough for either logit type
  const size_t a = plan_sampling(num_seqs, gamma, vocab, 2).ws_bytes;
  const size_t b = plan_sampling(num_seqs, gamma, vocab, 4).ws_bytes;
  return a > b ? a : b;
}

S3R_EXPORT s3r_status s3r_page_summaries_checked(const s3r_paged_kv* kv, int32_t tail_only, void* kmin,
                                                 void* kmax, uint32_t* status_word, void* stream) {
  s3r_status s = check_kv(kv);
  if (s != S3R_OK) return s;
  if (!kmin || !kmax || !aligned16(kmin) || !aligned16(kmax)) return S3R_ERR_INVALID_ARG;
  if (tail_only != 0 && tail_only != 1) return S3R_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (status_word) {
    s = from_cuda(cudaMemsetAsync(status_word, 0, sizeof(uint32_t), st));
    if (s != S3R_OK) return s;
  }
  return from_cuda(launch_summaries(*kv, tail_only, kmin, kmax, status_word, st));
}

S3R_EXPORT s3r_status s3r_page_summaries(const s3r_paged_kv* kv, int32_t tail_only, void* kmin, void* kmax,
                                         void* stream) {
  return s3r_page_summaries_checked(kv, tail_only, kmin, kmax, nullptr, stream);
}

S3R_EXPORT s3r_status s3r_sparse_draft_attn(const s3r_paged_kv* kv, const void* kmin, const void* kmax,
                                            const void* q, int32_t budget_pages, float scale, int32_t* selected,
                                            void* out, float* lse, void* workspace, size_t workspace_bytes,
                                            void* stream) {
  s3r_status s = check_attn(kv, 1, budget_pages, true);
  if (s != S3R_OK) return s;
  if (!kmin || !kmax || !q || !selected || !out) return S3R_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(kmin) || !aligned16(kmax) || !std::isfinite(scale))
    return S3R_ERR_INVALID_ARG;
  const AttnPlan pl = plan_attention(*kv, 1, budget_pages);
  if (!workspace || workspace_bytes < pl.ws_bytes) return S3R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p = make_attn_params(kv, pl, q, out, lse, 1, budget_pages, selected, scale, workspace);
  if (draft_fused_supported(*kv, budget_pages)) {
    // one kernel: page scoring, top-B and attention (everything host-side is
    // prepared before the launch)
    DraftLaunch dl;
    s = from_cuda(prepare_draft_fused(*kv, budget_pages, &dl));
    if (s != S3R_OK) return s;
    p.page_list = nullptr;
    p.kmin = kmin;
    p.kmax = kmax;
    p.selected_out = selected;
    p.parts = dl.parts;
    return from_cuda(launch_draft_fused(*kv, dl, p, st));
  }
  // selection kernel, then attention over the selected pages; the tensor maps
  // the attention needs are checked before anything is enqueued
  if (kv->dtype == S3R_BF16) {
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, kv->k_cache, *kv) || !make_cache_map(&mv, kv->v_cache, *kv)) return S3R_ERR_CUDA;
  }
  uint32_t* status = static_cast<uint32_t*>(workspace);
  int32_t* phys = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + pl.off_phys);
  if (select_only_supported(*kv, budget_pages)) {
    AttnParams ps = p;
    ps.kmin = kmin;
    ps.kmax = kmax;
    ps.selected_out = selected;
    uint32_t* work = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + kWsSelWork);
    s = from_cuda(launch_select_only(*kv, ps, phys, work, st));
  } else {
    s = from_cuda(launch_select(*kv, kmin, kmax, q, budget_pages, selected, phys, status, st));
  }
  if (s != S3R_OK) return s;
  p.page_phys = phys;
  s3r_status api;
  cudaError_t e = launch_attention(*kv, p, st, &api);
  if (api != S3R_OK) return api;
  return from_cuda(e);
}

S3R_EXPORT s3r_status s3r_verify_attn(const s3r_paged_kv* kv, const void* q, int32_t rows, float scale, void* out,
                                      float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  s3r_status s = check_attn(kv, rows, 0, false);
  if (s != S3R_OK) return s;
  if (!q || !out || !aligned16(q) || !aligned16(out) || !std::isfinite(scale)) return S3R_ERR_INVALID_ARG;
  const AttnPlan pl = plan_attention(*kv, rows, 0);
  if (!workspace || workspace_bytes < pl.ws_bytes) return S3R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p = make_attn_params(kv, pl, q, out, lse, rows, 0, nullptr, scale, workspace);
  s3r_status api;
  cudaError_t e = launch_attention(*kv, p, st, &api);
  if (api != S3R_OK) return api;
  return from_cuda(e);
}

S3R_EXPORT s3r_status s3r_verify_attn_tree(const s3r_paged_kv* kv, const void* q, int32_t nodes,
                                           const int32_t* parents, float scale, void* out, float* lse,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  s3r_status s = check_kv(kv);
  if (s != S3R_OK) return s;
  if (nodes < 1 || !parents) return S3R_ERR_INVALID_ARG;
  const int G = kv->num_q_heads / kv->num_kv_heads;
  if (nodes > kMaxTreeNodes || kv->num_seqs > kMaxSeqs) return S3R_ERR_UNSUPPORTED;
  // bf16: the token-major kernel (all packed rows of a unit in one MMA of at
  // most 64 columns); f32: up to 128 packed rows
  if ((int64_t)G * nodes > (kv->dtype == S3R_BF16 ? 64 : 128)) return S3R_ERR_UNSUPPORTED;
  if (!q || !out || !aligned16(q) || !aligned16(out) || !std::isfinite(scale)) return S3R_ERR_INVALID_ARG;
  const AttnPlan pl = plan_attention(*kv, nodes, 0);
  if (!workspace || workspace_bytes < pl.ws_bytes) return S3R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p = make_attn_params(kv, pl, q, out, lse, nodes, 0, nullptr, scale, workspace);
  p.tree_parent = parents;
  s3r_status api;
  cudaError_t e = launch_attention(*kv, p, st, &api);
  if (api != S3R_OK) return api;
  return from_cuda(e);
}

S3R_EXPORT size_t s3r_tree_sample_workspace_bytes(int32_t num_seqs, int32_t nodes, int32_t vocab) {
  if (num_seqs < 1 || nodes < 1 || nodes > kMaxTreeNodes || vocab < 1) return 0;
  return kWsHeader;
}

S3R_EXPORT s3r_status s3r_tree_spec_sample(const void* target_logits, const void* draft_logits,
                                           s3r_dtype logit_dtype, const int32_t* tokens, const int32_t* parents,
                                           const float* u_accept, const float* u_sample, int32_t num_seqs,
                                           int32_t nodes, int32_t vocab, float temperature, int32_t* out_tokens,
                                           int32_t* num_accepted, int32_t* path, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (!target_logits || !draft_logits || !tokens || !parents || !u_accept || !u_sample || !out_tokens ||
      !num_accepted)
    return S3R_ERR_INVALID_ARG;
  if (logit_dtype != S3R_F32 && logit_dtype != S3R_BF16) return S3R_ERR_INVALID_ARG;
  if (num_seqs < 1 || nodes < 1 || vocab < 1 || !(temperature > 0.0f) || !std::isfinite(temperature))
    return S3R_ERR_INVALID_ARG;
  if (nodes > kMaxTreeNodes || num_seqs > 65535) return S3R_ERR_UNSUPPORTED;
  if ((int64_t)num_seqs * nodes * vocab >= (1ll << 40)) return S3R_ERR_UNSUPPORTED;
  const size_t need = s3r_tree_sample_workspace_bytes(num_seqs, nodes, vocab);
  if (!workspace || workspace_bytes < need) return S3R_ERR_WORKSPACE;
  const size_t es = logit_dtype == S3R_BF16 ? 2 : 4;
  const bool vec = aligned16(target_logits) && aligned16(draft_logits) && ((size_t)vocab * es) % 16 == 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  return from_cuda(launch_tree_sample(target_logits, draft_logits, logit_dtype, tokens, parents, u_accept, u_sample,
                                      num_seqs, nodes, vocab, 1.0 / static_cast<double>(temperature), out_tokens,
                                      num_accepted, path, status, vec, st));
}

S3R_EXPORT int32_t s3r_tree_node_budget(int64_t capacity, int32_t active, int32_t n_min, int32_t n_max) {
  if (active < 1 || n_min < 1 || n_max < n_min || capacity < 0) return -1;
  const int64_t n = capacity / active;
  return (int32_t)(n < n_min ? n_min : (n > n_max ? n_max : n));
}

namespace {
SampleParams make_sample_params(const SamplePlan& pl, void* ws, int32_t nseq, int32_t gamma, int32_t vocab,
                                float temperature) {
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.nseq = nseq;
  p.gamma = gamma;
  p.vocab = vocab;
  p.inv_temp = 1.0f / temperature;
  p.inv_temp_d = 1.0 / static_cast<double>(temperature);
  bind_sample_workspace(&p, pl, ws);
  return p;
}
}  // namespace

S3R_EXPORT s3r_status s3r_spec_sample_ex(const void* target_logits, const void* draft_logits,
                                         s3r_dtype logit_dtype, const int32_t* draft_tokens, const float* u_accept,
                                         const float* u_sample, const double* draft_stats, int32_t num_seqs,
                                         int32_t gamma, int32_t vocab, float temperature, int32_t* out_tokens,
                                         int32_t* num_accepted, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  if (!target_logits || !draft_logits || !draft_tokens || !u_accept || !u_sample || !out_tokens || !num_accepted)
    return S3R_ERR_INVALID_ARG;
  if (logit_dtype != S3R_F32 && logit_dtype != S3R_BF16) return S3R_ERR_INVALID_ARG;
  if (num_seqs < 1 || vocab < 1 || gamma < 1) return S3R_ERR_INVALID_ARG;
  if (!(temperature > 0.0f) || !std::isfinite(temperature)) return S3R_ERR_INVALID_ARG;
  if (draft_stats && (reinterpret_cast<uintptr_t>(draft_stats) & 7u)) return S3R_ERR_INVALID_ARG;
  if (gamma > kMaxGamma) return S3R_ERR_UNSUPPORTED;
  const SamplePlan pl = plan_sampling(num_seqs, gamma, vocab, logit_dtype == S3R_BF16 ? 2 : 4);
  if (!workspace || workspace_bytes < pl.ws_bytes) return S3R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SampleParams p = make_sample_params(pl, workspace, num_seqs, gamma, vocab, temperature);
  p.target = target_logits;
  p.draft = draft_logits;
  p.draft_tokens = draft_tokens;
  p.u_accept = u_accept;
  p.u_sample = u_sample;
  p.out_tokens = out_tokens;
  p.num_accepted = num_accepted;
  p.draft_stats = draft_stats;
  return from_cuda(launch_sampling(p, logit_dtype, true, st));
}

S3R_EXPORT s3r_status s3r_spec_sample(const void* target_logits, const void* draft_logits, s3r_dtype logit_dtype,
                                      const int32_t* draft_tokens, const float* u_accept, const float* u_sample,
                                      int32_t num_seqs, int32_t gamma, int32_t vocab, float temperature,
                                      int32_t* out_tokens, int32_t* num_accepted, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  return s3r_spec_sample_ex(target_logits, draft_logits, logit_dtype, draft_tokens, u_accept, u_sample, nullptr,
                            num_seqs, gamma, vocab, temperature, out_tokens, num_accepted, workspace,
                            workspace_bytes, stream);
}

S3R_EXPORT s3r_status s3r_sample_tokens_ex(const void* logits, s3r_dtype logit_dtype, int32_t num_rows,
                                           int32_t vocab, float temperature, const float* u, int32_t* tokens,
                                           double* row_stats, void* workspace, size_t workspace_bytes,
                                           void* stream) {
  if (!logits || !u || !tokens) return S3R_ERR_INVALID_ARG;
  if (logit_dtype != S3R_F32 && logit_dtype != S3R_BF16) return S3R_ERR_INVALID_ARG;
  if (num_rows < 1 || vocab < 1) return S3R_ERR_INVALID_ARG;
  if (!(temperature > 0.0f) || !std::isfinite(temperature)) return S3R_ERR_INVALID_ARG;
  if (row_stats && (reinterpret_cast<uintptr_t>(row_stats) & 7u)) return S3R_ERR_INVALID_ARG;
  const SamplePlan pl = plan_sampling(num_rows, 0, vocab, logit_dtype == S3R_BF16 ? 2 : 4);
  if (!workspace || workspace_bytes < pl.ws_bytes) return S3R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SampleParams p = make_sample_params(pl, workspace, num_rows, 0, vocab, temperature);
  p.target = logits;
  p.u_sample = u;
  p.out_tokens = tokens;
  p.row_stats_out = row_stats;
  return from_cuda(launch_sampling(p, logit_dtype, false, st));
}

S3R_EXPORT s3r_status s3r_sample_tokens(const void* logits, s3r_dtype logit_dtype, int32_t num_rows, int32_t vocab,
                                        float temperature, const float* u, int32_t* tokens, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  return s3r_sample_tokens_ex(logits, logit_dtype, num_rows, vocab, temperature, u, tokens, nullptr, workspace,
                              workspace_bytes, stream);
}

S3R_EXPORT size_t s3r_kv_workspace_bytes(int32_t num_seqs) {
  if (num_seqs < 1) return 0;
  return kv_workspace_bytes(num_seqs);
}

namespace {
s3r_status check_kv_upkeep(const s3r_paged_kv* kv, int32_t* context_lens, void* kmin, void* kmax, void* workspace,
                           size_t workspace_bytes) {
  s3r_status s = check_kv(kv);
  if (s != S3R_OK) return s;
  if (!context_lens || !kmin || !kmax || !aligned16(kmin) || !aligned16(kmax)) return S3R_ERR_INVALID_ARG;
  if (reinterpret_cast<const void*>(context_lens) != reinterpret_cast<const void*>(kv->context_lens))
    return S3R_ERR_INVALID_ARG;                          // the lengths are updated where the cache reads them
  if (!workspace || workspace_bytes < kv_workspace_bytes(kv->num_seqs)) return S3R_ERR_WORKSPACE;
  return S3R_OK;
}
}  // namespace

S3R_EXPORT s3r_status s3r_kv_append(const s3r_paged_kv* kv, int32_t* context_lens, const void* k_new,
                                    const void* v_new, int32_t n, int32_t overwrite, void* kmin, void* kmax,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  s3r_status s = check_kv_upkeep(kv, context_lens, kmin, kmax, workspace, workspace_bytes);
  if (s != S3R_OK) return s;
  if (n < 0 || overwrite < 0 || n > kMaxAppendRows || overwrite > kMaxAppendRows) return S3R_ERR_INVALID_ARG;
  if (n > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))) return S3R_ERR_INVALID_ARG;
  if (n == 0 && overwrite == 0) return S3R_OK;
  return from_cuda(launch_kv_append(*kv, context_lens, k_new, v_new, n, overwrite, kmin, kmax, workspace,
                                    static_cast<cudaStream_t>(stream)));
}

S3R_EXPORT s3r_status s3r_kv_rollback(const s3r_paged_kv* kv, int32_t* context_lens, const int32_t* num_accepted,
                                      int32_t rows, void* kmin, void* kmax, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  s3r_status s = check_kv_upkeep(kv, context_lens, kmin, kmax, workspace, workspace_bytes);
  if (s != S3R_OK) return s;
  if (!num_accepted || rows < 1 || rows > kMaxGamma + 1) return S3R_ERR_INVALID_ARG;
  return from_cuda(launch_kv_rollback(*kv, context_lens, num_accepted, rows, kmin, kmax, workspace,
                                      static_cast<cudaStream_t>(stream)));
}

S3R_EXPORT s3r_status s3r_debug_exp64(const double* x, double* y_tbl, double* y_ref, int32_t n, void* stream) {
  if (!x || !y_tbl || !y_ref || n < 1) return S3R_ERR_INVALID_ARG;
  return from_cuda(launch_exp64_probe(x, y_tbl, y_ref, n, static_cast<cudaStream_t>(stream)));
}

S3R_EXPORT int32_t s3r_sparse_draft_kernels(const s3r_paged_kv* kv, int32_t budget_pages) {
  if (check_attn(kv, 1, budget_pages, true) != S3R_OK) return 0;
  return draft_fused_supported(*kv, budget_pages) ? 1 : 2;
}

S3R_EXPORT s3r_status s3r_device_status(const void* workspace, uint32_t* bits, void* stream) {
  if (!workspace) return S3R_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return S3R_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return S3R_ERR_CUDA;
  // the word is sticky until read: clear it for the calls that follow
  if (w != 0 && cudaMemset(const_cast<void*>(workspace), 0, sizeof(w)) != cudaSuccess) return S3R_ERR_CUDA;
  if (bits) *bits = w;
  return w == 0 ? S3R_OK : S3R_ERR_DEVICE_CHECK;
}
