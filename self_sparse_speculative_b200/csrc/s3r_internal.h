// Host-side interface between the C ABI (s3r_api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "s3r.h"

namespace s3r {

// Tokens per pipeline stage of the tensor-core attention kernel (one 64-token
// page, or four 16-token pages).
constexpr int kStageTokens = 64;
// Upper bound on the pages one fp32 attention CTA processes.
constexpr int kMaxSplitPages = 512;
constexpr int kMaxPagesPerSeq = 8192;
constexpr int kMaxGamma = 16;
// Rows one s3r_kv_append call writes (or overwrites) per sequence, at most.
constexpr int kMaxAppendRows = 1024;
// Sequences per call (the tensor-core attention keeps a per-sequence prefix
// of page counts in shared memory).
constexpr int kMaxSeqs = 1024;
// Upper bound on the persistent attention grid (one CTA per SM); sizes the
// partial-result slots of the workspace.
constexpr int kMaxPersistentCtas = 160;
constexpr int kMaxTreeNodes = 64;         // tree verification: nodes per sequence (one 64-bit mask)

// Workspace header: word 0 is the device status word; words 32 and 33 are
// the two-kernel sparse draft's selection counters (next unit, CTAs done);
// the rest is reserved.
constexpr size_t kWsHeader = 256;
constexpr size_t kWsSelWork = 128;        // byte offset of the selection counters

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct AttnParams {
  const void* q;
  void* out;
  float* lse;
  const int32_t* block_table;
  const int32_t* context_lens;
  const int32_t* page_list;   // sparse: selected [S, Hkv, budget]; dense: nullptr
  const int32_t* page_phys;   // sparse: physical ids of page_list's pages (written by the selector); else nullptr
  const void* k_cache;
  const void* v_cache;
  int32_t S, Hq, Hkv, G, D, P, R, rows;
  int32_t max_pages, num_pages_total, budget;
  int32_t nsplit, chunk_pages;   // fp32 path: grid splits per (seq, kv head) and pages per split
  float scale_log2;              // scale * log2(e)
  uint32_t* status;
  uint32_t* tickets;             // [S * Hkv]
  float* part_ml;                // [slots, rows, 2]  (running max in log2 units, sum)
  float* part_o;                 // [slots, rows, D]  (unnormalised)
  // fused sparse draft (page selection inside the attention kernel)
  const void* kmin;              // [num_pages_total, Hkv, D] page summaries
  const void* kmax;
  int32_t* selected_out;         // [S, Hkv, budget] logical ids of the kept pages
  int32_t parts;                 // CTAs sharing one (sequence, KV head) unit
  // tree verification: parent of each of the R round nodes [S, R] (null: the causal chain)
  const int32_t* tree_parent;
};

// Split plan shared by the workspace-size query and the launch.
struct AttnPlan {
  int32_t nsplit;
  int32_t chunk_pages;
  size_t ws_bytes;
  size_t off_tickets, off_ml, off_o;
  size_t off_phys;   // sparse: [S, Hkv, budget] physical page ids of the selection (0: none)
};
AttnPlan plan_attention(const s3r_paged_kv& kv, int32_t rows, int32_t budget_pages);

cudaError_t launch_summaries(const s3r_paged_kv& kv, int tail_only, void* kmin, void* kmax,
                             uint32_t* status, cudaStream_t st);
cudaError_t launch_select(const s3r_paged_kv& kv, const void* kmin, const void* kmax,
                          const void* q, int32_t budget, int32_t* selected, int32_t* selected_phys,
                          uint32_t* status, cudaStream_t st);
// Launch with programmatic dependent launch allowed (the kernel orders
// itself after its predecessor with griddepcontrol.wait) and, when
// cluster_x > 1, thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_attention(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st,
                             s3r_status* api_status);
cudaError_t launch_attention_tc(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st,
                                s3r_status* api_status);
cudaError_t launch_attention_tok(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st,
                                s3r_status* api_status);
// Whether the fused sparse draft kernel (selection and attention in one
// launch) serves this cache and budget; else select + attention kernels.
bool draft_fused_supported(const s3r_paged_kv& kv, int32_t budget_pages);
// Host-side preparation of the fused draft launch (tensor maps, shared
// memory size, grid): done before anything is enqueued, so a failure
// enqueues nothing.
struct DraftLaunch {
  CUtensorMap mk, mv;
  int grid;
  int parts;
  size_t smem;
};
cudaError_t prepare_draft_fused(const s3r_paged_kv& kv, int32_t budget_pages, DraftLaunch* dl);
cudaError_t launch_draft_fused(const s3r_paged_kv& kv, const DraftLaunch& dl, const AttnParams& p, cudaStream_t st);
// Selection alone (the fused kernel's selection, persistent CTAs taking units
// from the counters `work` [2] of the workspace header) for the two-kernel
// sparse draft: kept pages to p.selected_out, their physical ids to phys_out
// ([S, Hkv, budget]).
bool select_only_supported(const s3r_paged_kv& kv, int32_t budget_pages);
cudaError_t launch_select_only(const s3r_paged_kv& kv, const AttnParams& p, int32_t* phys_out, uint32_t* work,
                               cudaStream_t st);
bool make_cache_map(CUtensorMap* map, const void* base, const s3r_paged_kv& kv);
int device_sm_count();

// KV-cache upkeep (s3r_kv.cu): workspace = status word + per-sequence tickets.
size_t kv_workspace_bytes(int32_t num_seqs);
cudaError_t launch_kv_append(const s3r_paged_kv& kv, int32_t* lens, const void* k_new, const void* v_new, int32_t n,
                             int32_t overwrite, void* kmin, void* kmax, void* ws, cudaStream_t st);
cudaError_t launch_kv_rollback(const s3r_paged_kv& kv, int32_t* lens, const int32_t* num_accepted, int32_t rows,
                               void* kmin, void* kmax, void* ws, cudaStream_t st);

struct SamplePlan {
  int32_t nrows;        // rows with statistics (2*gamma+1 per sequence, or num_rows)
  int32_t nseq;         // sequences (or rows for plain sampling)
  int32_t c1, ch1;      // pass-1 chunks per row and elements per chunk
  int32_t c2, ch2;      // pass-2 chunks per sequence and elements per chunk
  size_t ws_bytes;
  size_t off_tk_row, off_tk_seq1, off_tk_seq2, off_tk_seq3, off_j;
  size_t off_part1, off_stats, off_znorm, off_zpart, off_wpart, off_cmax;
  size_t memset_bytes;  // bytes from the start of the workspace cleared per call
};
// elt: bytes per logit (2 for bf16, 4 for fp32); the chunking depends on it.
SamplePlan plan_sampling(int32_t nseq, int32_t gamma, int32_t vocab, int32_t elt);

struct SampleParams {
  const void* target;      // spec: [S, R, V]; plain: [N, V]
  const void* draft;       // spec: [S, gamma, V]; plain: unused
  const int32_t* draft_tokens;
  const float* u_accept;
  const float* u_sample;   // spec: [S, R]; plain: [N]
  int32_t* out_tokens;     // spec: [S, R]; plain: [N]
  int32_t* num_accepted;   // spec only
  int32_t nseq, gamma, vocab;
  float inv_temp;          // 1 / T
  double inv_temp_d;
  uint32_t* status;
  uint32_t* tk_row;
  uint32_t* tk_seq1;
  uint32_t* tk_seq2;
  uint32_t* tk_seq3;
  int32_t* jsel;
  void* part1;             // [nrows, c1] {float max, float pad, double sum}
  double* stats;           // [nrows, 2] {max, Z}   (Z from float32 exponentials)
  double* znorm;           // [nseq, 2] exact float64 Z of the residual's two rows
  double* zpart;           // [nseq, c2, 2] chunk partials of znorm
  double* wpart;           // [nseq, c2, 8] per-warp partial sums of the draw weights
  float* cmax;             // [nseq, c2] chunk maxima (plain draws)
  int32_t c1, ch1, c2, ch2;
  double* row_stats_out;       // plain: [N, 2] {row max, exact float64 Z} written by the draw, or null
  const double* draft_stats;   // spec: [S, gamma, 2] the draft rows' {max, exact Z} (from a plain draw), or null
};
// Fill the workspace pointers and sizes of `p` from a plan and a workspace base.
void bind_sample_workspace(SampleParams* p, const SamplePlan& pl, void* ws);
cudaError_t launch_sampling(const SampleParams& p, s3r_dtype dt, bool spec, cudaStream_t st);
cudaError_t launch_tree_sample(const void* target, const void* draft, s3r_dtype dt, const int32_t* tokens,
                               const int32_t* parents, const float* u_accept, const float* u_sample, int32_t nseq,
                               int32_t nodes, int32_t vocab, double inv_temp, int32_t* out_tokens,
                               int32_t* num_accepted, int32_t* path, uint32_t* status, bool vec, cudaStream_t st);
cudaError_t launch_exp64_probe(const double* x, double* y_tbl, double* y_ref, int n, cudaStream_t st);

}  // namespace s3r
