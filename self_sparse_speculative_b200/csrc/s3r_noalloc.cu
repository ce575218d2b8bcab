// Speculative sampling without a caller-provided workspace.
//
// Some callers cannot hand the library scratch memory: a caller that runs
// inside a host framework whose device memory is owned by its own pooling
// allocator (so a bare cudaMalloc would fragment or exceed the pool's
// budget), a plug-in that is never given an allocator handle, or code that
// must not allocate while a stream is being captured into a CUDA graph. For
// them this file gives s3r_spec_sample a variant whose scratch lives in a
// statically sized device array that the library itself owns; the caller
// still passes every input and output buffer.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits. Its
// device address is looked up (cudaGetSymbolAddress) on the first call made
// with a device current and kept for that device's current CUDA context; a
// call from another context (after cudaDeviceReset, for instance, the module
// is loaded again at a new address) looks it up again. The host-side symbol
// itself is only a stand-in and is never passed to a kernel.
#include <cmath>
#include <cstring>
#include <mutex>

#include "s3r_internal.h"

#define S3R_EXPORT extern "C" __attribute__((visibility("default")))

using namespace s3r;

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;      // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's address in one context (per device; the context it was looked
// up in, and the address).
struct ScratchSlot {
  std::mutex m;
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
ScratchSlot g_scratch_slot[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn get_ctx_fn() {
  static CtxGetCurrentFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(ptr);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

// Device address of the scratch array in the current device's current
// context (nullptr on error).
void* scratch_on_current_device(s3r_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { *st = S3R_ERR_CUDA; return nullptr; }
  if (dev < 0 || dev >= kMaxDevices) { *st = S3R_ERR_UNSUPPORTED; return nullptr; }
  CtxGetCurrentFn ctx_fn = get_ctx_fn();
  if (!ctx_fn) { *st = S3R_ERR_CUDA; return nullptr; }
  CUcontext ctx = nullptr;
  if (ctx_fn(&ctx) != CUDA_SUCCESS) { *st = S3R_ERR_CUDA; return nullptr; }   // null before any context exists
  ScratchSlot& slot = g_scratch_slot[dev];
  std::lock_guard<std::mutex> lock(slot.m);
  if (!ctx || slot.ctx != ctx || !slot.addr) {
    // the lookup also makes the runtime's context current, so read it after
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) { *st = S3R_ERR_CUDA; return nullptr; }
    if (ctx_fn(&ctx) != CUDA_SUCCESS || !ctx) { *st = S3R_ERR_CUDA; return nullptr; }
    slot.ctx = ctx;
    slot.addr = p;
  }
  *st = S3R_OK;
  return slot.addr;
}

}  // namespace

S3R_EXPORT s3r_status s3r_spec_sample_noalloc(const void* target_logits, const void* draft_logits,
                                              s3r_dtype logit_dtype, const int32_t* draft_tokens,
                                              const float* u_accept, const float* u_sample, int32_t num_seqs,
                                              int32_t gamma, int32_t vocab, float temperature,
                                              int32_t* out_tokens, int32_t* num_accepted, void* stream) {
  if (!target_logits || !draft_logits || !draft_tokens || !u_accept || !u_sample || !out_tokens || !num_accepted)
    return S3R_ERR_INVALID_ARG;
  if (logit_dtype != S3R_F32 && logit_dtype != S3R_BF16) return S3R_ERR_INVALID_ARG;
  if (num_seqs < 1 || vocab < 1 || gamma < 1) return S3R_ERR_INVALID_ARG;
  if (!(temperature > 0.0f) || !std::isfinite(temperature)) return S3R_ERR_INVALID_ARG;
  if (gamma > kMaxGamma) return S3R_ERR_UNSUPPORTED;
  const SamplePlan pl = plan_sampling(num_seqs, gamma, vocab, logit_dtype == S3R_BF16 ? 2 : 4);
  if (pl.ws_bytes > kStaticScratchBytes) return S3R_ERR_UNSUPPORTED;     // batch too large for the array
  s3r_status s;
  uint8_t* w = static_cast<uint8_t*>(scratch_on_current_device(&s));
  if (!w) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // tickets and the status word must start at zero on every call
  if (cudaMemsetAsync(w, 0, pl.memset_bytes, st) != cudaSuccess) return S3R_ERR_CUDA;
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.target = target_logits;
  p.draft = draft_logits;
  p.draft_tokens = draft_tokens;
  p.u_accept = u_accept;
  p.u_sample = u_sample;
  p.out_tokens = out_tokens;
  p.num_accepted = num_accepted;
  p.nseq = num_seqs;
  p.gamma = gamma;
  p.vocab = vocab;
  p.inv_temp = 1.0f / temperature;
  p.inv_temp_d = 1.0 / static_cast<double>(temperature);
  bind_sample_workspace(&p, pl, w);
  return launch_sampling(p, logit_dtype, true, st) == cudaSuccess ? S3R_OK : S3R_ERR_CUDA;
}
