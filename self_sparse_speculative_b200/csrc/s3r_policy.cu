// Draft-length policy: acceptance-aware gamma with a regime toggle (host
// code; no kernel). The researchpod.app page on EfficientRollout (another
// self-drafting method for RL rollouts) describes drafting only when it
// speeds the step up, which depends on whether the step is limited by compute
// or by memory bandwidth, and a draft length adapted to how often drafts are
// accepted; the expected tokens of a round come from the speculative-decoding
// papers on the mlsanity.com page's reference list.
//
//   alpha      = accepted / tested draft positions, each round's counts
//                weighted by decay^age, started from a prior
//   E(gamma)   = sum_{i=0}^{gamma} alpha^i committed tokens per sequence
//   rate       = E(gamma) / cost(gamma); rate(0) = 1 / cost(0) (plain decode)
//   gamma*     = the best rate over 0..gamma_max (the smaller on ties);
//                gamma* = 0 switches drafting off
//   cost model = max(HBM bytes / bandwidth, tensor flops / peak) per call
#include <cmath>

#include "s3r_internal.h"

#define S3R_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

double expected_tokens(double alpha, int gamma) {
  double e = 0.0;
  for (int i = 0; i <= gamma; ++i) e += std::pow(alpha, (double)i);
  return e;
}

double policy_alpha(const s3r_gamma_policy* p) { return p->tested > 0.0 ? p->accepted / p->tested : 0.0; }

double policy_rate(const s3r_gamma_policy* p, int gamma) {
  if (gamma == 0) return 1.0 / p->cost_us[0];
  return expected_tokens(policy_alpha(p), gamma) / p->cost_us[gamma];
}

bool finite_pos(double x) { return std::isfinite(x) && x > 0.0; }

}  // namespace

S3R_EXPORT s3r_status s3r_gamma_policy_init(s3r_gamma_policy* p, int32_t gamma_max, double decay,
                                            double prior_accept, double prior_weight, const double* cost_us) {
  if (!p || !cost_us) return S3R_ERR_INVALID_ARG;
  if (gamma_max < 1 || gamma_max > s3r::kMaxGamma) return S3R_ERR_UNSUPPORTED;
  if (!(decay >= 0.0 && decay <= 1.0) || !(prior_accept >= 0.0 && prior_accept <= 1.0) ||
      !(prior_weight >= 0.0) || !std::isfinite(prior_weight))
    return S3R_ERR_INVALID_ARG;
  for (int g = 0; g <= gamma_max; ++g)
    if (!finite_pos(cost_us[g])) return S3R_ERR_INVALID_ARG;
  p->gamma_max = gamma_max;
  p->decay = decay;
  p->accepted = prior_accept * prior_weight;
  p->tested = prior_weight;
  for (int g = 0; g <= s3r::kMaxGamma; ++g) p->cost_us[g] = g <= gamma_max ? cost_us[g] : 0.0;
  return S3R_OK;
}

S3R_EXPORT s3r_status s3r_gamma_policy_update(s3r_gamma_policy* p, const int32_t* num_accepted, int32_t num_seqs,
                                              int32_t gamma_used) {
  if (!p || !num_accepted || num_seqs < 1 || gamma_used < 1 || gamma_used > s3r::kMaxGamma)
    return S3R_ERR_INVALID_ARG;
  double a = 0.0, t = 0.0;
  for (int b = 0; b < num_seqs; ++b) {
    const int n = num_accepted[b];
    if (n < 0 || n > gamma_used) return S3R_ERR_INVALID_ARG;
    a += (double)n;
    t += (double)(n + 1 < gamma_used ? n + 1 : gamma_used);   // the accepted drafts and the first rejection
  }
  p->accepted = p->decay * p->accepted + a;
  p->tested = p->decay * p->tested + t;
  return S3R_OK;
}

S3R_EXPORT s3r_status s3r_gamma_policy_choose(const s3r_gamma_policy* p, int32_t* gamma, double* alpha,
                                              double* rate) {
  if (!p || !gamma || p->gamma_max < 1 || p->gamma_max > s3r::kMaxGamma) return S3R_ERR_INVALID_ARG;
  int best = 0;
  double best_rate = policy_rate(p, 0);
  for (int g = 1; g <= p->gamma_max; ++g) {
    const double r = policy_rate(p, g);
    if (r > best_rate) {
      best = g;
      best_rate = r;
    }
  }
  *gamma = best;
  if (alpha) *alpha = policy_alpha(p);
  if (rate) *rate = best_rate;
  return S3R_OK;
}

S3R_EXPORT double s3r_attend_cost_us(int32_t num_seqs, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                     int32_t kv_bytes, double mean_context, int32_t rows, double hbm_gbs,
                                     double tensor_tflops) {
  if (num_seqs < 1 || q_heads < 1 || kv_heads < 1 || head_dim < 1 || kv_bytes < 1 || rows < 1 ||
      !finite_pos(mean_context) || !finite_pos(hbm_gbs) || !finite_pos(tensor_tflops))
    return NAN;
  const double kv = num_seqs * 2.0 * kv_heads * head_dim * kv_bytes * mean_context;
  const double flops = 4.0 * num_seqs * q_heads * rows * mean_context * head_dim;
  return std::fmax(kv / (hbm_gbs * 1e9), flops / (tensor_tflops * 1e12)) * 1e6;
}

S3R_EXPORT double s3r_round_cost_us(int32_t num_seqs, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                    int32_t page_size, int32_t kv_bytes, double mean_context, int32_t budget_pages,
                                    int32_t vocab, int32_t logit_bytes, int32_t gamma, double hbm_gbs,
                                    double tensor_tflops) {
  if (page_size < 1 || budget_pages < 0 || vocab < 0 || logit_bytes < 1 || gamma < 0 || gamma > s3r::kMaxGamma)
    return NAN;
  const double bw = hbm_gbs * 1e9;
  const double attend1 =
      s3r_attend_cost_us(num_seqs, q_heads, kv_heads, head_dim, kv_bytes, mean_context, gamma + 1, hbm_gbs,
                         tensor_tflops) * 1e-6;
  if (std::isnan(attend1)) return NAN;
  const double S = num_seqs, H = kv_heads, D = head_dim, P = page_size;
  if (gamma == 0) return (attend1 + S * vocab * logit_bytes / bw) * 1e6;
  const double pages = std::ceil(mean_context / P);
  const double draft = S * H * (pages * 2.0 * D * kv_bytes + std::fmin((double)budget_pages, pages) * P * 2.0 * D * kv_bytes) / bw;
  const double sample = S * ((2 * gamma + 1) + 2) * (double)vocab * logit_bytes / bw;
  const double draws = S * gamma * (double)vocab * logit_bytes / bw;
  return (gamma * draft + attend1 + sample + draws) * 1e6;
}
