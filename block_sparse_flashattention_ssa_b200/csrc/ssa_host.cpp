// Host-side pieces of the C ABI: threshold model resolve/fit, q-block count,
// status strings. No CUDA calls.
#include <cmath>
#include <cstdint>
#include <limits>

#include "ssa.h"

// threshold_scale_factor = a * exp(b * target_sparsity) (Model-Optimizer README,
// "Calibrated threshold"; TRT-LLM VisualGen docs, "Checkpoint Config").
extern "C" double ssa_resolve(double a, double b, double target_sparsity) {
  if (!(a > 0.0) || !std::isfinite(a) || !std::isfinite(b) || !(target_sparsity >= 0.0 && target_sparsity <= 1.0))
    return std::numeric_limits<double>::quiet_NaN();
  return a * std::exp(b * target_sparsity);
}

// Ordinary least squares of y = ln(scale_factor) on x = sparsity over the
// usable points, in two passes (means first) for accuracy.
extern "C" int ssa_fit_logspace(const double* sparsity, const double* scale_factor, int n, double* a, double* b,
                                double* s_min, double* s_max) {
  if (!sparsity || !scale_factor || !a || !b || !s_min || !s_max || n < 0) return SSA_ERR_INVALID_ARG;
  auto usable = [&](int i) {
    return sparsity[i] > 0.0 && sparsity[i] < 1.0 && scale_factor[i] > 0.0 && std::isfinite(scale_factor[i]);
  };
  int m = 0;
  double sx = 0.0, sy = 0.0, lo = 1.0, hi = 0.0;
  for (int i = 0; i < n; ++i) {
    if (!usable(i)) continue;
    ++m;
    sx += sparsity[i];
    sy += std::log(scale_factor[i]);
    lo = std::fmin(lo, sparsity[i]);
    hi = std::fmax(hi, sparsity[i]);
  }
  if (m < 2 || !(hi > lo)) return SSA_ERR_INVALID_ARG;
  const double mx = sx / m, my = sy / m;
  double sxx = 0.0, sxy = 0.0;
  for (int i = 0; i < n; ++i) {
    if (!usable(i)) continue;
    const double dx = sparsity[i] - mx;
    sxx += dx * dx;
    sxy += dx * (std::log(scale_factor[i]) - my);
  }
  if (!(sxx > 0.0)) return SSA_ERR_INVALID_ARG;
  *b = sxy / sxx;
  *a = std::exp(my - *b * mx);
  *s_min = lo;
  *s_max = hi;
  return SSA_OK;
}

extern "C" int ssa_num_qblocks(const int32_t* cu, int batch) {
  if (!cu || batch < 1 || cu[0] < 0) return SSA_ERR_INVALID_ARG;
  int64_t q = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t len = static_cast<int64_t>(cu[b + 1]) - cu[b];
    if (len < 0) return SSA_ERR_INVALID_ARG;
    q += (len + SSA_TILE - 1) / SSA_TILE;
  }
  if (q > 0x7FFFFFFF) return SSA_ERR_INVALID_ARG;
  return static_cast<int>(q);
}

extern "C" const char* ssa_status_string(int status) {
  switch (status) {
    case SSA_OK: return "ok";
    case SSA_ERR_INVALID_ARG: return "invalid argument";
    case SSA_ERR_UNSUPPORTED: return "unsupported head_dim or misaligned pointer";
    case SSA_ERR_CUDA: return "CUDA runtime or launch error";
    case SSA_ERR_TIMEOUT: return "a device-side wait exceeded its time limit";
    case SSA_ERR_DEVICE_ARG: return "cu_seqlens inconsistent with total_tokens/max_seqlen (found on the device)";
    default: return "unknown status";
  }
}
