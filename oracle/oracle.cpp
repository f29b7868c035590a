// CPU oracle for BLASST skip-softmax attention. TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously correct restatement of what the GPU path computes.
// Only the tests, the package's smoke check and the benchmark's CPU-baseline
// leg may load it; the product path never does. It shares no code, header or
// constant with the CUDA library.
//
// Method (BLASST skip-softmax, as described in the Model-Optimizer pages
// "Skip-Softmax Sparse Attention for Diffusion Models", section "Threshold
// Modes", and the commit page's "Triton kernels" section): FlashAttention
// walks the KV tiles of one query tile in order; a KV tile whose scores are
// all far below the running softmax max is skipped whole (no V load, no
// softmax, no accumulation). The threshold lambda = threshold_scale_factor /
// seq_k is used as log2(lambda) (Model-Optimizer README, "Threshold Modes";
// TRT-LLM VisualGen docs, "Skip Softmax Attention"). The calibration kernel
// computes dense attention while counting, for N thresholds at once, the
// tiles that would have been skipped (commit page, "Triton kernels").
//
// Readings where the pages are silent (all fixed here, used by both sides):
//  * tiles are 128 x 128 (Br = Bc = 128, the eager config of Model-Optimizer
//    PR #1166, "Usage");
//  * scores in the log2 domain: s2 = fp32(q.k) * fp32(softmax_scale*log2 e),
//    the dot product exact in double and rounded once to fp32;
//  * m_r is the running max BEFORE the tile; the tile statistic is
//    d = max over valid rows of fp32(tilemax_r - m_r); skip iff d < L (strict),
//    L = fp32(log2 lambda); tile 0 has d = +inf; tsf <= 0 means L = -inf;
//  * rows past the sequence end do not vote, columns past it are -inf;
//  * no clamp of lambda to 1;
//  * probabilities and accumulators in double.
// The 8-bit P.V reading (the variant with E4M3 Q, K and V): V arrives decoded
// (each E4M3 value is exact in bf16) and its per-tensor scale multiplies the
// output; each kept tile's probabilities are taken against a per-row integer
// reference exponent r and shifted by sigma, P = 2^(s2 - r + sigma), and the
// P.V product uses P rounded to the nearest E4M3 value (ties to even,
// saturating at 448) while the row sum l adds the unrounded P. r starts at
// ceil of the first kept tile's max and moves to ceil(m) whenever the
// running max m rises above r + tau, rescaling O and l by 2^(r_old - r_new)
// (a power of two). With tau = 0 and sigma = 8 every P lies in (0, 256].
// Parity pins for every function live in tests/test_oracle.py.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr int kTile = 128;
constexpr double kLog2e = 1.4426950408889634073599246810019;

inline double bf16_to_double(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

struct Problem {
  const uint16_t *q, *k, *v;
  const int32_t* cu;
  int batch, H, D;
  float c;  // fp32(softmax_scale * log2 e)
  int p_e4m3;        // 1: the 8-bit P.V reading above
  double p_shift;    // sigma
  double p_lag;      // tau
  double out_scale;  // multiplies O / l (the V descale)
};

// Nearest E4M3 value of x >= 0 (OCP 8-bit floating point without infinities:
// 4 exponent bits with bias 7 and 3 mantissa bits, so a binade 2^e holds 8
// values 2^(e-3) apart, e >= -6, the subnormals continuing the spacing 2^-9
// down to 0; the largest finite value is 448). Ties go to the even multiple of
// the spacing; values from 448 up saturate to 448.
double e4m3_nearest(double x) {
  if (!(x > 0.0)) return 0.0;
  if (x >= 448.0) return 448.0;
  int e2;
  std::frexp(x, &e2);  // x = f * 2^e2 with f in [0.5, 1): the binade is 2^(e2 - 1)
  const int e = std::max(e2 - 1, -6);
  const double spacing = std::ldexp(1.0, e - 3);
  const double q = std::nearbyint(x / spacing);  // round half to even (default rounding mode)
  return std::min(q * spacing, 448.0);
}

struct UnitResult {
  float* out;        // [128][D]
  float* dstat;      // [max_tiles] or null
  uint8_t* decision; // [max_tiles] or null
  int32_t* skips;    // scalar or null
  int32_t* counts;   // [n_cal] or null
};

// One (sequence, head, query block) unit: the tiled online-softmax walk.
void walk_unit(const Problem& P, int seq, int head, int qb, int mode, float L, const float* Lcal, int n_cal,
               const int8_t* forced, int max_tiles, const UnitResult& R) {
  const int64_t base = P.cu[seq];
  const int S = P.cu[seq + 1] - P.cu[seq];
  const int D = P.D, H = P.H;
  const int r0 = qb * kTile, r1 = std::min(r0 + kTile, S);
  const int nrows = r1 - r0;
  const int ntiles = (S + kTile - 1) / kTile;
  const float inf = std::numeric_limits<float>::infinity();

  std::vector<double> qrow(static_cast<size_t>(nrows) * D);
  for (int r = 0; r < nrows; ++r)
    for (int d = 0; d < D; ++d)
      qrow[static_cast<size_t>(r) * D + d] = bf16_to_double(P.q[((base + r0 + r) * H + head) * D + d]);

  std::vector<float> m(nrows, -inf);
  std::vector<double> l(nrows, 0.0), O(static_cast<size_t>(nrows) * D, 0.0);
  std::vector<double> ref(nrows, -std::numeric_limits<double>::infinity());  // integer reference (8-bit P)
  std::vector<float> s2(static_cast<size_t>(nrows) * kTile);
  std::vector<double> kcol(D), vrow(D);
  int skips = 0;
  std::vector<int32_t> counts(std::max(n_cal, 0), 0);

  for (int j = 0; j < ntiles; ++j) {
    const int c0 = j * kTile, c1 = std::min(c0 + kTile, S);
    // Scores of the tile, log2 domain, fp32.
    for (int c = c0; c < c1; ++c) {
      for (int d = 0; d < D; ++d) kcol[d] = bf16_to_double(P.k[((base + c) * H + head) * D + d]);
      for (int r = 0; r < nrows; ++r) {
        double dot = 0.0;
        const double* qr = &qrow[static_cast<size_t>(r) * D];
        for (int d = 0; d < D; ++d) dot += qr[d] * kcol[d];
        const float sf = static_cast<float>(dot);
        s2[static_cast<size_t>(r) * kTile + (c - c0)] = sf * P.c;
      }
    }
    // Row maxima of the tile and the tile statistic against the running max.
    std::vector<float> tmax(nrows, -inf);
    for (int r = 0; r < nrows; ++r)
      for (int c = c0; c < c1; ++c) tmax[r] = std::max(tmax[r], s2[static_cast<size_t>(r) * kTile + (c - c0)]);
    float dj = -inf;
    for (int r = 0; r < nrows; ++r) {
      const float diff = tmax[r] - m[r];  // fp32 subtraction; +inf while m = -inf
      dj = std::max(dj, diff);
    }
    if (R.dstat) R.dstat[j] = dj;

    bool skip = false;
    if (mode == 0) {
      skip = dj < L;
      if (forced && forced[j] >= 0) skip = forced[j] != 0;
    } else {
      for (int kk = 0; kk < n_cal; ++kk)
        if (dj < Lcal[kk]) ++counts[kk];
    }
    if (R.decision) R.decision[j] = skip ? 1 : 0;
    if (skip) {
      ++skips;
      continue;
    }
    // Online softmax update with this tile.
    for (int r = 0; r < nrows; ++r) {
      const float mn = std::max(m[r], tmax[r]);
      double* orow = &O[static_cast<size_t>(r) * D];
      // reference the probabilities are taken against, and the O/l rescale
      double refp = mn, alpha = std::exp2(static_cast<double>(m[r]) - static_cast<double>(mn));  // 0 when m = -inf
      if (P.p_e4m3) {
        alpha = 1.0;
        if (std::isinf(ref[r]) || static_cast<double>(mn) > ref[r] + P.p_lag) {
          const double nr = std::ceil(static_cast<double>(mn));
          alpha = std::isinf(ref[r]) ? 0.0 : std::exp2(ref[r] - nr);
          ref[r] = nr;
        }
        refp = ref[r] - P.p_shift;
      }
      double rowsum = 0.0;
      for (int d = 0; d < D; ++d) orow[d] *= alpha;
      for (int c = c0; c < c1; ++c) {
        const double p = std::exp2(static_cast<double>(s2[static_cast<size_t>(r) * kTile + (c - c0)]) - refp);
        rowsum += p;
        const double pv = P.p_e4m3 ? e4m3_nearest(p) : p;  // the factor the P.V product uses
        const uint16_t* vr = &P.v[((base + c) * H + head) * D];
        for (int d = 0; d < D; ++d) orow[d] += pv * bf16_to_double(vr[d]);
      }
      l[r] = l[r] * alpha + rowsum;
      m[r] = mn;
    }
  }
  for (int j = ntiles; j < max_tiles; ++j) {
    if (R.dstat) R.dstat[j] = std::numeric_limits<float>::quiet_NaN();
    if (R.decision) R.decision[j] = 0;
  }
  for (int r = 0; r < kTile; ++r)
    for (int d = 0; d < D; ++d)
      R.out[static_cast<size_t>(r) * D + d] =
          r < nrows ? static_cast<float>(O[static_cast<size_t>(r) * D + d] / l[r] * P.out_scale) : 0.0f;
  if (R.skips) *R.skips = skips;
  if (R.counts)
    for (int kk = 0; kk < n_cal; ++kk) R.counts[kk] = counts[kk];
}

}  // namespace

extern "C" {

// L = fp32(log2(tsf / s_kv)); tsf <= 0 (or s_kv <= 0) gives -inf: the dense path.
float oracle_threshold_log2(double threshold_scale_factor, int64_t s_kv) {
  if (!(threshold_scale_factor > 0.0) || s_kv <= 0) return -std::numeric_limits<float>::infinity();
  return static_cast<float>(std::log2(threshold_scale_factor / static_cast<double>(s_kv)));
}

// L for a raw lambda (calibration trials): fp32(log2(lambda)).
float oracle_lambda_log2(double lambda) {
  if (!(lambda > 0.0)) return -std::numeric_limits<float>::infinity();
  return static_cast<float>(std::log2(lambda));
}

// fp32(softmax_scale * log2 e); softmax_scale <= 0 means 1/sqrt(D).
float oracle_score_scale(double softmax_scale, int D) {
  const double s = softmax_scale > 0.0 ? softmax_scale : 1.0 / std::sqrt(static_cast<double>(D));
  return static_cast<float>(s * kLog2e);
}

// threshold_scale_factor = a * exp(b * target_sparsity) (Model-Optimizer README,
// "Calibrated threshold"; TRT-LLM docs, "Checkpoint Config"). NaN when a <= 0,
// s outside [0, 1] or any argument is not finite.
double oracle_resolve(double a, double b, double s) {
  if (!(a > 0.0) || !std::isfinite(a) || !std::isfinite(b) || !(s >= 0.0 && s <= 1.0))
    return std::numeric_limits<double>::quiet_NaN();
  return a * std::exp(b * s);
}

// Log-space least squares of ln(scale_factor) = ln(a) + b * s (commit page,
// "Calibration": fit_logspace minimises relative error). Points with s outside
// the open interval (0, 1) or scale_factor <= 0 carry no information and are
// dropped. Returns 0, or -1 when fewer than two distinct s remain.
int oracle_fit_logspace(const double* s, const double* sf, int n, double* a, double* b, double* s_min,
                        double* s_max) {
  std::vector<double> x, y;
  for (int i = 0; i < n; ++i) {
    if (!(s[i] > 0.0 && s[i] < 1.0) || !(sf[i] > 0.0) || !std::isfinite(sf[i])) continue;
    x.push_back(s[i]);
    y.push_back(std::log(sf[i]));
  }
  if (x.size() < 2) return -1;
  double mx = 0, my = 0;
  for (size_t i = 0; i < x.size(); ++i) { mx += x[i]; my += y[i]; }
  mx /= x.size();
  my /= x.size();
  double sxx = 0, sxy = 0;
  for (size_t i = 0; i < x.size(); ++i) {
    sxx += (x[i] - mx) * (x[i] - mx);
    sxy += (x[i] - mx) * (y[i] - my);
  }
  if (!(sxx > 0.0)) return -1;
  const double bb = sxy / sxx;
  *b = bb;
  *a = std::exp(my - bb * mx);
  *s_min = *std::min_element(x.begin(), x.end());
  *s_max = *std::max_element(x.begin(), x.end());
  return 0;
}

// Nearest E4M3 value (exported for its pins).
double oracle_e4m3_nearest(double x) { return e4m3_nearest(x); }

// Walk a list of (sequence, head, query-block) units.
//   mode 0: forward with skipping; L_seq[b] is sequence b's threshold.
//   mode 1: calibration; never skips, counts d < L_cal[k] for each k.
// forced (nullable, [n_units][max_tiles]): -1 decide, 0 keep, 1 skip (mode 0).
// Outputs per unit: out [128][D] fp32 (rows past the end are 0), dstat
// [max_tiles] (+inf at tile 0, NaN past the end), decision [max_tiles],
// skips, counts [n_cal]. p_e4m3 selects the 8-bit P.V reading (p_shift =
// sigma, p_lag = tau); out_scale multiplies every output (1 for bf16 V).
// Returns 0, or -1 on a bad argument.
int oracle_walk(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_seqlens, int batch,
                int H, int D, double softmax_scale, int mode, const float* L_seq, const float* L_cal, int n_cal,
                int n_units, const int32_t* units, int max_tiles, const int8_t* forced, float* out, float* dstat,
                uint8_t* decision, int32_t* skips, int32_t* cal_counts, int p_e4m3, double p_shift, double p_lag,
                double out_scale, int nthreads) {
  if (!q || !k || !v || !cu_seqlens || !units || !out || batch <= 0 || H <= 0 || D <= 0) return -1;
  if (p_e4m3 && !(p_lag >= 0.0 && std::isfinite(p_shift))) return -1;
  if (mode == 0 && !L_seq) return -1;
  if (mode == 1 && (n_cal <= 0 || !L_cal)) return -1;
  for (int i = 0; i < n_units; ++i) {
    const int sq = units[3 * i], hd = units[3 * i + 1], qb = units[3 * i + 2];
    if (sq < 0 || sq >= batch || hd < 0 || hd >= H || qb < 0) return -1;
    const int S = cu_seqlens[sq + 1] - cu_seqlens[sq];
    if (qb * kTile >= S || (S + kTile - 1) / kTile > max_tiles) return -1;
  }
  Problem P{q, k, v, cu_seqlens, batch, H, D, oracle_score_scale(softmax_scale, D), p_e4m3, p_shift, p_lag, out_scale};
  std::atomic<int> next{0};
  auto worker = [&]() {
    for (int i = next++; i < n_units; i = next++) {
      UnitResult R{out + static_cast<size_t>(i) * kTile * D,
                   dstat ? dstat + static_cast<size_t>(i) * max_tiles : nullptr,
                   decision ? decision + static_cast<size_t>(i) * max_tiles : nullptr,
                   skips ? skips + i : nullptr,
                   (mode == 1 && cal_counts) ? cal_counts + static_cast<size_t>(i) * n_cal : nullptr};
      const int sq = units[3 * i];
      walk_unit(P, sq, units[3 * i + 1], units[3 * i + 2], mode, mode == 0 ? L_seq[sq] : 0.0f, L_cal, n_cal,
                forced ? forced + static_cast<size_t>(i) * max_tiles : nullptr, max_tiles, R);
    }
  };
  const int nt = std::max(1, std::min(nthreads, n_units));
  std::vector<std::thread> th;
  for (int t = 1; t < nt; ++t) th.emplace_back(worker);
  worker();
  for (auto& t : th) t.join();
  return 0;
}

}  // extern "C"
