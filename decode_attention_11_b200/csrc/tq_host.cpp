// Host-side parts of the tq C ABI: status strings, thread-local error detail, argument
// validation, and the Lloyd-Max codebook builder.
#include <cfenv>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "tq_internal.h"

namespace tq {

static thread_local std::string g_last_error;

tq_status fail(tq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

void clear_error() { g_last_error.clear(); }

NvtxRange::NvtxRange(const char* name) { nvtxRangePushA(name); }
NvtxRange::~NvtxRange() { nvtxRangePop(); }

tq_status check_cache(const tq_cache* c) {
  if (!c) return fail(TQ_ERR_INVALID_ARG, "cache is NULL");
  if (c->head_dim != kHeadDim) return fail(TQ_ERR_UNSUPPORTED, "head_dim %d (only 128)", c->head_dim);
  if (c->k_bits < 2 || c->k_bits > 4 || c->v_bits < 2 || c->v_bits > 4)
    return fail(TQ_ERR_UNSUPPORTED, "k_bits %d / v_bits %d (2..4)", c->k_bits, c->v_bits);
  if (c->qjl_m != 0 && c->qjl_m != kQjlRows)
    return fail(TQ_ERR_UNSUPPORTED, "qjl_m %d (0 or 128)", c->qjl_m);
  if (c->layout != TQ_LAYOUT_PLAIN && c->layout != TQ_LAYOUT_MIXED)
    return fail(TQ_ERR_UNSUPPORTED, "layout %d", c->layout);
  if (c->layout == TQ_LAYOUT_MIXED && (c->k_bits != 4 || c->v_bits != 4))
    return fail(TQ_ERR_UNSUPPORTED, "mixed layout with k_bits %d / v_bits %d (only 4 / 4: halves of 4 and 3 bits)",
                c->k_bits, c->v_bits);
  if (c->B < 1 || c->Hkv < 1 || c->T_cap < 1)
    return fail(TQ_ERR_INVALID_ARG, "cache shape B=%d Hkv=%d T_cap=%d", c->B, c->Hkv, c->T_cap);
  if ((int64_t)c->B * c->Hkv * c->T_cap > (int64_t)1 << 40)
    return fail(TQ_ERR_INVALID_ARG, "cache too large");
  if (!c->k_codes || !c->k_norm || !c->v_codes || !c->v_norm)
    return fail(TQ_ERR_INVALID_ARG, "cache array is NULL");
  if (c->qjl_m && (!c->k_signs || !c->k_rnorm))
    return fail(TQ_ERR_INVALID_ARG, "k_signs / k_rnorm NULL with qjl_m=%d", c->qjl_m);
  if (!aligned16(c->k_codes) || !aligned16(c->k_norm) || !aligned16(c->v_codes) ||
      !aligned16(c->v_norm) || (c->qjl_m && (!aligned16(c->k_signs) || !aligned16(c->k_rnorm))))
    return fail(TQ_ERR_INVALID_ARG, "cache arrays must be 16-byte aligned");
  return TQ_OK;
}

tq_status check_params(const tq_params* p, const tq_cache* c) {
  if (!p) return fail(TQ_ERR_INVALID_ARG, "params is NULL");
  if (!p->Pi || !p->k_centroids || !p->k_thresholds || !p->v_centroids || !p->v_thresholds)
    return fail(TQ_ERR_INVALID_ARG, "params array is NULL");
  if (c->qjl_m && !p->S) return fail(TQ_ERR_INVALID_ARG, "S is NULL with qjl_m=%d", c->qjl_m);
  if (!aligned16(p->Pi) || (c->qjl_m && !aligned16(p->S)) || !aligned16(p->S_Pi))
    return fail(TQ_ERR_INVALID_ARG, "Pi / S / S_Pi must be 16-byte aligned");
  if (c->layout == TQ_LAYOUT_MIXED) {
    if (!p->k_centroids_lo || !p->k_thresholds_lo || !p->v_centroids_lo || !p->v_thresholds_lo)
      return fail(TQ_ERR_INVALID_ARG, "mixed layout: a codebook of the non-outlier half is NULL");
    int bits = 0;
    for (int w = 0; w < 4; ++w) bits += __builtin_popcount(p->outlier_mask[w]);
    if (bits != kHeadDim / 2)
      return fail(TQ_ERR_INVALID_ARG, "mixed layout: outlier_mask has %d channels (needs %d)", bits, kHeadDim / 2);
  }
  return TQ_OK;
}

// ---------------------------------------------------------------------------------------------
// Lloyd-Max quantizer of N(0,1).
// ai-news.ru overview, "second idea": for a known distribution the optimal (non-uniform) grid is
// computed once in advance; tproger.ru "Step 1: PolarQuant": applied to every coordinate.
// ---------------------------------------------------------------------------------------------

static double normal_pdf(double x) {
  if (std::isinf(x)) return 0.0;
  return std::exp(-0.5 * x * x) * 0.39894228040143267794;  // 1/sqrt(2 pi)
}

static double normal_cdf(double x) {
  if (x == INFINITY) return 1.0;
  if (x == -INFINITY) return 0.0;
  return 0.5 * std::erfc(-x * 0.70710678118654752440);
}

// Quantile by bisection on the cdf (only used for the starting grid).
static double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

// Round a double to the nearest fp16 value (ties to even), for |x| in the normal fp16 range.
static double round_to_half(double x) {
  if (x == 0.0) return 0.0;
  int e;
  const double m = std::frexp(x, &e);         // x = m * 2^e, 0.5 <= |m| < 1
  const double scaled = std::ldexp(m, 11);    // 11 significant bits
  const int old = std::fegetround();
  std::fesetround(FE_TONEAREST);
  const double r = std::nearbyint(scaled);
  std::fesetround(old);
  return std::ldexp(r, e - 11);
}

}  // namespace tq

extern "C" {

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG: invalid argument";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED: unsupported configuration";
    case TQ_ERR_NO_CONVERGENCE: return "TQ_ERR_NO_CONVERGENCE: Lloyd iteration did not converge";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE: workspace too small";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA: CUDA runtime error";
    default: return "unknown tq_status";
  }
}

const char* tq_last_error(void) { return tq::g_last_error.c_str(); }

int tq_version(void) { return 100; }

tq_status tq_build_codebook(int bits, int max_iter, double tol, float* centroids,
                            float* thresholds, double* distortion) {
  using namespace tq;
  clear_error();
  if (bits < 1 || bits > 8) return fail(TQ_ERR_INVALID_ARG, "bits %d (1..8)", bits);
  if (max_iter < 1 || !(tol > 0.0)) return fail(TQ_ERR_INVALID_ARG, "max_iter/tol");
  if (!centroids || !thresholds) return fail(TQ_ERR_INVALID_ARG, "output array is NULL");
  const int L = 1 << bits;
  std::vector<double> c(L), t(L + 1), next(L);
  for (int k = 0; k < L; ++k) c[k] = normal_quantile((k + 0.5) / L);
  bool converged = false;
  for (int it = 0; it < max_iter; ++it) {
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int i = 1; i < L; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
    double move = 0.0;
    for (int k = 0; k < L; ++k) {
      // centroid condition: conditional mean of N(0,1) on [t_k, t_{k+1})
      next[k] = (normal_pdf(t[k]) - normal_pdf(t[k + 1])) / (normal_cdf(t[k + 1]) - normal_cdf(t[k]));
      move = std::fmax(move, std::fabs(next[k] - c[k]));
    }
    c.swap(next);
    if (move < tol) { converged = true; break; }
  }
  if (!converged) return fail(TQ_ERR_NO_CONVERGENCE, "bits=%d after %d iterations", bits, max_iter);
  for (int k = 0; k < L / 2; ++k) {  // exact symmetry
    const double s = 0.5 * (c[L - 1 - k] - c[k]);
    c[L - 1 - k] = s;
    c[k] = -s;
  }
  if (distortion) {
    double acc = 0.0;
    for (int k = 0; k < L; ++k) {
      const double lo = k == 0 ? -INFINITY : 0.5 * (c[k - 1] + c[k]);
      const double hi = k == L - 1 ? INFINITY : 0.5 * (c[k] + c[k + 1]);
      acc += (normal_cdf(hi) - normal_cdf(lo)) * c[k] * c[k];
    }
    *distortion = 1.0 - acc;
  }
  std::vector<double> stored(L);
  for (int k = 0; k < L; ++k) stored[k] = round_to_half(c[k]);
  for (int k = 0; k < L; ++k) centroids[k] = (float)stored[k];
  for (int i = 0; i + 1 < L; ++i) {
    const double mid = 0.5 * (stored[i] + stored[i + 1]);
    if ((double)(float)mid != mid) return fail(TQ_ERR_NO_CONVERGENCE, "midpoint not exact in fp32");
    thresholds[i] = (float)mid;
  }
  return TQ_OK;
}

// Structured rotation D1 H D2 H D3 / 128 (see tq.h).  Signs from SplitMix64 (Steele, Lea and
// Flood, OOPSLA 2014): output n of a generator started at `seed`.
tq_status tq_build_hadamard_rotation(uint64_t seed, float* Pi) {
  tq::clear_error();
  if (!Pi) return tq::fail(TQ_ERR_INVALID_ARG, "Pi is NULL");
  constexpr int d = tq::kHeadDim;
  auto splitmix = [seed](uint64_t n) {
    uint64_t z = seed + (n + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  };
  auto had = [](int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1; };
  int sgn[3][d];
  for (int k = 0; k < 3; ++k)
    for (int i = 0; i < d; ++i) sgn[k][i] = (splitmix((uint64_t)(k * d + i)) & 1) ? -1 : 1;
  // (D1 H D2 H D3)[i][j] = s1[i] s3[j] sum_m H[i][m] s2[m] H[m][j]: an integer, exact in fp32
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      int acc = 0;
      for (int m = 0; m < d; ++m) acc += had(i, m) * sgn[1][m] * had(m, j);
      Pi[i * d + j] = (float)(sgn[0][i] * sgn[2][j] * acc) / (float)d;
    }
  return TQ_OK;
}

}  // extern "C"
