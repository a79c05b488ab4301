// Power-spaced selection of the past latent frames kept resident by the
// bounded-history path (host code).
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "The 4090 preset": with T past latent frames
// and a budget N = min(budget, T), frame distances from the newest frame are
// d_i = i + rint((T - N) * u_i^gamma), u_i = i / (N - 1), and the kept frames
// are T - 1 - d_i; d always ends at T - 1, so frame 0 is always kept.  rint
// rounds half to even (the default rounding mode).  For N = 1, u_0 is taken
// as 0.  The output feeds nomas_kvcache_select.
#include <cfenv>
#include <cmath>

#include "nomas.h"

extern "C" nomas_status nomas_temporal_context_frames(int32_t n_past, int32_t budget,
                                                      float gamma, int32_t *out,
                                                      int32_t out_capacity, int32_t *n_out) {
  if (n_out == nullptr) return NOMAS_ERR_INVALID_ARG;
  *n_out = 0;
  if (n_past < 0 || budget < 0 || !(gamma >= 0.f) || !std::isfinite(gamma))
    return NOMAS_ERR_INVALID_ARG;
  const int32_t n = budget < n_past ? budget : n_past;
  if (n == 0) return NOMAS_OK;
  if (out == nullptr || out_capacity < n) return NOMAS_ERR_CAPACITY;
  const int saved = std::fegetround();
  std::fesetround(FE_TONEAREST);
  // d_i grows with i, so writing T - 1 - d_i from the last i down gives an
  // ascending list.
  for (int32_t i = 0; i < n; ++i) {
    const double u = n > 1 ? (double)i / (double)(n - 1) : 0.0;
    const double d = (double)i + std::rint((double)(n_past - n) * std::pow(u, (double)gamma));
    out[n - 1 - i] = (int32_t)((double)(n_past - 1) - d);
  }
  std::fesetround(saved);
  *n_out = n;
  return NOMAS_OK;
}
