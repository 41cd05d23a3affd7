// Span rule of MoA ("Mixture of Attention" project page, "Finding two":
// S = alpha + beta * N; "Method design / Elastic search space": spans respect
// the kernel's block size; heads A/B/C panel: a span longer than the input is
// clamped to it).  Host code, compiled with -ffp-contract=off so that beta*N
// and the following addition round separately, as the C ABI documents.
#include <cmath>

#include "internal.h"

extern "C" moa_status moa_rules_eval(const double* alpha, const double* beta, int32_t n_heads,
                                     int64_t N, int32_t block, int32_t* spans_out) {
  if (!alpha || !beta || !spans_out || n_heads < 1) return MOA_ERR_INVALID_ARG;
  if (N < 1 || N > INT32_MAX || block < 1) return MOA_ERR_INVALID_ARG;
  for (int32_t h = 0; h < n_heads; ++h) {
    const double a = alpha[h], b = beta[h];
    if (!std::isfinite(a) || !std::isfinite(b) || a < 0.0 || b < 0.0) return MOA_ERR_INVALID_ARG;
  }
  const double n = (double)N;
  const double bs = (double)block;
  for (int32_t h = 0; h < n_heads; ++h) {
    volatile double prod = beta[h] * n;   // first rounding
    volatile double x = alpha[h] + prod;  // second rounding
    volatile double r = x / bs;
    volatile double r_half = r + 0.5;
    double s = bs * std::floor(r_half);   // nearest multiple of the block, ties up
    if (s < bs) s = bs;                   // at least one block
    if (s > n) s = n;                     // never longer than the input
    spans_out[h] = (int32_t)s;
  }
  return MOA_OK;
}
