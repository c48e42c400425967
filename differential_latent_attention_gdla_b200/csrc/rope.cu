// rope.cu -- the RoPE cos/sin tables the kernels take as inputs, built on the
// host in double precision (model set-up, like loading weights; not part of a
// forward call).
//
// RoPE ("Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and
// Motif-2", section 2, the rotation-matrix equation): the pair of rotary
// dimensions (k, k + d_R/2) of a token at position m is rotated by the angle
// m * theta_k with theta_k = base^(-2k/d_R) (rotate-half pairing).
//
// YaRN (same section, the three-regime Scale(i) equation): extending a model
// trained on L_orig tokens by a factor s multiplies each frequency by a scale
// chosen from the band its wavelength lambda_k = 2 pi / theta_k falls in:
//   lambda_k < L_orig / beta_fast   scale 1         (high frequencies, kept)
//   lambda_k > L_orig / beta_slow   scale 1 / s     (low frequencies, interpolated)
//   in between                      scale (1 - a) + a / s, with the blend a
//                                   growing linearly with the wavelength from 0
//                                   at the lower edge to 1 at the upper edge.
// The logit temperature belongs to the softmax scale, not to the tables.
#include <math.h>

#include "../../include/gdla.h"

namespace {

// The YaRN scale of one frequency band.
double yarn_band_scale(double wavelength, double lo_edge, double hi_edge, double factor) {
  if (wavelength < lo_edge) return 1.0;
  if (wavelength > hi_edge) return 1.0 / factor;
  if (hi_edge <= lo_edge) return 1.0;  // an empty middle band: the wavelength sits on the edge
  const double a = (wavelength - lo_edge) / (hi_edge - lo_edge);
  return (1.0 - a) + a / factor;
}

void fill_tables(int max_pos, int half, const double* theta, float* cos_tab, float* sin_tab) {
  for (long p = 0; p < max_pos; ++p)
    for (int k = 0; k < half; ++k) {
      const double ang = (double)p * theta[k];
      cos_tab[p * half + k] = (float)cos(ang);
      sin_tab[p * half + k] = (float)sin(ang);
    }
}

constexpr int kMaxHalf = 512;

}  // namespace

extern "C" {

gdla_status gdla_rope_tables(int max_pos, int d_rope, double base, float* cos_tab, float* sin_tab) {
  if (max_pos < 1 || d_rope < 2 || d_rope % 2 || d_rope / 2 > kMaxHalf || !(base > 1.0) || !cos_tab || !sin_tab)
    return GDLA_ERR_INVALID_ARG;
  const int half = d_rope / 2;
  double theta[kMaxHalf];
  for (int k = 0; k < half; ++k) theta[k] = pow(base, -2.0 * k / (double)d_rope);
  fill_tables(max_pos, half, theta, cos_tab, sin_tab);
  return GDLA_OK;
}

gdla_status gdla_yarn_rope_tables(int max_pos, int d_rope, double base, double factor, int original_max_pos,
                                  double beta_fast, double beta_slow, float* cos_tab, float* sin_tab) {
  if (max_pos < 1 || d_rope < 2 || d_rope % 2 || d_rope / 2 > kMaxHalf || !(base > 1.0) || !(factor > 0.0) ||
      original_max_pos < 1 || !(beta_fast > 0.0) || !(beta_slow > 0.0) || !cos_tab || !sin_tab)
    return GDLA_ERR_INVALID_ARG;
  const int half = d_rope / 2;
  const double lo_edge = original_max_pos / beta_fast, hi_edge = original_max_pos / beta_slow;
  const double two_pi = 2.0 * acos(-1.0);
  double theta[kMaxHalf];
  for (int k = 0; k < half; ++k) {
    const double t = pow(base, -2.0 * k / (double)d_rope);
    theta[k] = t * yarn_band_scale(two_pi / t, lo_edge, hi_edge, factor);
  }
  fill_tables(max_pos, half, theta, cos_tab, sin_tab);
  return GDLA_OK;
}

double gdla_yarn_mscale(double factor) { return factor > 1.0 ? 1.0 + 0.1 * log(factor) : 1.0; }

}  // extern "C"
