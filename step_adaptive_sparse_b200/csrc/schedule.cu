// Host-side AReA schedule: the Phase I pooling ramp, the Phase II window
// sides, the noise-level switch between the two phases and the lattice of
// the global-KV bridge.  Pure host arithmetic (no device code); the attention
// calls of each step are issued by the caller on its stream.
//
// Pages:
//   ai.info summary, "Methodology in Plain English": Phase I (the pooling
//     factor ramps down linearly from f0 to a floor f_min = 2, each value
//     snapped to a valid grid divisor), Phase II (windows shrink
//     geometrically from w_start to w_min; bridge R = (rho w)^2, rho = 0.5),
//     "Scheduling the switch" (Phase I ends at a noise level sigma*, not at a
//     step count; in practice the first 8 of FLUX.1's steps);
//   gpt-diffusion.com, "Las dos fases de AReA" (the ramp [4,4,4,4,2,2,2,2] at a
//     256 x 256 patch grid);
//   github.com/KooroshRH/AReA wiki, usage notes (sigma* between 0.86 and
//     0.96 for the tuned models; 28 sampling steps in the FLUX.1 example).
#include <math.h>

#include "area.h"

extern "C" {

int area_pool_ramp(int f0, int f_min, int steps, int Hg, int Wg, int* ramp) {
  if (!ramp || steps < 1 || f0 < 1 || f_min < 1 || Hg < 1 || Wg < 1) return AREA_EINVAL;
  const int lim = Hg < Wg ? Hg : Wg;
  for (int t = 0; t < steps; ++t) {
    const double frac = steps > 1 ? (double)t / (double)(steps - 1) : 0.0;
    const double target = (double)f0 + (double)(f_min - f0) * frac;
    int best = 1;
    double bd = fabs(1.0 - target);
    for (int d = 2; d <= lim; ++d) {
      if (Hg % d || Wg % d) continue;
      const double dd = fabs((double)d - target);
      if (dd <= bd) {                     // equal distance: the larger divisor
        best = d;
        bd = dd;
      }
    }
    ramp[t] = best;
  }
  return AREA_OK;
}

int area_window_sides(int w0, int w_min, int steps, int* sides) {
  if (!sides || steps < 1 || w0 < 1 || w_min < 1) return AREA_EINVAL;
  for (int t = 0; t < steps; ++t) {
    const double e = steps > 1 ? (double)t / (double)(steps - 1) : 0.0;
    const double w = (double)w0 * pow((double)w_min / (double)w0, e);
    const int r = 8 * (int)floor(w / 8.0 + 0.5);
    sides[t] = r > 0 ? r : 8;
  }
  return AREA_OK;
}

int area_bridge_lattice(int w, int Hg, int Wg, int* ry, int* rx) {
  if (!ry || !rx || w < 1 || Hg < 1 || Wg < 1) return AREA_EINVAL;
  const int hy = w < Hg ? w : Hg, wx = w < Wg ? w : Wg;
  int a = (int)floor(0.5 * hy + 0.5), b = (int)floor(0.5 * wx + 0.5);
  a = a < 1 ? 1 : (a > Hg ? Hg : a);
  b = b < 1 ? 1 : (b > Wg ? Wg : b);
  *ry = a;
  *rx = b;
  return AREA_OK;
}

int area_phase_switch(const float* sigmas, int steps, float sigma_star, int* n_phase1) {
  if (!sigmas || !n_phase1 || steps < 0) return AREA_EINVAL;
  int n = 0;
  while (n < steps && sigmas[n] >= sigma_star) ++n;
  *n_phase1 = n;
  return AREA_OK;
}

int area_schedule(const float* sigmas, int steps, float sigma_star, int f0, int f_min, int w0,
                  int w_min, int Hg, int Wg, int* kind, int* param) {
  if (!sigmas || !kind || !param || steps < 1) return AREA_EINVAL;
  int n1 = 0;
  int st = area_phase_switch(sigmas, steps, sigma_star, &n1);
  if (st != AREA_OK) return st;
  if (n1 > 0) {
    st = area_pool_ramp(f0, f_min, n1, Hg, Wg, param);
    if (st != AREA_OK) return st;
    for (int t = 0; t < n1; ++t) kind[t] = AREA_PHASE_COARSE;
  }
  if (steps > n1) {
    st = area_window_sides(w0, w_min, steps - n1, param + n1);
    if (st != AREA_OK) return st;
    for (int t = n1; t < steps; ++t) kind[t] = AREA_PHASE_WINDOW;
  }
  return AREA_OK;
}

}  // extern "C"
