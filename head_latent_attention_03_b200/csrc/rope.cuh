// rope.cuh — rotary frequencies of the decoupled RoPE carrier (q^R, k^R).
//
// DeepSeek-V2 explainer (adg.csdn.net) section 2.2.2: RoPE rides on extra
// per-head queries q^R and one shared key k^R; section 3.1.3: YaRN (scale s,
// alpha, beta over the original 4K window) is applied to that key.
// Pair k of a d_h^R-wide vector turns by pos * theta_k with
// theta_k = base^(-2k/d_h^R); with YaRN, pairs whose rotation count r_k over
// the original window is below alpha are slowed by s, above beta kept, and
// blended linearly in between ("NTK-by-parts").  Angles are formed in fp64:
// at position 131072 an fp32 product pos * theta would be off by ~1e-2 rad.
#pragma once

#include <math.h>

namespace mla {

struct RopeParams {
  double base, yarn_scale, yarn_alpha, yarn_beta;
  int yarn_orig_ctx;
};

__host__ __device__ inline double rope_theta(const RopeParams& rp, int d_hr, int k) {
  const double theta = pow(rp.base, -2.0 * (double)k / (double)d_hr);
  if (rp.yarn_scale == 1.0) return theta;
  const double turns = (double)rp.yarn_orig_ctx * theta / (2.0 * 3.14159265358979323846);
  if (turns < rp.yarn_alpha) return theta / rp.yarn_scale;
  if (turns > rp.yarn_beta) return theta;
  const double g = (turns - rp.yarn_alpha) / (rp.yarn_beta - rp.yarn_alpha);
  return (1.0 - g) * theta / rp.yarn_scale + g * theta;
}

__device__ inline void rope_cos_sin_theta(double theta, long long pos, float* c, float* s) {
  double sd, cd;
  sincos((double)pos * theta, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

__device__ inline void rope_cos_sin(const RopeParams& rp, int d_hr, int k, long long pos, float* c, float* s) {
  rope_cos_sin_theta(rope_theta(rp, d_hr, k), pos, c, s);
}

// Frequencies theta_k of one layer, computed once on the host (fp64).
constexpr int ROPE_MAX_PAIRS = 64;
struct RopeTable {
  double theta[ROPE_MAX_PAIRS];
};
inline RopeTable rope_table(const RopeParams& rp, int d_hr) {
  RopeTable t{};
  for (int k = 0; k < d_hr / 2 && k < ROPE_MAX_PAIRS; ++k) t.theta[k] = rope_theta(rp, d_hr, k);
  return t;
}

// cos/sin of pos * theta for the bf16 path: the angle is formed in fp64 and
// reduced modulo 2 pi with Cody and Waite's two-constant scheme (2 pi split
// into a double head and the double nearest to the remainder), then the
// reduced angle in [-pi, pi] goes to the fp32 hardware sine/cosine, whose
// absolute error on that interval is about 4e-7 — far below bf16
// resolution, at a fraction of an fp64 sincos.
__device__ inline void rope_cos_sin_reduced(double theta, long long pos, float* c, float* s) {
  constexpr double kTwoPiHead = 6.283185307179586;        // 2 pi rounded to double
  constexpr double kTwoPiTail = 2.4492935982947064e-16;   // 2 pi - kTwoPiHead
  constexpr double kInvTwoPi = 0.15915494309189535;       // 1 / (2 pi)
  const double a = (double)pos * theta;
  const double n = rint(a * kInvTwoPi);
  double r = fma(-n, kTwoPiHead, a);
  r = fma(-n, kTwoPiTail, r);
  __sincosf((float)r, s, c);
}

}  // namespace mla
