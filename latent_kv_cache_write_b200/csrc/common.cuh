// Shared device helpers: storage-type loads/stores, token positions, RoPE angles,
// and the library's device-side error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

using bf16 = __nv_bfloat16;

// Codes OR-ed into the library's device-side error word (defined in mla_api.cu and
// handed to kernels as a pointer) by a kernel that gave up a bounded wait.
enum : unsigned int { kErrNone = 0, kErrTimeout = 1 };

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// Geometry of one problem, copied by value into kernels.
struct Geo {
  int32_t B, H, Dn, Dc, Dr;   // batch, heads, d_nope, d_latent, d_rope
  int32_t pairs[3];           // rope pairs on t, y, x
  double theta;
  int32_t gh, gw;             // frame grid
  int64_t F;                  // tokens per frame
  int64_t S;                  // ring slots
  int32_t row;                // d_latent + d_rope
};

// RoPE angle of rope pair p (0 <= p < d_rope/2) for global token g.
// Pair j of an axis segment holding n pairs turns by pos * theta^(-j/n).
__device__ __forceinline__ double rope_angle(const Geo& G, int64_t g, int p) {
  int64_t t = g / G.F;
  int64_t r = g - t * G.F;
  int64_t y = r / G.gw;
  int64_t x = r - y * G.gw;
  int64_t pos;
  int j, n;
  if (p < G.pairs[0]) {
    pos = t; j = p; n = G.pairs[0];
  } else if (p < G.pairs[0] + G.pairs[1]) {
    pos = y; j = p - G.pairs[0]; n = G.pairs[1];
  } else {
    pos = x; j = p - G.pairs[0] - G.pairs[1]; n = G.pairs[2];
  }
  return (double)pos * pow(G.theta, -(double)j / (double)n);
}

// Rotate the pair (a, b) by angle ang: (a cos - b sin, a sin + b cos).
__device__ __forceinline__ void rope_rotate(float& a, float& b, double ang) {
  double s, c;
  sincos(ang, &s, &c);
  double na = (double)a * c - (double)b * s;
  double nb = (double)a * s + (double)b * c;
  a = (float)na;
  b = (float)nb;
}

// The three axis positions (t, y, x) of token g, as doubles, computed once per token;
// rope_axis_pos picks the one RoPE pair p turns by.
struct RopeAxes {
  double t, y, x;
};
__device__ __forceinline__ RopeAxes rope_axes(const Geo& G, int64_t g) {
  const int64_t t = g / G.F;
  const int64_t r = g - t * G.F;
  const int64_t y = r / G.gw;
  return RopeAxes{(double)t, (double)y, (double)(r - y * G.gw)};
}
__device__ __forceinline__ double rope_axis_pos(const Geo& G, const RopeAxes& ax, int p) {
  return p < G.pairs[0] ? ax.t : (p < G.pairs[0] + G.pairs[1] ? ax.y : ax.x);
}
// The frequency theta^(-j/n) of RoPE pair p (pair j of an axis segment with n pairs).
__device__ __forceinline__ double rope_inv_freq(const Geo& G, int p) {
  int j, n;
  if (p < G.pairs[0]) {
    j = p; n = G.pairs[0];
  } else if (p < G.pairs[0] + G.pairs[1]) {
    j = p - G.pairs[0]; n = G.pairs[1];
  } else {
    j = p - G.pairs[0] - G.pairs[1]; n = G.pairs[2];
  }
  return pow(G.theta, -(double)j / (double)n);
}

// Rotate (a, b) by the angle pos * inv_freq: the product is formed in double, reduced
// modulo 2*pi in double (Cody-Waite with a two-part 2*pi) to [-pi, pi], where the
// hardware sin/cos approximations (__sincosf) are accurate to ~4e-7 absolute; the
// rotated pair is then rounded to bf16 (2^-9 relative).
__device__ __forceinline__ void rope_rotate_fast(float& a, float& b, double pos, double inv_freq) {
  const double ang = pos * inv_freq;
  const double k = rint(ang * 0.15915494309189535);          // 1 / (2 pi)
  double r = fma(-k, 6.283185307179586, ang);                 // 2 pi, leading part
  r = fma(-k, 2.4492935982947064e-16, r);                     // 2 pi, trailing part
  float s, c;
  __sincosf((float)r, &s, &c);
  const float na = a * c - b * s;
  const float nb = a * s + b * c;
  a = na;
  b = nb;
}

}  // namespace mla
