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

__device__ __forceinline__ void set_device_error(unsigned int* err, unsigned int code) {
  if (err) atomicOr(err, code);
}

}  // namespace mla
