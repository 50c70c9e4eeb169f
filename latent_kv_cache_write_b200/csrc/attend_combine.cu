// Merge of the split-key partials of the tensor-core attention: a tile whose key blocks
// were cut between clusters left one normalised bf16 partial output and one fp32
// log-sum-exp per CTA half for each piece in the workspace.
#include "attend_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace mla {
namespace attn {
namespace {

using tc::pack_bf16;

// CSPLIT warps per row of a split tile, 8 / CSPLIT rows per CTA: warp k of a row merges
// pieces p0 + k, p0 + k + CSPLIT, ... (with several warps per row, four pieces' loads in
// flight at a time) and the row's warps add their sums in shared memory.  One warp per
// row suits tiles cut in a few pieces (the chunk shapes); more suit a tile cut across
// every cluster (decode of a few sequences).  Lane l holds latent dims [16 l, 16 l + 16)
// (d_c = 512).  The output is the partials weighted by exp(lse_p - lse),
// lse = log sum_p exp(lse_p), each half of the dims with the log-sum-exps of the CTA half
// that computed it.
template <int CSPLIT>
__global__ void __launch_bounds__(256)
    combine_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CombineList cl) {
  constexpr int CROWS = 8 / CSPLIT;
  __shared__ float red[CSPLIT > 1 ? 8 * 32 * 17 : 1];     // [row][warp][lane][16 sums + w]
  tc::grid_dep_wait();                             // the attention's partials are visible
  tc::grid_dep_launch();
  const int i = blockIdx.x / (TM / CROWS);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = wid / CSPLIT, part = wid % CSPLIT;
  const int r = (blockIdx.x % (TM / CROWS)) * CROWS + rr;
  const TileGeo tg =
      tile_geo(a.g, a.n_q, a.q_first, a.k_first, a.n_keys, a.tiles_per_batch, cl.tile[i], a.bn);
  const bool row_ok = tg.row0 + r < tg.rows_b;
  const int p0 = cl.piece0[i], p1 = cl.piece0[i + 1];
  const int d = lane * 16;
  const int half = d / HALF;                 // the CTA half these dims were computed in
  // each half's largest log-sum-exp over the row's pieces, the lanes taking pieces in turn
  float m0 = -INFINITY, m1 = -INFINITY;
  if (row_ok)
    for (int p = p0 + lane; p < p1; p += 32) {
      m0 = fmaxf(m0, a.ws_lse[((int64_t)p * 2) * TM + r]);
      m1 = fmaxf(m1, a.ws_lse[((int64_t)p * 2 + 1) * TM + r]);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
  }
  const float mx = half ? m1 : m0;
  const float* lse_h = a.ws_lse + half * TM + r;   // + p * 2 * TM: piece p
  float acc[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) acc[q] = 0.f;
  float wsum = 0.f;
  // a piece's 16 dims of this lane: two 16-byte vectors of bf16
  auto add = [&](float lp, const uint4 (&v)[2]) {
    const float w = lp > -INFINITY ? expf(lp - mx) : 0.f;
    wsum += w;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t u[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[8 * q + 2 * e] += w * __uint_as_float(u[e] << 16);
        acc[8 * q + 2 * e + 1] += w * __uint_as_float(u[e] & 0xffff0000u);
      }
    }
  };
  if (row_ok && mx > -INFINITY) {
    int p = p0 + part;
    if constexpr (CSPLIT > 1) {
      for (; p + 3 * CSPLIT < p1; p += 4 * CSPLIT) {
        float lp[4];
        uint4 v[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int pu = p + u * CSPLIT;
          lp[u] = lse_h[(int64_t)pu * 2 * TM];
          const uint4* o =
              reinterpret_cast<const uint4*>(a.ws_o + ((int64_t)pu * TM + r) * a.g.Dc + d);
#pragma unroll
          for (int q = 0; q < 2; ++q) v[u][q] = o[q];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) add(lp[u], v[u]);
      }
    }
    for (; p < p1; p += CSPLIT) {
      uint4 v[2];
      const uint4* o = reinterpret_cast<const uint4*>(a.ws_o + ((int64_t)p * TM + r) * a.g.Dc + d);
#pragma unroll
      for (int q = 0; q < 2; ++q) v[q] = o[q];
      add(lse_h[(int64_t)p * 2 * TM], v);
    }
  }
  if constexpr (CSPLIT > 1) {
    float* mine = red + ((rr * CSPLIT + part) * 32 + lane) * 17;
#pragma unroll
    for (int q = 0; q < 16; ++q) mine[q] = acc[q];
    mine[16] = wsum;
    __syncthreads();
    if (part != 0 || !row_ok) return;
    for (int k = 1; k < CSPLIT; ++k) {
      const float* other = red + ((rr * CSPLIT + k) * 32 + lane) * 17;
#pragma unroll
      for (int q = 0; q < 16; ++q) acc[q] += other[q];
      wsum += other[16];
    }
  } else {
    if (!row_ok) return;
  }
  const int64_t grow = tg.grow0 + r;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(a.o_lat + grow * a.g.Dc + d);
#pragma unroll
  for (int q = 0; q < 2; ++q)
    dst[q] = make_uint4(pack_bf16(acc[8 * q] * inv, acc[8 * q + 1] * inv),
                        pack_bf16(acc[8 * q + 2] * inv, acc[8 * q + 3] * inv),
                        pack_bf16(acc[8 * q + 4] * inv, acc[8 * q + 5] * inv),
                        pack_bf16(acc[8 * q + 6] * inv, acc[8 * q + 7] * inv));
  if (lane == 0 && a.lse) a.lse[grow] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const AttnArgs& a, const CombineList& cl, cudaStream_t st) {
  if (cl.n == 0) return cudaSuccess;
  int most = 0;                                    // the most pieces of one tile
  for (int k = 0; k < cl.n; ++k)
    most = cl.piece0[k + 1] - cl.piece0[k] > most ? cl.piece0[k + 1] - cl.piece0[k] : most;
  if (most >= 32)
    return launch_dependent(combine_kernel<8>, (unsigned)(cl.n * TM), 256, 0, st, 1u, a, cl);
  if (most >= 8)
    return launch_dependent(combine_kernel<4>, (unsigned)(cl.n * (TM / 2)), 256, 0, st, 1u, a, cl);
  return launch_dependent(combine_kernel<1>, (unsigned)(cl.n * (TM / 8)), 256, 0, st, 1u, a, cl);
}

}  // namespace attn
}  // namespace mla
