// Merge of the split-key partials of the tensor-core attention: a tile whose key blocks
// were cut between clusters left one normalised fp32 partial output and one log-sum-exp
// per CTA half for each piece in the workspace.
#include "attend_common.cuh"
#include "tc_ptx.cuh"

namespace mla {
namespace attn {
namespace {

using tc::pack_bf16;

// One warp per row of a split tile, 8 rows per CTA; lane l merges latent dims
// [16 l, 16 l + 16) (d_c = 512).  The output is the partials weighted by exp(lse_p - lse),
// lse = log sum_p exp(lse_p), each half of the dims with the log-sum-exps of the CTA half
// that computed it.
constexpr int CROWS = 8;
__global__ void __launch_bounds__(32 * CROWS) combine_kernel(const __grid_constant__ AttnArgs a,
                                                             const __grid_constant__ CombineList cl) {
  const int i = blockIdx.x / (TM / CROWS);
  const int r = (blockIdx.x % (TM / CROWS)) * CROWS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const TileGeo tg =
      tile_geo(a.g, a.n_q, a.q_first, a.k_first, a.n_keys, a.tiles_per_batch, cl.tile[i], a.bn);
  if (tg.row0 + r >= tg.rows_b) return;
  const int64_t grow = tg.grow0 + r;
  const int p0 = cl.piece0[i], p1 = cl.piece0[i + 1];
  const int d = lane * 16;
  const int half = d / HALF;                 // the CTA half these dims were computed in
  const float* lse_h = a.ws_lse + half * TM + r;   // + p * 2 * TM: piece p
  float mx = -INFINITY;
  for (int p = p0; p < p1; ++p) mx = fmaxf(mx, lse_h[(int64_t)p * 2 * TM]);
  float acc[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) acc[q] = 0.f;
  float wsum = 0.f;
  if (mx > -INFINITY) {
    for (int p = p0; p < p1; ++p) {
      const float lp = lse_h[(int64_t)p * 2 * TM];
      if (!(lp > -INFINITY)) continue;
      const float w = expf(lp - mx);
      wsum += w;
      const float4* o = reinterpret_cast<const float4*>(a.ws_o + ((int64_t)p * TM + r) * a.g.Dc + d);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = o[q];
        acc[4 * q] += w * v.x;
        acc[4 * q + 1] += w * v.y;
        acc[4 * q + 2] += w * v.z;
        acc[4 * q + 3] += w * v.w;
      }
    }
  }
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
  combine_kernel<<<(unsigned)(cl.n * (TM / CROWS)), 32 * CROWS, 0, st>>>(a, cl);
  return cudaGetLastError();
}

}  // namespace attn
}  // namespace mla
