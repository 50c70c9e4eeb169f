// Definitions shared by the tensor-core attention kernel (tc_attend.cu) and the merge of
// its split-key partials (attend_combine.cu).
#pragma once

#include "launch.h"

namespace mla {
namespace attn {

constexpr int TM = 128;                               // rows per tile
constexpr int HALF = 256;                             // latent dims per CTA of a cluster
constexpr int MAXC = 128;                             // clusters one launch can schedule

struct AttnArgs {
  Geo g;
  int64_t n_q, q_first, k_first, n_keys;
  float scale_log2;
  const bf16* q_abs;
  bf16* o_lat;
  float* lse;
  bf16* ws_o;               // partial outputs [slot][TM][Dc], bf16, normalised by their l
  float* ws_lse;            // their natural log-sum-exps, one per CTA half [slot][2][TM]
  int tiles_per_batch;
  int bn;                   // keys per block of the launch
  int pf;                   // L2 look-ahead of the key loads in blocks (0: none)
  float xthr;               // largest raw partial score magnitude a row's 16-bit score
                            // exchange carries; a row with a larger one is sent exactly
  // the low-bit ring (packed variant only): codes of both paths, per-row float32 scales
  const uint8_t* pk_c;      // [B][S][d_c * cbits / 8]
  const uint8_t* pk_r;      // [B][S][d_R * rbits / 8]
  const float* sc_c;        // [B][S]
  const float* sc_r;        // [B][S]
  int cbits, rbits;
  unsigned int* err;
};

// Key blocks of one tile: its rows see the keys k_first .. k_first + L - 1 (frame-
// block-causal bound of its last row), stored in the ring as two contiguous slot runs.
struct Blocks {
  int64_t k_first, p1, n1, L;
  int bn;                   // keys per block
  int nb1, nblk;
  // block j: first ring slot, first global token, number of keys
  __device__ void get(int j, int64_t& slot0, int64_t& g0, int& valid) const {
    if (j < nb1) {
      slot0 = p1 + (int64_t)j * bn;
      g0 = k_first + (int64_t)j * bn;
      const int64_t v = n1 - (int64_t)j * bn;
      valid = v < bn ? (int)v : bn;
    } else {
      const int64_t jj = j - nb1;
      slot0 = jj * bn;
      g0 = k_first + n1 + jj * bn;
      const int64_t v = L - n1 - jj * bn;
      valid = v < bn ? (int)v : bn;
    }
  }
};

struct TileGeo {
  int b;
  int64_t rows_b, row0, grow0, i_last;
  Blocks blk;
};

// one past the last key query i sees (frame-block-causal, clipped to the key window)
__host__ __device__ inline int64_t key_end(const Geo& G, int64_t q_first, int64_t k_lim,
                                           int64_t i) {
  const int64_t e = ((q_first + i) / G.F + 1) * G.F;
  return e < k_lim ? e : k_lim;
}

__host__ __device__ inline TileGeo tile_geo(const Geo& G, int64_t n_q, int64_t q_first,
                                            int64_t k_first, int64_t n_keys,
                                            int tiles_per_batch, int tile, int bn) {
  TileGeo t;
  t.b = tile / tiles_per_batch;
  const int tb = tile - t.b * tiles_per_batch;
  t.rows_b = n_q * G.H;
  t.row0 = (int64_t)tb * TM;
  t.grow0 = (int64_t)t.b * t.rows_b + t.row0;
  const int64_t last_row = (t.row0 + TM < t.rows_b ? t.row0 + TM : t.rows_b) - 1;
  t.i_last = last_row / G.H;
  Blocks& k = t.blk;
  k.k_first = k_first;
  k.L = key_end(G, q_first, k_first + n_keys, t.i_last) - k_first;
  k.p1 = k_first % G.S;
  k.n1 = k.L < G.S - k.p1 ? k.L : G.S - k.p1;
  k.bn = bn;
  k.nb1 = (int)((k.n1 + bn - 1) / bn);
  k.nblk = k.nb1 + (int)((k.L - k.n1 + bn - 1) / bn);
  return t;
}

// Split tiles to merge: tile[i] has the partial segments in workspace slots
// [piece0[i], piece0[i + 1]).
struct CombineList {
  int32_t n;
  int32_t tile[MAXC];
  int32_t piece0[MAXC + 1];
};

// Merge the partials of the split tiles listed in `cl` into o_lat (and lse).
cudaError_t launch_combine(const AttnArgs& a, const CombineList& cl, cudaStream_t st);

}  // namespace attn
}  // namespace mla
