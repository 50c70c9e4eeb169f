// Absorbed MLA attention on tcgen05 tensor cores (bf16, d_c = 512, d_R = 64).
//
// Rows of the problem are (query, head) pairs; all heads share the cached rows
// [c_KV || k_R], which serve both as keys (all 576 dims) and as values (the 512 latent
// dims): S = Q_abs . [c || k_R]^T, P = softmax(S), O_lat = P . c.
//
// A 128 x 512 fp32 output accumulator fills a whole SM's tensor memory, so each 128-row
// tile is handled by a cluster of two CTAs that split the latent dimension: CTA 0 owns
// latent dims [0, 256), CTA 1 owns [256, 512) plus the 64 RoPE dims.  Per block of 64
// keys each CTA
//   - TMA-loads its columns of the 64 cached rows (one load serves as K and as V),
//   - computes its partial score S_c = Q_c . K_c^T with tcgen05.mma (Q's latent half
//     resident in TMEM as the A operand, the RoPE part from shared memory),
//   - exchanges partial scores through distributed shared memory: CTA c finishes the
//     softmax of rows [64c, 64c + 64) and receives the peer's partials for them,
//   - writes its P rows (bf16) into both CTAs' shared memory with the rescale factors,
//   - accumulates O_c += P . V_c (M=128, N=256) into its TMEM.
// The online softmax keeps a running max per row and rescales O only when the max grows
// by more than 8 (log2 units).  Masking is frame-block-causal per row; a ring that
// wraps is walked as two contiguous slot segments.
//
// Warp roles (192 threads): warps 0-3 softmax / exchange / epilogue (thread = row =
// TMEM lane), warp 4 TMA producer, warp 5 MMA issuer and TMEM owner.
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace mla {
namespace {

using namespace tc;

constexpr int TM = 128;                               // rows per tile
constexpr int BN = 64;                                // keys per block
constexpr int NST = 3;                                // K/V pipeline stages
constexpr int HALF = 256;                             // latent dims per CTA
constexpr int BOX_BYTES = BN * 64 * 2;                // 64 keys x 64 dims, 8 KB
constexpr int LAT_BYTES = 4 * BOX_BYTES;              // 32 KB
constexpr int STAGE_BYTES = LAT_BYTES + BOX_BYTES;    // + RoPE box (CTA 1)
constexpr int QR_BYTES = TM * 64 * 2;                 // Q RoPE part, 16 KB
constexpr int P_BYTES = TM * BN * 2;                  // 16 KB
constexpr int X_BYTES = 64 * BN * 4;                  // 16 KB

constexpr int OFF_KV = 0;
constexpr int OFF_QR = OFF_KV + NST * STAGE_BYTES;
constexpr int OFF_P = OFF_QR + QR_BYTES;
constexpr int OFF_X = OFF_P + 2 * P_BYTES;
constexpr int OFF_F = OFF_X + 2 * X_BYTES;            // factors [2][128] + final 1/l [128]
constexpr int OFF_BAR = OFF_F + 3 * TM * 4;

enum {
  B_KVF = 0,                // K/V stage loaded (TMA)
  B_KVE = B_KVF + NST,      // K/V stage free (MMA commit after PV)
  B_QR = B_KVE + NST,       // Q RoPE tile loaded
  B_QREADY,                 // Q latent half written to TMEM (128 threads)
  B_SF,                     // S buffer full (MMA commit)          [2]
  B_SE = B_SF + 2,          // S buffer read (128 threads)         [2]
  B_XF = B_SE + 2,          // peer partials landed in my X        [2] 64 remote
  B_XE = B_XF + 2,          // peer consumed my partials           [2] 64 remote
  B_RF = B_XE + 2,          // peer P rows + factors landed        [2] 64 remote
  B_PF = B_RF + 2,          // P buffer complete, O rescaled       [2] 128
  B_PE = B_PF + 2,          // PV done with P buffer               [2] commit
  B_PPE = B_PE + 2,         // peer's P buffer free for my rows    [2] 64 remote
  B_FIN = B_PPE + 2,        // peer's final 1/l landed                 64 remote
  B_DONE,                   // every MMA finished
  NBAR
};
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int ATT_SMEM = OFF_MISC + 16 + 1024;

constexpr uint32_t O_COL = 0, Q_COL = 256, S_COL = 384;
constexpr unsigned FULL = 0xffffffffu;

struct AttnArgs {
  Geo g;
  int64_t n_q, q_first, k_first, n_keys;
  float scale_log2;
  const bf16* q_abs;
  bf16* o_lat;
  float* lse;
  int tiles_per_batch;
  unsigned int* err;
};

struct Blocks {
  int64_t k_first, p1, n1, L;
  int nb1, nblk;
  // block j: first ring slot, first global token, number of keys
  __device__ void get(int j, int64_t& slot0, int64_t& g0, int& valid) const {
    if (j < nb1) {
      slot0 = p1 + (int64_t)j * BN;
      g0 = k_first + (int64_t)j * BN;
      const int64_t v = n1 - (int64_t)j * BN;
      valid = v < BN ? (int)v : BN;
    } else {
      const int64_t jj = j - nb1;
      slot0 = jj * BN;
      g0 = k_first + n1 + jj * BN;
      const int64_t v = L - n1 - jj * BN;
      valid = v < BN ? (int)v : BN;
    }
  }
};

__device__ __forceinline__ void rescale_row(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < HALF; c += 16) {
    uint32_t v[16];
    tmem_ld16(taddr + c, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * f);
    tmem_st16(taddr + c, v);
  }
  tmem_wait_st();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                  AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  float* F = reinterpret_cast<float*>(sm + OFF_F);

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geo& G = a.g;
  const int tile = blockIdx.x >> 1;
  const int b = tile / a.tiles_per_batch;
  const int tb = tile - b * a.tiles_per_batch;
  const int64_t rows_b = a.n_q * G.H;
  const int64_t row0 = (int64_t)tb * TM;
  const int64_t grow0 = (int64_t)b * rows_b + row0;
  const int64_t k_lim = a.k_first + a.n_keys;
  auto k_end_of = [&](int64_t i) {
    const int64_t e = ((a.q_first + i) / G.F + 1) * G.F;
    return e < k_lim ? e : k_lim;
  };
  const int64_t last_row = (row0 + TM < rows_b ? row0 + TM : rows_b) - 1;
  const int64_t i_last = last_row / G.H;
  Blocks blk;
  blk.k_first = a.k_first;
  blk.L = k_end_of(i_last) - a.k_first;
  blk.p1 = a.k_first % G.S;
  blk.n1 = blk.L < G.S - blk.p1 ? blk.L : G.S - blk.p1;
  blk.nb1 = (int)((blk.n1 + BN - 1) / BN);
  blk.nblk = blk.nb1 + (int)((blk.L - blk.n1 + BN - 1) / BN);
  const int nblk = blk.nblk;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar[B_KVF + s], 1);
      mbar_init(&bar[B_KVE + s], 1);
    }
    mbar_init(&bar[B_QR], 1);
    mbar_init(&bar[B_QREADY], 128);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bar[B_SF + q], 1);
      mbar_init(&bar[B_SE + q], 128);
      mbar_init(&bar[B_XF + q], 64);
      mbar_init(&bar[B_XE + q], 64);
      mbar_init(&bar[B_RF + q], 64);
      mbar_init(&bar[B_PF + q], 128);
      mbar_init(&bar[B_PE + q], 1);
      mbar_init(&bar[B_PPE + q], 64);
    }
    mbar_init(&bar[B_FIN], 64);
    mbar_init(&bar[B_DONE], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();          // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      if (rank == 1) {
        prefetch_tmap(&tmQ);
        mbar_expect_tx(&bar[B_QR], QR_BYTES);
        tma_load_2d(sm + OFF_QR, &tmQ, &bar[B_QR], G.Dc, (int32_t)grow0);
      }
      const uint32_t bytes = rank == 1 ? STAGE_BYTES : LAT_BYTES;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NST;
        if (!mbar_wait(&bar[B_KVE + s], ((j / NST) & 1) ^ 1, abort, a.err, 0x101, j)) break;
        int64_t slot0, g0;
        int valid;
        blk.get(j, slot0, g0, valid);
        uint8_t* st = sm + OFF_KV + s * STAGE_BYTES;
        mbar_expect_tx(&bar[B_KVF + s], bytes);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_3d(st + q * BOX_BYTES, &tmK, &bar[B_KVF + s], (int)rank * HALF + q * 64,
                      (int32_t)slot0, b);
        if (rank == 1)
          tma_load_3d(st + LAT_BYTES, &tmK, &bar[B_KVF + s], G.Dc, (int32_t)slot0, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, BN, false, false);
      const uint32_t id_pv = idesc_bf16(128, HALF, false, true);
      bool ok = mbar_wait(&bar[B_QREADY], 0, abort, a.err, 0x102, 0);
      if (ok && rank == 1) ok = mbar_wait(&bar[B_QR], 0, abort, a.err, 0x103, 0);
      tc_fence_after();
      auto pv = [&](int jj) -> bool {
        const int pb = jj & 1;
        if (!mbar_wait(&bar[B_PF + pb], (jj >> 1) & 1, abort, a.err, 0x104, jj)) return false;
        tc_fence_after();
        const uint32_t st = smem_u32(sm + OFF_KV + (jj % NST) * STAGE_BYTES);
        const uint32_t pa = smem_u32(sm + OFF_P + pb * P_BYTES);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_ss(tmem + O_COL, desc_sw128(pa + ks * 32, 16, 1024),
                 desc_sw128(st + ks * 2048, BOX_BYTES, 1024), id_pv, (jj > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar[B_PE + pb]);
        mma_commit(&bar[B_KVE + jj % NST]);
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % NST, sb = j & 1;
        if (!mbar_wait(&bar[B_KVF + s], (j / NST) & 1, abort, a.err, 0x105, j)) break;
        if (!mbar_wait(&bar[B_SE + sb], ((j >> 1) & 1) ^ 1, abort, a.err, 0x106, j)) break;
        tc_fence_after();
        const uint32_t d = tmem + S_COL + sb * BN;
        const uint32_t st = smem_u32(sm + OFF_KV + s * STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HALF / 16; ++kk)
          mma_ts(d, tmem + Q_COL + kk * 8,
                 desc_sw128(st + (kk >> 2) * BOX_BYTES + (kk & 3) * 32, 16, 1024), id_qk,
                 kk > 0 ? 1u : 0u);
        if (rank == 1) {
          const uint32_t qa = smem_u32(sm + OFF_QR);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            mma_ss(d, desc_sw128(qa + w * 32, 16, 1024),
                   desc_sw128(st + LAT_BYTES + w * 32, 16, 1024), id_qk, 1u);
        }
        mma_commit(&bar[B_SF + sb]);
        if (j > 0 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok && nblk > 0) pv(nblk - 1);
      mma_commit(&bar[B_DONE]);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int t = tid;                         // row of the tile == TMEM lane
    const bool owner = (uint32_t)(t >> 6) == rank;
    const int64_t r_in_b = row0 + t;
    const bool row_valid = r_in_b < rows_b;
    const int64_t grow = grow0 + t;
    const int64_t k_end_row = k_end_of(row_valid ? r_in_b / G.H : i_last);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t peer_bar0 = mapa(smem_u32(bar), peer);
    auto peer_bar = [&](int idx) { return peer_bar0 + idx * 8; };

    // Q latent half -> TMEM (A operand of the score MMA), bf16 pairs per column
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q_abs + grow * G.row + rank * HALF);
#pragma unroll 1
      for (int c = 0; c < HALF / 32; ++c) {
        uint32_t v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 x = row_valid ? src[c * 4 + q] : make_uint4(0, 0, 0, 0);
          v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
        }
        tmem_st16(tmem + lane_base + Q_COL + c * 16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[B_QREADY]);
    }

    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      const uint32_t kph = (j >> 1) & 1;
      if (!__all_sync(FULL, mbar_wait(&bar[B_SF + sb], kph, abort, a.err, 0x201, (t << 16) | j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + S_COL + sb * BN, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(v[c]);
        tmem_ld32(tmem + lane_base + S_COL + sb * BN + 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(v[c]);
      }
      tc_fence_before();
      mbar_arrive(&bar[B_SE + sb]);
      int64_t slot0, g0;
      int valid;
      blk.get(j, slot0, g0, valid);

      if (!owner) {
        // partial scores of the peer's rows -> peer's exchange buffer
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XE + sb], kph ^ 1, abort, a.err, 0x202,
                                                 (t << 16) | j))) {
          ok = false;
          break;
        }
        const uint32_t dst = mapa(smem_u32(sm + OFF_X + sb * X_BYTES), peer) +
                             (uint32_t)(t - (int)peer * 64) * (BN * 4);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          st_cluster_v4(dst + q * 16, __float_as_uint(s[4 * q]), __float_as_uint(s[4 * q + 1]),
                        __float_as_uint(s[4 * q + 2]), __float_as_uint(s[4 * q + 3]));
        mbar_arrive_cluster(peer_bar(B_XF + sb));
        // a partial block: zero this CTA's latent rows past the last key so that masked
        // keys contribute exact zeros to P.V whatever the ring holds there
        if (valid < BN) {
          const int s_idx = j % NST;
          if (!__all_sync(FULL, mbar_wait(&bar[B_KVF + s_idx], (j / NST) & 1, abort, a.err, 0x203,
                                          (t << 16) | j))) {
            ok = false;
            break;
          }
          const int u = t - (int)peer * 64;               // 0..63
          if (u >= valid) {
            uint8_t* st = sm + OFF_KV + s_idx * STAGE_BYTES + u * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4* p = reinterpret_cast<uint4*>(st + q * BOX_BYTES);
#pragma unroll
              for (int w = 0; w < 8; ++w) p[w] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        // this row's P and rescale factor from the owner
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_RF + sb], kph, abort, a.err, 0x204,
                                                 (t << 16) | j))) {
          ok = false;
          break;
        }
        const float fac = F[sb * TM + t];
        if (j > 0) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort,
                                          a.err, 0x205, (t << 16) | j))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // warp-collective TMEM access: every lane runs it, factor 1 where nothing grew
          if (__any_sync(FULL, fac != 1.f)) rescale_row(tmem + lane_base + O_COL, fac);
          // my P buffer of block j-1 is free again: the peer may write block j+1 rows
          mbar_arrive_cluster(peer_bar(B_PPE + ((j - 1) & 1)));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_PF + sb]);
      } else {
        // full scores: add the peer's partial
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XF + sb], kph, abort, a.err, 0x301,
                                                 (t << 16) | j))) {
          ok = false;
          break;
        }
        const float4* xr = reinterpret_cast<const float4*>(sm + OFF_X + sb * X_BYTES +
                                                           (t - (int)rank * 64) * (BN * 4));
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 x = xr[q];
          s[4 * q] += x.x; s[4 * q + 1] += x.y; s[4 * q + 2] += x.z; s[4 * q + 3] += x.w;
        }
        mbar_arrive_cluster(peer_bar(B_XE + sb));
        float mb = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const bool vis = c < valid && g0 + c < k_end_row;
          s[c] = vis ? s[c] * a.scale_log2 : -INFINITY;
          mb = fmaxf(mb, s[c]);
        }
        float fac = 1.f;
        if (j == 0) {
          m = mb;
        } else if (mb > m + 8.f) {
          fac = exp2f(m - mb);
          m = mb;
        }
        const float msub = m == -INFINITY ? 0.f : m;
        uint32_t pk[32];
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = exp2f(s[2 * c] - msub), p1 = exp2f(s[2 * c + 1] - msub);
          sum += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
        l = l * fac + sum;
        // warp-collective TMEM access: the whole warp rescales if any of its rows grew
        if (j > 0 && __any_sync(FULL, fac != 1.f)) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort,
                                          a.err, 0x302, (t << 16) | j))) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_row(tmem + lane_base + O_COL, fac);
        } else if (j >= 2) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + sb], kph ^ 1, abort, a.err, 0x303,
                                          (t << 16) | j))) {
            ok = false;
            break;
          }
        }
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_PPE + sb], kph ^ 1, abort, a.err, 0x304,
                                                 (t << 16) | j))) {
          ok = false;
          break;
        }
        uint8_t* prow = sm + OFF_P + sb * P_BYTES + t * 128;
        const uint32_t prem = mapa(smem_u32(prow), peer);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int pos = (c ^ (t & 7)) * 16;
          *reinterpret_cast<uint4*>(prow + pos) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          st_cluster_v4(prem + pos, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        st_cluster_f32(mapa(smem_u32(&F[sb * TM + t]), peer), fac);
        fence_proxy_async_cluster();
        fence_proxy_async_smem();
        mbar_arrive_cluster(peer_bar(B_RF + sb));
        tc_fence_before();
        mbar_arrive(&bar[B_PF + sb]);
      }
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait(&bar[B_DONE], 0, abort, a.err, 0x401, t);
    tc_fence_after();
    float inv = 0.f;
    if (owner) {
      inv = l > 0.f ? 1.f / l : 0.f;
      st_cluster_f32(mapa(smem_u32(&F[2 * TM + t]), peer), inv);
      mbar_arrive_cluster(peer_bar(B_FIN));
      if (a.lse && row_valid && ok) a.lse[grow] = (m + log2f(l)) * 0.69314718055994530942f;
    } else {
      if (ok) ok = mbar_wait_cluster(&bar[B_FIN], 0, abort, a.err, 0x402, t);
      inv = F[2 * TM + t];
    }
    bf16* dst = a.o_lat + grow * G.Dc + rank * HALF;
#pragma unroll 1
    for (int c = 0; c < HALF; c += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + O_COL + c, v);
      tmem_wait_ld();
      if (ok && row_valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
          w.y = pack_bf16(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
          w.z = pack_bf16(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
          w.w = pack_bf16(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
          reinterpret_cast<uint4*>(dst + c)[q] = w;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();          // no remote access into this CTA is still pending
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool tc_attend_supported(const Geo& g) { return g.Dc == 2 * HALF && g.Dr == 64; }

cudaError_t tc_attend(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                      const void* cache, int64_t k_first, int64_t n_keys, float scale,
                      void* o_lat, float* lse, unsigned int* err, cudaStream_t st) {
  CUtensorMap K, Q;
  {
    uint64_t d[3] = {(uint64_t)g.row, (uint64_t)g.S, (uint64_t)g.B};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.S * g.row * 2};
    uint32_t b[3] = {64, BN, 1};
    if (!make_tmap_bf16(&K, cache, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[2] = {(uint64_t)g.row, (uint64_t)g.B * n_q * g.H};
    uint64_t s[1] = {(uint64_t)g.row * 2};
    uint32_t b[2] = {64, TM};
    if (!make_tmap_bf16(&Q, q_abs, 2, d, s, b)) return cudaErrorInvalidValue;
  }
  static bool attr = false;
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  AttnArgs a{};
  a.g = g;
  a.n_q = n_q; a.q_first = q_first; a.k_first = k_first; a.n_keys = n_keys;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_abs = (const bf16*)q_abs;
  a.o_lat = (bf16*)o_lat;
  a.lse = lse;
  a.tiles_per_batch = (int)((n_q * g.H + TM - 1) / TM);
  a.err = err;
  const int64_t tiles = (int64_t)g.B * a.tiles_per_batch;
  attend_kernel<<<(unsigned)(2 * tiles), 192, ATT_SMEM, st>>>(K, Q, a);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
