// Absorbed MLA attention on tcgen05 tensor cores (bf16, d_c = 512, d_R = 64).
//
// Rows of the problem are (query, head) pairs; all heads share the cached rows
// [c_KV || k_R], which serve both as keys (all 576 dims) and as values (the 512 latent
// dims): S = Q_abs . [c || k_R]^T, P = softmax(S), O_lat = P . c.
//
// A 128 x 512 fp32 output accumulator fills a whole SM's tensor memory, so each 128-row
// tile is handled by a cluster of two CTAs that split the latent dimension: CTA c owns
// latent dims [256c, 256c + 256) and RoPE dims [32c, 32c + 32).  Per block of 64 keys
// each CTA
//   - TMA-loads its columns of the 64 cached rows (one load serves as K and as V),
//   - computes its partial score S_c = Q_c . K_c^T with tcgen05.mma (Q's latent half
//     resident in TMEM as the A operand, the RoPE part from shared memory),
//   - swaps partial scores (rounded to fp16) with its peer through distributed shared
//     memory, so both CTAs hold the full scores of all 128 rows,
//   - runs the online softmax of all 128 rows itself (both CTAs take bit-identical
//     decisions: each adds the same two fp16-rounded partials),
//   - accumulates O_c += P . V_c (M=128, N=256) into its TMEM.
//
// Two softmax warpgroups take alternate key blocks, so the exchange of one block
// overlaps the exponentials of the other; they hand the running row maximum to each
// other through shared memory.  An exchange buffer is handed back to the peer as soon as
// its scores are read.  O is rescaled only when a row maximum grows by more than 8 (log2
// units).  Masking is frame-block-causal per row; a ring that wraps is walked as two
// contiguous slot segments.
//
// Warp roles (320 threads): warps 0-3 and 4-7 are the two softmax warpgroups (thread =
// row = TMEM lane), warp 8 is the TMA producer, warp 9 the MMA issuer and TMEM owner.
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.h"

#include <cuda_fp16.h>

namespace mla {
namespace {

using namespace tc;

constexpr int TM = 128;                               // rows per tile
constexpr int BN = 64;                                // keys per block
constexpr int NST = 4;                                // K/V pipeline stages
constexpr int HALF = 256;                             // latent dims per CTA
constexpr int BOX_BYTES = BN * 64 * 2;                // 64 keys x 64 dims, 8 KB
constexpr int LAT_BYTES = 4 * BOX_BYTES;              // 32 KB of latent per stage
constexpr int RBOX_BYTES = BN * 32 * 2;               // 64 keys x 32 RoPE dims, 4 KB
constexpr int STAGE_BYTES = LAT_BYTES + RBOX_BYTES;   // bytes one stage's loads bring
// Shared-memory K/V ring, box-major: latent box q (dims 64q..64q+63 of this CTA's half,
// 128-byte swizzle) of stage s at OFF_KV + (q * NST + s) * BOX_BYTES, RoPE box of stage
// s (64-byte swizzle) at OFF_KVR + s * RBOX_BYTES.  Stages 2i and 2i+1 are adjacent
// within every box column, so one N=128 score MMA covers two consecutive 64-key blocks.
constexpr int QR_BYTES = TM * 32 * 2;                 // this CTA's Q RoPE part, 8 KB
constexpr int X_BYTES = TM * BN * 2;                  // exchange buffer, 16 KB: the peer's
                                                      // partial scores as fp16, chunk-major
                                                      // [8 x 16 B][128 rows]
constexpr int P_BYTES = TM * BN * 2;                  // P, bf16, 128-byte swizzled rows
constexpr int NTHREADS = 320;

constexpr int OFF_KV = 0;
constexpr int OFF_KVR = OFF_KV + NST * LAT_BYTES;
constexpr int OFF_QR = OFF_KVR + NST * RBOX_BYTES;
constexpr int OFF_X = OFF_QR + QR_BYTES;              // [2] exchange buffers
constexpr int OFF_P = OFF_X + 2 * X_BYTES;            // [2] P buffers
constexpr int OFF_M = OFF_P + 2 * P_BYTES;            // running max handoff [2][128]
constexpr int OFF_L = OFF_M + 2 * TM * 4;             // final (l, m) per warpgroup [2][2][128]
constexpr int OFF_BAR = OFF_L + 4 * TM * 4;

enum {
  B_KVF = 0,                // K/V stage loaded (TMA)
  B_KVE = B_KVF + NST,      // K/V stage free (MMA commit after PV)
  B_QR = B_KVE + NST,       // Q RoPE tile loaded
  B_QREADY,                 // Q latent half written to TMEM (256 threads)
  B_SF,                     // S buffer full (MMA commit)                  [2]
  B_SE = B_SF + 2,          // S buffer read (128 threads)                 [2]
  B_XF = B_SE + 2,          // peer's partial scores landed (tx bytes)     [2]
  B_XE = B_XF + 2,          // peer read the scores sent it (1 remote)    [2]
  B_PF = B_XE + 2,          // P complete, O rescaled (128)                [2]
  B_PE = B_PF + 2,          // PV done (MMA commit)                        [2]
  B_M = B_PE + 2,           // running max of a block published (128)      [2]
  B_DONE = B_M + 2,         // every MMA finished
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKR,
                  const __grid_constant__ CUtensorMap tmQR, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);

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
    mbar_init(&bar[B_QREADY], 256);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bar[B_SF + q], 1);
      mbar_init(&bar[B_SE + q], 128);
      mbar_init(&bar[B_XF + q], 1);
      mbar_init(&bar[B_XE + q], 1);
      mbar_init(&bar[B_PF + q], 128);
      mbar_init(&bar[B_PE + q], 1);
      mbar_init(&bar[B_M + q], 128);
    }
    mbar_init(&bar[B_DONE], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();          // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmKR);
      prefetch_tmap(&tmQR);
      mbar_expect_tx(&bar[B_QR], QR_BYTES);
      tma_load_2d(sm + OFF_QR, &tmQR, &bar[B_QR], G.Dc + (int)rank * 32, (int32_t)grow0);
      const uint32_t bytes = STAGE_BYTES;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NST;
        if (!mbar_wait(&bar[B_KVE + s], ((j / NST) & 1) ^ 1, abort, a.err, 0x101, j)) break;
        int64_t slot0, g0;
        int valid;
        blk.get(j, slot0, g0, valid);
        mbar_expect_tx(&bar[B_KVF + s], bytes);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_3d(sm + OFF_KV + (q * NST + s) * BOX_BYTES, &tmK, &bar[B_KVF + s],
                      (int)rank * HALF + q * 64, (int32_t)slot0, b);
        tma_load_3d(sm + OFF_KVR + s * RBOX_BYTES, &tmKR, &bar[B_KVF + s], G.Dc + (int)rank * 32,
                    (int32_t)slot0, b);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Scores of blocks 2i and 2i+1 are one N=128 series (S buffers 0 and 1 are adjacent);
    // a score series is issued as soon as its data and S buffers are ready, since the
    // scores start the softmax chains.  PV products are issued in block order, as soon as
    // their P is ready whenever the issuer would otherwise wait: that frees the K/V stage
    // for the next load and the exchange buffer for the peer early.
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, 2 * BN, false, false);
      const uint32_t id_pv = idesc_bf16(128, HALF, false, true);
      bool ok = mbar_wait(&bar[B_QREADY], 0, abort, a.err, 0x102, 0);
      if (ok) ok = mbar_wait(&bar[B_QR], 0, abort, a.err, 0x103, 0);
      tc_fence_after();
      int next_pv = 0;                         // next block whose PV is to be issued
      auto issue_pv = [&](int jj) {
        const int pb = jj & 1;
        const int s = jj % NST;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sm + OFF_KV + s * BOX_BYTES);
        const uint32_t pa = smem_u32(sm + OFF_P + pb * P_BYTES);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_ss(tmem + O_COL, desc_sw128(pa + ks * 32, 16, 1024),
                 desc_sw128(v0 + ks * 2048, NST * BOX_BYTES, 1024), id_pv,
                 (jj > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar[B_PE + pb]);
        mma_commit(&bar[B_KVE + s]);
      };
      // issue every PV whose P is ready, for blocks below `limit`, without blocking
      auto pv_ready = [&](int limit) {
        while (next_pv < limit &&
               mbar_test_wait(&bar[B_PF + (next_pv & 1)], (next_pv >> 1) & 1)) {
          issue_pv(next_pv);
          ++next_pv;
        }
      };
      // wait for a phase while keeping the PV stream moving
      auto wait_pv = [&](uint64_t* w, uint32_t parity, int limit, uint32_t site, int j) -> bool {
        if (mbar_test_wait(w, parity)) return true;
        const long long c0 = clock64();
        for (uint32_t it = 1;; ++it) {
          pv_ready(limit);
          if (mbar_test_wait(w, parity)) return true;
          if ((it & 255u) == 0) {
            if (*abort) return false;
            if (clock64() - c0 > 4000000000ll) {
              *abort = 1;
              report_timeout(a.err, site, (uint32_t)j);
              return false;
            }
          }
        }
      };
      const int npair = (nblk + 1) / 2;
      for (int i = 0; ok && i < npair; ++i) {
        const int j0 = 2 * i, s0 = j0 % NST;
        const bool two = j0 + 1 < nblk;
        const uint32_t ph = (i & 1) ^ 1;
        if (!wait_pv(&bar[B_KVF + s0], (j0 / NST) & 1, j0, 0x105, j0)) { ok = false; break; }
        if (two && !wait_pv(&bar[B_KVF + s0 + 1], (j0 / NST) & 1, j0, 0x105, j0 + 1)) {
          ok = false;
          break;
        }
        if (!wait_pv(&bar[B_SE], ph, j0, 0x106, j0)) { ok = false; break; }
        if (!wait_pv(&bar[B_SE + 1], ph, j0, 0x106, j0 + 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + S_COL;
        // descriptor of K box column 0 at stage s0; the 16-dim steps only add offsets
        const uint64_t kd = desc_sw128(smem_u32(sm + OFF_KV + s0 * BOX_BYTES), 16, 1024);
        mma_ts(d, tmem + Q_COL, kd, id_qk, 0u);
#pragma unroll
        for (int kk = 1; kk < HALF / 16; ++kk)
          mma_ts(d, tmem + Q_COL + kk * 8,
                 kd + (uint64_t)(((kk >> 2) * NST * BOX_BYTES + (kk & 3) * 32) >> 4), id_qk, 1u);
        const uint64_t qd = desc_sw64(smem_u32(sm + OFF_QR), 512);
        const uint64_t rd = desc_sw64(smem_u32(sm + OFF_KVR + s0 * RBOX_BYTES), 512);
        mma_ss(d, qd, rd, id_qk, 1u);
        mma_ss(d, qd + 2, rd + 2, id_qk, 1u);           // second 16-dim step: +32 bytes
        mma_commit(&bar[B_SF]);
        mma_commit(&bar[B_SF + 1]);
        pv_ready(j0);
      }
      // remaining PV products
      while (ok && next_pv < nblk) {
        if (!mbar_wait(&bar[B_PF + (next_pv & 1)], (next_pv >> 1) & 1, abort, a.err, 0x104,
                       next_pv)) {
          ok = false;
          break;
        }
        issue_pv(next_pv);
        ++next_pv;
      }
      mma_commit(&bar[B_DONE]);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;                  // warpgroup: even (0) or odd (1) blocks
    const int t = tid & (TM - 1);              // row of the tile == TMEM lane
    const int64_t r_in_b = row0 + t;
    const bool row_valid = r_in_b < rows_b;
    const int64_t grow = grow0 + t;
    const int64_t k_end_row = k_end_of(row_valid ? r_in_b / G.H : i_last);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float* m_sh = reinterpret_cast<float*>(sm + OFF_M);
    float* l_sh = reinterpret_cast<float*>(sm + OFF_L);

    // Q latent half -> TMEM (A operand of the score MMA), bf16 pairs per column; each
    // warpgroup loads half of the row
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q_abs + grow * G.row + rank * HALF +
                                                        wg * (HALF / 2));
#pragma unroll 1
      for (int c = 0; c < HALF / 64; ++c) {
        uint32_t v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 x = row_valid ? src[c * 4 + q] : make_uint4(0, 0, 0, 0);
          v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
        }
        tmem_st16(tmem + lane_base + Q_COL + wg * (HALF / 4) + c * 16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[B_QREADY]);
    }

    const uint32_t peer_x = mapa(smem_u32(sm + OFF_X + wg * X_BYTES), peer) + (uint32_t)t * 16;
    const uint32_t peer_xf = mapa(smem_u32(&bar[B_XF + wg]), peer);
    const uint4* my_x = reinterpret_cast<const uint4*>(sm + OFF_X + wg * X_BYTES) + t;
    uint8_t* prow = sm + OFF_P + wg * P_BYTES + t * 128;     // P row t
    const uint32_t peer_xe = mapa(smem_u32(&bar[B_XE + wg]), peer);
    const float c2 = a.scale_log2;
    float m_last = -INFINITY, l = 0.f;         // this warpgroup's running sum and its max
    bool ok = true;
    for (int j = wg; j < nblk; j += 2) {
      const uint32_t kph = (j >> 1) & 1;
      // arm this block's exchange: the peer's asynchronous stores complete X_BYTES of
      // transactions on it (they may land before or after this arrive)
      if (t == 0) mbar_expect_tx(&bar[B_XF + wg], X_BYTES);
      if (!__all_sync(FULL, mbar_wait(&bar[B_SF + wg], kph, abort, a.err, 0x201, (t << 16) | j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + S_COL + wg * BN, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(v[c]);
        tmem_ld32(tmem + lane_base + S_COL + wg * BN + 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(v[c]);
      }
      tc_fence_before();
      mbar_arrive(&bar[B_SE + wg]);

      // send this CTA's partial scores into the peer's buffer once the peer's PV of two
      // blocks ago no longer reads it
      if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XE + wg], kph ^ 1, abort, a.err, 0x202,
                                               (t << 16) | j))) {
        ok = false;
        break;
      }
      // both CTAs add the same two fp16-rounded partials, so their softmax agrees bit
      // for bit; the rounding is ~2^-11 of a partial score
      uint32_t hs[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        __half2 h2 = __floats2half2_rn(s[2 * c], s[2 * c + 1]);
        hs[c] = *reinterpret_cast<uint32_t*>(&h2);
        const float2 back = __half22float2(h2);
        s[2 * c] = back.x;
        s[2 * c + 1] = back.y;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st_async_v4(peer_x + q * (TM * 16), hs[4 * q], hs[4 * q + 1], hs[4 * q + 2],
                    hs[4 * q + 3], peer_xf);

      int64_t slot0, g0;
      int valid;
      blk.get(j, slot0, g0, valid);
      if (valid < BN && t < BN && t >= valid) {
        // a partial block: zero this CTA's latent rows past the last key so that masked
        // keys contribute exact zeros to P.V whatever the ring holds there (the stage has
        // landed: QK of this block has completed)
        uint8_t* st = sm + OFF_KV + (j % NST) * BOX_BYTES + t * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4* p = reinterpret_cast<uint4*>(st + q * NST * BOX_BYTES);
#pragma unroll
          for (int w = 0; w < 8; ++w) p[w] = make_uint4(0, 0, 0, 0);
        }
      }

      // full scores: add the peer's partial
      if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XF + wg], kph, abort, a.err, 0x203,
                                               (t << 16) | j))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 x = my_x[q * TM];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
          s[8 * q + 2 * e] += f.x;
          s[8 * q + 2 * e + 1] += f.y;
        }
      }
      named_bar(1 + wg, TM);            // the whole buffer is read: hand it back
      if (t == 0) mbar_arrive_cluster_relaxed(peer_xe);

      // masked raw maximum (scores are scaled inside the exponent)
      const int64_t lim64 = k_end_row - g0;
      const int lim = lim64 < valid ? (lim64 < 0 ? 0 : (int)lim64) : valid;
      if (lim < BN) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = c < lim ? s[c] : -INFINITY;
      }
      float rmax = s[0];
#pragma unroll
      for (int c = 1; c < 64; ++c) rmax = fmaxf(rmax, s[c]);
      const float mb = rmax * c2;

      // running maximum after the previous block (published by the other warpgroup)
      float m_prev = -INFINITY;
      if (j > 0) {
        if (!__all_sync(FULL, mbar_wait(&bar[B_M + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort,
                                        a.err, 0x204, (t << 16) | j))) {
          ok = false;
          break;
        }
        m_prev = m_sh[((j - 1) & 1) * TM + t];
      }
      float m = m_prev, fac = 1.f;
      if (j == 0) {
        m = mb;
      } else if (mb > m_prev + 8.f) {
        m = mb;
        fac = ex2(m_prev - m);
      }
      m_sh[wg * TM + t] = m;
      mbar_arrive(&bar[B_M + wg]);

      const float msub = m == -INFINITY ? 0.f : m;
      uint32_t pk[32];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ex2(fmaf(s[2 * c], c2, -msub));
        const float p1 = ex2(fmaf(s[2 * c + 1], c2, -msub));
        sum += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l = l * ex2(m_last - msub) + sum;
      m_last = m;
      // P buffer of this warpgroup is free once PV of its previous block has finished;
      // O is rescaled (warp-collective TMEM access) after PV of the previous block
      if (j > 0 && __any_sync(FULL, fac != 1.f)) {
        if (!__all_sync(FULL, mbar_wait(&bar[B_PE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort,
                                        a.err, 0x205, (t << 16) | j))) {
          ok = false;
          break;
        }
        tc_fence_after();
        rescale_row(tmem + lane_base + O_COL, fac);
      } else if (j >= 2) {
        if (!__all_sync(FULL, mbar_wait(&bar[B_PE + wg], kph ^ 1, abort, a.err, 0x206,
                                        (t << 16) | j))) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (t & 7)) * 16)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar[B_PF + wg]);
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait(&bar[B_DONE], 0, abort, a.err, 0x401, t);
    ok = __all_sync(FULL, ok);
    tc_fence_after();
    l_sh[(wg * 2) * TM + t] = l;
    l_sh[(wg * 2 + 1) * TM + t] = m_last;
    named_bar(3, 2 * TM);
    const float l0 = l_sh[t], m0 = l_sh[TM + t], l1 = l_sh[2 * TM + t], m1 = l_sh[3 * TM + t];
    const float mf = fmaxf(m0, m1);
    const float lt = l0 * ex2(m0 - mf) + l1 * ex2(m1 - mf);
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    if (wg == 0 && rank == 0 && a.lse && row_valid && ok)
      a.lse[grow] = (mf + log2f(lt)) * 0.69314718055994530942f;
    bf16* dst = a.o_lat + grow * G.Dc + rank * HALF;
#pragma unroll 1
    for (int c = wg * (HALF / 2); c < (wg + 1) * (HALF / 2); c += 32) {
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool tc_attend_supported(const Geo& g) { return g.Dc == 2 * HALF && g.Dr == 64; }

cudaError_t tc_attend(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                      const void* cache, int64_t k_first, int64_t n_keys, float scale,
                      void* o_lat, float* lse, unsigned int* err, cudaStream_t st) {
  CUtensorMap K, KR, QR;
  {
    uint64_t d[3] = {(uint64_t)g.row, (uint64_t)g.S, (uint64_t)g.B};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.S * g.row * 2};
    uint32_t b[3] = {64, BN, 1};
    if (!make_tmap_bf16(&K, cache, 3, d, s, b)) return cudaErrorInvalidValue;
    uint32_t br[3] = {32, BN, 1};
    if (!make_tmap_bf16(&KR, cache, 3, d, s, br, true)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[2] = {(uint64_t)g.row, (uint64_t)g.B * n_q * g.H};
    uint64_t s[1] = {(uint64_t)g.row * 2};
    uint32_t b[2] = {32, TM};
    if (!make_tmap_bf16(&QR, q_abs, 2, d, s, b, true)) return cudaErrorInvalidValue;
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
  attend_kernel<<<(unsigned)(2 * tiles), NTHREADS, ATT_SMEM, st>>>(K, KR, QR, a);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
