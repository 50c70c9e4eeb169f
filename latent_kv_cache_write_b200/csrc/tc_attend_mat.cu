// Non-absorbed ("materialised") MLA attention on tcgen05 tensor cores (bf16, d_nope = 128,
// d_R = 64 or 512).
//
// The per-head keys and values are rebuilt from the latent beforehand for every ring slot
// (tc_materialise: K_h = c . W_UK[h]^T and V_h = c . W_UV[h]^T, into the caller's
// workspace), so attention runs per head in head space, with the query and key the
// concatenation of the content and RoPE channels:
//   s = scale * ([q_nope || RoPE(q_R)] . [K_h[slot] || k_R[slot]]),  o = softmax(s) . V_h.
// A tile is 128 queries of one head, and one CTA holds it whole: O (128 x 128 fp32) and
// the query (128 x (128 + d_R) bf16) stay in TMEM beside two score buffers, so the CTAs
// share nothing.  Blocks are 64 keys for d_R = 64; for d_R = 512 the query takes 320 of the
// 512 TMEM columns, so blocks are 32 keys (two 32-column score buffers).  Per block the CTA
//   - TMA-loads the block's K_h rows (two 64-dim boxes), its cached k_R rows (one box, or
//     eight for d_R = 512) and its V_h rows (two boxes),
//   - computes S = Q . [K_h || k_R]^T with tcgen05.mma (the query as the TMEM A operand),
//   - runs the online softmax of the 128 rows (two warpgroups take alternate blocks and
//     hand each other the running row maximum),
//   - accumulates O += P . V_h (M=128, N=128) in TMEM.
// The CTAs are persistent over whole tiles, ordered (sequence, head, query block), so
// that the CTAs running at one time read the keys of a few heads from L2.
//
// Warp roles (352 threads): warps 0-3 and 4-7 are the softmax warpgroups (thread = row =
// TMEM lane), warp 8 is the TMA producer, warp 9 issues the score MMAs and owns the TMEM
// allocation, warp 10 issues the PV MMAs.
#include "attend_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.h"

#include <mutex>

namespace mla {
namespace {

using namespace tc;
using attn::Blocks;
using attn::key_end;
using attn::TM;

constexpr int NTHREADS = 352;
constexpr int DN = 128;                        // d_nope: per-head key and value width
constexpr int NST = 4;                         // K/V ring stages

// Layout of one variant (d_R = 64 or 512).  The ring is box-major: box q of stage s at
// OFF + (q * NST + s) * BOX, a box being 64 dims of the block's BN rows (128-byte rows).
template <int DRV>
struct MLay {
  static constexpr int DR = DRV;
  static constexpr int BN = DRV == 512 ? 32 : 64;        // keys per block
  static constexpr int BOX = BN * 64 * 2;                // one 64-dim box of a block
  static constexpr int NRB = DR / 64;                    // k_R boxes per stage
  static constexpr int STAGE = (4 + NRB) * BOX;          // K_h (2 boxes), k_R, V_h (2 boxes)
  static constexpr int PBUF = TM * BN * 2;               // P of one block
  static constexpr int OFF_K = 0;
  static constexpr int OFF_KR = OFF_K + 2 * NST * BOX;
  static constexpr int OFF_V = OFF_KR + NRB * NST * BOX;
  static constexpr int OFF_P = OFF_V + 2 * NST * BOX;    // [2]
  static constexpr int OFF_M = OFF_P + 2 * PBUF;         // running max [2][128]
  static constexpr int OFF_FREQ = OFF_M + 2 * TM * 4;    // RoPE frequencies [DR / 2] (double)
  static constexpr int OFF_BAR = OFF_FREQ + DR / 2 * 8;
  static constexpr int NBAR = 4 * 2 + 4 + 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static_assert(SMEM <= 227 * 1024, "dynamic shared memory of one CTA");
  static_assert(OFF_P % 1024 == 0, "P buffers on the swizzle atom");
  // TMEM columns: O (128), the query (64 for q_nope + DR / 2 for the RoPE part), S [2]
  static constexpr uint32_t O_COL = 0, Q_COL = 128, S_COL = DRV == 512 ? 448 : 256;
  static_assert(S_COL + 2 * BN <= 512 && Q_COL + (DN + DR) / 2 <= S_COL, "TMEM columns");
};
constexpr int B_KVF = 0;                       // stage loaded (TMA)                   [NST]
constexpr int B_KVE = B_KVF + NST;             // stage free (MMA commit after PV)    [NST]
constexpr int B_QREADY = B_KVE + NST;          // the tile's query in TMEM (256)
constexpr int B_QKDONE = B_QREADY + 1;         // every score MMA of a tile finished
constexpr int B_SEGDONE = B_QREADY + 2;        // every PV MMA of a tile finished
constexpr int B_OFREE = B_QREADY + 3;          // O of a tile read out of TMEM (256)
constexpr int B_SF = B_QREADY + 4;             // S buffer full (MMA commit)           [2]
constexpr int B_SE = B_SF + 2;                 // S buffer read (128)                  [2]
constexpr int B_PF = B_SE + 2;                 // P written, O rescaled (128)          [2]
constexpr int B_PE = B_PF + 2;                 // PV done (MMA commit)                 [2]
constexpr int B_M = B_PE + 2;                  // running max of a block published (128) [2]
static_assert(B_M + 2 == MLay<64>::NBAR, "barrier count");

constexpr unsigned FULL = 0xffffffffu;

struct MatArgs {
  Geo g;
  int64_t n_q, q_first, k_first, n_keys;
  float scale_log2;
  const bf16* q_nope;       // [B, n_q, H, DN]
  const bf16* q_rope;       // [B, n_q, H, d_R], un-rotated
  bf16* out;                // [B, n_q, H, DN]
  float* lse;               // [B, n_q, H] or null
  int qblocks;              // 128-query blocks per (sequence, head)
  int tiles;
  unsigned int* err;
};

// Tile t = ((b * H) + h) * qblocks + qb: queries [128 qb, 128 qb + 128) of head h.
struct MatTile {
  int b, h;
  int64_t i0, n_rows, i_last;
  Blocks blk;
};

template <int BN>
__device__ __forceinline__ MatTile mat_tile(const MatArgs& a, int t) {
  const Geo& G = a.g;
  MatTile m;
  const int qb = t % a.qblocks;
  const int bh = t / a.qblocks;
  m.h = bh % G.H;
  m.b = bh / G.H;
  m.i0 = (int64_t)qb * TM;
  m.n_rows = a.n_q - m.i0 < TM ? a.n_q - m.i0 : TM;
  m.i_last = m.i0 + m.n_rows - 1;
  Blocks& k = m.blk;
  k.k_first = a.k_first;
  k.L = key_end(G, a.q_first, a.k_first + a.n_keys, m.i_last) - a.k_first;
  k.p1 = a.k_first % G.S;
  k.n1 = k.L < G.S - k.p1 ? k.L : G.S - k.p1;
  k.bn = BN;
  k.nb1 = (int)((k.n1 + BN - 1) / BN);
  k.nblk = k.nb1 + (int)((k.L - k.n1 + BN - 1) / BN);
  return m;
}

// The tiles of one CTA, in order, with the running counts that barrier phases and ring
// stages derive from (every role walks the same sequence).
template <int BN>
struct TileWalk {
  int t, k, gbase, nbase0, nbase1;
  MatTile m;
  __device__ void begin(const MatArgs& a) {
    t = blockIdx.x;
    k = gbase = nbase0 = nbase1 = 0;
    if (valid(a)) m = mat_tile<BN>(a, t);
  }
  __device__ bool valid(const MatArgs& a) const { return t < a.tiles; }
  __device__ int nb() const { return m.blk.nblk; }
  __device__ int done_by(int w) const { return w ? nbase1 : nbase0; }
  __device__ void next(const MatArgs& a) {
    const int n = nb();
    gbase += n;
    nbase0 += (n + 1) >> 1;
    nbase1 += n >> 1;
    ++k;
    t += gridDim.x;
    if (valid(a)) m = mat_tile<BN>(a, t);
  }
};

__device__ __forceinline__ void rescale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < DN; c += 16) {
    uint32_t v[16];
    tmem_ld16(taddr + c, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * f);
    tmem_st16(taddr + c, v);
  }
  tmem_wait_st();
}

// The query of row i of the tile into TMEM from column tq: warpgroup 0 writes q_nope
// (64 columns of bf16 pairs), warpgroup 1 the RoPE'd q_R (DR / 2 columns), rotated by the
// query token's (t, y, x) position.
template <int DR>
__device__ __forceinline__ void load_q(const MatArgs& a, const MatTile& m, uint32_t tq,
                                       int t, int wg, const double* inv_freq) {
  const Geo& G = a.g;
  const int64_t i = m.i0 + t;
  const bool ok = t < m.n_rows;
  const int64_t row = ((int64_t)m.b * a.n_q + i) * G.H + m.h;
  if (wg == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(a.q_nope + row * DN);
    uint4 x[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) x[q] = ok ? src[q] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] = x[4 * c + q].x; v[4 * q + 1] = x[4 * c + q].y;
        v[4 * q + 2] = x[4 * c + q].z; v[4 * q + 3] = x[4 * c + q].w;
      }
      tmem_st16(tq + c * 16, v);
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(a.q_rope + row * DR);
    const RopeAxes ax = rope_axes(G, a.q_first + i);
    // 32 dims (16 pairs, 16 TMEM columns) at a time
#pragma unroll 1
    for (int c = 0; c < DR / 32; ++c) {
      uint4 x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) x[q] = ok ? src[4 * c + q] : make_uint4(0, 0, 0, 0);
      uint32_t v[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t w[4] = {x[q].x, x[q].y, x[q].z, x[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int p = 16 * c + 4 * q + e;            // RoPE pair: elements (2p, 2p + 1)
          float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
          rope_rotate_fast(lo, hi, rope_axis_pos(G, ax, p), inv_freq[p]);
          v[4 * q + e] = pack_bf16(lo, hi);
        }
      }
      tmem_st16(tq + 64 + c * 16, v);
    }
  }
  tmem_wait_st();
}

template <int DRV>
__global__ void __launch_bounds__(NTHREADS, 1)
    attend_mat_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKR,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ MatArgs a) {
  using LY = MLay<DRV>;
  constexpr int BN = LY::BN, DR = LY::DR, BOX = LY::BOX, NRB = LY::NRB, STAGE = LY::STAGE;
  constexpr int PBUF = LY::PBUF, OFF_K = LY::OFF_K, OFF_KR = LY::OFF_KR, OFF_V = LY::OFF_V;
  constexpr int OFF_P = LY::OFF_P, OFF_M = LY::OFF_M, OFF_FREQ = LY::OFF_FREQ;
  constexpr int OFF_BAR = LY::OFF_BAR, OFF_MISC = LY::OFF_MISC;
  constexpr uint32_t O_COL = LY::O_COL, Q_COL = LY::Q_COL, S_COL = LY::S_COL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  double* inv_freq = reinterpret_cast<double*>(sm + OFF_FREQ);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geo& G = a.g;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar[B_KVF + s], 1);
      mbar_init(&bar[B_KVE + s], 1);
    }
    mbar_init(&bar[B_QREADY], 256);
    mbar_init(&bar[B_QKDONE], 1);
    mbar_init(&bar[B_SEGDONE], 1);
    mbar_init(&bar[B_OFREE], 256);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bar[B_SF + q], 1);
      mbar_init(&bar[B_SE + q], 128);
      mbar_init(&bar[B_PF + q], 128);
      mbar_init(&bar[B_PE + q], 1);
      mbar_init(&bar[B_M + q], 128);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (tid < DR / 2) inv_freq[tid] = rope_inv_freq(G, tid);
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();                               // the previous kernel's outputs are visible
  grid_dep_launch();

  TileWalk<BN> tw;
  tw.begin(a);

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmKR);
      prefetch_tmap(&tmV);
      bool ok = true;
      for (; ok && tw.valid(a); tw.next(a)) {
        const MatTile& m = tw.m;
        for (int j = 0; j < m.blk.nblk; ++j) {
          const int g = tw.gbase + j, s = g % NST;
          ok = mbar_wait(&bar[B_KVE + s], ((g / NST) & 1) ^ 1, abort, a.err, 0x501, g);
          if (!ok) break;
          int64_t slot0, g0;
          int valid;
          m.blk.get(j, slot0, g0, valid);
          const int32_t r = (int32_t)((int64_t)m.b * G.S + slot0);   // row of K_h / V_h
          mbar_expect_tx(&bar[B_KVF + s], STAGE);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            tma_load_3d(sm + OFF_K + (q * NST + s) * BOX, &tmK, &bar[B_KVF + s], q * 64, m.h, r);
            tma_load_3d(sm + OFF_V + (q * NST + s) * BOX, &tmV, &bar[B_KVF + s], q * 64, m.h, r);
          }
#pragma unroll
          for (int q = 0; q < NRB; ++q)
            tma_load_3d(sm + OFF_KR + (q * NST + s) * BOX, &tmKR, &bar[B_KVF + s], G.Dc + 64 * q,
                        (int32_t)slot0, m.b);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ score MMA issuer
    // The scores of a block are one N=BN series into the S buffer of the warpgroup that
    // takes it: 8 K-steps over K_h and DR / 16 over k_R, the query as the TMEM A operand.
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, BN, false, false);
      bool ok = true;
      for (; ok && tw.valid(a); tw.next(a)) {
        ok = mbar_wait(&bar[B_QREADY], tw.k & 1, abort, a.err, 0x502, tw.k);
        if (!ok) break;
        tc_fence_after();
        const int n = tw.nb();
        for (int jl = 0; jl < n; ++jl) {
          const int w = jl & 1;                             // S buffer = warpgroup
          const int g = tw.gbase + jl, s = g % NST;
          const int q = tw.done_by(w) + (jl >> 1);           // S buffer use
          ok = mbar_wait(&bar[B_KVF + s], (g / NST) & 1, abort, a.err, 0x503, g);
          if (ok) ok = mbar_wait(&bar[B_SE + w], (q & 1) ^ 1, abort, a.err, 0x504, g);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + S_COL + w * BN;
          const uint64_t kd = desc_sw128(smem_u32(sm + OFF_K + s * BOX), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < DN / 16; ++kk)
            mma_ts(d, tmem + Q_COL + kk * 8,
                   kd + (uint64_t)(((kk >> 2) * NST * BOX + (kk & 3) * 32) >> 4), id_qk,
                   kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kr = 0; kr < DR / 16; ++kr) {
            const uint64_t rd =
                desc_sw128(smem_u32(sm + OFF_KR + ((kr >> 2) * NST + s) * BOX), 16, 1024);
            mma_ts(d, tmem + Q_COL + DN / 2 + kr * 8, rd + (uint64_t)(((kr & 3) * 32) >> 4),
                   id_qk, 1u);
          }
          mma_commit(&bar[B_SF + w]);
        }
        mma_commit(&bar[B_QKDONE]);
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ PV issuer
    // O += P . V_h in block order as each P is ready; the commits free the stage and the
    // P buffer and let the softmax rescale O.  A tile starts once the previous tile's O
    // has been read out; its last commit also covers its score MMAs.
    if (lane == 0) {
      const uint32_t id_pv = idesc_bf16(128, DN, false, true);
      bool ok = true;
      for (; ok && tw.valid(a); tw.next(a)) {
        if (tw.k > 0) ok = mbar_wait(&bar[B_OFREE], (tw.k - 1) & 1, abort, a.err, 0x505, tw.k);
        const int n = tw.nb();
        for (int jl = 0; ok && jl < n; ++jl) {
          const int pb = jl & 1, seq = tw.done_by(pb) + (jl >> 1);
          const int g = tw.gbase + jl, s = g % NST;
          ok = mbar_wait(&bar[B_PF + pb], seq & 1, abort, a.err, 0x506, g);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v0 = smem_u32(sm + OFF_V + s * BOX);
          const uint32_t pa = smem_u32(sm + OFF_P + pb * PBUF);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            // P is K-major: rows of BN keys, 128-byte swizzle (64 keys) or 64-byte (32 keys)
            const uint64_t pd = BN == 64 ? desc_sw128(pa + ks * 32, 16, 1024)
                                         : desc_sw64(pa, 512) + (uint64_t)((ks * 32) >> 4);
            mma_ss(tmem + O_COL, pd, desc_sw128(v0 + ks * 2048, NST * BOX, 1024), id_pv,
                   (jl > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_PE + pb]);
          mma_commit(&bar[B_KVE + s]);
        }
        if (ok) mma_commit(&bar[B_SEGDONE]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;                  // even (0) or odd (1) blocks
    const int t = tid & (TM - 1);              // row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float* m_sh = reinterpret_cast<float*>(sm + OFF_M);
    uint8_t* prow = sm + OFF_P + wg * PBUF + t * (BN * 2);
    const float c2 = a.scale_log2;
    bool ok = true;

    if (tw.valid(a)) {
      load_q<DR>(a, tw.m, tmem + lane_base + Q_COL, t, wg, inv_freq);
      tc_fence_before();
      mbar_arrive(&bar[B_QREADY]);
    }
    for (; tw.valid(a); tw.next(a)) {
      const MatTile& m = tw.m;
      const bool row_valid = t < m.n_rows;
      const int64_t i = m.i0 + t;
      const int64_t k_end_row =
          key_end(G, a.q_first, a.k_first + a.n_keys, row_valid ? i : m.i_last);
      const int n = tw.nb();
      float m_last = -INFINITY, l = 0.f;       // this warpgroup's running sum and its max
      for (int jl = wg; jl < n; jl += 2) {
        const int seq = tw.done_by(wg) + (jl >> 1);
        const uint32_t kph = seq & 1;
        if (!__all_sync(FULL, mbar_wait(&bar[B_SF + wg], kph, abort, a.err, 0x601, (t << 16) | jl))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
        {
          uint32_t v[BN / 32][32];
#pragma unroll
          for (int h = 0; h < BN / 32; ++h) tmem_ld32(tmem + lane_base + S_COL + wg * BN + 32 * h, v[h]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < BN / 32; ++h)
#pragma unroll
            for (int c = 0; c < 32; ++c) s[32 * h + c] = __uint_as_float(v[h][c]);
        }
        tc_fence_before();
        mbar_arrive(&bar[B_SE + wg]);

        int64_t slot0, g0;
        int valid;
        m.blk.get(jl, slot0, g0, valid);
        if (valid < BN && t < BN && t >= valid) {
          // a partial block: zero the V_h rows past the last key, so that masked keys add
          // exact zeros to P.V whatever those rows hold (the stage has landed: this
          // block's score MMAs have completed)
          uint8_t* st = sm + OFF_V + ((tw.gbase + jl) % NST) * BOX + t * 128;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint4* p = reinterpret_cast<uint4*>(st + q * NST * BOX);
#pragma unroll
            for (int w = 0; w < 8; ++w) p[w] = make_uint4(0, 0, 0, 0);
          }
        }

        // masked raw maximum (scores are scaled inside the exponent)
        const int64_t lim64 = k_end_row - g0;
        const int lim = lim64 < valid ? (lim64 < 0 ? 0 : (int)lim64) : valid;
        if (lim < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = c < lim ? s[c] : -INFINITY;
        }
        float rmax = s[0];
#pragma unroll
        for (int c = 1; c < BN; ++c) rmax = fmaxf(rmax, s[c]);
        const float mb = rmax * c2;

        // running maximum after the previous block (published by the other warpgroup)
        const int ow = wg ^ 1, oseq = tw.done_by(ow) + ((jl - 1) >> 1);
        float m_prev = -INFINITY;
        if (jl > 0) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_M + ow], oseq & 1, abort, a.err, 0x602,
                                          (t << 16) | jl))) {
            ok = false;
            break;
          }
          m_prev = m_sh[ow * TM + t];
        }
        float mx = m_prev, fac = 1.f;
        if (jl == 0) {
          mx = mb;
        } else if (mb > m_prev + 8.f) {
          mx = mb;
          fac = ex2(m_prev - mx);
        }
        m_sh[wg * TM + t] = mx;
        mbar_arrive(&bar[B_M + wg]);

        const float msub = mx == -INFINITY ? 0.f : mx;
        uint32_t pk[BN / 2];
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) {
          const float p0 = ex2(fmaf(s[2 * c], c2, -msub));
          const float p1 = ex2(fmaf(s[2 * c + 1], c2, -msub));
          sum += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
        l = l * ex2(m_last - msub) + sum;
        m_last = mx;
        // O is rescaled (warp-collective TMEM access) after PV of the previous block; the
        // P buffer is free once PV of this warpgroup's previous block has read it
        if (jl > 0 && __any_sync(FULL, fac != 1.f)) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + ow], oseq & 1, abort, a.err, 0x603,
                                          (t << 16) | jl))) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_o(tmem + lane_base + O_COL, fac);
        }
        if (!__all_sync(FULL, mbar_wait(&bar[B_PE + wg], kph ^ 1, abort, a.err, 0x604,
                                        (t << 16) | jl))) {
          ok = false;
          break;
        }
        // P row t, 16-byte chunks in the hardware swizzle: chunk ^ (row & 7) for 128-byte
        // rows (64 keys), chunk ^ ((row / 2) & 3) for 64-byte rows (32 keys)
#pragma unroll
        for (int c = 0; c < BN / 8; ++c) {
          const int cs = BN == 64 ? (c ^ (t & 7)) : (c ^ ((t >> 1) & 3));
          *reinterpret_cast<uint4*>(prow + cs * 16) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_PF + wg]);
      }
      if (!__all_sync(FULL, ok)) break;

      // the next tile's query may enter TMEM once this tile's score MMAs are done
      const uint32_t kph = tw.k & 1;
      {
        TileWalk<BN> nx = tw;
        nx.next(a);
        if (nx.valid(a)) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_QKDONE], kph, abort, a.err, 0x701, t))) break;
          tc_fence_after();
          load_q<DR>(a, nx.m, tmem + lane_base + Q_COL, t, wg, inv_freq);
          tc_fence_before();
          mbar_arrive(&bar[B_QREADY]);
        }
      }

      // ---------------------------------------------------------- tile epilogue
      if (!__all_sync(FULL, mbar_wait(&bar[B_SEGDONE], kph, abort, a.err, 0x702, t))) break;
      tc_fence_after();
      // the two warpgroups' (l, m) meet in the running-max array, which no block of this
      // tile reads any more: the maxima, then the sums at the common maximum
      m_sh[wg * TM + t] = m_last;
      named_bar(3, 2 * TM);
      const float mf = fmaxf(m_last, m_sh[(wg ^ 1) * TM + t]);
      named_bar(3, 2 * TM);
      m_sh[wg * TM + t] = m_last > -INFINITY ? l * ex2(m_last - mf) : 0.f;
      named_bar(3, 2 * TM);
      const float lt = m_sh[t] + m_sh[TM + t];
      named_bar(3, 2 * TM);                  // both have read: the array is the next tile's
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const int64_t orow = ((int64_t)m.b * a.n_q + i) * G.H + m.h;
      if (wg == 0 && row_valid && a.lse)
        a.lse[orow] = lt > 0.f ? (mf + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      // each warpgroup writes half of the row's d_nope outputs
      uint32_t v[2][32];
      tmem_ld32(tmem + lane_base + O_COL + wg * (DN / 2), v[0]);
      tmem_ld32(tmem + lane_base + O_COL + wg * (DN / 2) + 32, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar[B_OFREE]);
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + orow * DN + wg * (DN / 2));
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t* w = &v[hh][8 * q];
            dst[4 * hh + q] = make_uint4(
                pack_bf16(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                pack_bf16(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                pack_bf16(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                pack_bf16(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
          }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DRV>
int sm_count() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 0;
  if (cudaFuncSetAttribute(attend_mat_kernel<DRV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           MLay<DRV>::SMEM) != cudaSuccess)
    return 0;
  if (dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

bool tc_attend_mat_supported(const Geo& g) {
  return g.Dn == DN && (g.Dr == 64 || g.Dr == 512) && g.Dc % 128 == 0 &&
         (int64_t)g.B * g.S < INT32_MAX;
}

cudaError_t tc_attend_mat(const Geo& g, const void* q_nope, const void* q_rope, int64_t n_q,
                          int64_t q_first, const void* cache, const void* k_mat,
                          const void* v_mat, int64_t k_first, int64_t n_keys, float scale,
                          void* out, float* lse, unsigned int* err, cudaStream_t st) {
  const bool wide = g.Dr == 512;
  const int bn = wide ? MLay<512>::BN : MLay<64>::BN;
  CUtensorMap K, KR, V;
  {
    // K_h / V_h as (d_nope, heads, slots of all sequences): 64-dim boxes of 64 slots
    uint64_t d[3] = {(uint64_t)DN, (uint64_t)g.H, (uint64_t)g.B * g.S};
    uint64_t s[2] = {(uint64_t)DN * 2, (uint64_t)g.H * DN * 2};
    uint32_t b[3] = {64, 1, (uint32_t)bn};
    if (!make_tmap_bf16(&K, k_mat, 3, d, s, b)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&V, v_mat, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    // the cached rows, for their k_R columns: (row, slots, sequences)
    uint64_t d[3] = {(uint64_t)g.row, (uint64_t)g.S, (uint64_t)g.B};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.S * g.row * 2};
    uint32_t b[3] = {64, (uint32_t)bn, 1};
    if (!make_tmap_bf16(&KR, cache, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  const int nsm = wide ? sm_count<512>() : sm_count<64>();
  if (nsm == 0) return cudaErrorInvalidDevice;
  MatArgs a{};
  a.g = g;
  a.n_q = n_q; a.q_first = q_first; a.k_first = k_first; a.n_keys = n_keys;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_nope = (const bf16*)q_nope;
  a.q_rope = (const bf16*)q_rope;
  a.out = (bf16*)out;
  a.lse = lse;
  a.qblocks = (int)((n_q + TM - 1) / TM);
  const int64_t tiles = (int64_t)g.B * g.H * a.qblocks;
  if (tiles > INT32_MAX / 2) return cudaErrorInvalidValue;
  a.tiles = (int)tiles;
  a.err = err;
  if (a.tiles == 0) return cudaSuccess;
  const int grid = a.tiles < nsm ? a.tiles : nsm;
  cudaError_t e =
      wide ? launch_dependent(attend_mat_kernel<512>, (unsigned)grid, NTHREADS, MLay<512>::SMEM,
                              st, 1u, K, KR, V, a)
           : launch_dependent(attend_mat_kernel<64>, (unsigned)grid, NTHREADS, MLay<64>::SMEM,
                              st, 1u, K, KR, V, a);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
