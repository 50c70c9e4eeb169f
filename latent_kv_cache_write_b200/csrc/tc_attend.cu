// Absorbed MLA attention on tcgen05 tensor cores (bf16, d_c = 512, d_R = 64 or 512).
//
// Rows of the problem are (query, head) pairs; all heads share the cached rows
// [c_KV || k_R], which serve both as keys (all 576 dims) and as values (the 512 latent
// dims): S = Q_abs . [c || k_R]^T, P = softmax(S), O_lat = P . c.
//
// A 128 x 512 fp32 output accumulator fills a whole SM's tensor memory, so each 128-row
// tile is handled by a cluster of two CTAs that split the latent dimension: CTA c owns
// latent dims [256c, 256c + 256) and half of the RoPE dims ([32c, 32c + 32) for d_R = 64,
// [256c, 256c + 256) for d_R = 512).  Per block of 64 keys each CTA
//   - TMA-loads its columns of the 64 cached rows (one load serves as K and as V),
//   - computes its partial score S_c = Q_c . K_c^T with tcgen05.mma (Q's latent half
//     resident in TMEM as the A operand, the RoPE part from shared memory),
//   - swaps partial scores with its peer through distributed shared memory, so both
//     CTAs hold the full scores of all 128 rows: a row's partials go rounded to fp16
//     while none exceeds a bound (a few tenths of a percent of a softmax weight at most),
//     else as exact fp32 in two rounds,
//   - runs the online softmax of all 128 rows itself (its own fp32 partial plus the
//     peer's; the CTAs' row sums may differ in the last bits, and each normalises its own
//     half of O with its own sum),
//   - accumulates O_c += P . V_c (M=128, N=256) into its TMEM.
//
// Two softmax warpgroups take alternate key blocks, so the exchange of one block
// overlaps the exponentials of the other; they hand the running row maximum to each
// other through shared memory.  In the wide variant the buffer the peer's partial scores
// land in takes P once they are read.  O is rescaled only when a row maximum grows by
// more than 8 (log2 units).  Masking is frame-block-causal per row; a ring that wraps is
// walked as two contiguous slot segments.  The kernel is launched dependent on the
// previous kernel of the stream: its prologue (barriers, TMEM) runs while that kernel
// finishes, and it waits for it before touching any buffer.
//
// Scheduling is persistent and split-key ("stream-K"): the launch has one cluster per
// pair of SMs, and the key blocks of all tiles, laid end to end, are cut into one equal
// range per cluster.  A cluster walks its range as segments (blocks [jb, je) of one
// tile); a segment that covers its whole tile writes the final output, any other writes
// its normalised partial output and log-sum-exp to the workspace, and a combine kernel
// merges the partials of each split tile.  Without a workspace the cuts fall on tile
// boundaries only.
//
// Warp roles (352 threads): warps 0-3 and 4-7 are the two softmax warpgroups (thread =
// row = TMEM lane), warp 8 is the TMA producer, warp 9 issues the score MMAs, loads the
// Q RoPE tiles and owns the TMEM allocation, warp 10 issues the PV MMAs.
#include "attend_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.h"

#include <cuda_fp16.h>

#include <mutex>
#include <vector>

namespace mla {
namespace {

using namespace tc;
using namespace attn;

// Three variants of one kernel, chosen per call by the host; all take 64-key blocks.
//   V = 0: d_R = 64: 4 K/V stages, separate exchange and P buffers; a warpgroup hands its
//          exchange buffer back to the peer as soon as it has read it.
//   V = 1: d_R = 512 (the wide positional key): each CTA's 256 RoPE dims as four 64-dim
//          boxes, Q's RoPE half (64 KB) in shared memory.  The latent half of a block
//          (32 KB, held until its PV product) and its RoPE boxes (32 KB, read by the score
//          MMAs only) have rings of their own: 3 latent stages and one RoPE slot, which
//          is reloaded as soon as a block's scores are done.  P is written over the
//          exchange buffer once the scores are read, and the PV product's commit,
//          multicast to the peer, hands the buffer back.
//   V = 2: d_R = 64 over the low-bit ring: as V = 0 with 3 K/V stages, and the stages are
//          not loaded but written.  TMA brings each block's packed codes and scales into a
//          3-slot staging ring, and two warps (one key row per lane; 384 threads) write the
//          dequantised bf16 rows into the stage in the layout the TMA loads would have.
// K/V ring, box-major: latent box q (dims 64q..64q+63 of this CTA's half, 128-byte
// swizzle) of stage s at OFF_KV + (q * NST + s) * BOXB; RoPE box q of RoPE slot r at
// OFF_KVR + (q * NSTR + r) * RBB (NSTR = NST and r = s except for V = 1).
// A per-block barrier completes once per use of its buffer, a per-segment one once per
// segment; a waiter counts the uses and waits on the parity of the count.
template <int V>
struct Lay {
  static constexpr bool WIDE = V == 1;
  static constexpr bool PACKED = V == 2;
  static constexpr int NT = PACKED ? 384 : 352;              // threads
  static constexpr int NST = WIDE ? 3 : (PACKED ? 3 : 4);     // latent stages
  static constexpr int NSTR = WIDE ? 1 : NST;                  // RoPE slots
  static constexpr bool MERGED = WIDE;
  static constexpr int BNK = 64;                             // keys per block
  static constexpr int BOXB = BNK * 64 * 2;                  // latent box: BNK keys x 64 dims
  static constexpr int LATB = 4 * BOXB;                      // this CTA's latent half
  static constexpr int NRB = WIDE ? 4 : 1;                   // RoPE boxes per stage
  static constexpr int RDIMS = WIDE ? 64 : 32;               // dims per RoPE box
  static constexpr int RBB = BNK * RDIMS * 2;                // RoPE box bytes
  static constexpr int STAGEB = LATB + NRB * RBB;            // bytes one stage's loads bring
  static constexpr int RHALF = NRB * RDIMS;                  // RoPE dims per CTA
  static constexpr int QRB = TM * RHALF * 2;                 // this CTA's Q RoPE part
  static constexpr int XPB = TM * BNK * 2;                   // exchange / P buffer (128-byte rows)
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_KVR = OFF_KV + NST * LATB;
  // packed variant: staging slots of one block's codes (this CTA's half of 64 rows; content
  // slots 1024-byte aligned for the swizzle) and scales (68 floats from a 16-byte aligned
  // row, per path)
  static constexpr int NSG = PACKED ? 3 : 0;
  static constexpr int SGC = 64 * 128, SGR = 64 * 16, SGS = 2 * 384;   // 128-byte aligned boxes
  static constexpr int OFF_SG = OFF_KVR + NSTR * NRB * RBB;         // content [NSG]
  static constexpr int OFF_SGR = OFF_SG + NSG * SGC;                // RoPE codes [NSG]
  static constexpr int OFF_SGS = OFF_SGR + NSG * SGR;               // scales [NSG]
  static constexpr int OFF_QR = (OFF_SGS + NSG * SGS + 1023) / 1024 * 1024;
  static constexpr int OFF_X = OFF_QR + QRB;                 // [2] exchange buffers
  static constexpr int OFF_P = MERGED ? OFF_X : OFF_X + 2 * XPB;   // [2] P buffers
  static constexpr int OFF_M = OFF_P + 2 * XPB;              // running max [2][128]
  static constexpr int OFF_BAR = OFF_M + 2 * TM * 4;
  static constexpr int B_KVF = 0;               // K/V stage loaded (TMA)                [NST]
  static constexpr int B_KVE = B_KVF + NST;     // K/V stage free (MMA commit after PV) [NST]
  static constexpr int B_QR = B_KVE + NST;      // Q RoPE tile of a segment loaded (TMA)
  static constexpr int B_QREADY = B_QR + 1;     // Q latent half of a segment in TMEM (256)
  static constexpr int B_QKDONE = B_QR + 2;     // every score MMA of a segment finished
  static constexpr int B_SEGDONE = B_QR + 3;    // every PV MMA of a segment finished
  static constexpr int B_OFREE = B_QR + 4;      // O of a segment read out of TMEM (256)
  static constexpr int B_SF = B_QR + 5;         // S buffer full (MMA commit)            [2]
  static constexpr int B_SE = B_SF + 2;         // S buffer read (128)                   [2]
  static constexpr int B_XF = B_SE + 2;         // peer's partial scores landed (tx)     [2]
  static constexpr int B_XE = B_XF + 2;         // exchange buffer in the peer free       [2]
  static constexpr int B_PF = B_XE + 2;         // P complete, O rescaled (128)          [2]
  static constexpr int B_PE = B_PF + 2;         // PV done (MMA commit)                  [2]
  static constexpr int B_M = B_PE + 2;          // running max of a block published (128) [2]
  static constexpr int B_KRE = B_M + 2;         // RoPE slot free (wide; MMA commit after the
                                                // scores)                                [NSTR]
  static constexpr int B_KRF = B_KRE + NSTR;    // RoPE slot loaded (wide; TMA)           [NSTR]
  static constexpr int B_SGF = B_KRF + NSTR;   // staging slot loaded (TMA)           [NSG]
  static constexpr int B_SGE = B_SGF + NSG;    // staging slot read (64)               [NSG]
  static constexpr int NBAR = B_SGE + NSG;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 48 + 1024;   // TMEM slot, abort flag, votes [2][4]
  static_assert(SMEM <= 227 * 1024, "dynamic shared memory of one CTA");
  static_assert(OFF_SG % 1024 == 0 && OFF_SGR % 128 == 0 && OFF_SGS % 128 == 0 &&
                OFF_QR % 1024 == 0 && OFF_X % 1024 == 0 && OFF_P % 1024 == 0,
                "TMA and swizzled boxes start on their alignment");
};

constexpr uint32_t O_COL = 0, Q_COL = 256, S_COL = 384;
constexpr int PF_BLOCKS = 1;                  // L2 look-ahead of the key loads (decode)
constexpr unsigned FULL = 0xffffffffu;

// Cluster c walks the key blocks from (cut_tile[c], cut_blk[c]) up to, not including,
// (cut_tile[c + 1], cut_blk[c + 1]) in tile-major order; its partial segments take the
// workspace slots slot0[c], slot0[c] + 1, ...
struct Sched {
  int32_t cut_tile[MAXC + 1];
  int32_t cut_blk[MAXC + 1];
  int32_t slot0[MAXC];
};

// The segments of one cluster's range, in order.  Every role walks the same sequence
// and keeps the running counts that barrier phases and ring stages derive from.
struct SegWalk {
  int tile, jb, je, tend, bend;
  int k;                    // segment index within this cluster
  int gbase;                // blocks of earlier segments (K/V ring position)
  int nbase[2];             // blocks of earlier segments taken by each warpgroup
  int slot;                 // workspace slot of the next partial segment
  TileGeo tg;

  __device__ void begin(const Sched& sc, const AttnArgs& a, int c) {
    tile = sc.cut_tile[c];
    jb = sc.cut_blk[c];
    tend = sc.cut_tile[c + 1];
    bend = sc.cut_blk[c + 1];
    k = 0;
    gbase = 0;
    nbase[0] = nbase[1] = 0;
    slot = sc.slot0[c];
    load(a);
  }
  __device__ bool valid() const { return tile < tend || (tile == tend && jb < bend); }
  __device__ void load(const AttnArgs& a) {
    if (!valid()) return;
    tg = tile_geo(a.g, a.n_q, a.q_first, a.k_first, a.n_keys, a.tiles_per_batch, tile, a.bn);
    je = tile == tend ? bend : tg.blk.nblk;
  }
  __device__ int nb() const { return je - jb; }
  // blocks of earlier segments taken by warpgroup w (a select, not an indexed load)
  __device__ int done_by(int w) const { return w ? nbase[1] : nbase[0]; }
  __device__ bool partial() const { return jb > 0 || je < tg.blk.nblk; }
  __device__ void next(const AttnArgs& a) {
    const int n = nb();
    gbase += n;
    nbase[0] += (n + 1) >> 1;
    nbase[1] += n >> 1;
    if (partial()) ++slot;
    ++k;
    ++tile;
    jb = 0;
    load(a);
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

// s[0..7] -= the eight fp16 values packed in x.
__device__ __forceinline__ void sub_f16x8(const uint4& x, float* s) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
    s[2 * e] -= f.x;
    s[2 * e + 1] -= f.y;
  }
}

// This thread's row of a 64-column S buffer (fp32 partial scores) -> s.
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&s)[64]) {
  uint32_t v[2][32];
  tmem_ld32(taddr, v[0]);
  tmem_ld32(taddr + 32, v[1]);
  tmem_wait_ld();
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int c = 0; c < 32; ++c) s[32 * h + c] = __uint_as_float(v[h][c]);
}

// Q latent half of row `grow` -> TMEM columns from `tq` (A operand of the score MMA),
// bf16 pairs per column; each warpgroup loads half of the row.  All 16 vector loads are
// issued before the first TMEM store, so their latencies overlap.
__device__ __forceinline__ void load_q(const AttnArgs& a, uint32_t tq, int64_t grow,
                                       bool row_ok, uint32_t rank, int wg) {
  const uint4* src = reinterpret_cast<const uint4*>(a.q_abs + grow * a.g.row + rank * HALF +
                                                    wg * (HALF / 2));
  uint4 x[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) x[q] = row_ok ? src[q] : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int c = 0; c < HALF / 64; ++c) {
    uint32_t v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[4 * q] = x[4 * c + q].x; v[4 * q + 1] = x[4 * c + q].y;
      v[4 * q + 2] = x[4 * c + q].z; v[4 * q + 3] = x[4 * c + q].w;
    }
    tmem_st16(tq + wg * (HALF / 4) + c * 16, v);
  }
  tmem_wait_st();
}

// Dequantise one key's packed row of this CTA's half into K/V stage rows (one lane = one
// key row k of the block).  A code pair becomes the bf16 pair (bias + c0, bias + c1) by
// placing the biased fields in the low mantissa bits of 128.0 (exact), then c = that - bias
// (exact) and c * s with s the row's scale rounded to bf16: one rounding of the product to
// bf16, as the MMA operand needs.
__device__ __forceinline__ uint32_t dq_pair(uint32_t biased_pair, uint32_t bias2, uint32_t s2) {
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&biased_pair);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&bias2);
  const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162*>(&s2);
  v = __hmul2(__hsub2(v, b), sc);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// eight INT4 codes (one 32-bit word, code i at bits 4i) -> eight bf16 (one 16-byte chunk)
__device__ __forceinline__ uint4 dq8_int4(uint32_t w, uint32_t s2) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;   // codes 2k, 2k+1 in byte k
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // byte k of lo to bits 0-7, byte k of hi to bits 16-23; then 0x4300 | (code ^ 8)
    const uint32_t pr = __byte_perm(lo, hi, (uint32_t)(k | (k << 4) | ((k + 4) << 8) | ((k + 4) << 12)));
    o[k] = dq_pair((pr & 0x000F000Fu) ^ 0x43084308u, 0x43084308u, s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}
// eight INT2 codes (the low 16 bits of w, code i at bits 2i) -> eight bf16
__device__ __forceinline__ uint4 dq8_int2(uint32_t w, uint32_t s2) {
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t f = (w >> (4 * k)) & 0xFu;               // codes 2k (bits 0-1), 2k+1 (2-3)
    o[k] = dq_pair(((f & 3u) | ((f >> 2) << 16)) ^ 0x43024302u, 0x43024302u, s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int V>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Lay<V>::NT, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKR,
                  const __grid_constant__ CUtensorMap tmQR, const __grid_constant__ CUtensorMap tmSC,
                  const __grid_constant__ CUtensorMap tmSR, const __grid_constant__ AttnArgs a,
                  const __grid_constant__ Sched sc) {
  using LY = Lay<V>;
  constexpr int NST = LY::NST, NSTR = LY::NSTR;
  constexpr int BN = LY::BNK, BOX_BYTES = LY::BOXB, RBOX_BYTES = LY::RBB;
  constexpr int STAGE_BYTES = LY::STAGEB, QR_BYTES = LY::QRB, XP_BYTES = LY::XPB;
  constexpr int OFF_KV = LY::OFF_KV, OFF_KVR = LY::OFF_KVR, OFF_QR = LY::OFF_QR;
  constexpr int OFF_X = LY::OFF_X, OFF_P = LY::OFF_P, OFF_M = LY::OFF_M;
  constexpr int B_KVF = LY::B_KVF, B_KVE = LY::B_KVE, B_QR = LY::B_QR, B_QREADY = LY::B_QREADY;
  constexpr int B_QKDONE = LY::B_QKDONE, B_SEGDONE = LY::B_SEGDONE, B_OFREE = LY::B_OFREE;
  constexpr int B_SF = LY::B_SF, B_SE = LY::B_SE, B_XF = LY::B_XF, B_XE = LY::B_XE;
  constexpr int B_PF = LY::B_PF, B_PE = LY::B_PE, B_M = LY::B_M, B_KRE = LY::B_KRE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + LY::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + LY::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + LY::OFF_MISC + 4);

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geo& G = a.g;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar[B_KVF + s], LY::PACKED ? 64 : 1);   // TMA, or the two dequantising warps
      mbar_init(&bar[B_KVE + s], 1);
    }
    for (int r = 0; r < NSTR; ++r) {
      mbar_init(&bar[B_KRE + r], 1);
      mbar_init(&bar[LY::B_KRF + r], 1);
    }
    for (int q = 0; q < LY::NSG; ++q) {
      mbar_init(&bar[LY::B_SGF + q], 1);
      mbar_init(&bar[LY::B_SGE + q], 64);
    }
    mbar_init(&bar[B_QR], 1);
    mbar_init(&bar[B_QREADY], 256);
    mbar_init(&bar[B_QKDONE], 1);
    mbar_init(&bar[B_SEGDONE], 1);
    mbar_init(&bar[B_OFREE], 256);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bar[B_SF + q], 1);
      mbar_init(&bar[B_SE + q], 128);
      mbar_init(&bar[B_XF + q], 1);
      mbar_init(&bar[B_XE + q], 1);
      mbar_init(&bar[B_PF + q], 128);
      mbar_init(&bar[B_PE + q], 1);
      mbar_init(&bar[B_M + q], 128);
    }
    *abort = 0;
    for (int q = 0; q < 8; ++q) reinterpret_cast<uint32_t*>(sm + LY::OFF_MISC + 16)[q] = 0u;
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
  grid_dep_wait();                               // the previous kernel's outputs are visible
  grid_dep_launch();

  SegWalk sw;
  sw.begin(sc, a, blockIdx.x >> 1);

  if (LY::PACKED && (warp == 8 || warp == 11)) {
    // ------------------------------------------------------------ dequantising producers
    // Lane 0 of warp 8 keeps the staging ring NSG blocks ahead with TMA: the block's
    // content codes (this CTA's half of 64 rows, 128- or 64-byte swizzle), its RoPE codes and
    // both paths' scales.  Lane `lane` of warp 8 turns key row `lane` of every block into
    // bf16 stage rows, warp 11 row 32 + lane.
    constexpr int NSG = LY::NSG > 0 ? LY::NSG : 1;   // (the branch is dead for V = 0, 1)
    const int kr = (warp == 8 ? 0 : 32) + lane;
    const int cb = a.cbits;                       // 4 or 2; RoPE codes are 4 bits
    const int chalf = HALF * cb / 8;              // content bytes of a row for this CTA
    const bool issuer = warp == 8 && lane == 0;
    SegWalk iw = sw;                              // the issuer's walk, NSG blocks ahead
    int ij = iw.valid() ? iw.jb : 0, issued = 0;
    auto issue_next = [&]() -> bool {
      if (!iw.valid()) return true;
      const int q = issued % NSG;
      if (!mbar_wait(&bar[LY::B_SGE + q], ((issued / NSG) & 1) ^ 1, abort, a.err, 0x10B, issued))
        return false;
      int64_t slot0, g0;
      int valid;
      iw.tg.blk.get(ij, slot0, g0, valid);
      const int32_t row0 = (int32_t)((int64_t)iw.tg.b * G.S + slot0);
      const int32_t row4 = row0 & ~3;             // scales from a 16-byte aligned element
      uint8_t* scl = sm + LY::OFF_SGS + q * LY::SGS;
      mbar_expect_tx(&bar[LY::B_SGF + q], 64 * chalf + LY::SGR + 2 * 68 * 4);
      tma_load_2d(sm + LY::OFF_SG + q * LY::SGC, &tmK, &bar[LY::B_SGF + q], (int)rank * chalf, row0);
      tma_load_2d(sm + LY::OFF_SGR + q * LY::SGR, &tmKR, &bar[LY::B_SGF + q], (int)rank * 16, row0);
      tma_load_1d(scl, &tmSC, &bar[LY::B_SGF + q], row4);
      tma_load_1d(scl + 384, &tmSR, &bar[LY::B_SGF + q], row4);
      ++issued;
      if (++ij >= iw.je) {
        iw.next(a);
        ij = iw.valid() ? iw.jb : 0;
      }
      return true;
    };
    bool ok = true;
    if (issuer) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmKR);
      prefetch_tmap(&tmSC);
      prefetch_tmap(&tmSR);
      for (int q = 0; ok && q < NSG; ++q) ok = issue_next();
    }
    for (; ok && sw.valid(); sw.next(a)) {
      for (int j = sw.jb; j < sw.je; ++j) {
        const int g = sw.gbase + (j - sw.jb);
        const int s = g % NST, q = g % NSG;
        int64_t slot0, g0;
        int valid;
        sw.tg.blk.get(j, slot0, g0, valid);
        ok = mbar_wait(&bar[LY::B_SGF + q], (g / NSG) & 1, abort, a.err, 0x10A, (kr << 16) | j);
        if (ok) ok = mbar_wait(&bar[B_KVE + s], ((g / NST) & 1) ^ 1, abort, a.err, 0x109,
                               (kr << 16) | j);
        if (!ok) break;
        const uint8_t* scl = sm + LY::OFF_SGS + q * LY::SGS;
        const bool live = kr < valid;
        const int r4 = (int)(((int64_t)sw.tg.b * G.S + slot0) & 3) + kr;   // scale index
        const float scc = live ? reinterpret_cast<const float*>(scl)[r4] : 0.f;
        const float scr = live ? reinterpret_cast<const float*>(scl + 384)[r4] : 0.f;
        const uint32_t s2c = pack_bf16(scc, scc), s2r = pack_bf16(scr, scr);
        // this row's codes in the staging slot: 16-byte chunk c of a 128-byte row at chunk
        // c ^ (kr % 8) (INT4), of a 64-byte row at c ^ ((kr / 2) % 4) (INT2)
        const uint8_t* crow = sm + LY::OFF_SG + q * LY::SGC + kr * chalf;
        // the four 64-dim latent boxes, one per iteration (a compact loop: the unrolled body
        // would crowd the instruction cache the softmax warps share); row kr, 16-byte chunk c
        // at chunk c ^ (kr % 8)
#pragma unroll 1
        for (int bq = 0; bq < 4; ++bq) {
          uint8_t* box = sm + OFF_KV + (bq * NST + s) * BOX_BYTES + kr * 128;
          uint32_t ww[8];
          if (cb == 4) {
            // box bq holds codes 64 bq .. 64 bq + 63: staging chunks 2 bq, 2 bq + 1
            const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * bq) ^ (kr & 7)) * 16));
            const uint4 c1 =
                *reinterpret_cast<const uint4*>(crow + (((2 * bq + 1) ^ (kr & 7)) * 16));
            ww[0] = c0.x; ww[1] = c0.y; ww[2] = c0.z; ww[3] = c0.w;
            ww[4] = c1.x; ww[5] = c1.y; ww[6] = c1.z; ww[7] = c1.w;
          } else {
            const uint4 c0 = *reinterpret_cast<const uint4*>(crow + ((bq ^ ((kr >> 1) & 3)) * 16));
            const uint32_t hw[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) ww[c] = (c & 1) ? (hw[c >> 1] >> 16) : (hw[c >> 1] & 0xFFFFu);
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (live) v = cb == 4 ? dq8_int4(ww[c], s2c) : dq8_int2(ww[c], s2c);
            *reinterpret_cast<uint4*>(box + ((c ^ (kr & 7)) * 16)) = v;
          }
        }
        // the 32-dim RoPE box (64-byte rows, 64-byte swizzle: chunk c at c ^ ((kr / 2) % 4))
        {
          uint8_t* box = sm + OFF_KVR + s * RBOX_BYTES + kr * 64;
          const uint4 rw = *reinterpret_cast<const uint4*>(sm + LY::OFF_SGR + q * LY::SGR + kr * 16);
          const uint32_t rws[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(box + ((c ^ ((kr >> 1) & 3)) * 16)) =
                live ? dq8_int4(rws[c], s2r) : make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bar[B_KVF + s]);
        mbar_arrive(&bar[LY::B_SGE + q]);          // the staging slot may be refilled
        if (issuer) ok = issue_next();
        if (!__all_sync(FULL, ok)) {
          ok = false;
          break;
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmKR);
      // With a.pf > 0 the boxes of block j + a.pf are asked into L2 while block j's stage
      // is awaited: keys that no other tile reads come from HBM, and a stage is held from
      // its load to its PV product, so the stages alone keep too few loads in flight.
      auto prefetch_block = [&](int j) {
        int64_t slot0, g0;
        int valid;
        sw.tg.blk.get(j, slot0, g0, valid);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_prefetch_l2_3d(&tmK, (int)rank * HALF + q * 64, (int32_t)slot0, sw.tg.b);
        if constexpr (LY::WIDE) {
#pragma unroll
          for (int q = 0; q < LY::NRB; ++q)
            tma_prefetch_l2_3d(&tmK, G.Dc + (int)rank * LY::RHALF + q * 64, (int32_t)slot0,
                               sw.tg.b);
        } else {
          tma_prefetch_l2_3d(&tmKR, G.Dc + (int)rank * LY::RHALF, (int32_t)slot0, sw.tg.b);
        }
      };
      bool ok = true;
      for (; ok && sw.valid(); sw.next(a)) {
        if (a.pf > 0)
          for (int j = sw.jb; j < sw.je && j < sw.jb + a.pf; ++j) prefetch_block(j);
        for (int j = sw.jb; j < sw.je; ++j) {
          if (a.pf > 0 && j + a.pf < sw.je) prefetch_block(j + a.pf);
          const int g = sw.gbase + (j - sw.jb);
          const int s = g % NST;
          const uint32_t fph = ((g / NST) & 1) ^ 1;
          int64_t slot0, g0;
          int valid;
          sw.tg.blk.get(j, slot0, g0, valid);
          ok = mbar_wait(&bar[B_KVE + s], fph, abort, a.err, 0x101, g);
          if (!ok) break;
          mbar_expect_tx(&bar[B_KVF + s], LY::WIDE ? LY::LATB : STAGE_BYTES);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tma_load_3d(sm + OFF_KV + (q * NST + s) * BOX_BYTES, &tmK, &bar[B_KVF + s],
                        (int)rank * HALF + q * 64, (int32_t)slot0, sw.tg.b);
          if constexpr (LY::WIDE) {
            // the block's RoPE boxes, read only by its score MMAs: the slot is refilled as
            // soon as the previous block's scores are done
            const int r = g % NSTR;
            ok = mbar_wait(&bar[B_KRE + r], ((g / NSTR) & 1) ^ 1, abort, a.err, 0x109, g);
            if (!ok) break;
            mbar_expect_tx(&bar[LY::B_KRF + r], LY::NRB * RBOX_BYTES);
#pragma unroll
            for (int q = 0; q < LY::NRB; ++q)
              tma_load_3d(sm + OFF_KVR + (q * NSTR + r) * RBOX_BYTES, &tmK, &bar[LY::B_KRF + r],
                          G.Dc + (int)rank * LY::RHALF + q * 64, (int32_t)slot0, sw.tg.b);
          } else {
            tma_load_3d(sm + OFF_KVR + s * RBOX_BYTES, &tmKR, &bar[B_KVF + s],
                        G.Dc + (int)rank * LY::RHALF, (int32_t)slot0, sw.tg.b);
          }
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ score MMA issuer
    // The scores of a block are one N=64 series into the S buffer of the warpgroup that
    // takes it, issued as soon as the block's stage has landed and the buffer has been
    // read: the scores start the softmax chains.  An MMA issue blocks while the tensor
    // pipe is busy, so the PV products have their own issuing thread.  A segment's Q RoPE
    // tile is loaded once every score MMA of the previous segment has finished.
    if (lane == 0) {
      prefetch_tmap(&tmQR);
      const uint32_t id_qk1 = idesc_bf16(128, BN, false, false);
      // one score series: S columns [d, d + N) for the keys of stage s (RoPE slot r); the
      // wide variant waits for its RoPE slot between the latent and the RoPE steps
      auto qk_series = [&](uint32_t d, int s, int r, int g, uint32_t id) -> bool {
        // descriptor of K box column 0 at stage s; the 16-dim steps only add offsets
        const uint64_t kd = desc_sw128(smem_u32(sm + OFF_KV + s * BOX_BYTES), 16, 1024);
        mma_ts(d, tmem + Q_COL, kd, id, 0u);
#pragma unroll
        for (int kk = 1; kk < HALF / 16; ++kk)
          mma_ts(d, tmem + Q_COL + kk * 8,
                 kd + (uint64_t)(((kk >> 2) * NST * BOX_BYTES + (kk & 3) * 32) >> 4), id, 1u);
        if constexpr (LY::WIDE) {
          if (!mbar_wait(&bar[LY::B_KRF + r], (g / NSTR) & 1, abort, a.err, 0x10A, g))
            return false;
          tc_fence_after();
          // 256 RoPE dims: Q's from its four 128-row boxes, K's from the slot's four boxes
#pragma unroll
          for (int kr = 0; kr < LY::RHALF / 16; ++kr) {
            const int q = kr >> 2;
            const uint64_t qd = desc_sw128(smem_u32(sm + OFF_QR + q * (TM * 128)) + (kr & 3) * 32,
                                           16, 1024);
            const uint64_t rd =
                desc_sw128(smem_u32(sm + OFF_KVR + (q * NSTR + r) * RBOX_BYTES) + (kr & 3) * 32,
                           16, 1024);
            mma_ss(d, qd, rd, id, 1u);
          }
        } else {
          const uint64_t qd = desc_sw64(smem_u32(sm + OFF_QR), 512);
          const uint64_t rd = desc_sw64(smem_u32(sm + OFF_KVR + s * RBOX_BYTES), 512);
          mma_ss(d, qd, rd, id, 1u);
          mma_ss(d, qd + 2, rd + 2, id, 1u);            // second 16-dim step: +32 bytes
        }
        return true;
      };
      bool ok = true;
      for (; ok && sw.valid(); sw.next(a)) {
        const uint32_t kph = sw.k & 1;
        if (sw.k > 0) ok = mbar_wait(&bar[B_QKDONE], kph ^ 1, abort, a.err, 0x107, sw.k);
        if (!ok) break;
        mbar_expect_tx(&bar[B_QR], QR_BYTES);
        if constexpr (LY::WIDE) {
#pragma unroll
          for (int q = 0; q < LY::NRB; ++q)
            tma_load_2d(sm + OFF_QR + q * (TM * 128), &tmQR, &bar[B_QR],
                        G.Dc + (int)rank * LY::RHALF + q * 64, (int32_t)sw.tg.grow0);
        } else {
          tma_load_2d(sm + OFF_QR, &tmQR, &bar[B_QR], G.Dc + (int)rank * LY::RHALF,
                      (int32_t)sw.tg.grow0);
        }
        ok = mbar_wait(&bar[B_QREADY], kph, abort, a.err, 0x102, sw.k);
        if (ok) ok = mbar_wait(&bar[B_QR], kph, abort, a.err, 0x103, sw.k);
        if (!ok) break;
        tc_fence_after();
        const int n = sw.nb();
        for (int jl = 0; jl < n; ++jl) {
          const int w = jl & 1;                          // S buffer = warpgroup
          const int g = sw.gbase + jl, s = g % NST;
          const int q = sw.done_by(w) + (jl >> 1);         // S buffer use
          ok = mbar_wait(&bar[B_KVF + s], (g / NST) & 1, abort, a.err, 0x105, g);
          if (ok) ok = mbar_wait(&bar[B_SE + w], (q & 1) ^ 1, abort, a.err, 0x106, g);
          if (!ok) break;
          tc_fence_after();
          ok = qk_series(tmem + S_COL + w * BN, s, g % NSTR, g, id_qk1);
          if (!ok) break;
          mma_commit(&bar[B_SF + w]);
          if constexpr (LY::WIDE) mma_commit(&bar[B_KRE + g % NSTR]);
        }
        mma_commit(&bar[B_QKDONE]);
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ PV issuer
    // O += P . V in block order as each P is ready; the commits free the K/V stage for
    // the next load and the P buffer, let the softmax rescale O, and with merged
    // exchange/P buffers (multicast to the peer) let the peer send its next partial
    // scores into the buffer that held P.  A segment starts
    // once the previous segment's O has been read out (its first PV overwrites O); its
    // last commit also covers its score MMAs: a block's P exists only after its scores
    // were read.
    if (lane == 0) {
      const uint32_t id_pv = idesc_bf16(128, HALF, false, true);
      bool ok = true;
      for (; ok && sw.valid(); sw.next(a)) {
        if (sw.k > 0) ok = mbar_wait(&bar[B_OFREE], (sw.k - 1) & 1, abort, a.err, 0x108, sw.k);
        const int n = sw.nb();
        for (int jl = 0; ok && jl < n; ++jl) {
          const int pb = jl & 1, seq = sw.done_by(pb) + (jl >> 1);
          const int g = sw.gbase + jl, s = g % NST;
          ok = mbar_wait(&bar[B_PF + pb], seq & 1, abort, a.err, 0x104, g);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v0 = smem_u32(sm + OFF_KV + s * BOX_BYTES);
          const uint32_t pa = smem_u32(sm + OFF_P + pb * XP_BYTES);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            // P is K-major: 128-byte swizzled rows of 64 keys
            mma_ss(tmem + O_COL, desc_sw128(pa + ks * 32, 16, 1024),
                   desc_sw128(v0 + ks * 2048, NST * BOX_BYTES, 1024), id_pv,
                   (jl > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_PE + pb]);
          mma_commit(&bar[B_KVE + s]);
          if constexpr (LY::MERGED) mma_commit_cluster(&bar[B_XE + pb], (uint16_t)(1u << peer));
        }
        if (ok) mma_commit(&bar[B_SEGDONE]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;                  // warpgroup: even (0) or odd (1) blocks
    const int t = tid & (TM - 1);              // row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float* m_sh = reinterpret_cast<float*>(sm + OFF_M);
    const uint32_t peer_x = mapa(smem_u32(sm + OFF_X + wg * XP_BYTES), peer) + (uint32_t)t * 16;
    const uint32_t peer_xf = mapa(smem_u32(&bar[B_XF + wg]), peer);
    const uint32_t peer_xe = mapa(smem_u32(&bar[B_XE + wg]), peer);
    const uint4* my_x = reinterpret_cast<const uint4*>(sm + OFF_X + wg * XP_BYTES) + t;
    uint8_t* prow = sm + OFF_P + wg * XP_BYTES + t * (BN * 2);   // P row t
    const float c2 = a.scale_log2;
    bool ok = true;
    uint32_t xc = 0;        // exchange rounds this warpgroup has taken part in (barrier phases)
    uint32_t nd = 0;        // blocks this warpgroup has decided the exchange of
    uint32_t* xvote = reinterpret_cast<uint32_t*>(sm + LY::OFF_MISC + 16);

    if (sw.valid()) {
      load_q(a, tmem + lane_base + Q_COL, sw.tg.grow0 + t, sw.tg.row0 + t < sw.tg.rows_b, rank,
             wg);
      tc_fence_before();
      mbar_arrive(&bar[B_QREADY]);
    }
    for (; sw.valid(); sw.next(a)) {
      const TileGeo& tg = sw.tg;
      const int64_t r_in_b = tg.row0 + t;
      const bool row_valid = r_in_b < tg.rows_b;
      const int64_t grow = tg.grow0 + t;
      const int64_t k_end_row =
          key_end(G, a.q_first, a.k_first + a.n_keys, row_valid ? r_in_b / G.H : tg.i_last);
      const int n = sw.nb();
      {
        // the next segment's Q rows (this CTA's latent half, this warpgroup's half of it)
        // into L2 now, so that their load into TMEM at the segment's end is short
        SegWalk nx = sw;
        nx.next(a);
        if (nx.valid() && nx.tg.row0 + t < nx.tg.rows_b) {
          const char* qrow = reinterpret_cast<const char*>(
              a.q_abs + (nx.tg.grow0 + t) * G.row + rank * HALF + wg * (HALF / 2));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow + 128));
        }
      }
      float m_last = -INFINITY, l = 0.f;       // this warpgroup's running sum and its max
      for (int jl = wg; jl < n; jl += 2) {
        const int j = sw.jb + jl;              // block of the tile
        const int seq = sw.done_by(wg) + (jl >> 1);
        const uint32_t kph = seq & 1;
        // arm this block's first exchange round: the peer's asynchronous stores complete
        // XP_BYTES of transactions on it (they may land before or after this arrive)
        if (t == 0) mbar_expect_tx(&bar[B_XF + wg], XP_BYTES);
        if (!__all_sync(FULL, mbar_wait(&bar[B_SF + wg], kph, abort, a.err, 0x201, (t << 16) | j))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
        load_scores(tmem + lane_base + S_COL + wg * BN, s);
        tc_fence_before();
        mbar_arrive(&bar[B_SE + wg]);

        // send this CTA's partial scores into the peer's buffer once the peer is done
        // with it: it has read what was sent in this warpgroup's previous round (and,
        // with merged buffers, its PV has read the P held there)
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XE + wg], (xc & 1) ^ 1, abort, a.err,
                                                 0x202, (t << 16) | j))) {
          ok = false;
          break;
        }
        // The partials go rounded to fp16 (saturating: within 2^-11 of each partial).  A row
        // with a partial beyond a.xthr in magnitude sets bit 0 of its last 16-byte chunk (the
        // lowest mantissa bit of key 56), found while the first seven chunks travel; if any
        // row of either CTA did, both CTAs' warpgroups exchange exact fp32 partials below.
        bool need;
        {
          uint32_t hs[BN / 2];
#pragma unroll
          for (int c = 0; c < BN / 2; ++c) hs[c] = f16x2_satfinite(s[2 * c], s[2 * c + 1]);
#pragma unroll
          for (int q = 0; q < BN / 8 - 1; ++q)
            st_async_v4(peer_x + q * (TM * 16), hs[4 * q], hs[4 * q + 1], hs[4 * q + 2],
                        hs[4 * q + 3], peer_xf);
          float hi[4], lo[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            hi[c] = fmax3(s[16 * c], s[16 * c + 1], s[16 * c + 2]);
            lo[c] = fmin3(s[16 * c], s[16 * c + 1], s[16 * c + 2]);
#pragma unroll
            for (int e = 3; e < 15; e += 2) {
              hi[c] = fmax3(hi[c], s[16 * c + e], s[16 * c + e + 1]);
              lo[c] = fmin3(lo[c], s[16 * c + e], s[16 * c + e + 1]);
            }
            hi[c] = fmaxf(hi[c], s[16 * c + 15]);
            lo[c] = fminf(lo[c], s[16 * c + 15]);
          }
          need = fmaxf(fmax3(hi[0], hi[1], fmaxf(hi[2], hi[3])),
                       -fmin3(lo[0], lo[1], fminf(lo[2], lo[3]))) > a.xthr;
          constexpr int QL = BN / 8 - 1;
          st_async_v4(peer_x + QL * (TM * 16), (hs[4 * QL] & ~1u) | (need ? 1u : 0u),
                      hs[4 * QL + 1], hs[4 * QL + 2], hs[4 * QL + 3], peer_xf);
        }

        int64_t slot0, g0;
        int valid;
        tg.blk.get(j, slot0, g0, valid);
        if (valid < BN && t < BN && t >= valid) {
          // a partial block: zero this CTA's latent rows past the last key so that masked
          // keys contribute exact zeros to P.V whatever the ring holds there (the stage
          // has landed: the score MMAs of this block have completed)
          uint8_t* st = sm + OFF_KV + ((sw.gbase + jl) % NST) * BOX_BYTES + t * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4* p = reinterpret_cast<uint4*>(st + q * NST * BOX_BYTES);
#pragma unroll
            for (int w = 0; w < 8; ++w) p[w] = make_uint4(0, 0, 0, 0);
          }
        }

        // full scores: add the peer's partial
        if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XF + wg], xc & 1, abort, a.err, 0x203,
                                                 (t << 16) | j))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int q = 0; q < BN / 8; ++q) {
          const uint4 x = my_x[q * TM];
          if (q == BN / 8 - 1) need = need || (x.x & 1u) != 0u;
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            s[8 * q + 2 * e] = add_f32_f16(s[8 * q + 2 * e], w[e] & 0xFFFFu);
            s[8 * q + 2 * e + 1] = add_f32_f16(s[8 * q + 2 * e + 1], w[e] >> 16);
          }
        }
        ++xc;
        // The decision: a word per warpgroup and block (four in turn, each cleared two blocks
        // before its next use) collects the rows' flags across the barrier that also
        // marks the buffer as read.  Both CTAs see the same pairs of flags.
        volatile uint32_t* vote = xvote + wg * 4;
        if (need) atomicOr(const_cast<uint32_t*>(&vote[nd & 3]), 1u);
        named_bar(1 + wg, TM);
        const bool exact = vote[nd & 3] != 0u;
        if (t == 0) vote[(nd + 2) & 3] = 0u;
        ++nd;
        if (exact) {
          // Rounds two and three: undo the fp16 addend (s then holds this CTA's partial to
          // within one float32 rounding) and swap exact fp32 partials, keys 0-31 then 32-63.
#pragma unroll
          for (int q = 0; q < BN / 8; ++q) sub_f16x8(my_x[q * TM], s + 8 * q);
          named_bar(1 + wg, TM);                 // the buffer is read again before hand-back
          if (t == 0) {
            mbar_expect_tx(&bar[B_XF + wg], XP_BYTES);
            mbar_arrive_cluster_relaxed(peer_xe);
          }
          for (int h = 0; ok && h < 2; ++h) {
            if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XE + wg], (xc & 1) ^ 1, abort, a.err,
                                                     0x207, (t << 16) | j))) {
              ok = false;
              break;
            }
#pragma unroll
            for (int q = 0; q < BN / 8; ++q)
              st_async_v4(peer_x + q * (TM * 16), __float_as_uint(s[32 * h + 4 * q]),
                          __float_as_uint(s[32 * h + 4 * q + 1]),
                          __float_as_uint(s[32 * h + 4 * q + 2]),
                          __float_as_uint(s[32 * h + 4 * q + 3]), peer_xf);
            if (!__all_sync(FULL, mbar_wait_cluster(&bar[B_XF + wg], xc & 1, abort, a.err, 0x208,
                                                     (t << 16) | j))) {
              ok = false;
              break;
            }
#pragma unroll
            for (int q = 0; q < BN / 8; ++q) {
              const uint4 x = my_x[q * TM];
              s[32 * h + 4 * q] += __uint_as_float(x.x);
              s[32 * h + 4 * q + 1] += __uint_as_float(x.y);
              s[32 * h + 4 * q + 2] += __uint_as_float(x.z);
              s[32 * h + 4 * q + 3] += __uint_as_float(x.w);
            }
            ++xc;
            named_bar(1 + wg, TM);
            if (h == 0 && t == 0) mbar_expect_tx(&bar[B_XF + wg], XP_BYTES);   // round three
            // with merged buffers the last round's buffer is handed back by the PV commit
            if (!LY::MERGED || h == 0) {
              if (t == 0) mbar_arrive_cluster_relaxed(peer_xe);
            }
          }
          if (!ok) break;
        } else if constexpr (!LY::MERGED) {
          if (t == 0) mbar_arrive_cluster_relaxed(peer_xe);   // hand the buffer back
        }

        // masked raw maximum (scores are scaled inside the exponent)
        const int64_t lim64 = k_end_row - g0;
        const int lim = lim64 < valid ? (lim64 < 0 ? 0 : (int)lim64) : valid;
        if (lim < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = c < lim ? s[c] : -INFINITY;
        }
        float rm[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) rm[c] = s[c];
#pragma unroll
        for (int c = 8; c < BN; ++c) rm[c & 7] = fmaxf(rm[c & 7], s[c]);
        const float rmax = fmaxf(fmaxf(fmaxf(rm[0], rm[1]), fmaxf(rm[2], rm[3])),
                                 fmaxf(fmaxf(rm[4], rm[5]), fmaxf(rm[6], rm[7])));
        const float mb = rmax * c2;

        // running maximum after the previous block (published by the other warpgroup)
        const int ow = wg ^ 1, oseq = sw.done_by(ow) + ((jl - 1) >> 1);
        float m_prev = -INFINITY;
        if (jl > 0) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_M + ow], oseq & 1, abort, a.err, 0x204,
                                          (t << 16) | j))) {
            ok = false;
            break;
          }
          m_prev = m_sh[ow * TM + t];
        }
        float m = m_prev, fac = 1.f;
        if (jl == 0) {
          m = mb;
        } else if (mb > m_prev + 8.f) {
          m = mb;
          fac = ex2(m_prev - m);
        }
        m_sh[wg * TM + t] = m;
        mbar_arrive(&bar[B_M + wg]);

        const float msub = m == -INFINITY ? 0.f : m;
        uint32_t pk[BN / 2];
        float sums[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) {
          const float p0 = ex2(fmaf(s[2 * c], c2, -msub));
          const float p1 = ex2(fmaf(s[2 * c + 1], c2, -msub));
          sums[c & 3] += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
        const float sum = (sums[0] + sums[1]) + (sums[2] + sums[3]);
        l = l * ex2(m_last - msub) + sum;
        m_last = m;
        // O is rescaled (warp-collective TMEM access) after PV of the previous block.
        // The P buffer is free once PV of this warpgroup's previous block has read it
        // (with merged buffers that is implied: the peer sent this block's scores into
        // it only then).
        if (jl > 0 && __any_sync(FULL, fac != 1.f)) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + ow], oseq & 1, abort, a.err, 0x205,
                                          (t << 16) | j))) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_row(tmem + lane_base + O_COL, fac);
        }
        if constexpr (!LY::MERGED) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_PE + wg], kph ^ 1, abort, a.err, 0x206,
                                          (t << 16) | j))) {
            ok = false;
            break;
          }
        }
        // P row t, 16-byte chunks in the 128-byte hardware swizzle (chunk ^ (row & 7))
#pragma unroll
        for (int c = 0; c < BN / 8; ++c) {
          const int cs = c ^ (t & 7);
          *reinterpret_cast<uint4*>(prow + cs * 16) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_PF + wg]);
      }
      if (!__all_sync(FULL, ok)) break;

      // the next segment's Q may enter TMEM once this segment's score MMAs are done
      const uint32_t kph = sw.k & 1;
      {
        SegWalk nx = sw;
        nx.next(a);
        if (nx.valid()) {
          if (!__all_sync(FULL, mbar_wait(&bar[B_QKDONE], kph, abort, a.err, 0x301, t))) break;
          tc_fence_after();
          load_q(a, tmem + lane_base + Q_COL, nx.tg.grow0 + t, nx.tg.row0 + t < nx.tg.rows_b,
                 rank, wg);
          tc_fence_before();
          mbar_arrive(&bar[B_QREADY]);
        }
      }

      // ---------------------------------------------------------- segment epilogue
      if (!__all_sync(FULL, mbar_wait(&bar[B_SEGDONE], kph, abort, a.err, 0x401, t))) break;
      tc_fence_after();
      // the two warpgroups' (l, m) meet in the running-max array, which no block of this
      // segment reads any more (a warpgroup that gets here first rewrites its slot with
      // the value it published last): the maxima, then the sums at the common maximum
      m_sh[wg * TM + t] = m_last;
      named_bar(3, 2 * TM);
      const float mf = fmaxf(m_last, m_sh[(wg ^ 1) * TM + t]);
      named_bar(3, 2 * TM);
      m_sh[wg * TM + t] = m_last > -INFINITY ? l * ex2(m_last - mf) : 0.f;
      named_bar(3, 2 * TM);
      const float lt = m_sh[t] + m_sh[TM + t];
      named_bar(3, 2 * TM);                  // both have read: the array is the next segment's
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float lse_v = lt > 0.f ? (mf + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      const bool part = sw.partial();
      if (wg == 0 && row_valid) {
        if (part)
          a.ws_lse[((int64_t)sw.slot * 2 + rank) * TM + t] = lse_v;
        else if (a.lse && rank == 0)
          a.lse[grow] = lse_v;
      }
#pragma unroll 1
      for (int c = wg * (HALF / 2); c < (wg + 1) * (HALF / 2); c += 32) {
        uint32_t v[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_base + O_COL + c, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = 0u;
        }
        if (!row_valid) continue;
        if (part) {
          // the normalised partial, rounded to bf16 like a final output (the merge adds the
          // pieces of a row in fp32)
          uint4* dst = reinterpret_cast<uint4*>(a.ws_o + ((int64_t)sw.slot * TM + t) * G.Dc +
                                                rank * HALF + c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(
                pack_bf16(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv),
                pack_bf16(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv),
                pack_bf16(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv),
                pack_bf16(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv));
        } else {
          bf16* dst = a.o_lat + grow * G.Dc + rank * HALF + c;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
            reinterpret_cast<uint4*>(dst)[q] = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[B_OFREE]);
    }
    // with merged buffers the peer's last PV commit arrives on this CTA's barrier: let it
    // land before exit
    if constexpr (LY::MERGED) {
      if (ok && !sw.valid() && xc > 0)
        mbar_wait_cluster(&bar[B_XE + wg], (xc - 1) & 1, abort, a.err, 0x402, t);
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

// Clusters of the attention kernel that can be resident at once on the current device
// (one CTA per SM; a cluster needs two SMs of one GPC), capped at MAXC.  The first call
// on a device also opts the kernel in to its shared memory.  0 on failure.
int cluster_slots() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  // every variant is resident at one CTA per SM; the schedule (and the workspace size)
  // uses the smallest count any of them reaches
  int n = MAXC;
  bool ok = true;
  auto probe = [&](auto kern, int smem, int threads) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess) {
      ok = false;
      return;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * MAXC);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) != cudaSuccess || c < 1) c = 0;
    n = c < n ? c : n;
  };
  probe(attend_kernel<0>, Lay<0>::SMEM, Lay<0>::NT);
  probe(attend_kernel<1>, Lay<1>::SMEM, Lay<1>::NT);
  probe(attend_kernel<2>, Lay<2>::SMEM, Lay<2>::NT);
  if (!ok) return 0;
  if (n < 1) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    n = sms / 2;
  }
  n = n < 1 ? 1 : (n > MAXC ? MAXC : n);
  if (dev < 64) cached[dev] = n;
  return n;
}

// one partial slot: 128 rows of d_latent bf16 outputs and two fp32 log-sum-exps
size_t slot_bytes(const Geo& g) { return (size_t)TM * ((size_t)g.Dc * 2 + 2 * sizeof(float)); }

}  // namespace

bool tc_attend_supported(const Geo& g) {
  return g.Dc == 2 * HALF && (g.Dr == 2 * Lay<0>::RHALF || g.Dr == 2 * Lay<1>::RHALF);
}

size_t tc_attend_workspace(const Geo& g) { return 2 * (size_t)cluster_slots() * slot_bytes(g); }


bool tc_attend_packed_supported(const Geo& g, int cbits, int rbits) {
  return g.Dc == 2 * HALF && g.Dr == 2 * Lay<2>::RHALF && (cbits == 4 || cbits == 2) &&
         rbits == 4;
}

cudaError_t tc_attend(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                      const void* cache, int64_t k_first, int64_t n_keys, float scale,
                      void* o_lat, float* lse, void* workspace, size_t workspace_bytes,
                      unsigned int* err, cudaStream_t st) {
  return tc_attend_ring(g, q_abs, n_q, q_first, cache, nullptr, k_first, n_keys, scale, o_lat,
                        lse, workspace, workspace_bytes, err, st);
}

cudaError_t tc_attend_ring(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                           const void* cache, const PackedRing* pk, int64_t k_first,
                           int64_t n_keys, float scale, void* o_lat, float* lse,
                           void* workspace, size_t workspace_bytes, unsigned int* err,
                           cudaStream_t st) {
  const int tiles_per_batch = (int)((n_q * g.H + TM - 1) / TM);
  // the low-bit ring, the wide positional key, or d_R = 64
  const int variant = pk ? 2 : (g.Dr == 2 * Lay<1>::RHALF ? 1 : 0);
  const int bn = variant == 1 ? Lay<1>::BNK : Lay<0>::BNK;
  CUtensorMap K{}, KR{}, QR, SC{}, SR{};
  if (pk) {
    // the packed ring: content codes (this CTA's half of a row per box row), RoPE codes,
    // and the two paths' float32 scales
    const uint64_t rows = (uint64_t)g.B * g.S;
    const uint64_t crow = (uint64_t)g.Dc * pk->cbits / 8, rrow = (uint64_t)g.Dr * pk->rbits / 8;
    const uint32_t chalf = (uint32_t)(crow / 2);
    {
      uint64_t d[2] = {crow, rows};
      uint64_t st2[1] = {crow};
      uint32_t b[2] = {chalf, 64};
      if (!make_tmap_raw(&K, pk->codes_c, false, 2, d, st2, b, chalf == 128 ? 128 : 64))
        return cudaErrorInvalidValue;
    }
    {
      uint64_t d[2] = {rrow, rows};
      uint64_t st2[1] = {rrow};
      uint32_t b[2] = {(uint32_t)(rrow / 2), 64};
      if (!make_tmap_raw(&KR, pk->codes_r, false, 2, d, st2, b, 0)) return cudaErrorInvalidValue;
    }
    {
      uint64_t d[1] = {rows};
      uint32_t b[1] = {68};
      if (!make_tmap_raw(&SC, pk->scale_c, true, 1, d, nullptr, b, 0) ||
          !make_tmap_raw(&SR, pk->scale_r, true, 1, d, nullptr, b, 0))
        return cudaErrorInvalidValue;
    }
  } else {
    // K: 64-dim boxes of bn cached rows (the latent boxes, and the wide RoPE boxes);
    // KR: the 32-dim RoPE box of d_R = 64 (64-byte swizzle)
    uint64_t d[3] = {(uint64_t)g.row, (uint64_t)g.S, (uint64_t)g.B};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.S * g.row * 2};
    uint32_t b[3] = {64, (uint32_t)bn, 1};
    if (!make_tmap_bf16(&K, cache, 3, d, s, b)) return cudaErrorInvalidValue;
    uint32_t br[3] = {32, (uint32_t)bn, 1};
    if (!make_tmap_bf16(&KR, cache, 3, d, s, br, true)) return cudaErrorInvalidValue;
  }
  {
    // Q's RoPE part: one 32-dim box (64-byte swizzle), or 64-dim boxes (wide)
    uint64_t d[2] = {(uint64_t)g.row, (uint64_t)g.B * n_q * g.H};
    uint64_t s[1] = {(uint64_t)g.row * 2};
    uint32_t b[2] = {variant == 1 ? 64u : 32u, TM};
    if (!make_tmap_bf16(&QR, q_abs, 2, d, s, b, variant != 1)) return cudaErrorInvalidValue;
  }
  const int ncl = cluster_slots();
  if (ncl == 0) return cudaErrorInvalidDevice;
  AttnArgs a{};
  a.g = g;
  a.n_q = n_q; a.q_first = q_first; a.k_first = k_first; a.n_keys = n_keys;
  a.scale_log2 = scale * 1.4426950408889634f;
  {
    // The 16-bit exchange rounds a partial score to within 2^-11 of itself.  Up to
    // XCHG_LOG2 in the exponent's log2 units that error stays below 2^-8 of one such unit
    // (a few tenths of a percent of a softmax weight, like the bf16 rounding of P); rows
    // with larger partials get the exact exchange.  Capped well inside the fp16 range.
    constexpr float XCHG_LOG2 = 8.f;
    float thr = XCHG_LOG2 / a.scale_log2;
    if (!(thr <= 32768.f)) thr = 32768.f;
    a.xthr = thr;
  }
  a.q_abs = (const bf16*)q_abs;
  a.o_lat = (bf16*)o_lat;
  a.lse = lse;
  a.tiles_per_batch = tiles_per_batch;
  a.bn = bn;
  // a sequence's keys are read by its tiles only: with one or two tiles (decode) each key
  // block comes from HBM once, and the producer looks PF_BLOCKS blocks ahead
  a.pf = !pk && tiles_per_batch <= 2 ? PF_BLOCKS : 0;
  if (pk) {
    a.pk_c = static_cast<const uint8_t*>(pk->codes_c);
    a.pk_r = static_cast<const uint8_t*>(pk->codes_r);
    a.sc_c = pk->scale_c;
    a.sc_r = pk->scale_r;
    a.cbits = pk->cbits;
    a.rbits = pk->rbits;
  }
  a.err = err;
  const bool split = workspace != nullptr && workspace_bytes >= tc_attend_workspace(g);

  // ---- batches per launch.  Every tile of a sequence reads that sequence's keys.  With
  // all sequences in one launch, each cluster walks its own run of consecutive tiles, so
  // the clusters spread over every sequence at once and, when the sequences' keys
  // together crowd L2, they are read from HBM again and again.  Sequences then go in
  // groups whose keys fit a third of L2, as long as a group's tiles still give every
  // cluster several; groups run one after another (stream order also keeps the
  // workspace of one group's merge apart from the next group's partials).
  int group = g.B;
  {
    int dev = 0, l2 = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) == cudaSuccess && l2 > 0) {
      const double key_bytes = pk ? (double)g.Dc * pk->cbits / 8 + g.Dr * pk->rbits / 8 + 8
                                  : (double)g.row * 2;
      const double keys_bytes = (double)n_keys * key_bytes;     // one sequence's keys
      if (keys_bytes * g.B > l2 / 3.0) {
        const int by_l2 = (int)((l2 / 3.0) / keys_bytes);                  // fit a third of L2
        const int fill = (4 * ncl + tiles_per_batch - 1) / tiles_per_batch;   // >= 4 tiles each
        const int want = by_l2 > fill ? by_l2 : fill;
        group = want < 1 ? 1 : (want < g.B ? want : g.B);
      }
    }
  }

  // Every group's schedule is built and checked before the first launch, so an error
  // leaves nothing enqueued.
  struct Plan {
    Sched sc;
    CombineList cl;
    int G;
  };
  std::vector<Plan> plans;
  bool any_partial = false;
  for (int b0 = 0; b0 < g.B; b0 += group) {
    const int t_lo = b0 * tiles_per_batch;
    const int t_hi = (b0 + group < g.B ? b0 + group : g.B) * tiles_per_batch;
    const int Tg = t_hi - t_lo;

    // ---- schedule: the blocks of the group's tiles end to end, one equal range per
    // cluster (tile indices are absolute)
    std::vector<int64_t> pre(Tg + 1, 0);
    std::vector<int> nbt(Tg);
    for (int t = 0; t < Tg; ++t) {
      nbt[t] = tile_geo(g, n_q, q_first, k_first, n_keys, a.tiles_per_batch, t_lo + t, bn).blk.nblk;
      pre[t + 1] = pre[t] + nbt[t];
    }
    const int64_t W = pre[Tg];
    // Two candidate schedules, costed in key blocks: a cluster's blocks plus SEG_COST per
    // segment it walks (the switch: Q reload, output epilogue, pipeline refill), plus
    // COMBINE_COST when tiles are split (the merge launch).  Both costs were measured on
    // B200 (video chunk, long window and decode shapes).
    constexpr int64_t SEG_COST = 7, COMBINE_COST = 16;
    // schedules below are in group-relative tiles until they are shifted for the launch
    auto cost = [&](const Sched& c, int nc) {
      int64_t worst = 0;
      bool any_split = false;
      for (int k = 0; k < nc; ++k) {
        const int t0 = c.cut_tile[k], b0_ = c.cut_blk[k], t1 = c.cut_tile[k + 1], b1 = c.cut_blk[k + 1];
        const int64_t blocks = (pre[t1] + b1) - (pre[t0] + b0_);
        const int64_t segs = (int64_t)(t1 - t0) + (b1 > 0 ? 1 : 0);
        any_split = any_split || b0_ > 0 || b1 > 0;
        worst = blocks + SEG_COST * segs > worst ? blocks + SEG_COST * segs : worst;
      }
      return worst + (any_split ? COMBINE_COST : 0);
    };
    // cuts on tile boundaries: the first one at or past an equal share of the blocks (of
    // the tiles when there are no blocks)
    Sched whole{};
    const int G_whole = Tg < ncl ? Tg : ncl;
    {
      int t = 0;
      for (int c = 1; c <= G_whole; ++c) {
        if (c == G_whole) {
          t = Tg;
        } else if (W > 0) {
          const int64_t pos = W * c / G_whole;
          while (t < Tg && pre[t] < pos) ++t;
        } else {
          t = (int)((int64_t)Tg * c / G_whole);
        }
        whole.cut_tile[c] = t;
        whole.cut_blk[c] = 0;
      }
    }
    Sched sc = whole;
    int G = G_whole;
    if (split && W > 0) {
      // cut c at block W*c/G; tiles without blocks go with the range before them
      Sched sk{};
      const int G_split = (int)(W < ncl ? W : ncl);
      int t = 0;
      for (int c = 1; c <= G_split; ++c) {
        const int64_t pos = W * c / G_split;
        while (t < Tg && pre[t + 1] <= pos) ++t;      // tile holding block `pos`
        sk.cut_tile[c] = t;
        sk.cut_blk[c] = t < Tg ? (int)(pos - pre[t]) : 0;
      }
      if (cost(sk, G_split) < cost(whole, G_whole)) {
        sc = sk;
        G = G_split;
      }
    }
    sc.cut_tile[0] = 0;
    sc.cut_blk[0] = 0;
    // partial segments: their workspace slots, and the tiles to combine
    CombineList cl{};
    int nslot = 0;
    for (int c = 0; c < G; ++c) {
      sc.slot0[c] = nslot;
      int t = sc.cut_tile[c], jb = sc.cut_blk[c];
      const int tend = sc.cut_tile[c + 1], bend = sc.cut_blk[c + 1];
      while (t < tend || (t == tend && jb < bend)) {
        const int je = t == tend ? bend : nbt[t];
        if (jb > 0 || je < nbt[t]) {
          if (cl.n == 0 || cl.tile[cl.n - 1] != t_lo + t) {
            if (cl.n == MAXC) return cudaErrorInvalidValue;   // at most G - 1 cuts split
            cl.piece0[cl.n] = nslot;
            cl.tile[cl.n++] = t_lo + t;
          }
          ++nslot;
        }
        ++t;
        jb = 0;
      }
    }
    cl.piece0[cl.n] = nslot;
    if (nslot > 2 * ncl) return cudaErrorInvalidValue;    // at most two per cluster
    any_partial = any_partial || nslot > 0;
    if (G == 0) continue;
    for (int c = 0; c <= G; ++c) sc.cut_tile[c] += t_lo;
    plans.push_back(Plan{sc, cl, G});
  }
  if (any_partial) {
    a.ws_o = (bf16*)workspace;
    a.ws_lse = reinterpret_cast<float*>(a.ws_o + (size_t)2 * ncl * TM * g.Dc);
  }
  for (const Plan& p : plans) {
    cudaError_t e;
    if (variant == 2)
      e = launch_dependent(attend_kernel<2>, (unsigned)(2 * p.G), Lay<2>::NT, Lay<2>::SMEM, st, 1u,
                           K, KR, QR, SC, SR, a, p.sc);
    else if (variant == 1)
      e = launch_dependent(attend_kernel<1>, (unsigned)(2 * p.G), Lay<1>::NT, Lay<1>::SMEM, st, 1u,
                           K, KR, QR, SC, SR, a, p.sc);
    else
      e = launch_dependent(attend_kernel<0>, (unsigned)(2 * p.G), Lay<0>::NT, Lay<0>::SMEM, st, 1u,
                           K, KR, QR, SC, SR, a, p.sc);
    if (e != cudaSuccess) return e;
    count_launches(1);
    if (p.cl.n > 0) {
      e = launch_combine(a, p.cl, st);
      if (e != cudaSuccess) return e;
      count_launches(1);
    }
  }
  return cudaSuccess;
}

}  // namespace mla
