// Tensor-core (tcgen05) GEMMs of the path, bf16 in, fp32 accumulation in TMEM:
//   cache write:  [h] x [W_DKV | W_KR]  -> RoPE on the W_KR columns -> bf16 -> ring slot
//   absorb:       q_nope[:, h] x W_UK[h] -> q_lat (plus RoPE of q_R in the same CTAs)
//   up-projection: o_lat[:, h] x W_UV[h]^T -> out
//   materialisation: c[slot] x W[h]^T -> per-head keys or values of every ring slot
// Persistent: one CTA per SM walks the 128 x 128 output tiles (M fastest, so CTAs that
// run together share the weight tile in L2).  Warp 0 lane 0 streams TMA loads through a
// 4-stage shared-memory ring, warp 1 lane 0 issues tcgen05.mma (M=128, N=128, K=16 steps)
// into one of two TMEM accumulators, and warps 2-5 drain the other accumulator (one row
// per thread) through the fused epilogue, so a tile's epilogue overlaps the next tile's
// main loop.
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.h"

#include <mutex>

namespace mla {
namespace {

using namespace tc;

constexpr int GBM = 128, GBK = 64, GBN = 128;

constexpr int GTHREADS = 192;
constexpr int A_BYTES = GBM * GBK * 2;           // 16 KB
constexpr int B_BYTES = GBN * GBK * 2;           // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MAX_PAIRS = 512;                   // RoPE pairs with a table entry (d_R <= 1024)
constexpr int STG_BYTES = 32 * 64;                // per epilogue warp: 32 rows x 32 cols bf16
constexpr int RB_BYTES = GBM * GBN * 4;          // split-K partial accumulator, 64 KB
// Shared memory: the stage ring, barriers, the RoPE frequency table, epilogue staging and,
// with split-K, the buffer the other CTA of the pair sends its fp32 partial tile into.
constexpr int OBOX_BYTES = GBM * 64 * 2;         // TMA-store box: 128 rows x 64 cols bf16
template <int ST, bool SK> struct GLay {
  static constexpr int OFF_TAB = ST * STAGE_BYTES + 256;
  static constexpr int OFF_STG = OFF_TAB + MAX_PAIRS * 8;
  static constexpr int OFF_RB = OFF_STG + 4 * STG_BYTES;
  // output boxes for the TMA stores of the absorption and the up-projection [2]
  static constexpr int OFF_OST = (OFF_RB + (SK ? RB_BYTES : 0) + 1023) & ~1023;
  static constexpr int SMEM = OFF_OST + (SK ? 0 : 2 * OBOX_BYTES) + 1024;
};

enum Mode { MODE_CACHE = 0, MODE_ABSORB = 1, MODE_UPV = 2, MODE_MAT = 3 };

struct TcGemm {
  int M, N, K, Z;
  int mode;
  int b_mn;                 // B is MN-major (N contiguous) instead of K-major
  int n_split;              // cache: tiles at n >= n_split read tmB2 at n - n_split
  bf16* out;
  int64_t rows_per_batch;   // cache: tokens per sequence in the call (n_tok)
  Geo geo;
  int64_t first_tok;        // cache: first token; absorb: first query token
  int32_t* slots;
  const bf16* q_rope;       // absorb: RoPE part input
  unsigned int* err;
};

// GSTAGES-deep TMA ring.  Four stages (one CTA per SM) suit long K loops; two stages let
// two CTAs share an SM, which hides the latency of short-K tiles (the absorption).
// SPLITK: launched in clusters of two CTAs that share each tile, rank r taking half of
// the K blocks; rank 1 sends its fp32 accumulator to rank 0 through distributed shared
// memory (st.async, completion counted in bytes) and rank 0 adds it before the epilogue.
// For few tiles with long K (the cache write: 65 tiles of K = 4096) it brings twice the
// SMs' load bandwidth to the same tiles.
template <int GSTAGES, bool SPLITK>
__global__ void __launch_bounds__(GTHREADS, GSTAGES == 2 ? 2 : 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmO,
                   TcGemm p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + GSTAGES * STAGE_BYTES);
  uint64_t* empty = full + GSTAGES;
  uint64_t* accf = empty + GSTAGES;              // accumulator ready [2]
  uint64_t* acce = accf + 2;                     // accumulator drained [2]
  uint64_t* rbf = acce + 2;                      // split-K: partial landed (rank 0, tx bytes)
  uint64_t* rbe = acce + 3;                      // split-K: rank 0 has read it (rank 1)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 4);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  using GL = GLay<GSTAGES, SPLITK>;
  double* inv_freq = reinterpret_cast<double*>(smem + GL::OFF_TAB);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nm = (p.M + GBM - 1) / GBM, nn = (p.N + GBN - 1) / GBN;
  const int ntiles = nm * nn * p.Z;
  const int nk = (p.K + GBK - 1) / GBK;
  // tiles this CTA (or CTA pair) walks, and its K blocks
  const uint32_t crank = SPLITK ? cluster_ctarank() : 0u;
  const int t_first = SPLITK ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int t_step = SPLITK ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int kb0 = SPLITK && crank ? nk / 2 : 0;
  const int kb1 = SPLITK && !crank ? nk / 2 : nk;

  if (tid == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 128);
    }
    mbar_init(rbf, 1);
    mbar_init(rbe, 1);
    *abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * GBN);
    tmem_relinquish();
  }
  for (int q = tid; q < p.geo.Dr / 2 && q < MAX_PAIRS; q += GTHREADS)
    inv_freq[q] = rope_inv_freq(p.geo, q);
  tc_fence_before();
  __syncthreads();
  if constexpr (SPLITK) cluster_sync();        // the pair's barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();                               // the previous kernel's outputs are visible
  grid_dep_launch();

  auto tile_coords = [&](int t, int& m0, int& n0, int& z) {
    z = t / (nm * nn);
    const int r = t - z * nm * nn;
    m0 = (r % nm) * GBM;
    n0 = (r / nm) * GBN;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int t = t_first; t < ntiles; t += t_step) {
        int m0, n0, z;
        tile_coords(t, m0, n0, z);
        const bool second = p.mode == MODE_CACHE && n0 >= p.n_split;
        const CUtensorMap* mB = second ? &tmB2 : &tmB;
        const int nb = second ? n0 - p.n_split : n0;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % GSTAGES;
          if (!mbar_wait(&empty[s], ((it / GSTAGES) & 1) ^ 1, abort, p.err, 0x11, kb)) break;
          uint8_t* a = smem + s * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          mbar_expect_tx(&full[s], STAGE_BYTES);
          // the cache write's and the materialisation's A rows serve every head
          tma_load_3d(a, &tmA, &full[s], kb * GBK,
                      p.mode == MODE_CACHE || p.mode == MODE_MAT ? 0 : z, m0);
          if (p.b_mn) {
            tma_load_3d(b, mB, &full[s], nb, kb * GBK, z);
            tma_load_3d(b + B_BYTES / 2, mB, &full[s], nb + 64, kb * GBK, z);
          } else {
            tma_load_3d(b, mB, &full[s], kb * GBK, nb, z);
          }
        }
        if (*abort) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(GBM, GBN, false, p.b_mn != 0);
      uint32_t it = 0, tc = 0;
      for (int t = t_first; t < ntiles; t += t_step, ++tc) {
        const int acc = tc & 1;
        if (!mbar_wait(&acce[acc], ((tc >> 1) & 1) ^ 1, abort, p.err, 0x14, tc)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * GBN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % GSTAGES;
          if (!mbar_wait(&full[s], (it / GSTAGES) & 1, abort, p.err, 0x12, kb)) break;
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b = a + A_BYTES;
          const uint64_t da = desc_sw128(a, 16, 1024);
          const uint64_t db = p.b_mn ? desc_sw128(b, B_BYTES / 2, 1024) : desc_sw128(b, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < GBK / 16; ++ks) {
            // K-major operands advance 32 bytes per 16-element K step inside the swizzle
            // atom; the MN-major B advances 16 rows of 128 bytes.
            const uint64_t bstep = p.b_mn ? (uint64_t)(ks * 2048 >> 4) : (uint64_t)(ks * 32 >> 4);
            mma_ss(d, da + (uint64_t)(ks * 32 >> 4), db + bstep, idesc,
                   (kb != kb0 || ks != 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        mma_commit(&accf[acc]);
        if (*abort) break;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    // Thread r drains TMEM row r of its warp's lane quarter 32 columns at a time, into a
    // per-warp staging buffer (2 KB, 16-byte chunks XOR-swizzled by row so that neither
    // the row-wise writes nor the chunk-wise reads conflict); the warp then writes the
    // 32 rows as 64-byte segments, four lanes per row, instead of one scattered row per
    // lane.
    const int r = (warp & 3) * 32 + lane;       // TMEM lane quarter = warp id % 4
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const Geo& G = p.geo;
    uint8_t* stg = smem + GL::OFF_STG + (warp - 2) * STG_BYTES;
    // split-K partial tile, chunk-major [32 chunks of 4 floats][128 rows]: conflict-free
    // for both the sending and the reading thread of a row
    const float4* rb = reinterpret_cast<const float4*>(smem + GL::OFF_RB) + r;
    uint32_t tc = 0, ost = 0;                   // ost: output boxes stored so far
    for (int t = t_first; t < ntiles; t += t_step, ++tc) {
      int m0, n0, z;
      tile_coords(t, m0, n0, z);
      const int acc = tc & 1;
      if constexpr (SPLITK) {
        if (crank == 1) {
          // drain this CTA's half-K accumulator into rank 0's buffer once rank 0 has read
          // the previous tile's
          bool okr = __all_sync(0xffffffffu, mbar_wait(&accf[acc], (tc >> 1) & 1, abort, p.err,
                                                         0x15, (r << 16) | tc));
          if (okr)
            okr = __all_sync(0xffffffffu, mbar_wait_cluster(rbe, (tc & 1) ^ 1, abort, p.err,
                                                             0x16, (r << 16) | tc));
          tc_fence_after();
          const uint32_t trow = tmem + lane_base + acc * GBN;
          const uint32_t dst = mapa(smem_u32(smem + GL::OFF_RB), 0) + (uint32_t)r * 16;
          const uint32_t dbar = mapa(smem_u32(rbf), 0);
          for (int c0 = 0; c0 < GBN; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(trow + c0, v);
            tmem_wait_ld();
            if (c0 + 32 == GBN) {
              tc_fence_before();
              mbar_arrive(&acce[acc]);          // accumulator may be overwritten
            }
            if (!okr) continue;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_async_v4(dst + (uint32_t)(c0 / 4 + q) * (GBM * 16), v[4 * q], v[4 * q + 1],
                          v[4 * q + 2], v[4 * q + 3], dbar);
          }
          if (!okr) break;
          continue;
        }
        // rank 0: the partial of this tile lands in its buffer (armed here, per tile)
        if (r == 0) mbar_expect_tx(rbf, RB_BYTES);
      }
      const int64_t m = m0 + r;
      const bool row_ok = m < p.M;
      // the absorption's share of RoPE(q_R) for this row: its loads are issued before the
      // wait for the accumulator, so that their latency overlaps it and the drain
      const bool rope_q = row_ok && p.mode == MODE_ABSORB && G.Dr > 0;
      int qa0 = 0, qa1 = 0;
      uint4 rin[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      const uint4* rsrc = nullptr;
      if (rope_q) {
        // the row's rotation pairs are shared out over the tiles of its row block, a
        // multiple of 4 pairs (one 16-byte vector) each
        const int nn = (p.N + GBN - 1) / GBN, npairs = G.Dr / 2;
        const int ppt = ((npairs + nn - 1) / nn + 3) & ~3;
        qa0 = (n0 / GBN) * ppt;
        qa1 = qa0 + ppt < npairs ? qa0 + ppt : npairs;
        rsrc = reinterpret_cast<const uint4*>(p.q_rope + (m * G.H + z) * G.Dr);
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (qa0 / 4 + u < qa1 / 4) rin[u] = rsrc[qa0 / 4 + u];
      }
      // this row's output base (element offset of column 0) and, for the cache, its token
      int64_t base = 0, g = 0;
      RopeAxes ax{0.0, 0.0, 0.0};
      if (p.mode == MODE_CACHE) {
        const int64_t b = m / p.rows_per_batch;
        g = p.first_tok + (m - b * p.rows_per_batch);
        base = (b * G.S + g % G.S) * G.row;
        if (row_ok && G.Dr > 0) ax = rope_axes(G, g);
      } else if (p.mode == MODE_ABSORB) {
        base = (m * G.H + z) * G.row;
      } else {
        base = (m * G.H + z) * G.Dn;
      }
      bool ok = __all_sync(0xffffffffu, mbar_wait(&accf[acc], (tc >> 1) & 1, abort, p.err,
                                                   0x13, (r << 16) | tc));
      if constexpr (SPLITK) {
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait_cluster(rbf, tc & 1, abort, p.err, 0x17,
                                                         (r << 16) | tc));
      }
      tc_fence_after();
      const uint32_t trow = tmem + lane_base + acc * GBN;
      // two 32-column TMEM loads in flight per wait
      for (int c0 = 0; c0 < GBN; c0 += 64) {
        uint32_t v[2][32];
        tmem_ld32(trow + c0, v[0]);
        tmem_ld32(trow + c0 + 32, v[1]);
        tmem_wait_ld();
        if (c0 + 64 == GBN) {
          tc_fence_before();
          mbar_arrive(&acce[acc]);              // accumulator may be overwritten
        }
        if (!SPLITK && p.mode != MODE_CACHE) {
          // The absorption's and the up-projection's outputs are plain 3-D tensors: the
          // warps fill one 128-row x 64-column box (128-byte swizzle) of a two-buffer
          // ring and one thread stores it with TMA, which writes the rows whole.
          uint8_t* ob = smem + GL::OFF_OST + (ost & 1) * OBOX_BYTES;
          ++ost;
          if (r == 0) bulk_wait_group_read<1>();   // the store that last read `ob` is done
          named_bar(1, 128);
          if (ok) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t* w = &v[hh][8 * q];
                *reinterpret_cast<uint4*>(ob + r * 128 + (((4 * hh + q) ^ (r & 7)) * 16)) =
                    make_uint4(pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                               pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                               pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                               pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
              }
          }
          fence_proxy_async_smem();
          named_bar(1, 128);
          if (ok && r == 0 && n0 + c0 < p.N) {
            tma_store_3d(&tmO, ob, n0 + c0, z, m0);
            bulk_commit_group();
          }
          continue;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = n0 + c0 + 32 * hh;      // output column of v[hh][0] (warp-uniform)
          if (!ok || n >= p.N) continue;
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[hh][j]);
          if constexpr (SPLITK) {
            // plus the other half of K, from the pair's rank 1
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 o = rb[((c0 + 32 * hh) / 4 + q) * GBM];
              f[4 * q] += o.x;
              f[4 * q + 1] += o.y;
              f[4 * q + 2] += o.z;
              f[4 * q + 3] += o.w;
            }
          }
          if (p.mode == MODE_CACHE && n >= p.n_split && row_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int q = (n + j - p.n_split) / 2;
              rope_rotate_fast(f[j], f[j + 1], rope_axis_pos(G, ax, q), inv_freq[q]);
            }
          }
          uint4* srow = reinterpret_cast<uint4*>(stg + lane * 64);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            srow[q ^ ((lane >> 1) & 3)] = make_uint4(
                pack_bf16(f[8 * q + 0], f[8 * q + 1]), pack_bf16(f[8 * q + 2], f[8 * q + 3]),
                pack_bf16(f[8 * q + 4], f[8 * q + 5]), pack_bf16(f[8 * q + 6], f[8 * q + 7]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 8 * i + (lane >> 2), j = lane & 3;      // row of the warp, chunk
            const int64_t rbase = __shfl_sync(0xffffffffu, base, rr);
            if (m0 + (warp & 3) * 32 + rr < p.M) {
              const uint4 w = reinterpret_cast<const uint4*>(stg + rr * 64)[j ^ ((rr >> 1) & 3)];
              *reinterpret_cast<uint4*>(p.out + rbase + n + 8 * j) = w;
            }
          }
          __syncwarp();
        }
      }
      if constexpr (SPLITK) {
        // every row of the partial is read: rank 1 may send the next tile's
        named_bar(1, 128);
        if (r == 0) mbar_arrive_cluster_relaxed(mapa(smem_u32(rbe), 1));
      }
      if (ok && row_ok && n0 == 0 && p.mode == MODE_CACHE && p.slots)
        p.slots[m] = (int32_t)(g % G.S);
      if (rope_q && ok && qa0 < qa1) {
        // q_abs[.., Dc:] = RoPE(q_R) for the pairs [qa0, qa1) of this row
        const RopeAxes qa = rope_axes(G, p.first_tok + m % p.rows_per_batch);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (m * G.H + z) * G.row + G.Dc);
        for (int c = qa0 / 4; c < qa1 / 4; c += 2) {
          uint4 in[2] = {rin[0], rin[1]};
          if (c > qa0 / 4) {
#pragma unroll
            for (int u = 0; u < 2; ++u) if (c + u < qa1 / 4) in[u] = rsrc[c + u];
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (c + u >= qa1 / 4) break;
            uint32_t w[4] = {in[u].x, in[u].y, in[u].z, in[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = (c + u) * 4 + e;
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
              float a = f.x, b = f.y;
              rope_rotate_fast(a, b, rope_axis_pos(G, qa, q), inv_freq[q]);
              w[e] = pack_bf16(a, b);
            }
            dst[c + u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (!ok) break;
    }
    // the output boxes' stores have finished with shared memory and landed before exit
    if (r == 0) bulk_wait_group<0>();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if constexpr (SPLITK) cluster_sync();        // no remote access into this CTA is pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * GBN);
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

template <int ST, bool SK>
cudaError_t launch_st(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& B2,
                      const CUtensorMap& O, const TcGemm& q, long long tiles, cudaStream_t st) {
  using GL = GLay<ST, SK>;
  {
    // the shared-memory opt-in is per device
    static std::mutex mu;
    static uint64_t done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 64 || !(done >> dev & 1)) {
      e = cudaFuncSetAttribute(tc_gemm_kernel<ST, SK>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, GL::SMEM);
      if (e != cudaSuccess) return e;
      if (dev < 64) done |= 1ull << dev;
    }
  }
  if (!SK) {
    const long long slots = (long long)sm_count() * (ST == 2 ? 2 : 1);
    const int grid = (int)(tiles < slots ? tiles : slots);
    if (grid == 0) return cudaSuccess;
    cudaError_t e = launch_dependent(tc_gemm_kernel<ST, SK>, (unsigned)grid, GTHREADS, GL::SMEM, st,
                                     1u, A, B, B2, O, q);
    if (e != cudaSuccess) return e;
  } else {
    // clusters of two CTAs, one cluster per tile up to one per SM pair
    const long long pairs = sm_count() / 2;
    const int nclu = (int)(tiles < pairs ? tiles : pairs);
    if (nclu == 0) return cudaSuccess;
    cudaError_t e = launch_dependent(tc_gemm_kernel<ST, SK>, (unsigned)(2 * nclu), GTHREADS,
                                     GL::SMEM, st, 2u, A, B, B2, O, q);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

cudaError_t launch(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& B2,
                   const CUtensorMap& O, const TcGemm& p, int zcount, cudaStream_t st) {
  TcGemm q = p;
  q.Z = zcount;
  const long long tiles =
      (long long)((p.M + GBM - 1) / GBM) * ((p.N + GBN - 1) / GBN) * zcount;
  const int nk = (p.K + GBK - 1) / GBK;
  // the absorption's tiles are two K-blocks long: two CTAs per SM hide their latency; so
  // do the materialisation's (eight K-blocks, but 1568 tiles; measured 2 % faster for the
  // whole non-absorbed call, while the up-projection measured slower that way)
  if (p.mode == MODE_ABSORB || p.mode == MODE_MAT)
    return launch_st<2, false>(A, B, B2, O, q, tiles, st);
  // fewer tiles than SMs and a long K loop (the cache write): split K over CTA pairs
  if (p.mode == MODE_CACHE && nk >= 2 && tiles < sm_count())
    return launch_st<4, true>(A, B, B2, O, q, tiles, st);
  return launch_st<4, false>(A, B, B2, O, q, tiles, st);
}

}  // namespace

bool tc_gemm_supported(const Geo& g, int d_model) {
  // every output width is a multiple of the epilogue's 32-column chunks
  return g.Dc % GBN == 0 && g.Dr % 64 == 0 && g.Dn % 64 == 0 && g.Dr / 2 <= MAX_PAIRS &&
         (d_model <= 0 || d_model % 64 == 0);
}

cudaError_t tc_cache_write(const Geo& g, const void* h, int d_model, int64_t n_tok,
                           int64_t first_tok, const void* w_dkv, const void* w_kr, void* cache,
                           int32_t* slots, unsigned int* err, cudaStream_t st) {
  CUtensorMap A, B, B2;
  const uint64_t rows = (uint64_t)g.B * n_tok;
  {
    uint64_t d[3] = {(uint64_t)d_model, 1, rows};
    uint64_t s[2] = {(uint64_t)d_model * 2, (uint64_t)d_model * 2};
    uint32_t b[3] = {64, 1, 128};
    if (!make_tmap_bf16(&A, h, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[3] = {(uint64_t)g.Dc, (uint64_t)d_model, 1};
    uint64_t s[2] = {(uint64_t)g.Dc * 2, (uint64_t)g.Dc * d_model * 2};
    uint32_t b[3] = {64, 64, 1};
    if (!make_tmap_bf16(&B, w_dkv, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  if (g.Dr > 0) {
    uint64_t d[3] = {(uint64_t)g.Dr, (uint64_t)d_model, 1};
    uint64_t s[2] = {(uint64_t)g.Dr * 2, (uint64_t)g.Dr * d_model * 2};
    uint32_t b[3] = {64, 64, 1};
    if (!make_tmap_bf16(&B2, w_kr, 3, d, s, b)) return cudaErrorInvalidValue;
  } else {
    B2 = B;
  }
  TcGemm p{};
  p.M = (int)rows; p.N = g.row; p.K = d_model; p.mode = MODE_CACHE; p.b_mn = 1;
  p.n_split = g.Dc; p.out = (bf16*)cache; p.rows_per_batch = n_tok; p.geo = g;
  p.first_tok = first_tok; p.slots = slots; p.err = err;
  return launch(A, B, B2, B, p, 1, st);       // the cache write stores without TMA
}

cudaError_t tc_absorb_q(const Geo& g, const void* q_nope, const void* q_rope, int64_t n_q,
                        int64_t q_first, const void* w_uk, void* q_abs, unsigned int* err,
                        cudaStream_t st) {
  CUtensorMap A, B;
  const uint64_t rows = (uint64_t)g.B * n_q;
  {
    uint64_t d[3] = {(uint64_t)g.Dn, (uint64_t)g.H, rows};
    uint64_t s[2] = {(uint64_t)g.Dn * 2, (uint64_t)g.H * g.Dn * 2};
    uint32_t b[3] = {64, 1, 128};
    if (!make_tmap_bf16(&A, q_nope, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[3] = {(uint64_t)g.Dc, (uint64_t)g.Dn, (uint64_t)g.H};
    uint64_t s[2] = {(uint64_t)g.Dc * 2, (uint64_t)g.Dc * g.Dn * 2};
    uint32_t b[3] = {64, 64, 1};
    if (!make_tmap_bf16(&B, w_uk, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  TcGemm p{};
  p.M = (int)rows; p.N = g.Dc; p.K = g.Dn; p.mode = MODE_ABSORB; p.b_mn = 1;
  p.n_split = 1 << 30; p.out = (bf16*)q_abs; p.rows_per_batch = n_q; p.geo = g;
  p.first_tok = q_first; p.q_rope = (const bf16*)q_rope; p.err = err;
  CUtensorMap O;
  {
    // q_abs as (d_c + d_R, heads, rows): 64-column boxes of 128 rows of one head
    uint64_t d[3] = {(uint64_t)g.row, (uint64_t)g.H, rows};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.H * g.row * 2};
    uint32_t b[3] = {64, 1, (uint32_t)GBM};
    if (!make_tmap_bf16(&O, q_abs, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  return launch(A, B, B, O, p, g.H, st);
}

cudaError_t tc_up_v(const Geo& g, const void* o_lat, int64_t n_q, const void* w_uv, void* out,
                    unsigned int* err, cudaStream_t st) {
  CUtensorMap A, B;
  const uint64_t rows = (uint64_t)g.B * n_q;
  {
    uint64_t d[3] = {(uint64_t)g.Dc, (uint64_t)g.H, rows};
    uint64_t s[2] = {(uint64_t)g.Dc * 2, (uint64_t)g.H * g.Dc * 2};
    uint32_t b[3] = {64, 1, 128};
    if (!make_tmap_bf16(&A, o_lat, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[3] = {(uint64_t)g.Dc, (uint64_t)g.Dn, (uint64_t)g.H};
    uint64_t s[2] = {(uint64_t)g.Dc * 2, (uint64_t)g.Dc * g.Dn * 2};
    uint32_t b[3] = {64, (uint32_t)GBN, 1};
    if (!make_tmap_bf16(&B, w_uv, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  TcGemm p{};
  p.M = (int)rows; p.N = g.Dn; p.K = g.Dc; p.mode = MODE_UPV; p.b_mn = 0;
  p.n_split = 1 << 30; p.out = (bf16*)out; p.rows_per_batch = n_q; p.geo = g; p.err = err;
  CUtensorMap O;
  {
    // out as (d_nope, heads, rows): 64-column boxes of 128 rows of one head
    uint64_t d[3] = {(uint64_t)g.Dn, (uint64_t)g.H, rows};
    uint64_t s[2] = {(uint64_t)g.Dn * 2, (uint64_t)g.H * g.Dn * 2};
    uint32_t b[3] = {64, 1, (uint32_t)GBM};
    if (!make_tmap_bf16(&O, out, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  return launch(A, B, B, O, p, g.H, st);
}

cudaError_t tc_materialise(const Geo& g, const void* cache, const void* w, void* out,
                           unsigned int* err, cudaStream_t st) {
  CUtensorMap A, B;
  const uint64_t rows = (uint64_t)g.B * g.S;
  {
    // the latent columns of every cached row, as (d_latent, 1, slots)
    uint64_t d[3] = {(uint64_t)g.Dc, 1, rows};
    uint64_t s[2] = {(uint64_t)g.row * 2, (uint64_t)g.row * 2};
    uint32_t b[3] = {64, 1, 128};
    if (!make_tmap_bf16(&A, cache, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[3] = {(uint64_t)g.Dc, (uint64_t)g.Dn, (uint64_t)g.H};
    uint64_t s[2] = {(uint64_t)g.Dc * 2, (uint64_t)g.Dc * g.Dn * 2};
    uint32_t b[3] = {64, (uint32_t)GBN, 1};
    if (!make_tmap_bf16(&B, w, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  TcGemm p{};
  p.M = (int)rows; p.N = g.Dn; p.K = g.Dc; p.mode = MODE_MAT; p.b_mn = 0;
  p.n_split = 1 << 30; p.out = (bf16*)out; p.rows_per_batch = g.S; p.geo = g; p.err = err;
  CUtensorMap O;
  {
    // out as (d_nope, heads, slots): 64-column boxes of 128 slots of one head
    uint64_t d[3] = {(uint64_t)g.Dn, (uint64_t)g.H, rows};
    uint64_t s[2] = {(uint64_t)g.Dn * 2, (uint64_t)g.H * g.Dn * 2};
    uint32_t b[3] = {64, 1, (uint32_t)GBM};
    if (!make_tmap_bf16(&O, out, 3, d, s, b)) return cudaErrorInvalidValue;
  }
  return launch(A, B, B, O, p, g.H, st);
}

}  // namespace mla
