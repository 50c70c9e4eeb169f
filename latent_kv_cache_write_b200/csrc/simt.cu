// SIMT (CUDA-core) kernels for every step of the path.  They serve the float32
// workloads (tensor cores would round to tf32) and any shape the tensor-core kernels
// do not take.  Accumulation is float32 throughout.
#include "launch.h"

namespace mla {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

enum Epi { EPI_STORE = 0, EPI_CACHE = 1 };

// C[z](m, n) = sum_k A[z](m, k) * B[z](k, n) for z = zb * zH + zh.
struct GemmArgs {
  const void* A; int64_t lda, a_sb, a_sh;
  const void* B; int64_t ldb, b_sh; int b_kmajor;   // B(k,n) = kmajor ? B[n*ldb+k] : B[k*ldb+n]
  const void* B2; int64_t ldb2; int n_split;        // columns >= n_split read B2 (K x N2)
  void* C; int64_t ldc, c_sb, c_sh;
  int M, N, K, zH;
  // cache epilogue
  Geo geo; int64_t first_tok; int32_t* slots;
};

template <typename T, int EPI>
__global__ void __launch_bounds__(NT) gemm_simt_kernel(GemmArgs a) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  const int z = blockIdx.z;
  const int zb = z / a.zH, zh = z % a.zH;
  const T* A = (const T*)a.A + zb * a.a_sb + zh * a.a_sh;
  const T* Bm = (const T*)a.B + zh * a.b_sh;
  const T* B2 = (const T*)a.B2;

  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += BK) {
    for (int e = tid; e < BM * BK; e += NT) {
      int r = e / BK, k = e % BK;
      int m = m0 + r, kk = k0 + k;
      As[k][r] = (m < a.M && kk < a.K) ? to_f32(A[(int64_t)m * a.lda + kk]) : 0.f;
    }
    for (int e = tid; e < BN * BK; e += NT) {
      int k = e / BN, c = e % BN;
      int n = n0 + c, kk = k0 + k;
      float v = 0.f;
      if (n < a.N && kk < a.K) {
        if (EPI == EPI_CACHE && n >= a.n_split)
          v = to_f32(B2[(int64_t)kk * a.ldb2 + (n - a.n_split)]);
        else
          v = to_f32(a.b_kmajor ? Bm[(int64_t)n * a.ldb + kk] : Bm[(int64_t)kk * a.ldb + n]);
      }
      Bs[k][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  T* C = (T*)a.C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
    if (EPI == EPI_CACHE) {
      const int64_t g = a.first_tok + m;
      const int64_t slot = g % a.geo.S;
      T* row = C + ((int64_t)zb * a.geo.S + slot) * a.ldc;
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        const int n = n0 + tx * 4 + j;
        if (n >= a.N) continue;
        float v0 = acc[i][j], v1 = acc[i][j + 1];
        if (n >= a.n_split) rope_rotate(v0, v1, rope_angle(a.geo, g, (n - a.n_split) / 2));
        row[n] = from_f32<T>(v0);
        if (n + 1 < a.N) row[n + 1] = from_f32<T>(v1);
      }
      if (a.slots && blockIdx.y == 0 && tx == 0) a.slots[(int64_t)zb * a.M + m] = (int32_t)slot;
    } else {
      T* row = C + zb * a.c_sb + zh * a.c_sh + (int64_t)m * a.ldc;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n < a.N) row[n] = from_f32<T>(acc[i][j]);
      }
    }
  }
}

template <typename T, int EPI>
cudaError_t run_gemm(const GemmArgs& a, int zcount, cudaStream_t st) {
  if (a.M == 0 || zcount == 0) return cudaSuccess;
  dim3 grid((a.M + BM - 1) / BM, (a.N + BN - 1) / BN, zcount);
  gemm_simt_kernel<T, EPI><<<grid, NT, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

// q_abs[b,i,h,Dc:] = RoPE(q_rope[b,i,h,:], q_first + i)
template <typename T>
__global__ void rope_q_kernel(Geo g, const T* q_rope, int64_t n_q, int64_t q_first, T* q_abs) {
  const int half = g.Dr / 2;
  const int64_t total = (int64_t)g.B * n_q * g.H * half;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(e % half);
    const int64_t bih = e / half;              // (b * n_q + i) * H + h
    const int64_t i = (bih / g.H) % n_q;
    float a = to_f32(q_rope[bih * g.Dr + 2 * p]);
    float b = to_f32(q_rope[bih * g.Dr + 2 * p + 1]);
    rope_rotate(a, b, rope_angle(g, q_first + i, p));
    T* dst = q_abs + bih * g.row + g.Dc;
    dst[2 * p] = from_f32<T>(a);
    dst[2 * p + 1] = from_f32<T>(b);
  }
}

// One warp per (b, query, head); the 8 warps of a block share the query and walk the
// same keys, so the key rows are served from L1 after the first warp.
template <typename T>
__global__ void __launch_bounds__(256) attend_simt_kernel(Geo g, const T* q_abs, int64_t n_q,
                                                          int64_t q_first, const T* cache,
                                                          int64_t k_first, int64_t n_keys,
                                                          float scale, T* o_lat, float* lse) {
  constexpr int MAXR = 40;                    // row width <= 32 * MAXR
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.x * 8 + warp;
  const int64_t i = blockIdx.y;
  const int b = blockIdx.z;
  if (h >= g.H) return;
  const int64_t gq = q_first + i;
  // visible keys: [k_first, k_end)
  int64_t k_end = (gq / g.F + 1) * g.F;
  if (k_end > k_first + n_keys) k_end = k_first + n_keys;
  const T* q = q_abs + (((int64_t)b * n_q + i) * g.H + h) * g.row;
  const int nr = (g.row + 31) / 32;
  const int nc = (g.Dc + 31) / 32;
  float qv[MAXR], acc[MAXR];
#pragma unroll
  for (int r = 0; r < MAXR; ++r) {
    const int d = lane + 32 * r;
    qv[r] = (r < nr && d < g.row) ? to_f32(q[d]) * scale : 0.f;
    acc[r] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const T* base = cache + (int64_t)b * g.S * g.row;
  for (int64_t k = k_first; k < k_end; ++k) {
    const T* row = base + (k % g.S) * g.row;
    float kv[MAXR];
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      const int d = lane + 32 * r;
      kv[r] = (r < nr && d < g.row) ? to_f32(row[d]) : 0.f;
      s = fmaf(qv[r], kv[r], s);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn);
    const float p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      const int d = lane + 32 * r;
      if (r < nc && d < g.Dc) acc[r] = fmaf(acc[r], corr, p * kv[r]);
    }
    m = mn;
  }
  T* out = o_lat + (((int64_t)b * n_q + i) * g.H + h) * g.Dc;
  const float inv = 1.f / l;
#pragma unroll
  for (int r = 0; r < MAXR; ++r) {
    const int d = lane + 32 * r;
    if (r < nc && d < g.Dc) out[d] = from_f32<T>(acc[r] * inv);
  }
  if (lse && lane == 0) lse[((int64_t)b * n_q + i) * g.H + h] = m + logf(l);
}

template <typename T>
cudaError_t run_cache_write(const Geo& g, const void* h, int d_model, int64_t n_tok,
                            int64_t first_tok, const void* w_dkv, const void* w_kr,
                            void* cache, int32_t* slots, cudaStream_t st) {
  GemmArgs a{};
  a.A = h; a.lda = d_model; a.a_sb = n_tok * d_model; a.a_sh = 0;
  a.B = w_dkv; a.ldb = g.Dc; a.b_sh = 0; a.b_kmajor = 0;
  a.B2 = w_kr; a.ldb2 = g.Dr; a.n_split = g.Dc;
  a.C = cache; a.ldc = g.row;
  a.M = (int)n_tok; a.N = g.row; a.K = d_model; a.zH = 1;
  a.geo = g; a.first_tok = first_tok; a.slots = slots;
  return run_gemm<T, EPI_CACHE>(a, g.B, st);
}

template <typename T>
cudaError_t run_absorb(const Geo& g, const void* q_nope, const void* q_rope, int64_t n_q,
                       int64_t q_first, const void* w_uk, void* q_abs, cudaStream_t st) {
  GemmArgs a{};
  a.A = q_nope; a.lda = (int64_t)g.H * g.Dn; a.a_sb = n_q * g.H * g.Dn; a.a_sh = g.Dn;
  a.B = w_uk; a.ldb = g.Dc; a.b_sh = (int64_t)g.Dn * g.Dc; a.b_kmajor = 0;
  a.C = q_abs; a.ldc = (int64_t)g.H * g.row; a.c_sb = n_q * g.H * g.row; a.c_sh = g.row;
  a.M = (int)n_q; a.N = g.Dc; a.K = g.Dn; a.zH = g.H;
  cudaError_t e = run_gemm<T, EPI_STORE>(a, g.B * g.H, st);
  if (e != cudaSuccess || g.Dr == 0) return e;
  const int64_t total = (int64_t)g.B * n_q * g.H * (g.Dr / 2);
  const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
  rope_q_kernel<T><<<blocks, 256, 0, st>>>(g, (const T*)q_rope, n_q, q_first, (T*)q_abs);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

template <typename T>
cudaError_t run_up_v(const Geo& g, const void* o_lat, int64_t n_q, const void* w_uv, void* out,
                     cudaStream_t st) {
  GemmArgs a{};
  a.A = o_lat; a.lda = (int64_t)g.H * g.Dc; a.a_sb = n_q * g.H * g.Dc; a.a_sh = g.Dc;
  a.B = w_uv; a.ldb = g.Dc; a.b_sh = (int64_t)g.Dn * g.Dc; a.b_kmajor = 1;
  a.C = out; a.ldc = (int64_t)g.H * g.Dn; a.c_sb = n_q * g.H * g.Dn; a.c_sh = g.Dn;
  a.M = (int)n_q; a.N = g.Dn; a.K = g.Dc; a.zH = g.H;
  return run_gemm<T, EPI_STORE>(a, g.B * g.H, st);
}

}  // namespace

cudaError_t simt_cache_write(const Geo& g, bool bf, const void* h, int d_model, int64_t n_tok,
                             int64_t first_tok, const void* w_dkv, const void* w_kr,
                             void* cache, int32_t* slots, cudaStream_t st) {
  return bf ? run_cache_write<bf16>(g, h, d_model, n_tok, first_tok, w_dkv, w_kr, cache, slots, st)
            : run_cache_write<float>(g, h, d_model, n_tok, first_tok, w_dkv, w_kr, cache, slots, st);
}

cudaError_t simt_absorb_q(const Geo& g, bool bf, const void* q_nope, const void* q_rope,
                          int64_t n_q, int64_t q_first, const void* w_uk, void* q_abs,
                          cudaStream_t st) {
  return bf ? run_absorb<bf16>(g, q_nope, q_rope, n_q, q_first, w_uk, q_abs, st)
            : run_absorb<float>(g, q_nope, q_rope, n_q, q_first, w_uk, q_abs, st);
}

cudaError_t simt_attend(const Geo& g, bool bf, const void* q_abs, int64_t n_q, int64_t q_first,
                        const void* cache, int64_t k_first, int64_t n_keys, float scale,
                        void* o_lat, float* lse, cudaStream_t st) {
  if (n_q == 0) return cudaSuccess;
  dim3 grid((g.H + 7) / 8, (unsigned)n_q, g.B);
  if (bf)
    attend_simt_kernel<bf16><<<grid, 256, 0, st>>>(g, (const bf16*)q_abs, n_q, q_first,
                                                   (const bf16*)cache, k_first, n_keys, scale,
                                                   (bf16*)o_lat, lse);
  else
    attend_simt_kernel<float><<<grid, 256, 0, st>>>(g, (const float*)q_abs, n_q, q_first,
                                                    (const float*)cache, k_first, n_keys, scale,
                                                    (float*)o_lat, lse);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

cudaError_t simt_up_v(const Geo& g, bool bf, const void* o_lat, int64_t n_q, const void* w_uv,
                      void* out, cudaStream_t st) {
  return bf ? run_up_v<bf16>(g, o_lat, n_q, w_uv, out, st)
            : run_up_v<float>(g, o_lat, n_q, w_uv, out, st);
}

}  // namespace mla
