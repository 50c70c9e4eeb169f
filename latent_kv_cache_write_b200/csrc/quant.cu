// Low-bit latent ring: per-row, per-path scale quantisation of cached rows, and its inverse
// (QuantMLA abstract on the "Multi-Head Latent Attention" topic page: the content latent and
// the RoPE key are cached at INT4, or the content at INT2 with the RoPE key at INT4, each
// path with a quantiser of its own).
//
// Each path of a row gets s = max|x| / q, q = 2^(bits-1) - 1, and codes x / s rounded to the
// nearest integer (ties to even), clipped to [-q, q]; a zero path has s = 0 and codes 0.
// Codes are two's-complement fields packed little-endian: element i at bits
// [i*bits, (i+1)*bits) of the packed row, so 8 elements fill exactly `bits` bytes.
// Memory-bound: one warp per cached row, each lane holding up to four 8-element chunks of a
// path in registers between the max reduction and the quantisation.
#include "launch.h"

namespace mla {
namespace {

constexpr int QT = 256;                       // threads per block: 8 rows
constexpr int MAXCH = 4;                      // 8-element chunks per lane and path
constexpr unsigned FULLMASK = 0xffffffffu;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<bf16>(bf16* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// the `bits` bytes of one packed chunk (bits is 2, 4 or 8: a naturally aligned word)
__device__ __forceinline__ void store_chunk(uint8_t* p, int bits, uint64_t w) {
  if (bits == 2)
    *reinterpret_cast<uint16_t*>(p) = (uint16_t)w;
  else if (bits == 4)
    *reinterpret_cast<uint32_t*>(p) = (uint32_t)w;
  else
    *reinterpret_cast<uint64_t*>(p) = w;
}
__device__ __forceinline__ uint64_t load_chunk(const uint8_t* p, int bits) {
  if (bits == 2) return *reinterpret_cast<const uint16_t*>(p);
  if (bits == 4) return *reinterpret_cast<const uint32_t*>(p);
  return *reinterpret_cast<const uint64_t*>(p);
}

// Quantise the d values at src (one path of one row) into dst (d * bits / 8 bytes) and *scale.
template <typename T>
__device__ __forceinline__ void quantise_path(const T* src, int d, int bits, uint8_t* dst,
                                              float* scale, int lane) {
  const int nch = d >> 3;
  float v[MAXCH][8];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < MAXCH; ++k) {
    const int ch = lane + 32 * k;
    if (ch < nch) {
      load8(src + 8 * ch, v[k]);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[k][e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULLMASK, amax, o));
  const int q = (1 << (bits - 1)) - 1;
  const float s = __fdiv_rn(amax, (float)q);
  if (lane == 0) *scale = s;
  const uint64_t field = (1ull << bits) - 1;
#pragma unroll
  for (int k = 0; k < MAXCH; ++k) {
    const int ch = lane + 32 * k;
    if (ch < nch) {
      uint64_t w = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int c = 0;
        if (s > 0.f) {
          const float r = rintf(__fdiv_rn(v[k][e], s));
          c = (int)fminf(fmaxf(r, (float)-q), (float)q);
        }
        w |= ((uint64_t)(int64_t)c & field) << (e * bits);
      }
      store_chunk(dst + (size_t)ch * bits, bits, w);
    }
  }
}

template <typename T>
__device__ __forceinline__ void dequantise_path(const uint8_t* src, float s, int d, int bits,
                                                T* dst, int lane) {
  const int nch = d >> 3;
  const uint64_t field = (1ull << bits) - 1;
  const int64_t half = 1ll << (bits - 1);
#pragma unroll
  for (int k = 0; k < MAXCH; ++k) {
    const int ch = lane + 32 * k;
    if (ch < nch) {
      const uint64_t w = load_chunk(src + (size_t)ch * bits, bits);
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int64_t c = (int64_t)((w >> (e * bits)) & field);
        if (c >= half) c -= 2 * half;                    // sign of the two's-complement field
        v[e] = (float)c * s;
      }
      store8(dst + 8 * ch, v);
    }
  }
}

struct QuantRing {
  uint8_t* qc;                // [B, S, Dc * cbits / 8]
  uint8_t* qr;                // [B, S, Dr * rbits / 8]
  float* sc;                  // [B, S]
  float* sr;                  // [B, S]
  int cbits, rbits;
};

template <typename T>
__global__ void __launch_bounds__(QT) quantise_kernel(Geo G, const T* cache, QuantRing R,
                                                      int64_t first_tok, int64_t n_tok) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * (QT / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)G.B * n_tok) return;                // whole warps leave together
  const int64_t b = w / n_tok, i = w - b * n_tok;
  const int64_t row = b * G.S + (first_tok + i) % G.S;
  const T* src = cache + row * G.row;
  quantise_path(src, G.Dc, R.cbits, R.qc + row * ((int64_t)G.Dc * R.cbits / 8), R.sc + row,
                lane);
  quantise_path(src + G.Dc, G.Dr, R.rbits, R.qr + row * ((int64_t)G.Dr * R.rbits / 8),
                R.sr + row, lane);
}

template <typename T>
__global__ void __launch_bounds__(QT) dequantise_kernel(Geo G, QuantRing R, T* cache,
                                                        int64_t first_tok, int64_t n_tok) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * (QT / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)G.B * n_tok) return;
  const int64_t b = w / n_tok, i = w - b * n_tok;
  const int64_t row = b * G.S + (first_tok + i) % G.S;
  T* dst = cache + row * G.row;
  dequantise_path(R.qc + row * ((int64_t)G.Dc * R.cbits / 8), R.sc[row], G.Dc, R.cbits, dst,
                  lane);
  dequantise_path(R.qr + row * ((int64_t)G.Dr * R.rbits / 8), R.sr[row], G.Dr, R.rbits,
                  dst + G.Dc, lane);
}

}  // namespace

bool quant_supported(const Geo& g) {
  return g.Dc % 8 == 0 && g.Dr % 8 == 0 && g.Dc <= 8 * 32 * MAXCH && g.Dr <= 8 * 32 * MAXCH;
}

cudaError_t quantise_ring(const Geo& g, bool bf, const void* cache, int64_t first_tok,
                          int64_t n_tok, int cbits, int rbits, void* qc, void* qr, float* sc,
                          float* sr, cudaStream_t st) {
  const int64_t rows = (int64_t)g.B * n_tok;
  if (rows == 0) return cudaSuccess;
  const QuantRing R{(uint8_t*)qc, (uint8_t*)qr, sc, sr, cbits, rbits};
  const unsigned blocks = (unsigned)((rows + QT / 32 - 1) / (QT / 32));
  if (bf)
    quantise_kernel<bf16><<<blocks, QT, 0, st>>>(g, (const bf16*)cache, R, first_tok, n_tok);
  else
    quantise_kernel<float><<<blocks, QT, 0, st>>>(g, (const float*)cache, R, first_tok, n_tok);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

cudaError_t dequantise_ring(const Geo& g, bool bf, const void* qc, const void* qr,
                            const float* sc, const float* sr, int cbits, int rbits,
                            int64_t first_tok, int64_t n_tok, void* cache, cudaStream_t st) {
  const int64_t rows = (int64_t)g.B * n_tok;
  if (rows == 0) return cudaSuccess;
  const QuantRing R{(uint8_t*)qc, (uint8_t*)qr, (float*)sc, (float*)sr, cbits, rbits};
  const unsigned blocks = (unsigned)((rows + QT / 32 - 1) / (QT / 32));
  if (bf)
    dequantise_kernel<bf16><<<blocks, QT, 0, st>>>(g, R, (bf16*)cache, first_tok, n_tok);
  else
    dequantise_kernel<float><<<blocks, QT, 0, st>>>(g, R, (float*)cache, first_tok, n_tok);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
