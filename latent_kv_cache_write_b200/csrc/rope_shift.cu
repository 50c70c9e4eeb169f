// Whole-frame re-indexing of cached RoPE keys: the delta-rotation that the Irminsul
// abstract on the "Multi-Head Latent Attention" topic page gives for reused tokens at
// shifted positions.  The cached row is a position-free latent plus a RoPE key rotated
// by the token's own (t, y, x) position, so moving a token delta frames later turns its
// RoPE key by the angles of position (delta, 0, 0): the t-axis pairs turn by
// delta * theta^(-j/n), and the y and x pairs and the latent stay as they are.
// Memory-bound.  Every row turns by the same angles, so a block computes the n_t rotations
// (cos, sin in double) once, and each thread then turns one pair of one row in place.
#include "launch.h"

namespace mla {
namespace {

constexpr int SHIFT_THREADS = 256;
constexpr int MAX_T_PAIRS = 640;             // d_rope / 2 of every shape the ABI accepts

template <typename T>
__global__ void __launch_bounds__(SHIFT_THREADS)
    shift_frames_kernel(Geo G, T* cache, int64_t first_tok, int64_t n_tok, int64_t delta) {
  __shared__ double rot[MAX_T_PAIRS][2];
  const int n = G.pairs[0];
  for (int j = threadIdx.x; j < n; j += SHIFT_THREADS) {
    double sn, cs;
    sincos((double)delta * pow(G.theta, -(double)j / (double)n), &sn, &cs);
    rot[j][0] = cs;
    rot[j][1] = sn;
  }
  __syncthreads();
  const int64_t idx = (int64_t)blockIdx.x * SHIFT_THREADS + threadIdx.x;
  if (idx >= (int64_t)G.B * n_tok * n) return;
  const int j = (int)(idx % n);
  const int64_t w = idx / n;                          // (sequence, token) of the row
  const int64_t b = w / n_tok, i = w - b * n_tok;
  T* pr = cache + (b * G.S + (first_tok + i) % G.S) * G.row + G.Dc + 2 * j;
  const double a = to_f32(pr[0]), c = to_f32(pr[1]);
  pr[0] = from_f32<T>((float)(a * rot[j][0] - c * rot[j][1]));
  pr[1] = from_f32<T>((float)(a * rot[j][1] + c * rot[j][0]));
}

}  // namespace

cudaError_t shift_frames(const Geo& g, bool bf, void* cache, int64_t first_tok, int64_t n_tok,
                         int64_t delta_frames, cudaStream_t st) {
  const int64_t work = (int64_t)g.B * n_tok * g.pairs[0];
  if (work == 0 || delta_frames == 0) return cudaSuccess;
  if (g.pairs[0] > MAX_T_PAIRS) return cudaErrorInvalidValue;
  const unsigned blocks = (unsigned)((work + SHIFT_THREADS - 1) / SHIFT_THREADS);
  if (bf)
    shift_frames_kernel<bf16><<<blocks, SHIFT_THREADS, 0, st>>>(g, (bf16*)cache, first_tok,
                                                               n_tok, delta_frames);
  else
    shift_frames_kernel<float><<<blocks, SHIFT_THREADS, 0, st>>>(g, (float*)cache, first_tok,
                                                                n_tok, delta_frames);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
