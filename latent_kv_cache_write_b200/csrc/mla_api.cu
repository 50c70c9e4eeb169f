// The C ABI: argument validation, then dispatch to the kernels.  Nothing is launched
// unless every check passes.
#include <stdio.h>

#include <atomic>
#include <mutex>

#include "launch.h"

namespace mla {

// Device-side error words: [0] status bits ORed by a kernel that gave up a bounded wait,
// [1] site id of the first such wait, [2] its CTA index, [3] its (thread, block) tag.
__device__ unsigned int g_device_error[4] = {0, 0, 0, 0};
static unsigned int g_last_error_info[4] = {0, 0, 0, 0};

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

unsigned int* device_error_word() {
  // One lookup per device: the symbol's address differs between devices.
  static std::mutex mu;
  static unsigned int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

mla_status check_shape(const mla_shape* s, Geo* g) {
  if (!s) return MLA_ERR_ARG;
  if (s->batch < 1 || s->n_heads < 1 || s->d_nope < 1 || s->d_latent < 1 || s->d_rope < 0)
    return MLA_ERR_ARG;
  if (s->grid_h < 1 || s->grid_w < 1 || s->ring_slots < 1 || s->reserved != 0)
    return MLA_ERR_ARG;
  if (s->d_rope % 2 != 0 || s->d_latent % 2 != 0) return MLA_ERR_ARG;
  if (s->rope_pairs[0] < 0 || s->rope_pairs[1] < 0 || s->rope_pairs[2] < 0) return MLA_ERR_ARG;
  if ((int64_t)s->rope_pairs[0] + s->rope_pairs[1] + s->rope_pairs[2] != s->d_rope / 2)
    return MLA_ERR_ARG;
  if (!(s->rope_theta > 0.0)) return MLA_ERR_ARG;
  if (s->dtype != MLA_F32 && s->dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)s->d_latent + s->d_rope > 32 * 40) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)s->batch * s->n_heads > 65535) return MLA_ERR_UNSUPPORTED;
  // ring rows are addressed with 32-bit tensor coordinates
  if ((int64_t)s->batch * s->ring_slots > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  g->B = s->batch; g->H = s->n_heads; g->Dn = s->d_nope; g->Dc = s->d_latent; g->Dr = s->d_rope;
  for (int i = 0; i < 3; ++i) g->pairs[i] = s->rope_pairs[i];
  g->theta = s->rope_theta;
  g->gh = s->grid_h; g->gw = s->grid_w;
  g->F = (int64_t)s->grid_h * s->grid_w;
  g->S = s->ring_slots;
  g->row = s->d_latent + s->d_rope;
  return MLA_OK;
}

mla_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  fprintf(stderr, "mla: CUDA error %s\n", cudaGetErrorString(e));
  return MLA_ERR_CUDA;
}


bool quant_bits_ok(int32_t b) { return b == 2 || b == 4 || b == 8; }

// the checks both directions of the low-bit ring share
mla_status check_quant(const mla_shape* shape, Geo* g, int64_t first_tok, int64_t n_tok,
                       int32_t cbits, int32_t rbits, const void* cache, const void* qc,
                       const void* qr, const float* sc, const float* sr) {
  mla_status st = check_shape(shape, g);
  if (st != MLA_OK) return st;
  if (!cache || !qc || !qr || !sc || !sr || n_tok < 0 || !quant_bits_ok(cbits) ||
      !quant_bits_ok(rbits))
    return MLA_ERR_ARG;
  if (!quant_supported(*g)) return MLA_ERR_UNSUPPORTED;
  if (first_tok < 0 || n_tok > g->S) return MLA_ERR_RANGE;
  if (!aligned16(cache) || !aligned16(qc) || !aligned16(qr) || !aligned16(sc) ||
      !aligned16(sr))
    return MLA_ERR_ALIGN;
  return MLA_OK;
}

// the checks of mla_attend and mla_attend_fixed_scratch, all but the workspace's
mla_status check_attend(const mla_shape* shape, Geo* g, const void* q_abs, int64_t n_q,
                        int64_t q_first_tok, const void* cache, int64_t k_first_tok,
                        int64_t n_keys, float softmax_scale, const void* o_lat,
                        const float* lse) {
  mla_status st = check_shape(shape, g);
  if (st != MLA_OK) return st;
  if (n_q < 0 || !q_abs || !cache || !o_lat) return MLA_ERR_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return MLA_ERR_ARG;
  if (n_keys < 1 || n_keys > g->S || k_first_tok < 0 || q_first_tok < k_first_tok ||
      q_first_tok + n_q > k_first_tok + n_keys)
    return MLA_ERR_RANGE;
  if (n_q > 65535 || (int64_t)g->B * n_q * g->H > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_abs) || !aligned16(cache) || !aligned16(o_lat) || (lse && !aligned16(lse)))
    return MLA_ERR_ALIGN;
  return MLA_OK;
}

// the launches of a checked attention call (n_q > 0)
mla_status run_attend(const mla_shape* shape, const Geo& g, const void* q_abs, int64_t n_q,
                      int64_t q_first_tok, const void* cache, int64_t k_first_tok,
                      int64_t n_keys, float softmax_scale, void* o_lat, float* lse,
                      void* workspace, size_t workspace_bytes, void* stream) {
  const bool bf = shape->dtype == MLA_BF16;
  if (bf && tc_attend_supported(g))
    return cuda_status(tc_attend(g, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                                 softmax_scale, o_lat, lse, workspace, workspace_bytes,
                                 device_error_word(), (cudaStream_t)stream));
  return cuda_status(simt_attend(g, bf, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                                 softmax_scale, o_lat, lse, (cudaStream_t)stream));
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_ARG: return "MLA_ERR_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN";
    case MLA_ERR_RANGE: return "MLA_ERR_RANGE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status mla_cache_write(const mla_shape* shape, const void* h, int32_t d_model,
                           int64_t n_tok, int64_t first_tok, const void* w_dkv,
                           const void* w_kr, void* cache, int32_t* slots_out, void* stream) {
  Geo g;
  mla_status st = check_shape(shape, &g);
  if (st != MLA_OK) return st;
  if (d_model < 1 || n_tok < 0) return MLA_ERR_ARG;
  if (!h || !w_dkv || !cache || (g.Dr > 0 && !w_kr)) return MLA_ERR_ARG;
  if (first_tok < 0 || n_tok > g.S) return MLA_ERR_RANGE;
  if (n_tok > INT32_MAX / 2) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(h) || !aligned16(w_dkv) || (w_kr && !aligned16(w_kr)) || !aligned16(cache) ||
      (slots_out && !aligned16(slots_out)))
    return MLA_ERR_ALIGN;
  if (n_tok == 0) return MLA_OK;
  const bool bf = shape->dtype == MLA_BF16;
  cudaStream_t s = (cudaStream_t)stream;
  if (bf && g.Dr > 0 && tc_gemm_supported(g, d_model))
    return cuda_status(tc_cache_write(g, h, d_model, n_tok, first_tok, w_dkv, w_kr, cache,
                                      slots_out, device_error_word(), s));
  return cuda_status(simt_cache_write(g, bf, h, d_model, n_tok, first_tok, w_dkv, w_kr, cache,
                                      slots_out, s));
}

mla_status mla_absorb_q(const mla_shape* shape, const void* q_nope, const void* q_rope,
                        int64_t n_q, int64_t q_first_tok, const void* w_uk, void* q_abs,
                        void* stream) {
  Geo g;
  mla_status st = check_shape(shape, &g);
  if (st != MLA_OK) return st;
  if (n_q < 0 || !q_nope || !w_uk || !q_abs || (g.Dr > 0 && !q_rope)) return MLA_ERR_ARG;
  if (q_first_tok < 0) return MLA_ERR_RANGE;
  if (n_q > INT32_MAX / 2 || (int64_t)g.B * n_q * g.H > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_nope) || (q_rope && !aligned16(q_rope)) || !aligned16(w_uk) ||
      !aligned16(q_abs))
    return MLA_ERR_ALIGN;
  if (n_q == 0) return MLA_OK;
  const bool bf = shape->dtype == MLA_BF16;
  if (bf && tc_gemm_supported(g, 0))
    return cuda_status(tc_absorb_q(g, q_nope, q_rope, n_q, q_first_tok, w_uk, q_abs,
                                   device_error_word(), (cudaStream_t)stream));
  return cuda_status(simt_absorb_q(g, bf, q_nope, q_rope, n_q, q_first_tok, w_uk, q_abs,
                                   (cudaStream_t)stream));
}

size_t mla_attend_workspace_size(const mla_shape* shape, int64_t n_q, int64_t n_keys) {
  (void)n_q; (void)n_keys;
  Geo g;
  if (check_shape(shape, &g) != MLA_OK) return 0;
  if (shape->dtype == MLA_BF16 && tc_attend_supported(g)) return tc_attend_workspace(g);
  return 0;
}

mla_status mla_attend(const mla_shape* shape, const void* q_abs, int64_t n_q,
                      int64_t q_first_tok, const void* cache, int64_t k_first_tok,
                      int64_t n_keys, float softmax_scale, void* o_lat, float* lse,
                      void* workspace, size_t workspace_bytes, void* stream) {
  Geo g;
  mla_status st = check_attend(shape, &g, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                               softmax_scale, o_lat, lse);
  if (st != MLA_OK) return st;
  // no workspace at all is allowed (the schedule then keeps tiles whole); a workspace
  // that is given must be large enough
  const size_t need = mla_attend_workspace_size(shape, n_q, n_keys);
  if ((workspace || workspace_bytes > 0) && (!workspace || workspace_bytes < need))
    return MLA_ERR_ARG;
  if (workspace && !aligned16(workspace)) return MLA_ERR_ALIGN;
  if (n_q == 0) return MLA_OK;
  return run_attend(shape, g, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                    softmax_scale, o_lat, lse, workspace, workspace_bytes, stream);
}

mla_status mla_attend_fixed_scratch(const mla_shape* shape, const void* q_abs, int64_t n_q,
                                    int64_t q_first_tok, const void* cache,
                                    int64_t k_first_tok, int64_t n_keys, float softmax_scale,
                                    void* o_lat, float* lse, void* stream) {
  Geo g;
  mla_status st = check_attend(shape, &g, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                               softmax_scale, o_lat, lse);
  if (st != MLA_OK) return st;
  if (n_q == 0) return MLA_OK;
  // the static array replaces the caller's workspace; a shape and device that would
  // need more is refused rather than run with a smaller schedule
  const size_t need = mla_attend_workspace_size(shape, n_q, n_keys);
  if (need > MLA_FIXED_SCRATCH_BYTES) return MLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  size_t bytes = 0;
  if (need > 0) {
    if (fixed_scratch(&scratch) != cudaSuccess) return MLA_ERR_CUDA;
    bytes = MLA_FIXED_SCRATCH_BYTES;
  }
  return run_attend(shape, g, q_abs, n_q, q_first_tok, cache, k_first_tok, n_keys,
                    softmax_scale, o_lat, lse, scratch, bytes, stream);
}

mla_status mla_attend_quantised(const mla_shape* shape, const void* q_abs, int64_t n_q,
                                int64_t q_first_tok, const void* q_content, const void* q_rope,
                                const float* scale_c, const float* scale_r,
                                int32_t content_bits, int32_t rope_bits, int64_t k_first_tok,
                                int64_t n_keys, float softmax_scale, void* o_lat, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream) {
  Geo g;
  // the packed ring stands where mla_attend takes the bf16 cache
  mla_status st = check_attend(shape, &g, q_abs, n_q, q_first_tok, q_content, k_first_tok,
                               n_keys, softmax_scale, o_lat, lse);
  if (st != MLA_OK) return st;
  if (!q_rope || !scale_c || !scale_r || !quant_bits_ok(content_bits) ||
      !quant_bits_ok(rope_bits))
    return MLA_ERR_ARG;
  if (shape->dtype != MLA_BF16 || !tc_attend_packed_supported(g, content_bits, rope_bits))
    return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_rope) || !aligned16(scale_c) || !aligned16(scale_r)) return MLA_ERR_ALIGN;
  const size_t need = mla_attend_workspace_size(shape, n_q, n_keys);
  if ((workspace || workspace_bytes > 0) && (!workspace || workspace_bytes < need))
    return MLA_ERR_ARG;
  if (workspace && !aligned16(workspace)) return MLA_ERR_ALIGN;
  if (n_q == 0) return MLA_OK;
  const PackedRing pk{q_content, q_rope, scale_c, scale_r, content_bits, rope_bits};
  return cuda_status(tc_attend_ring(g, q_abs, n_q, q_first_tok, nullptr, &pk, k_first_tok,
                                    n_keys, softmax_scale, o_lat, lse, workspace,
                                    workspace_bytes, device_error_word(), (cudaStream_t)stream));
}

mla_status mla_up_v(const mla_shape* shape, const void* o_lat, int64_t n_q, const void* w_uv,
                    void* out, void* stream) {
  Geo g;
  mla_status st = check_shape(shape, &g);
  if (st != MLA_OK) return st;
  if (n_q < 0 || !o_lat || !w_uv || !out) return MLA_ERR_ARG;
  if (n_q > INT32_MAX / 2 || (int64_t)g.B * n_q * g.H > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(o_lat) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_ALIGN;
  if (n_q == 0) return MLA_OK;
  const bool bf = shape->dtype == MLA_BF16;
  if (bf && tc_gemm_supported(g, 0))
    return cuda_status(tc_up_v(g, o_lat, n_q, w_uv, out, device_error_word(),
                               (cudaStream_t)stream));
  return cuda_status(simt_up_v(g, bf, o_lat, n_q, w_uv, out, (cudaStream_t)stream));
}

mla_status mla_cache_shift_frames(const mla_shape* shape, void* cache, int64_t first_tok,
                                  int64_t n_tok, int64_t delta_frames, void* stream) {
  Geo g;
  mla_status st = check_shape(shape, &g);
  if (st != MLA_OK) return st;
  if (!cache || n_tok < 0) return MLA_ERR_ARG;
  if (first_tok < 0 || n_tok > g.S) return MLA_ERR_RANGE;
  if (!aligned16(cache)) return MLA_ERR_ALIGN;
  if (n_tok == 0) return MLA_OK;
  return cuda_status(shift_frames(g, shape->dtype == MLA_BF16, cache, first_tok, n_tok,
                                  delta_frames, (cudaStream_t)stream));
}

mla_status mla_cache_quantise(const mla_shape* shape, const void* cache, int64_t first_tok,
                              int64_t n_tok, int32_t content_bits, int32_t rope_bits,
                              void* q_content, void* q_rope, float* scale_c, float* scale_r,
                              void* stream) {
  Geo g;
  mla_status st = check_quant(shape, &g, first_tok, n_tok, content_bits, rope_bits, cache,
                              q_content, q_rope, scale_c, scale_r);
  if (st != MLA_OK) return st;
  if (n_tok == 0) return MLA_OK;
  return cuda_status(quantise_ring(g, shape->dtype == MLA_BF16, cache, first_tok, n_tok,
                                   content_bits, rope_bits, q_content, q_rope, scale_c,
                                   scale_r, (cudaStream_t)stream));
}

mla_status mla_cache_dequantise(const mla_shape* shape, const void* q_content,
                                const void* q_rope, const float* scale_c,
                                const float* scale_r, int32_t content_bits, int32_t rope_bits,
                                int64_t first_tok, int64_t n_tok, void* cache, void* stream) {
  Geo g;
  mla_status st = check_quant(shape, &g, first_tok, n_tok, content_bits, rope_bits, cache,
                              q_content, q_rope, scale_c, scale_r);
  if (st != MLA_OK) return st;
  if (n_tok == 0) return MLA_OK;
  return cuda_status(dequantise_ring(g, shape->dtype == MLA_BF16, q_content, q_rope, scale_c,
                                     scale_r, content_bits, rope_bits, first_tok, n_tok, cache,
                                     (cudaStream_t)stream));
}

size_t mla_attend_materialised_workspace_size(const mla_shape* shape) {
  Geo g;
  if (check_shape(shape, &g) != MLA_OK) return 0;
  if (shape->dtype != MLA_BF16 || !tc_attend_mat_supported(g) || !tc_gemm_supported(g, 0))
    return 0;
  return (size_t)2 * g.B * g.S * g.H * g.Dn * 2;
}

mla_status mla_attend_materialised(const mla_shape* shape, const void* q_nope,
                                   const void* q_rope, int64_t n_q, int64_t q_first_tok,
                                   const void* cache, int64_t k_first_tok, int64_t n_keys,
                                   float softmax_scale, const void* w_uk, const void* w_uv,
                                   void* out, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  Geo g;
  mla_status st = check_shape(shape, &g);
  if (st != MLA_OK) return st;
  if (n_q < 0 || !q_nope || !q_rope || !cache || !w_uk || !w_uv || !out) return MLA_ERR_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return MLA_ERR_ARG;
  if (n_keys < 1 || n_keys > g.S || k_first_tok < 0 || q_first_tok < k_first_tok ||
      q_first_tok + n_q > k_first_tok + n_keys)
    return MLA_ERR_RANGE;
  const size_t need = mla_attend_materialised_workspace_size(shape);
  if (need == 0 || n_q > 65535 || (int64_t)g.B * n_q * g.H > INT32_MAX)
    return MLA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < need) return MLA_ERR_ARG;
  if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(cache) || !aligned16(w_uk) ||
      !aligned16(w_uv) || !aligned16(out) || (lse && !aligned16(lse)) || !aligned16(workspace))
    return MLA_ERR_ALIGN;
  if (n_q == 0) return MLA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int* err = device_error_word();
  uint8_t* k_mat = static_cast<uint8_t*>(workspace);
  uint8_t* v_mat = k_mat + need / 2;
  cudaError_t e = tc_materialise(g, cache, w_uk, k_mat, err, s);
  if (e == cudaSuccess) e = tc_materialise(g, cache, w_uv, v_mat, err, s);
  if (e == cudaSuccess)
    e = tc_attend_mat(g, q_nope, q_rope, n_q, q_first_tok, cache, k_mat, v_mat, k_first_tok,
                      n_keys, softmax_scale, out, lse, err, s);
  return cuda_status(e);
}

mla_status mla_check_wait_timeout(void* stream) {
  unsigned int* err = device_error_word();
  if (!err) return MLA_ERR_CUDA;
  return cuda_status(wait_check(err, (cudaStream_t)stream));
}

void mla_device_error_info(uint32_t info[4]) {
  for (int i = 0; i < 4; ++i) info[i] = g_last_error_info[i];
}

uint64_t mla_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

mla_status mla_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned int words[4] = {0, 0, 0, 0}, zero[4] = {0, 0, 0, 0};
  e = cudaMemcpyFromSymbol(words, g_device_error, sizeof(words));
  if (e != cudaSuccess) return cuda_status(e);
  if (words[0] != 0) {
    for (int i = 0; i < 4; ++i) g_last_error_info[i] = words[i];
    e = cudaMemcpyToSymbol(g_device_error, zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_status(e);
    return MLA_ERR_TIMEOUT;
  }
  return MLA_OK;
}

}  // extern "C"
