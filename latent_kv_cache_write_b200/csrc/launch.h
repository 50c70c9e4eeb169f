// Internal launchers behind the C ABI (host side).  Each returns the CUDA error of its
// launch.  Arguments have been validated by the ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

// Launch a kernel so that it may start while the previous kernel on the stream finishes
// (programmatic dependent launch): its CTAs set up barriers and tensor memory, then wait
// in grid_dep_wait before their first global access.  Hides each launch's latency and
// prologue behind the previous kernel's tail.  cluster_x > 1 sets the cluster size of a
// kernel that has none compiled in.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block,
                                    size_t smem, cudaStream_t st, unsigned cluster_x,
                                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Host-side count of kernels launched by the library (see mla_kernel_launches).
void count_launches(int n);

// SIMT CUDA-core path: every dtype and shape (float32 storage uses it throughout).
cudaError_t simt_cache_write(const Geo& g, bool bf, const void* h, int d_model, int64_t n_tok,
                             int64_t first_tok, const void* w_dkv, const void* w_kr,
                             void* cache, int32_t* slots, cudaStream_t st);
cudaError_t simt_absorb_q(const Geo& g, bool bf, const void* q_nope, const void* q_rope,
                          int64_t n_q, int64_t q_first, const void* w_uk, void* q_abs,
                          cudaStream_t st);
cudaError_t simt_attend(const Geo& g, bool bf, const void* q_abs, int64_t n_q, int64_t q_first,
                        const void* cache, int64_t k_first, int64_t n_keys, float scale,
                        void* o_lat, float* lse, cudaStream_t st);
cudaError_t simt_up_v(const Geo& g, bool bf, const void* o_lat, int64_t n_q, const void* w_uv,
                      void* out, cudaStream_t st);

// Tensor-core (tcgen05 + TMA) path for bf16 storage.
bool tc_gemm_supported(const Geo& g, int d_model);
cudaError_t tc_cache_write(const Geo& g, const void* h, int d_model, int64_t n_tok,
                           int64_t first_tok, const void* w_dkv, const void* w_kr, void* cache,
                           int32_t* slots, unsigned int* err, cudaStream_t st);
cudaError_t tc_absorb_q(const Geo& g, const void* q_nope, const void* q_rope, int64_t n_q,
                        int64_t q_first, const void* w_uk, void* q_abs, unsigned int* err,
                        cudaStream_t st);
cudaError_t tc_up_v(const Geo& g, const void* o_lat, int64_t n_q, const void* w_uv, void* out,
                    unsigned int* err, cudaStream_t st);
// out[b][slot][h] = w[h] . cache[b][slot][0 : d_latent] for every ring slot (the per-head
// keys with w = W_UK, the values with w = W_UV), bf16 [B, S, n_h, d_nope].
cudaError_t tc_materialise(const Geo& g, const void* cache, const void* w, void* out,
                           unsigned int* err, cudaStream_t st);

// Turn the cached RoPE keys of tokens first_tok .. + n_tok by a (delta_frames, 0, 0)
// position (rope_shift.cu).
cudaError_t shift_frames(const Geo& g, bool bf, void* cache, int64_t first_tok, int64_t n_tok,
                         int64_t delta_frames, cudaStream_t st);

// Low-bit latent ring (quant.cu): per-row, per-path scale quantisation of the ring rows of
// tokens first_tok .. first_tok + n_tok - 1 into packed codes and float32 scales, and the
// inverse.  quant_supported: both paths a multiple of 8 and at most 1024 wide.
bool quant_supported(const Geo& g);
cudaError_t quantise_ring(const Geo& g, bool bf, const void* cache, int64_t first_tok,
                          int64_t n_tok, int cbits, int rbits, void* qc, void* qr, float* sc,
                          float* sr, cudaStream_t st);
cudaError_t dequantise_ring(const Geo& g, bool bf, const void* qc, const void* qr,
                            const float* sc, const float* sr, int cbits, int rbits,
                            int64_t first_tok, int64_t n_tok, void* cache, cudaStream_t st);

// Non-absorbed attention over the materialised keys and values (tc_attend_mat.cu).
bool tc_attend_mat_supported(const Geo& g);
cudaError_t tc_attend_mat(const Geo& g, const void* q_nope, const void* q_rope, int64_t n_q,
                          int64_t q_first, const void* cache, const void* k_mat,
                          const void* v_mat, int64_t k_first, int64_t n_keys, float scale,
                          void* out, float* lse, unsigned int* err, cudaStream_t st);

bool tc_attend_supported(const Geo& g);
// Workspace for split-key partials on the current device (0 if it cannot be queried).
size_t tc_attend_workspace(const Geo& g);
// With workspace_bytes >= tc_attend_workspace(g) tiles may be split across clusters;
// otherwise (workspace may be null) the schedule cuts on tile boundaries only.
cudaError_t tc_attend(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                      const void* cache, int64_t k_first, int64_t n_keys, float scale,
                      void* o_lat, float* lse, void* workspace, size_t workspace_bytes,
                      unsigned int* err, cudaStream_t st);

// The low-bit ring the attention reads instead of a bf16 cache (packed codes of both paths
// and their per-row float32 scales, as mla_cache_quantise writes them).
struct PackedRing {
  const void* codes_c;
  const void* codes_r;
  const float* scale_c;
  const float* scale_r;
  int cbits, rbits;
};
// Content codes of 4 or 2 bits and RoPE codes of 4 bits, d_c = 512, d_R = 64.
bool tc_attend_packed_supported(const Geo& g, int cbits, int rbits);
// tc_attend over either ring: `cache` when pk is null, else the packed ring *pk.
cudaError_t tc_attend_ring(const Geo& g, const void* q_abs, int64_t n_q, int64_t q_first,
                           const void* cache, const PackedRing* pk, int64_t k_first,
                           int64_t n_keys, float scale, void* o_lat, float* lse,
                           void* workspace, size_t workspace_bytes, unsigned int* err,
                           cudaStream_t st);

// Address of the static split-key scratch (MLA_FIXED_SCRATCH_BYTES) on the current device.
cudaError_t fixed_scratch(void** ptr);

// Launch one thread whose bounded wait on a barrier nothing completes must expire
// (wait_check.cu).
cudaError_t wait_check(unsigned int* err, cudaStream_t st);

// Device address of the library's error word on the current device (nullptr on failure).
unsigned int* device_error_word();

}  // namespace mla
