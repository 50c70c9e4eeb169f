/*
 * mla.h — C ABI of the absorbed multi-head latent attention hot path over a
 * sliding-window latent KV ring, for NVIDIA B200 (sm_100a).
 *
 * The method (sources cited by page title and section):
 *   - Only a shared low-rank content latent c_KV (d_latent wide) and a shared
 *     decoupled RoPE key k_R (d_rope wide) are cached per token
 *     ("Multi-Head Latent Attention" concept page, "Low-rank joint compression" and
 *     "The RoPE problem, and the decoupled fix"; "Understanding Multi-Head Latent
 *     Attention and KV Compression", "Decoupling Rotary Position Embeddings (RoPE)").
 *   - The positional key encodes the 3-D (t, h, w) position of a video token with
 *     RoPE and the cache is a fixed-size sliding window over frames ("VideoMLA:
 *     Compressing Video Diffusion Memory by 92.7% with Low-Rank Latent Attention",
 *     "The Gap" and "Core Mechanism").
 *   - W_UK is absorbed into the query, so scores are taken against the latent
 *     directly; W_UV is applied after attention (concept page, "Low-rank joint
 *     compression": the absorption identity).
 *
 * Conventions shared by every call
 *   - Tensor arguments are DEVICE pointers to dense row-major arrays, 16-byte
 *     aligned, in the storage dtype of the shape (float32 or bfloat16) unless stated.
 *     The caller allocates and owns every buffer, workspace included; the library
 *     allocates nothing and keeps no per-call state.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *     and the call returns without synchronising.  Results are visible to later work
 *     on the same stream.  The tensor-core kernels are launched as programmatic
 *     dependent launches: their thread blocks may become resident while the previous
 *     kernel on the stream finishes, but they wait for it to complete (and for its
 *     writes to be visible) before they read or write any buffer, so stream order holds
 *     for every buffer, whatever kernel wrote or reads it.
 *   - Arguments are validated before anything is launched; on any error status no
 *     work has been enqueued.  MLA_ERR_CUDA reports a launch failure
 *     (cudaGetLastError after the launch).
 *   - Positions: global token g lies in frame t = g / F (F = grid_h * grid_w), row
 *     y = (g % F) / grid_w and column x = g % grid_w of that frame, and in ring slot
 *     g mod ring_slots.  A one-token frame (grid 1x1) gives plain token positions
 *     (1-D RoPE with rope_pairs = {d_rope/2, 0, 0}) and a token-causal mask.
 *   - 3-D RoPE: d_rope is split into contiguous t, y, x segments of 2*rope_pairs[a]
 *     elements; pair j of an axis segment with n pairs, elements (2j, 2j+1) of the
 *     segment, is rotated by pos_a * rope_theta^(-j/n) radians.
 *   - Accumulation is float32.  bfloat16 results are rounded to nearest even.
 *   - Sizes: batch * ring_slots, and for the calls that take queries
 *     batch * n_q * n_heads, are at most 2^31 - 1 (rows are addressed with 32-bit
 *     tensor coordinates); larger shapes return MLA_ERR_UNSUPPORTED.
 */
#ifndef MLA_H
#define MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_ARG = 1,          /* null pointer, non-positive size, inconsistent shape      */
  MLA_ERR_UNSUPPORTED = 2,  /* dtype or shape combination this library does not handle  */
  MLA_ERR_ALIGN = 3,        /* a tensor pointer is not 16-byte aligned                  */
  MLA_ERR_RANGE = 4,        /* token ranges outside the ring or the key window          */
  MLA_ERR_CUDA = 5,         /* a CUDA launch failed                                     */
  MLA_ERR_TIMEOUT = 6       /* a bounded device-side wait expired (see mla_device_error) */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Problem shape.  64 bytes, no padding holes. */
typedef struct {
  int32_t batch;          /* B, independent sequences                                  */
  int32_t n_heads;        /* n_h                                                       */
  int32_t d_nope;         /* d_h, per-head content query/key/value width               */
  int32_t d_latent;       /* d_c, shared content latent width                          */
  int32_t d_rope;         /* d_R, shared decoupled RoPE key width (even)               */
  int32_t rope_pairs[3];  /* rotation pairs on the t, y, x axes; sum = d_rope / 2      */
  double  rope_theta;     /* RoPE base                                                  */
  int32_t grid_h;         /* frame rows                                                 */
  int32_t grid_w;         /* frame columns; tokens per frame F = grid_h * grid_w        */
  int64_t ring_slots;     /* S, token slots per sequence in the ring                    */
  int32_t dtype;          /* mla_dtype of every tensor argument                         */
  int32_t reserved;       /* must be 0                                                   */
} mla_shape;

/*
 * mla_cache_write — step 1: fused down-projection, 3-D RoPE and store into the ring.
 * ("Multi-Head Latent Attention" concept page, "Low-rank joint compression": only
 * the joint latent is cached; "The RoPE problem, and the decoupled fix": a small
 * decoupled RoPE key is cached beside it, shared across heads.)
 *
 * For b < B and i < n_tok, with g = first_tok + i:
 *   cache[b][g mod S][0 : d_latent]          = h[b][i] . w_dkv
 *   cache[b][g mod S][d_latent : +d_rope]    = RoPE3D(h[b][i] . w_kr, position of g)
 *   slots_out[b][i]                          = g mod S          (if slots_out != NULL)
 *
 *   h        [B, n_tok, d_model]                 storage dtype, read
 *   w_dkv    [d_model, d_latent]                 storage dtype, read
 *   w_kr     [d_model, d_rope]                   storage dtype, read
 *   cache    [B, S, d_latent + d_rope]           storage dtype, written at n_tok slots
 *   slots_out[B, n_tok] int32 or NULL            written
 * Errors: MLA_ERR_RANGE if n_tok > S (a call may not overwrite its own rows) or
 * first_tok < 0; MLA_ERR_ARG for null tensors or non-positive sizes.
 */
mla_status mla_cache_write(const mla_shape* shape, const void* h, int32_t d_model,
                           int64_t n_tok, int64_t first_tok, const void* w_dkv,
                           const void* w_kr, void* cache, int32_t* slots_out,
                           void* stream);

/*
 * mla_absorb_q — step 2: query absorption through W_UK and RoPE of the query's
 * decoupled part (concept page, "Low-rank joint compression": W^UK folds into the
 * query side; "The RoPE problem, and the decoupled fix").
 *
 * For b, i < n_q, head h, with g = q_first_tok + i:
 *   q_abs[b][i][h][0 : d_latent]       = q_nope[b][i][h] . w_uk[h]     ([d_nope] x [d_nope, d_latent])
 *   q_abs[b][i][h][d_latent : +d_rope] = RoPE3D(q_rope[b][i][h], position of g)
 *
 *   q_nope [B, n_q, n_h, d_nope]           read
 *   q_rope [B, n_q, n_h, d_rope]           read (un-rotated)
 *   w_uk   [n_h, d_nope, d_latent]         read  (per-head key = w_uk[h] . c)
 *   q_abs  [B, n_q, n_h, d_latent + d_rope] written
 * Errors: MLA_ERR_ARG / MLA_ERR_RANGE (q_first_tok < 0).
 */
mla_status mla_absorb_q(const mla_shape* shape, const void* q_nope, const void* q_rope,
                        int64_t n_q, int64_t q_first_tok, const void* w_uk, void* q_abs,
                        void* stream);

/*
 * mla_attend_workspace_size — bytes of device workspace that lets mla_attend split the
 * key range of a tile across SMs (split-key partial outputs, bfloat16, and their float32
 * log-sum-exps, two slots per resident cluster of the current device).  May be 0 (the
 * float32 path, and shapes without the tensor-core kernel, never need one).
 */
size_t mla_attend_workspace_size(const mla_shape* shape, int64_t n_q, int64_t n_keys);

/*
 * mla_attend — steps 3 and 4: absorbed attention in latent space over the ring
 * (concept page, "Low-rank joint compression": one attends directly in latent space;
 * "The RoPE problem, and the decoupled fix": score = content term + positional term;
 * VideoMLA "The Gap": next-frame prediction over a sliding window).
 *
 * Keys are the global tokens k_first_tok .. k_first_tok + n_keys - 1, stored in slot
 * g mod S.  Query i is token q_first_tok + i; it sees key g iff frame(g) <=
 * frame(q) (frame-block-causal).  For every (b, i, h):
 *   s(g)   = softmax_scale * (q_abs[b][i][h] . cache[b][g mod S])   (all d_latent+d_rope)
 *   p      = softmax over the visible keys
 *   o_lat[b][i][h] = sum_g p(g) * cache[b][g mod S][0 : d_latent]
 *   lse[b][i][h]   = log(sum_g exp(s(g)))   (natural log, float32; if lse != NULL)
 *
 *   q_abs  [B, n_q, n_h, d_latent + d_rope]   read
 *   cache  [B, S, d_latent + d_rope]          read
 *   o_lat  [B, n_q, n_h, d_latent]            written
 *   lse    [B, n_q, n_h] float32 or NULL      written
 *   workspace: device scratch of at least mla_attend_workspace_size() bytes, or NULL
 *   with workspace_bytes 0; its contents on entry do not matter.  Without it the work
 *   is still spread over the SMs, but only in whole 128-row tiles (slower when there
 *   are few tiles or they do not divide evenly).  Calls that share a workspace must
 *   not run concurrently.
 * A single query per sequence (n_q == 1) is the decode case.
 * Score range: any inputs whose scores are finite in float32.  The bfloat16 tensor-core
 * path splits each score's dot product between two SMs and sums the two partials; a
 * partial whose magnitude times softmax_scale * log2(e) is at most 8 is passed on rounded
 * to fp16 (an error of at most 2^-8 in the exponent's log2 units, a fraction of a percent
 * of a softmax weight, like the bf16 rounding of P); larger partials, up to the float32
 * range, are passed on exactly, at the cost of two more exchanges for the key block.
 * Errors: MLA_ERR_RANGE if n_keys > S, n_keys < 1, or the queries are not inside the
 * key window (k_first_tok <= q_first_tok and q_first_tok + n_q <= k_first_tok +
 * n_keys); MLA_ERR_ARG if a workspace is given (or workspace_bytes > 0) and it is
 * NULL or smaller than mla_attend_workspace_size().
 */
mla_status mla_attend(const mla_shape* shape, const void* q_abs, int64_t n_q,
                      int64_t q_first_tok, const void* cache, int64_t k_first_tok,
                      int64_t n_keys, float softmax_scale, void* o_lat, float* lse,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * MLA_FIXED_SCRATCH_BYTES, mla_attend_fixed_scratch — mla_attend without a caller
 * workspace.  The pages have no counterpart: this is an interface matter, not part of
 * the method.
 *
 * For callers that cannot hand mla_attend a device workspace: a plain C host that
 * holds only the tensors it was given and no device allocator of its own, or a serving
 * loop that must not allocate between steps (cudaMalloc and cudaFree synchronise the
 * device).  Instead of the workspace, the split-key partials (bfloat16 partial outputs
 * and float32 log-sum-exps) go to one static device array of MLA_FIXED_SCRATCH_BYTES
 * inside the library, 40 MiB per device (two partial slots of 128 x d_latent bfloat16 and
 * 256 floats for each resident pair of SMs: 19 MiB on a 148-SM B200, 33 MiB for the
 * largest schedule of 128 clusters).  The call allocates nothing.
 *
 * Arguments, results and errors are those of mla_attend (without workspace and
 * workspace_bytes); the results equal mla_attend's with a full workspace.  In addition:
 *   - MLA_ERR_UNSUPPORTED if this shape on the current device would need more scratch
 *     than MLA_FIXED_SCRATCH_BYTES (mla_attend_workspace_size() > it);
 *   - MLA_ERR_CUDA if the array's device address cannot be obtained.
 * The first call on a device looks the array's address up (cudaGetSymbolAddress, with
 * that device current) and should come before any stream capture.  Under lazy module
 * loading (CUDA_MODULE_LOADING=LAZY, the CUDA 12 default) the array takes device memory
 * on a device only once the library's module is first used there; under eager loading
 * every context that loads the library holds the 40 MiB from the start.
 * All calls on a device share the one array: calls that overlap in time (on different
 * streams, or from different host threads without ordering) race on it and corrupt each
 * other's results; calls ordered on one stream do not.  Nothing in the array needs to
 * start at zero: every slot a call reads was written earlier in the same call.
 */
#define MLA_FIXED_SCRATCH_BYTES (40u * 1024u * 1024u)

mla_status mla_attend_fixed_scratch(const mla_shape* shape, const void* q_abs, int64_t n_q,
                                    int64_t q_first_tok, const void* cache,
                                    int64_t k_first_tok, int64_t n_keys, float softmax_scale,
                                    void* o_lat, float* lse, void* stream);

/*
 * mla_up_v — step 5: per-head W_UV up-projection of the latent attention output
 * (concept page, "Low-rank joint compression": W^UV is applied on the output side).
 *   out[b][i][h] = w_uv[h] . o_lat[b][i][h]     ([d_nope, d_latent] x [d_latent])
 *
 *   o_lat [B, n_q, n_h, d_latent]   read
 *   w_uv  [n_h, d_nope, d_latent]   read
 *   out   [B, n_q, n_h, d_nope]     written
 */
mla_status mla_up_v(const mla_shape* shape, const void* o_lat, int64_t n_q,
                    const void* w_uv, void* out, void* stream);

/*
 * mla_cache_shift_frames — whole-frame re-indexing of cached RoPE keys (the
 * delta-rotation for reused tokens at shifted positions, Irminsul abstract on the
 * "Multi-Head Latent Attention" topic page; positions as in VideoMLA "Core Mechanism").
 *
 * For b < B and the ring slots g mod S of g = first_tok .. first_tok + n_tok - 1, turn the
 * cached RoPE key as if its token had been written delta_frames frames later (or earlier,
 * for a negative delta_frames):
 *   cache[b][g mod S][d_latent : +d_rope] = RoPE3D-rotation by position (delta_frames, 0, 0)
 * A frame shift changes t only: the t-axis pairs turn by delta_frames * theta^(-j/n_t); the
 * y and x pairs and the latent are left as they are.  A row written for token g therefore
 * equals, up to rounding, what mla_cache_write stores for token g + delta_frames * F.  In
 * place: the rows stay in their slots, and the caller keeps track of the positions they
 * now stand for (shifts compose; a shift by a whole ring, delta_frames * F a multiple of S,
 * keeps the slot convention g mod S).
 *
 *   cache [B, S, d_latent + d_rope]   read and written at n_tok slots
 * Errors: MLA_ERR_RANGE if n_tok > S or first_tok < 0; MLA_ERR_ARG for a NULL cache or
 * n_tok < 0.
 */
mla_status mla_cache_shift_frames(const mla_shape* shape, void* cache, int64_t first_tok,
                                  int64_t n_tok, int64_t delta_frames, void* stream);

/*
 * mla_cache_quantise — the low-bit latent ring (QuantMLA abstract on the "Multi-Head Latent
 * Attention" topic page: the content latent and the RoPE key are cached at low bit width,
 * INT4 and INT4, or INT2 content with an INT4 RoPE key, each path with a quantiser of its
 * own).  The path's learned transformations are not applied: each path of each row has one
 * scale.
 *
 * For b < B and the slots r = g mod S of g = first_tok .. first_tok + n_tok - 1, the content
 * part x = cache[b][r][0 : d_latent] (and likewise the RoPE part cache[b][r][d_latent :]) is
 * quantised with q = 2^(bits-1) - 1:
 *   scale[b][r] = max|x| / q                              (float32, correctly rounded)
 *   code_i = x_i / scale rounded to the nearest integer (ties to even; float32 division),
 *            clipped to [-q, q]                           (all 0 when the scale is 0)
 * and the codes are stored as two's-complement fields of `bits` bits, little-endian: code i
 * at bits [i*bits, (i+1)*bits) of the packed row, byte k holding bits [8k, 8k + 8).
 *
 *   cache     [B, S, d_latent + d_rope]          read at n_tok slots (finite values)
 *   q_content [B, S, d_latent * content_bits / 8] bytes, written at those slots
 *   q_rope    [B, S, d_rope * rope_bits / 8]      bytes, written at those slots
 *   scale_c, scale_r [B, S] float32               written at those slots
 * content_bits and rope_bits are 2, 4 or 8.  Other slots are not touched.
 * Errors: MLA_ERR_ARG for a NULL pointer, n_tok < 0 or a bit width other than 2, 4, 8;
 * MLA_ERR_UNSUPPORTED unless d_latent and d_rope are multiples of 8 and at most 1024;
 * MLA_ERR_RANGE if n_tok > S or first_tok < 0; MLA_ERR_ALIGN for a pointer not 16-byte
 * aligned.
 */
mla_status mla_cache_quantise(const mla_shape* shape, const void* cache, int64_t first_tok,
                              int64_t n_tok, int32_t content_bits, int32_t rope_bits,
                              void* q_content, void* q_rope, float* scale_c, float* scale_r,
                              void* stream);

/*
 * mla_cache_dequantise — the rows a low-bit ring stands for (the inverse of
 * mla_cache_quantise): for the same slots,
 *   cache[b][r][i] = code_i * scale[b][r]   (the float32 product, rounded to the storage
 *                                            dtype to nearest even)
 * for both paths.  Arguments as in mla_cache_quantise, with the packed ring and scales read
 * and the cache written at n_tok slots; the same errors.
 */
mla_status mla_cache_dequantise(const mla_shape* shape, const void* q_content,
                                const void* q_rope, const float* scale_c,
                                const float* scale_r, int32_t content_bits, int32_t rope_bits,
                                int64_t first_tok, int64_t n_tok, void* cache, void* stream);

/*
 * mla_attend_quantised — steps 3 and 4 over the low-bit ring, with the dequantisation inside
 * the attention kernel (QuantMLA abstract on the "Multi-Head Latent Attention" topic page:
 * the attention unpacks and dequantises the INT4 / INT2 content codes and the INT4 RoPE
 * codes itself; the scores, softmax and output are those of mla_attend).
 *
 * The result is that of mla_attend over the ring whose rows are the dequantised values
 *   cache[b][r][i] = code_i * scale[b][r]      (both paths, as mla_cache_dequantise defines
 *                                              them),
 * up to rounding: inside the kernel a row's scale is rounded to bf16 and each product
 * code * scale to bf16 (the tensor cores' operand type), so an element can differ from the
 * float32 product rounded once by a unit in the last bf16 place.
 *
 *   q_abs      [B, n_q, n_h, d_latent + d_rope]            read
 *   q_content  [B, S, d_latent * content_bits / 8] bytes    read (mla_cache_quantise's layout)
 *   q_rope     [B, S, d_rope * rope_bits / 8] bytes         read
 *   scale_c, scale_r [B, S] float32                          read
 *   o_lat, lse, workspace: as in mla_attend (the same workspace size)
 * Supported: bfloat16, d_latent = 512, d_rope = 64, content_bits 4 or 2, rope_bits 4 (the
 * two configurations the QuantMLA abstract names).
 * Errors: those of mla_attend (the packed content codes stand where the cache does);
 * MLA_ERR_ARG for a NULL q_rope or scale, or a bit width other than 2, 4, 8;
 * MLA_ERR_UNSUPPORTED for other shapes, bit widths or float32; MLA_ERR_ALIGN for a pointer
 * not 16-byte aligned.
 */
mla_status mla_attend_quantised(const mla_shape* shape, const void* q_abs, int64_t n_q,
                                int64_t q_first_tok, const void* q_content, const void* q_rope,
                                const float* scale_c, const float* scale_r,
                                int32_t content_bits, int32_t rope_bits, int64_t k_first_tok,
                                int64_t n_keys, float softmax_scale, void* o_lat, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_attend_materialised_workspace_size — bytes of device workspace mla_attend_materialised
 * needs: the per-head keys and then the per-head values of every ring slot, bf16,
 * 2 * B * S * n_h * d_nope * 2 bytes.  0 for shapes the call does not support.
 */
size_t mla_attend_materialised_workspace_size(const mla_shape* shape);

/*
 * mla_attend_materialised — the non-absorbed form of steps 3 and 5 together: the
 * per-head keys and values are rebuilt from the latent ("Understanding Multi-Head
 * Latent Attention and KV Compression", "On-the-Fly Reconstruction and Matrix
 * Absorption"), and attention runs per head on the concatenation of the content and
 * RoPE channels (concept page, "The RoPE problem, and the decoupled fix").  Same result
 * as mla_absorb_q + mla_attend + mla_up_v up to rounding, with fewer flops whenever the
 * window holds more keys than a head has dimensions to absorb (chunks, not decode).
 *
 * For every ring slot r of every sequence b, and head h:
 *   K[b][r][h] = w_uk[h] . cache[b][r][0 : d_latent]     V[b][r][h] = w_uv[h] . cache[b][r][0 : d_latent]
 * (into the workspace, rounded to bf16); then for every (b, i, h), with the keys, window
 * and frame-block-causal mask of mla_attend:
 *   s(g)  = softmax_scale * (q_nope[b][i][h] . K[b][g mod S][h]
 *                            + RoPE3D(q_rope[b][i][h], position of q_first_tok + i) . cache[b][g mod S][d_latent :])
 *   out[b][i][h] = sum_g softmax(s)(g) * V[b][g mod S][h]
 *   lse[b][i][h] = log(sum_g exp(s(g)))   (natural log, float32; if lse != NULL)
 *
 *   q_nope [B, n_q, n_h, d_nope]      read
 *   q_rope [B, n_q, n_h, d_rope]      read (un-rotated)
 *   cache  [B, S, d_latent + d_rope]  read
 *   w_uk, w_uv [n_h, d_nope, d_latent] read
 *   out    [B, n_q, n_h, d_nope]      written
 *   lse    [B, n_q, n_h] float32 or NULL written
 *   workspace: at least mla_attend_materialised_workspace_size() bytes (required); its
 *   contents on entry do not matter, and calls sharing one must not run concurrently.
 * Supported: bf16 storage, d_nope = 128, d_rope = 64 or 512, d_latent a multiple of 128.
 * Errors: those of mla_attend; MLA_ERR_UNSUPPORTED for other shapes or float32;
 * MLA_ERR_ARG if the workspace is NULL or smaller than required.
 */
mla_status mla_attend_materialised(const mla_shape* shape, const void* q_nope,
                                   const void* q_rope, int64_t n_q, int64_t q_first_tok,
                                   const void* cache, int64_t k_first_tok, int64_t n_keys,
                                   float softmax_scale, const void* w_uk, const void* w_uv,
                                   void* out, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * mla_kernel_launches — number of kernels this library has launched in this process
 * (a host-side counter, incremented at every successful launch).  Diagnostic only.
 */
uint64_t mla_kernel_launches(void);

/* Human-readable name of a status. Never NULL. */
const char* mla_status_string(mla_status status);

/*
 * mla_device_error — synchronises `stream`, then reads and clears the library's
 * device-side error word.  Returns MLA_ERR_TIMEOUT if a kernel gave up a bounded
 * wait (on an mbarrier) since the last call, MLA_ERR_CUDA if the stream reports an
 * error, else MLA_OK.  The only call that synchronises.
 */
mla_status mla_device_error(void* stream);

/*
 * mla_check_wait_timeout — diagnostic of the failure path: enqueues one kernel whose single
 * thread waits, with the bounded wait every tensor-core kernel of the library uses, on a
 * barrier that nothing completes.  The wait gives up after its limit (about 2 s), records
 * site 0x7FF in the device error word and the kernel returns; mla_device_error on the same
 * stream then returns MLA_ERR_TIMEOUT, and the device stays usable.  Returns the launch
 * status (MLA_OK, or MLA_ERR_CUDA).
 */
mla_status mla_check_wait_timeout(void* stream);

/*
 * mla_device_error_info — details of the last device-side error that mla_device_error
 * reported: info[0] status bits, info[1] id of the first wait site that gave up,
 * info[2] its CTA index, info[3] a (thread << 16 | block) tag.  Zeros if none yet.
 */
void mla_device_error_info(uint32_t info[4]);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H */
