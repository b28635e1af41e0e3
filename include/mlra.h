/*
 * mlra.h -- C ABI of the MLRA / MLA latent-KV decode-attention library (libmlra.so).
 *
 * One decode step of one attention layer, in absorbed form, as described for
 * Multi-Head Low-Rank Attention ("Multi-Head Low-Rank Attention", ai.info AI
 * summary): Main Findings, "decoding reduces to three absorbable steps" --
 *   1. query-side weight absorption           -> mlra_absorb_q
 *   2. MQA-style attention over the shared latent KV cache, one softmax per
 *      latent branch (Methodology, second paragraph), split over the KV
 *      length (flash-decoding) and merged by log-sum-exp
 *                                              -> mlra_decode_attn + mlra_splitkv_combine
 *   3. output up-projection of every branch, summed over branches and scaled
 *      by the branch-count rescale (Key Contributions #2 and #3)
 *                                              -> mlra_out_proj
 * n_blocks = 1 is MLA (one latent head, one softmax), the comparison mode.
 *
 * Conventions shared by every call
 * --------------------------------
 * Pointers.  Every tensor pointer is a CUDA device pointer owned by the caller.
 *   The library allocates and frees no memory; scratch lives in a caller-owned
 *   workspace (mlra_workspace_size).  Tensors are dense, row-major, in the
 *   index order given, with no padding.
 * Streams.  Every call only enqueues work on `stream` (0 = legacy default
 *   stream) and returns; no call synchronises except mlra_get_device_error.
 * Errors.  Invalid arguments are detected on the host and returned as a status
 *   before anything is launched.  Launch failures return MLRA_ERR_CUDA.
 *   Problems only the device can see (an out-of-range page id, an mbarrier wait
 *   that exceeded its bound) are recorded in an error word inside the
 *   workspace; kernels never trap.  Nothing throws across this ABI.
 * Dtypes.  `dtype` is the storage type of the KV cache, W_uk, W_uv and
 *   q_nope / q_rope (MLRA_F32 or MLRA_BF16).  Absorbed queries, split
 *   partials, latent outputs, lse and the final output are always fp32.
 *   Arithmetic accumulates in fp32 throughout.
 * Index convention of the up-projections.  W[b, h, i, j] maps latent channel i
 *   of block b to head-dim channel j of head h:
 *     k_nope[t, j] = sum_i c_b[t, i] * W_uk[b, h, i, j]   (same for W_uv).
 * Cache row of one token.  D = n_blocks*d_cb + d_r elements:
 *   [ c_0 (d_cb) | c_1 (d_cb) | ... | c_{nb-1} (d_cb) | k_rope (d_r) ].
 *   With d_h = 128 and four blocks of 128 plus d_r = 64 this is 576 elements,
 *   4.5 d_h per token (Key Contributions #2; Main Findings, first bullet).
 * Logit of head h, branch b, token t (Key Contributions #2; shared RoPE key):
 *   z = (q_abs[h, b, :] . c_b[t] + q_rope[h, :] . k_rope[t]) * softmax_scale
 */
#ifndef MLRA_H_
#define MLRA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLRA_API __attribute__((visibility("default")))
#else
#define MLRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mlra_stream_t; /* == cudaStream_t */

typedef enum {
  MLRA_OK = 0,
  MLRA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent dims      */
  MLRA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (shape / dtype)      */
  MLRA_ERR_ALIGNMENT = 3,    /* a pointer is under-aligned (see each call)     */
  MLRA_ERR_WORKSPACE = 4,    /* workspace too small or misaligned              */
  MLRA_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed            */
  MLRA_ERR_BAD_PAGE = 6,     /* device: page id outside [0, num_pages)         */
  MLRA_ERR_TIMEOUT = 7,      /* device: a bounded wait expired                 */
  MLRA_ERR_NO_DEVICE = 8,    /* no usable sm_100 device                        */
  MLRA_ERR_RANGE = 9         /* device: a cache value of magnitude >= 65520 met
                                a tensor-core kernel that takes the tile as
                                fp16 (128 heads per CTA; MLA with a multiple
                                of 128 heads).  mlra_decode_attn then
                                recomputes the call with a kernel that keeps
                                the tile in bf16 (launched right after, it
                                returns at once unless needed) and the word
                                reads 0; it stays set, and the result is not
                                usable, only for MLRA with a multiple of 128
                                heads above 128, which no bf16 kernel takes */
} mlra_status_t;

typedef enum { MLRA_F32 = 0, MLRA_BF16 = 1 } mlra_dtype_t;

/* Shapes and scales of one attention layer. */
typedef struct {
  int32_t n_blocks;      /* latent branches nb: 4 (MLRA-4), 2 (MLRA-2), 1 (MLA)          */
  int32_t d_cb;          /* width of one latent block c_b                                */
  int32_t d_r;           /* width of the shared RoPE key (d_h / 2 in the paper's models) */
  int32_t n_heads;       /* query heads h                                                */
  int32_t d_h;           /* per-head NoPE key width = value width                        */
  int32_t page_size;     /* tokens per cache page when paged (must be 64); else ignored  */
  mlra_dtype_t dtype;    /* storage dtype, see above                                     */
  float softmax_scale;   /* multiplies the logit, e.g. 1/sqrt(d_h + d_r)                 */
  float branch_scale;    /* rescale of the summed branch outputs, e.g. 1/sqrt(n_blocks)  */
} mlra_config_t;

/* Human-readable name of a status code (static string). */
MLRA_API const char* mlra_status_string(mlra_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
MLRA_API int32_t mlra_version(void);

/*
 * Step 1: query absorption (Main Findings, "three absorbable steps", first step).
 *   q_abs[s, h, b, i] = sum_j W_uk[b, h, i, j] * q_nope[s, h, j]
 * so that q_abs . c_b[t] equals q_nope . k_nope[t] with the explicit key.
 *   q_nope : [batch, n_heads, d_h]            dtype
 *   w_uk   : [n_blocks, n_heads, d_cb, d_h]   dtype
 *   q_abs  : [batch, n_heads, n_blocks, d_cb] fp32 (written)
 * fp32 accumulation.  batch = 0 is a no-op.  w_uk must be 16-byte aligned.
 */
MLRA_API mlra_status_t mlra_absorb_q(const mlra_config_t* cfg, const void* q_nope, const void* w_uk,
                            float* q_abs, int32_t batch, mlra_stream_t stream);

/*
 * Step 1 with the query side of the calibration ("Multi-Head Low-Rank
 * Attention", Main Findings, variance bullet: the query is scaled by
 * alpha_q = sqrt(d / d_c'); Key Contributions #2: the decoupled RoPE query
 * meets the one shared RoPE key):
 *   q_abs[s, h, b, i]  = alpha_q * sum_j W_uk[b, h, i, j] * q_nope[s, h, j]   (fp32)
 *   q_rope_out[s, h, :] = RoPE(alpha_q * q_rope[s, h, :], positions[s])       (dtype)
 * RoPE pairs channel i with i + d_r/2 and rotates the pair by
 * p * rope_theta^(-2i / d_r), the same rotation mlra_cache_append gives the
 * key, so the RoPE logit depends only on the distance between the query's and
 * the key's positions.  q_rope_out then goes to mlra_decode_attn as q_rope.
 *   q_nope     : [batch, n_heads, d_h] dtype (before alpha_q)
 *   q_rope     : [batch, n_heads, d_r] dtype (before alpha_q and RoPE)
 *   positions  : [batch] int32 device memory: the query token's position
 *                (normally seqlens[s] - 1); any int32 is a valid angle
 *   w_uk, q_abs: as mlra_absorb_q
 *   q_rope_out : [batch, n_heads, d_r] dtype (written); must not overlap
 *                q_rope unless it is the same buffer (in place)
 * The angle and its sine and cosine are taken in fp64; the rotation in fp32,
 * rounded once to dtype.  With alpha_q = 1, q_abs equals mlra_absorb_q's bit
 * for bit.  d_r must be even and <= 512.  batch = 0 is a no-op.
 */
MLRA_API mlra_status_t mlra_absorb_q_rope(const mlra_config_t* cfg, const void* q_nope,
                                          const void* q_rope, const int32_t* positions,
                                          float alpha_q, float rope_theta, const void* w_uk,
                                          float* q_abs, void* q_rope_out, int32_t batch,
                                          mlra_stream_t stream);

/*
 * Workspace bytes needed by mlra_decode_attn / mlra_splitkv_combine for up to
 * `batch` sequences on the current CUDA device (depends on its SM count).
 * Writes the size to *bytes.  The workspace must be 256-byte aligned.  It holds
 * the split plan, the split partials (fp32) and the device error word.
 */
MLRA_API mlra_status_t mlra_workspace_size(const mlra_config_t* cfg, int32_t batch, size_t* bytes);

/*
 * Step 2a: split-KV attention over the latent cache, one softmax per branch
 * ("Multi-Head Low-Rank Attention": Main Findings, the MQA-style second of the
 * three absorbable steps; Methodology, second paragraph, attention on each
 * latent block separately; Key Contributions #2, the shared RoPE key).
 * For every sequence s the tokens t in [0, seqlens[s]) are cut into chunks
 * (planned on the device from seqlens, balanced over the SMs); for every chunk,
 * head h and branch b it computes, over that chunk's tokens,
 *   o_part = sum_t softmax(z)_t * c_b[t]        (latent output, fp32)
 *   lse_part = log sum_t exp(z_t)               (natural log)
 * and stores both in the workspace for mlra_splitkv_combine.
 *   q_abs      : [batch, n_heads, n_blocks, d_cb] fp32 (from mlra_absorb_q)
 *   q_rope     : [batch, n_heads, d_r] dtype
 *   kv_cache   : paged (page_table != NULL): [num_pages, page_size, D] dtype;
 *                contiguous (page_table == NULL): [batch, max_len, D] dtype
 *   num_pages  : paged: pages in kv_cache (page ids are checked against it);
 *                contiguous: ignored
 *   page_table : [batch, max_pages] int32 or NULL.  Entry p of row s holds the
 *                page of tokens [64p, 64p+64) of sequence s; entries past the
 *                sequence's last page are never read.
 *   max_pages  : paged: row stride of page_table; contiguous: max_len, the row
 *                stride of kv_cache in tokens
 *   seqlens    : [batch] int32, 0 <= seqlens[s] <= max_pages*page_size (paged)
 *                or <= max_len (contiguous); device memory
 *   workspace  : >= mlra_workspace_size bytes, 256-byte aligned, caller-owned
 * Cache rows at or beyond seqlens[s] never influence the result, whatever they
 * hold (they are zero-filled on chip before use).  The device error word is
 * reset at the start of every call.  kv_cache, q_abs and q_rope must be
 * 16-byte aligned (they are read in 16-byte units, the cache by the tensor
 * memory accelerator); seqlens and page_table 4-byte aligned.
 * Launches: the planner and the attention kernel; with bf16 data and 128 heads
 * (MLRA with d_cb = 128, or MLA with a multiple of 128 heads), whose kernel
 * takes the tile as fp16, a third launch that returns at once unless a cache
 * value left the fp16 range (MLRA_ERR_RANGE), in which case it recomputes the
 * call with a kernel that keeps the tile in bf16 and clears that error.
 */
MLRA_API mlra_status_t mlra_decode_attn(const mlra_config_t* cfg, const float* q_abs, const void* q_rope,
                               const void* kv_cache, int64_t num_pages, const int32_t* page_table,
                               int32_t max_pages, const int32_t* seqlens, int32_t batch,
                               void* workspace, size_t workspace_bytes, mlra_stream_t stream);

/*
 * Step 2b: merge the split partials of every (sequence, head, branch) -- the
 * chunks of step 2a split one softmax over all of a sequence's tokens
 * (Methodology, second paragraph: one softmax per branch), so their
 * log-sum-exp merge gives that softmax's output, up to rounding:
 *   lse = log sum_k exp(lse_k);   o_lat = sum_k exp(lse_k - lse) * o_k
 *   workspace : the one passed to the preceding mlra_decode_attn (same stream)
 *   o_latent  : [batch, n_heads, n_blocks, d_cb] fp32 (written)
 *   lse       : [batch, n_heads, n_blocks] fp32 natural log (written; may be NULL)
 * A sequence with seqlens = 0 gets o_latent = 0 and lse = -inf.
 */
MLRA_API mlra_status_t mlra_splitkv_combine(const mlra_config_t* cfg, const void* workspace,
                                   size_t workspace_bytes, int32_t batch, float* o_latent,
                                   float* lse, mlra_stream_t stream);

/*
 * Step 3: output up-projection, summed over branches and rescaled
 * (Key Contributions #2: block outputs are summed; #3: branch-count rescale):
 *   out[s, h, j] = branch_scale * sum_b sum_i o_latent[s, h, b, i] * W_uv[b, h, i, j]
 *   o_latent : [batch, n_heads, n_blocks, d_cb] fp32
 *   w_uv     : [n_blocks, n_heads, d_cb, d_h] dtype
 *   out      : [batch, n_heads, d_h] fp32 (written)
 * w_uv must be 16-byte aligned; d_h <= 128.
 */
MLRA_API mlra_status_t mlra_out_proj(const mlra_config_t* cfg, const float* o_latent, const void* w_uv,
                            float* out, int32_t batch, mlra_stream_t stream);

/*
 * Steps 2b + 3 in one launch: the split partials of the workspace are merged
 * (as mlra_splitkv_combine) while they are staged as the operand of the output
 * up-projection (as mlra_out_proj).  The paper describes the two steps, not
 * their fusion; the result is the same up to fp32 rounding order.
 *   workspace : the one passed to the preceding mlra_decode_attn (same stream)
 *   w_uv      : [n_blocks, n_heads, d_cb, d_h] dtype, 16-byte aligned
 *   out       : [batch, n_heads, d_h] fp32 (written)
 *   o_latent  : [batch, n_heads, n_blocks, d_cb] fp32, written when not NULL
 *               (16-byte aligned)
 *   lse       : [batch, n_heads, n_blocks] fp32, written when not NULL
 * Runs as one tensor-core kernel for bf16 with d_h = 128, d_cb a multiple of
 * 128 and n_blocks * d_cb <= 512 on sm_100; otherwise it runs the two steps
 * one after the other, which needs o_latent (MLRA_ERR_UNSUPPORTED if NULL).
 */
MLRA_API mlra_status_t mlra_combine_out_proj(const mlra_config_t* cfg, const void* workspace,
                                    size_t workspace_bytes, int32_t batch, const void* w_uv,
                                    float* out, float* o_latent, float* lse,
                                    mlra_stream_t stream);

/*
 * Workspace bytes mlra_decode_step needs for up to `batch` sequences on the
 * current device: the mlra_decode_attn workspace (first, so that
 * mlra_get_device_error reads the same error word) followed by the absorbed
 * query, the latent output and staging room for the step's inputs and output.
 */
MLRA_API mlra_status_t mlra_step_workspace_size(const mlra_config_t* cfg, int32_t batch,
                                                size_t* bytes);

/*
 * Steps 1, 2a, 2b and 3 in one call: absorb the query, split-KV attention,
 * merge and output up-projection (Main Findings, the three absorbable steps),
 * enqueued on `stream` in that order.  The result equals that of
 * mlra_absorb_q -> mlra_decode_attn -> mlra_combine_out_proj bit for bit.
 *   q_nope, q_rope, seqlens : as mlra_absorb_q / mlra_decode_attn
 *   w_uk, w_uv              : as mlra_absorb_q / mlra_out_proj (device)
 *   kv_cache, num_pages, page_table, max_pages : as mlra_decode_attn (device)
 *   out      : [batch, n_heads, d_h] fp32 (written)
 *   host_io  : 0 = q_nope, q_rope, seqlens and out are device memory;
 *              1 = they are host memory: the call enqueues the transfer of
 *              the inputs into the workspace, the kernels and the transfer of
 *              out back to the host, and returns without waiting (out is
 *              valid once `stream` has passed this call).  Page-locked host
 *              memory mapped into the device's address space (cudaHostAlloc /
 *              cudaMallocHost under unified addressing) is read by one
 *              staging kernel and out is written by the projection kernel in
 *              place; other host memory moves by cudaMemcpyAsync, which is
 *              synchronous for pageable memory.  The host must not modify
 *              the inputs or read out until the stream has passed the call.
 *   workspace : >= mlra_step_workspace_size bytes, 256-byte aligned
 * Errors as the three calls it makes; MLRA_ERR_INVALID_ARG for host_io not 0
 * or 1.  batch = 0 launches nothing.
 * Repeated calls: a call whose transfers are all kernels (device buffers, or
 * mapped host buffers) is recorded as a CUDA graph the second time the same
 * pointers, sizes and configuration are passed, and later calls replay it (one
 * graph launch instead of five kernel launches; the contents of every buffer
 * may change between calls, as with direct launches).  Nothing is recorded
 * while `stream` is being captured by the caller.  The library keeps up to 64
 * such graphs per process, until mlra_release_step_graphs.
 */
MLRA_API mlra_status_t mlra_decode_step(const mlra_config_t* cfg, const void* q_nope,
                                        const void* q_rope, const int32_t* seqlens, int32_t batch,
                                        const void* w_uk, const void* w_uv, const void* kv_cache,
                                        int64_t num_pages, const int32_t* page_table,
                                        int32_t max_pages, float* out, int32_t host_io,
                                        void* workspace, size_t workspace_bytes,
                                        mlra_stream_t stream);

/*
 * Destroy every CUDA graph mlra_decode_step has recorded in this process (no
 * counterpart in the paper: the recording is a property of this library).
 * Call it only when no mlra_decode_step call is executing on the GPU (after
 * synchronising the streams they were made on); later calls record afresh.
 * Returns MLRA_ERR_CUDA if a graph could not be destroyed (the record is
 * dropped all the same).
 */
MLRA_API mlra_status_t mlra_release_step_graphs(void);

/*
 * Cache write (the step before decode attention reads the cache; the paper
 * describes it in prose: Methodology, third paragraph, latent RMSNorm before
 * the up-projection; Main Findings, variance bullet, the KV latent scaled by
 * alpha_kv; Key Contributions #2, one decoupled RoPE key).  For every
 * sequence s, the row of its new token at position p = positions[s]:
 *   latent block b: alpha_kv * gamma * c_b / sqrt(mean(c_b^2) + rms_eps)
 *   RoPE key: channel i paired with i + d_r/2, rotated by p * theta^(-2i/d_r)
 *   c_new      : [batch, n_blocks * d_cb] dtype (latent before normalisation)
 *   k_rope_new : [batch, d_r] dtype (RoPE key before rotation; d_r even)
 *   rms_gamma  : [n_blocks * d_cb] fp32 gain
 *   alpha_kv   : the latent scale (sqrt(d_model / d_cb) in the paper's calibration)
 *   kv_cache, num_pages, page_table, max_pages : as mlra_decode_attn; the row
 *                of token p is written in place (page_table[s][p / 64], row p % 64)
 *   positions  : [batch] int32, 0 <= p < max_pages * 64 (paged) or < max_len
 *   device_status : one int32 in device memory or NULL; a position out of
 *                range (MLRA_ERR_INVALID_ARG) or a page id out of range
 *                (MLRA_ERR_BAD_PAGE) is recorded there (first error wins) and
 *                that sequence's row is not written.
 * Pointers must be aligned to their element type.  No counterpart to the
 * paper's kernels: it fixes no layout for this step.
 */
MLRA_API mlra_status_t mlra_cache_append(const mlra_config_t* cfg, const void* c_new,
                                const void* k_rope_new, const float* rms_gamma, float alpha_kv,
                                float rms_eps, float rope_theta, void* kv_cache,
                                int64_t num_pages, const int32_t* page_table, int32_t max_pages,
                                const int32_t* positions, int32_t batch, int32_t* device_status,
                                mlra_stream_t stream);

/*
 * Read (and then clear) the device error word of a workspace.  Synchronises
 * `stream`.  *device_status receives MLRA_OK or the first device-side error
 * (MLRA_ERR_BAD_PAGE, MLRA_ERR_TIMEOUT) recorded since the last decode call.
 */
MLRA_API mlra_status_t mlra_get_device_error(const void* workspace, size_t workspace_bytes,
                                    int32_t* device_status, mlra_stream_t stream);

/*
 * Steps 2a + 2b without a caller workspace (no counterpart in the paper: this
 * is a deployment convenience of the library).
 * Some callers cannot call cudaMalloc: a plugin running inside a host
 * framework that owns all device memory through its own allocator, or a
 * serving process that reserves all free HBM for the KV cache at start-up and
 * must not allocate later (cudaMalloc may also synchronise the device, which a
 * latency-bound decode loop cannot afford).  This call needs no workspace and
 * allocates nothing: its scratch (split plan, split partials, error word) is a
 * fixed 16 MiB array inside libmlra.so, held on every GPU that loads the
 * library until the process exits.
 *   Arguments as mlra_decode_attn, then as mlra_splitkv_combine:
 *   o_latent      : [batch, n_heads, n_blocks, d_cb] fp32 (written)
 *   lse           : [batch, n_heads, n_blocks] fp32 (written; may be NULL)
 *   device_status : one int32 in device memory (may be NULL); receives the
 *                   device error word of this call (MLRA_OK, MLRA_ERR_BAD_PAGE,
 *                   MLRA_ERR_TIMEOUT, MLRA_ERR_INVALID_ARG for clamped seqlens)
 * Returns MLRA_ERR_WORKSPACE, launching nothing, when the scratch this batch
 * needs (mlra_workspace_size) exceeds 16 MiB.  The first call on a device looks
 * up the array's device address with that device current (and again after the
 * device's context changed, e.g. after cudaDeviceReset); make that first call
 * before capturing any stream.  All calls share the one array and it
 * keeps the last call's contents: calls ordered on one stream are safe, calls
 * that overlap on the GPU (other streams, other host threads) race on it.
 */
MLRA_API mlra_status_t mlra_decode_attn_noalloc(const mlra_config_t* cfg, const float* q_abs,
                                                const void* q_rope, const void* kv_cache,
                                                int64_t num_pages, const int32_t* page_table,
                                                int32_t max_pages, const int32_t* seqlens,
                                                int32_t batch, float* o_latent, float* lse,
                                                int32_t* device_status, mlra_stream_t stream);

/*
 * Which decode kernel mlra_decode_attn would launch for cfg on the current
 * device: 1 = tensor-core kernel (tcgen05 / TMEM / TMA), 2 = fp32 SIMT kernel,
 * 0 = unsupported.  Host-only query, launches nothing.
 */
MLRA_API int32_t mlra_decode_kernel_kind(const mlra_config_t* cfg);

#ifdef __cplusplus
}
#endif

#endif /* MLRA_H_ */
