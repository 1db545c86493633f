/*
 * mla.h -- C ABI of libmla: Multi-head Latent Attention (MLA) decode over a
 * paged, low-rank joint-compressed KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek V2 MLA page, snabindia.com, sections 2.1-2.3): every
 * token caches only its joint latent c_KV = W_DKV x (width d_c) and one
 * decoupled RoPE key k_R = RoPE(W_KR x, pos) (width d_r) shared by all H
 * heads.  W_UK is absorbed into the query and W_UV into the output, so all
 * heads attend directly over the latent rows  row_j = c_KV_j (+) k_R_j  of
 * width D = d_c + d_r, with V = row[0:d_c].
 *
 * A decode step of one layer is, in order:
 *   mla_cache_append   write the new tokens' rows into the paged cache
 *   mla_absorb_q       q_lat = (W_UK^T q_nope) (+) RoPE(q_pe)
 *   mla_decode         split-KV attention over the latent rows + split merge
 *   mla_out_proj       y = W_O (W_UV o_lat)
 *
 * Conventions shared by every call
 * --------------------------------
 * - All pointers are device pointers unless a parameter says "host".  The
 *   caller allocates and owns every buffer (cache, page table, weights,
 *   workspace, outputs).  The library allocates device memory only inside
 *   mla_create (RoPE table, error word) and frees it in mla_destroy; no call
 *   on the decode path allocates, frees or synchronises.
 * - Calls are asynchronous on the given stream (0 = legacy default stream).
 * - Tensors are dense, row-major, innermost dimension last, no padding.
 *   bf16 tensors hold IEEE bfloat16 bit patterns, fp32 tensors IEEE binary32,
 *   fp8 tensors OCP E4M3 codes.  Activation tensors (c_kv, k_r, q_nope, q_pe,
 *   q_lat, o_lat, y, weights) use the handle's act_dtype; the cache uses
 *   cache_dtype.
 * - Device pointers to activations, weights, caches and workspaces must be
 *   16-byte aligned (vector and TMA access); int32 arrays 4-byte; the fp32
 *   cache_scale array 4-byte for the append calls and 16-byte for the decode
 *   calls (a page's 64 scales are fetched by one bulk copy).
 * - Return value: MLA_OK (0) or a negative mla_status_t.  A call that returns
 *   an error has launched nothing.  Invalid page-table entries or positions
 *   found by a kernel are reported through the device error word, read by
 *   mla_last_device_error; the offending access is skipped, never performed.
 * - No call exits, aborts or traps.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,  /* null pointer, bad size or bad config value        */
  MLA_ERR_UNSUPPORTED = -2,  /* dims/dtypes the library has no kernel for          */
  MLA_ERR_ALIGNMENT = -3,    /* a pointer is not 16-byte aligned                   */
  MLA_ERR_WORKSPACE = -4,    /* workspace null or smaller than the query call says */
  MLA_ERR_LAUNCH = -5,       /* a kernel launch failed (cudaGetLastError)          */
  MLA_ERR_BAD_INDEX = -6,    /* device: page-table entry or position out of range  */
  MLA_ERR_TIMEOUT = -7,      /* device: a bounded wait gave up                     */
  MLA_ERR_CUDA = -8,         /* another CUDA runtime error                         */
  MLA_ERR_RANGE = -9         /* device: a value beyond the range of an fp16 split partial */
} mla_status_t;

typedef enum { MLA_BF16 = 0, MLA_FP8_E4M3 = 1, MLA_FP32 = 2 } mla_dtype_t;

/* Layer configuration.  Dimension names follow the V2 page (section 3.1 table:
 * h = 128 heads, d = 128, d_c = 512, d_r = 64). */
typedef struct {
  int32_t num_heads;     /* H                                                    */
  int32_t d_c;           /* latent width (kv_lora_rank); multiple of 16          */
  int32_t d_r;           /* decoupled RoPE width; even, multiple of 8            */
  int32_t d_nope;        /* per-head non-RoPE query/key width                    */
  int32_t d_v;           /* per-head value width                                 */
  int32_t d_model;       /* model width (rows of W_O)                            */
  int32_t block_size;    /* tokens per cache page; 64                            */
  int32_t act_dtype;     /* MLA_BF16 or MLA_FP32                                 */
  int32_t cache_dtype;   /* MLA_BF16, MLA_FP8_E4M3 (act bf16) or MLA_FP32 (act fp32) */
  float softmax_scale;   /* multiplies q.k; the library reads it as given        */
  float rope_base;       /* RoPE base, 10000 on the pages                        */
  int32_t max_position;  /* positions must lie in [0, max_position)              */
} mla_config_t;

typedef struct mla_ctx* mla_handle_t;

/* Create a handle: validates the configuration, checks the current device is
 * sm_100, builds the RoPE table cos/sin(pos * theta_i), theta_i =
 * rope_base^(-2i/d_r) (V2 page section 2.2 apply_rope) on the host in double
 * precision, stores it as fp32 [max_position][d_r/2] on the current device,
 * and allocates the device error word.  *out is set only on success.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA. */
MLA_API int mla_create(const mla_config_t* cfg, mla_handle_t* out);

/* Free the handle's device memory.  Waits for nothing: the caller must not
 * destroy a handle while work that uses it is in flight.  NULL is a no-op. */
MLA_API int mla_destroy(mla_handle_t h);

/* Bytes of one cached token row, and of its scale (0 unless FP8). */
MLA_API size_t mla_cache_row_bytes(mla_handle_t h);
MLA_API size_t mla_cache_scale_bytes(mla_handle_t h);

/* mla_cache_append -- V2 page section 2.2 (mla_rope: k_r = apply_rope(k_r,
 * pos)) and section 2.3 (cache only KV_comp and k_R); V3 page MLA sketch
 * (kv_cache = cat(kv_cache, kv_latent)); paged memory, V2 page section 3.3.
 *
 * For token t (0 <= t < num_tokens): b = seq_idx ? seq_idx[t] : t,
 * p = pos[t], page = block_table[b * max_blocks_per_seq + p / block_size],
 * slot = page * block_size + p % block_size, and
 *   cache[slot][0:d_c]      = c_kv[t]
 *   cache[slot][d_c:d_c+d_r] = RoPE(k_r[t], p)   (rotate-half pairs (i, i+d_r/2))
 * computed in fp32 and rounded once to the cache dtype.  FP8 cache: the fp32
 * row is quantised per token: amax = max|row|, scale = amax/448,
 * code = e4m3_rn_satfinite(row * (448/amax)); cache_scale[slot] = scale
 * (amax = 0 gives scale 1 and zero codes).
 *
 * c_kv  [num_tokens, d_c] act dtype      k_r [num_tokens, d_r] act dtype (pre-RoPE)
 * seq_idx [num_tokens] int32 or NULL     pos [num_tokens] int32
 * block_table [batch, max_blocks_per_seq] int32 (the caller's page allocator
 *   must have mapped every page a token lands in)
 * cache [num_blocks, block_size, d_c+d_r] cache dtype (written in place)
 * cache_scale [num_blocks, block_size] fp32 for FP8, else NULL
 * Rows of tokens whose page or position is out of range are not written; the
 * error word records MLA_ERR_BAD_INDEX.  Two tokens mapping to one slot race.
 * Errors: INVALID_ARG, ALIGNMENT, LAUNCH. */
MLA_API int mla_cache_append(mla_handle_t h, const void* c_kv, const void* k_r,
                     const int32_t* seq_idx, const int32_t* pos, int32_t num_tokens,
                     const int32_t* block_table, int32_t max_blocks_per_seq, int32_t batch,
                     void* cache, float* cache_scale, int32_t num_blocks,
                     cudaStream_t stream);

/* mla_kv_project_append -- the step before mla_cache_append, fused with it
 * (V2 page section 2.1: KV_comp = W_D^KV X; V3 page sketch w_dkv / w_kr):
 *   c_kv[t] = W_DKV x[t],  k_raw[t] = W_KR x[t],  then exactly the row write of
 * mla_cache_append.  x [num_tokens, d_model]; w_dkv [d_c, d_model];
 * w_kr [d_r, d_model]; other arguments as mla_cache_append.  fp32 accumulation. */
MLA_API int mla_kv_project_append(mla_handle_t h, const void* x, const void* w_dkv, const void* w_kr,
                          const int32_t* seq_idx, const int32_t* pos, int32_t num_tokens,
                          const int32_t* block_table, int32_t max_blocks_per_seq, int32_t batch,
                          void* cache, float* cache_scale, int32_t num_blocks,
                          cudaStream_t stream);

/* mla_absorb_q -- V2 page section 2.3 ("absorb W_U^K into W_Q") and section
 * 4.1 optimize_for_inference, applied per head at run time:
 *   q_lat[b][h][0:d_c]       = W_UK[h]^T q_nope[b][h]      (sum over d_nope)
 *   q_lat[b][h][d_c:d_c+d_r] = RoPE(q_pe[b][h], pos[b])
 * q_nope [batch, H, d_nope]; q_pe [batch, H, d_r] (pre-RoPE); pos [batch]
 * int32; w_uk [H, d_nope, d_c] (so that K_nope = W_UK[h] c_KV);
 * q_lat [batch, H, d_c+d_r] out.  fp32 accumulation, one rounding.
 * Errors: INVALID_ARG, ALIGNMENT, LAUNCH; out-of-range pos -> BAD_INDEX. */
MLA_API int mla_absorb_q(mla_handle_t h, const void* q_nope, const void* q_pe, const int32_t* pos,
                 const void* w_uk, int32_t batch, void* q_lat, cudaStream_t stream);

/* Split count mla_decode picks for num_splits = 0, from the batch and the
 * longest sequence (host value).  Always >= 1. */
MLA_API int32_t mla_decode_auto_splits(mla_handle_t h, int32_t batch, int32_t max_seq_len);

/* Workspace bytes mla_decode / mla_decode_partial need for this batch and
 * split count (num_splits = 0: the automatic count for max_seq_len). */
MLA_API size_t mla_decode_workspace_bytes(mla_handle_t h, int32_t batch, int32_t num_splits,
                                  int32_t max_seq_len);

/* mla_decode -- absorbed MLA attention over the latent cache (V2 page section
 * 2.3: Softmax((Q_c (+) Q_R)(K_c^T (+) K_R^T)/sqrt(d)) with K_c = W_UK c_KV
 * folded into q_lat and V = W_UV c_KV folded into the output side).
 * For every sequence b and head h, over the seq_lens[b] tokens at positions
 * 0..seq_lens[b]-1 of sequence b:
 *   s_j = softmax_scale * q_lat[b][h] . row_j          (fp8: row_j = scale_j * code_j)
 *   o_lat[b][h] = sum_j softmax(s)_j row_j[0:d_c],   lse[b][h] = ln sum_j exp(s_j)
 * The tokens are cut into num_splits ranges per sequence (flash-decoding);
 * each range's normalised partial and log-sum-exp go to the workspace and a
 * second kernel merges them.  seq_lens[b] = 0 gives o_lat = 0, lse = -inf.
 * q_lat [batch, H, d_c+d_r] act dtype; cache / cache_scale / num_blocks as
 * mla_cache_append (pages outside [0, num_blocks) are skipped and reported);
 * block_table [batch, max_blocks_per_seq]; seq_lens [batch] int32 with
 * seq_lens[b] <= max_seq_len <= max_blocks_per_seq * block_size;
 * num_splits >= 0 (0 = automatic); workspace >= mla_decode_workspace_bytes;
 * o_lat [batch, H, d_c] act dtype out; lse [batch, H] fp32 out (may be NULL).
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, LAUNCH. */
MLA_API int mla_decode(mla_handle_t h, const void* q_lat, const void* cache, const float* cache_scale,
               int32_t num_blocks, const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
               int32_t batch, int32_t max_seq_len, int32_t num_splits,
               void* workspace, size_t workspace_bytes, void* o_lat, float* lse,
               cudaStream_t stream);

/* The two halves of mla_decode, for callers that time or schedule them
 * separately.  mla_decode_partial writes the workspace; mla_decode_combine
 * reads it (same batch / num_splits / max_seq_len) and writes o_lat and lse.
 * Workspace layout: o_part, then at the next 256-byte boundary lse_part fp32
 * [batch][S][H].  o_part holds each split's normalised partial output in
 * 16-byte groups of latent columns, heads next: with bf16 activations fp16
 * [batch][S][d_c/8][H][8] (o_part[b][s][c/8][h][c%8]), with fp32 activations
 * fp32 [batch][S][d_c/4][H][4].  An empty range stores lse_part = -inf,
 * o_part = 0.  An fp16 partial holds |value| <= 65504: a larger latent
 * output (only from cache values of that size) records MLA_ERR_RANGE in the
 * device error word. */
MLA_API int mla_decode_partial(mla_handle_t h, const void* q_lat, const void* cache,
                       const float* cache_scale, int32_t num_blocks, const int32_t* block_table,
                       int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                       int32_t max_seq_len, int32_t num_splits, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream);
MLA_API int mla_decode_combine(mla_handle_t h, int32_t batch, int32_t max_seq_len, int32_t num_splits,
                       const void* workspace, size_t workspace_bytes, void* o_lat, float* lse,
                       cudaStream_t stream);

/* mla_decode_noalloc -- mla_decode for callers that cannot allocate device
 * memory (for example a plugin inside a framework that owns every device
 * buffer through its own pool, or a loop that must not risk the implicit
 * device synchronisation of cudaMalloc).  The pages have no counterpart: this
 * is a deployment convenience of this library, not a step of the method.
 *
 * Same arguments and results as mla_decode minus the workspace: the split
 * partials go to a 32 MiB array compiled into the library, which stays
 * allocated on every GPU that loads the library until the process exits.
 * - A call whose workspace (mla_decode_workspace_bytes for the same batch,
 *   num_splits and max_seq_len) exceeds 32 MiB returns MLA_ERR_WORKSPACE and
 *   launches nothing.
 * - The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.
 * - Every call on a device shares the one array, which keeps the last call's
 *   contents; nothing in it needs clearing between calls, but calls that
 *   overlap on the GPU (other streams, other threads) race on it.
 * - It calls no cudaMalloc, cudaFree or other allocating routine. */
MLA_API int mla_decode_noalloc(mla_handle_t h, const void* q_lat, const void* cache,
                               const float* cache_scale, int32_t num_blocks,
                               const int32_t* block_table, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                               int32_t num_splits, void* o_lat, float* lse, cudaStream_t stream);

/* W_O in tile-major order, for a faster weight stream.  Writes
 * w_o_tiled[m/128][k/64][m%128][k%64] = w_o[m][k] for the handle's
 * [d_model, H*d_v] W_O (act dtype), so that every 128 x 64 tile is one
 * contiguous 16 KB (32 KB in fp32) run; the tensor-core output projection then
 * reads one contiguous run per request.  w_o_tiled is a separate buffer of the
 * same size, owned by the caller; both 16-byte aligned.  Asynchronous on
 * `stream`.  Errors: INVALID_ARG (null or identical pointers), UNSUPPORTED
 * (d_model not a multiple of 128 or H*d_v not a multiple of 64), ALIGNMENT,
 * LAUNCH. */
MLA_API int mla_pack_w_o(mla_handle_t h, const void* w_o, void* w_o_tiled, cudaStream_t stream);

/* Layout of the w_o argument of later mla_out_proj / mla_combine_out_proj
 * calls on this handle: 0 row-major (default), 1 tile-major (mla_pack_w_o).
 * Results do not depend on the layout beyond fp32 summation order.  Errors:
 * INVALID_ARG (null handle), UNSUPPORTED (shape not tileable). */
MLA_API int mla_set_w_o_layout(mla_handle_t h, int tiled);

/* Workspace bytes mla_out_proj needs for this batch. */
MLA_API size_t mla_out_proj_workspace_bytes(mla_handle_t h, int32_t batch);

/* mla_out_proj -- V2 page section 2.3 ("absorb W_U^V into W_O"), applied as
 * two contractions:  o[b][h] = W_UV[h] o_lat[b][h]  (d_v x d_c per head), then
 * y[b] = W_O concat_h o[b][h]  (d_model x H*d_v).  fp32 accumulation; o is
 * rounded to the act dtype between the two.
 * o_lat [batch, H, d_c]; w_uv [H, d_v, d_c]; w_o [d_model, H*d_v] row-major,
 * or tile-major after mla_set_w_o_layout(h, 1) (see mla_pack_w_o);
 * y [batch, d_model] out; o_out [batch, H, d_v] out, or NULL to keep o in the
 * workspace only.  Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, LAUNCH. */
MLA_API int mla_out_proj(mla_handle_t h, const void* o_lat, const void* w_uv, const void* w_o,
                 int32_t batch, void* workspace, size_t workspace_bytes, void* y, void* o_out,
                 cudaStream_t stream);

/* mla_combine_out_proj -- the split merge of mla_decode_combine followed by
 * mla_out_proj, in one call (V2 page section 2.3 for the output side; the merge
 * is the log-sum-exp combination of the split partials).  Where the tensor-core
 * path covers the batch, the merge runs inside the W_UV kernel: every head's
 * merged o_lat slice is built straight into that kernel's operand, which saves
 * the merge kernel and its round trip through memory; the results are bit-for-
 * bit those of the two separate calls.  Otherwise the two calls run in turn.
 * batch / max_seq_len / num_splits / workspace as for mla_decode_partial (its
 * workspace holds the partials); w_uv, w_o, op_workspace (at least
 * mla_out_proj_workspace_bytes), y and o_out as for mla_out_proj; o_lat
 * [batch, H, d_c] out (required); lse [batch, H] out or NULL.
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, LAUNCH. */
MLA_API int mla_combine_out_proj(mla_handle_t h, int32_t batch, int32_t max_seq_len, int32_t num_splits,
                                 const void* workspace, size_t workspace_bytes, const void* w_uv,
                                 const void* w_o, void* op_workspace, size_t op_workspace_bytes,
                                 void* o_lat, float* lse, void* y, void* o_out, cudaStream_t stream);

/* Synchronise the stream, then read and clear the handle's device error word:
 * MLA_OK, MLA_ERR_BAD_INDEX or MLA_ERR_TIMEOUT (or MLA_ERR_CUDA if the sync
 * itself failed).  Not for use inside stream capture. */
MLA_API int mla_last_device_error(mla_handle_t h, cudaStream_t stream);

/* Debug knob for tests of the bounded waits: the iteration limit of every
 * device-side wait loop (0 = the built-in default).  A limit so small that a
 * wait gives up makes the kernel record MLA_ERR_TIMEOUT and return. */
MLA_API int mla_set_wait_limit(mla_handle_t h, uint32_t limit);

/* Launch overlap (programmatic dependent launch), off by default.  When on,
 * each kernel of this handle is launched so that it may start while the
 * kernel issued before it on the same stream is still running: it sets up its
 * barriers and tensor memory and requests its first weight boxes (W_UK for
 * mla_absorb_q, W_UV and W_O for mla_out_proj / mla_combine_out_proj), then
 * waits for that kernel to complete before it reads any other input or writes
 * any output.  The caller's obligation: the weight operands of a call must not
 * be written by the kernel issued immediately before it on the stream.  Every
 * other input may come from that kernel.  Returns MLA_OK or
 * MLA_ERR_INVALID_ARG (null handle). */
MLA_API int mla_set_launch_overlap(mla_handle_t h, int enable);

/* Number of kernels this library has launched in this process (all handles,
 * all devices), for accounting of launches over a timed region. */
MLA_API uint64_t mla_launch_count(void);

/* Human-readable name of a status code (static storage). */
MLA_API const char* mla_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
