// Host side of libmla's C ABI (include/mla.h): handle life cycle, argument
// validation, workspace sizing and kernel dispatch.  No call on the decode
// path allocates, frees or synchronises.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "internal.h"
#include "umma_kernels.h"

using namespace mla;

namespace {

std::atomic<uint64_t> g_launches{0};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t act_bytes(int dt) { return dt == MLA_FP32 ? 4 : 2; }
size_t cache_elem_bytes(int dt) { return dt == MLA_FP32 ? 4 : (dt == MLA_BF16 ? 2 : 1); }

int map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  return MLA_ERR_LAUNCH;
}

// The handle belongs to the device that was current at mla_create.
bool on_handle_device(const mla_ctx* h) {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess && d == h->device;
}

int resolve_splits(const mla_ctx* h, int32_t batch, int32_t max_seq_len, int32_t num_splits) {
  if (num_splits > 0) return num_splits;
  return mla_decode_auto_splits(const_cast<mla_ctx*>(h), batch, max_seq_len);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bytes of one split partial value: fp16 with bf16 activations, fp32 with fp32.
size_t part_elem_bytes(const mla_ctx* h) { return h->cfg.act_dtype == MLA_FP32 ? 4 : 2; }

// Bytes of o_part for `parts` (sequence, split, head) rows, rounded to 256.
size_t opart_bytes(const mla_ctx* h, size_t parts) {
  return round_up(parts * h->cfg.d_c * part_elem_bytes(h), 256);
}

size_t decode_ws_bytes(const mla_ctx* h, int32_t batch, int32_t splits) {
  const size_t parts = static_cast<size_t>(batch) * splits * h->cfg.num_heads;
  return opart_bytes(h, parts) + round_up(parts * sizeof(float), 256);
}

}  // namespace

namespace mla {
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace mla

extern "C" {

uint64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* mla_status_string(int s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_LAUNCH: return "MLA_ERR_LAUNCH";
    case MLA_ERR_BAD_INDEX: return "MLA_ERR_BAD_INDEX";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_RANGE: return "MLA_ERR_RANGE";
    default: return "MLA_ERR_UNKNOWN";
  }
}

int mla_create(const mla_config_t* cfg, mla_handle_t* out) {
  if (cfg == nullptr || out == nullptr) return MLA_ERR_INVALID_ARG;
  const mla_config_t c = *cfg;
  if (c.num_heads <= 0 || c.d_c <= 0 || c.d_r <= 0 || c.d_nope <= 0 || c.d_v <= 0 ||
      c.d_model <= 0 || c.block_size <= 0 || c.max_position <= 0)
    return MLA_ERR_INVALID_ARG;
  if (c.d_r % 2 != 0) return MLA_ERR_INVALID_ARG;
  if (!(c.softmax_scale > 0.f) || !std::isfinite(c.softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!(c.rope_base > 1.f) || !std::isfinite(c.rope_base)) return MLA_ERR_INVALID_ARG;
  const bool dt_ok = (c.act_dtype == MLA_FP32 && c.cache_dtype == MLA_FP32) ||
                     (c.act_dtype == MLA_BF16 && c.cache_dtype == MLA_BF16) ||
                     (c.act_dtype == MLA_BF16 && c.cache_dtype == MLA_FP8_E4M3);
  if (!dt_ok) return MLA_ERR_UNSUPPORTED;
  // rows and per-token vectors must stay 16-byte aligned
  const size_t ab = act_bytes(c.act_dtype);
  if ((c.d_c * ab) % 16 || (c.d_r * ab) % 16 || (c.d_nope * ab) % 16 || (c.d_v * ab) % 16 ||
      (c.d_model * ab) % 16 || ((c.d_c + c.d_r) * cache_elem_bytes(c.cache_dtype)) % 16)
    return MLA_ERR_UNSUPPORTED;
  if (c.d_c > 512) return MLA_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (prop.major != 10) return MLA_ERR_UNSUPPORTED;

  // RoPE table: cos/sin(pos * theta_i), theta_i = base^(-2i/d_r), in double on the host
  const int half = c.d_r / 2;
  std::vector<float2> table(static_cast<size_t>(c.max_position) * half);
  for (int i = 0; i < half; ++i) {
    const double theta = std::pow(static_cast<double>(c.rope_base), -2.0 * i / c.d_r);
    for (int p = 0; p < c.max_position; ++p) {
      const double ang = static_cast<double>(p) * theta;
      table[static_cast<size_t>(p) * half + i] =
          make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
    }
  }
  mla_ctx* h = new (std::nothrow) mla_ctx();
  if (h == nullptr) return MLA_ERR_CUDA;
  h->cfg = c;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->cc_major = prop.major;
  h->cc_minor = prop.minor;
  h->wait_limit = kDefaultWaitLimit;
  h->overlap = 0;
  h->w_o_tiled = 0;
  if (cudaMalloc(&h->rope_cs, table.size() * sizeof(float2)) != cudaSuccess ||
      cudaMalloc(&h->err, 256) != cudaSuccess ||
      cudaMemcpy(h->rope_cs, table.data(), table.size() * sizeof(float2),
                 cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(h->err, 0, 256) != cudaSuccess) {
    if (h->rope_cs) cudaFree(h->rope_cs);
    if (h->err) cudaFree(h->err);
    delete h;
    return MLA_ERR_CUDA;
  }
  *out = h;
  return MLA_OK;
}

int mla_destroy(mla_handle_t h) {
  if (h == nullptr) return MLA_OK;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != h->device) cudaSetDevice(h->device);
  cudaFree(h->rope_cs);
  cudaFree(h->err);
  if (dev != h->device && dev >= 0) cudaSetDevice(dev);
  delete h;
  return MLA_OK;
}

size_t mla_cache_row_bytes(mla_handle_t h) {
  if (h == nullptr) return 0;
  return static_cast<size_t>(h->cfg.d_c + h->cfg.d_r) * cache_elem_bytes(h->cfg.cache_dtype);
}

size_t mla_cache_scale_bytes(mla_handle_t h) {
  if (h == nullptr) return 0;
  return h->cfg.cache_dtype == MLA_FP8_E4M3 ? sizeof(float) : 0;
}

static int append_common(mla_handle_t h, const void* c_kv, const void* k_r, const void* x,
                         const void* w_dkv, const void* w_kr, const int32_t* seq_idx,
                         const int32_t* pos, int32_t num_tokens, const int32_t* block_table,
                         int32_t max_blocks, int32_t batch, void* cache, float* cache_scale,
                         int32_t num_blocks, cudaStream_t stream, bool project) {
  if (h == nullptr || pos == nullptr || block_table == nullptr || cache == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (num_tokens < 0 || batch <= 0 || max_blocks <= 0 || num_blocks <= 0)
    return MLA_ERR_INVALID_ARG;
  if (seq_idx == nullptr && num_tokens > batch) return MLA_ERR_INVALID_ARG;
  const bool fp8 = h->cfg.cache_dtype == MLA_FP8_E4M3;
  if (fp8 != (cache_scale != nullptr)) return MLA_ERR_INVALID_ARG;
  if (project) {
    if (x == nullptr || w_dkv == nullptr || w_kr == nullptr) return MLA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_dkv, 16) || !aligned(w_kr, 16)) return MLA_ERR_ALIGNMENT;
  } else {
    if (c_kv == nullptr || k_r == nullptr) return MLA_ERR_INVALID_ARG;
    if (!aligned(c_kv, 16) || !aligned(k_r, 16)) return MLA_ERR_ALIGNMENT;
  }
  if (!aligned(cache, 16) || !aligned(pos, 4) || !aligned(block_table, 4) ||
      (seq_idx && !aligned(seq_idx, 4)) || (cache_scale && !aligned(cache_scale, 4)))
    return MLA_ERR_ALIGNMENT;
  if (!on_handle_device(h)) return MLA_ERR_INVALID_ARG;
  if (num_tokens == 0) return MLA_OK;
  AppendArgs a{};
  a.c_kv = c_kv;
  a.k_r = k_r;
  a.x = x;
  a.w_dkv = w_dkv;
  a.w_kr = w_kr;
  a.seq_idx = seq_idx;
  a.pos = pos;
  a.num_tokens = num_tokens;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.batch = batch;
  a.cache = cache;
  a.cache_scale = cache_scale;
  a.num_blocks = num_blocks;
  a.rope_cs = h->rope_cs;
  a.err = h->err;
  a.d_c = h->cfg.d_c;
  a.d_r = h->cfg.d_r;
  a.d_model = h->cfg.d_model;
  a.block_size = h->cfg.block_size;
  a.max_position = h->cfg.max_position;
  a.overlap = h->overlap;
  return map_cuda(launch_append(a, h->cfg.act_dtype, h->cfg.cache_dtype, project, stream));
}

int mla_cache_append(mla_handle_t h, const void* c_kv, const void* k_r, const int32_t* seq_idx,
                     const int32_t* pos, int32_t num_tokens, const int32_t* block_table,
                     int32_t max_blocks_per_seq, int32_t batch, void* cache, float* cache_scale,
                     int32_t num_blocks, cudaStream_t stream) {
  return append_common(h, c_kv, k_r, nullptr, nullptr, nullptr, seq_idx, pos, num_tokens,
                       block_table, max_blocks_per_seq, batch, cache, cache_scale, num_blocks,
                       stream, false);
}

int mla_kv_project_append(mla_handle_t h, const void* x, const void* w_dkv, const void* w_kr,
                          const int32_t* seq_idx, const int32_t* pos, int32_t num_tokens,
                          const int32_t* block_table, int32_t max_blocks_per_seq, int32_t batch,
                          void* cache, float* cache_scale, int32_t num_blocks,
                          cudaStream_t stream) {
  return append_common(h, nullptr, nullptr, x, w_dkv, w_kr, seq_idx, pos, num_tokens, block_table,
                       max_blocks_per_seq, batch, cache, cache_scale, num_blocks, stream, true);
}

int mla_absorb_q(mla_handle_t h, const void* q_nope, const void* q_pe, const int32_t* pos,
                 const void* w_uk, int32_t batch, void* q_lat, cudaStream_t stream) {
  if (h == nullptr || q_nope == nullptr || q_pe == nullptr || pos == nullptr || w_uk == nullptr ||
      q_lat == nullptr || batch < 0)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_nope, 16) || !aligned(q_pe, 16) || !aligned(w_uk, 16) || !aligned(q_lat, 16) ||
      !aligned(pos, 4))
    return MLA_ERR_ALIGNMENT;
  if (!on_handle_device(h)) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  AbsorbArgs a{};
  a.q_nope = q_nope;
  a.q_pe = q_pe;
  a.pos = pos;
  a.w_uk = w_uk;
  a.q_lat = q_lat;
  a.rope_cs = h->rope_cs;
  a.err = h->err;
  a.batch = batch;
  a.num_heads = h->cfg.num_heads;
  a.d_nope = h->cfg.d_nope;
  a.d_c = h->cfg.d_c;
  a.d_r = h->cfg.d_r;
  a.max_position = h->cfg.max_position;
  if (umma_absorb_supported(h, batch)) return map_cuda(launch_absorb_umma(h, a, stream));
  return map_cuda(launch_absorb_generic(a, h->cfg.act_dtype, stream));
}

int32_t mla_decode_auto_splits(mla_handle_t h, int32_t batch, int32_t max_seq_len) {
  if (h == nullptr || batch <= 0 || max_seq_len <= 0) return 1;
  const int pages = (max_seq_len + h->cfg.block_size - 1) / h->cfg.block_size;
  // the tensor-core decode runs one CTA pair per (sequence, split)
  const int pairs = h->num_sms / 2;
  int s = pairs / batch;
  if (s < 1) s = 1;
  if (s > pages) s = pages;
  return s;
}

size_t mla_decode_workspace_bytes(mla_handle_t h, int32_t batch, int32_t num_splits,
                                  int32_t max_seq_len) {
  if (h == nullptr || batch <= 0 || num_splits < 0) return 0;
  return decode_ws_bytes(h, batch, resolve_splits(h, batch, max_seq_len, num_splits));
}

static int decode_check(mla_handle_t h, int32_t batch, int32_t max_seq_len, int32_t num_splits,
                        const void* workspace, size_t ws_bytes, int* splits) {
  if (h == nullptr || batch < 0 || num_splits < 0 || max_seq_len < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const int s = resolve_splits(h, batch, max_seq_len, num_splits);
  if (workspace == nullptr || ws_bytes < decode_ws_bytes(h, batch, s)) return MLA_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return MLA_ERR_ALIGNMENT;
  if (!on_handle_device(h)) return MLA_ERR_INVALID_ARG;
  *splits = s;
  return MLA_OK;
}

int mla_decode_partial(mla_handle_t h, const void* q_lat, const void* cache,
                       const float* cache_scale, int32_t num_blocks, const int32_t* block_table,
                       int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                       int32_t max_seq_len, int32_t num_splits, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  int S = 0;
  int st = decode_check(h, batch, max_seq_len, num_splits, workspace, workspace_bytes, &S);
  if (st != MLA_OK || batch == 0) return st;
  if (q_lat == nullptr || cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      max_blocks_per_seq <= 0 || num_blocks <= 0)
    return MLA_ERR_INVALID_ARG;
  const bool fp8 = h->cfg.cache_dtype == MLA_FP8_E4M3;
  if (fp8 != (cache_scale != nullptr)) return MLA_ERR_INVALID_ARG;
  if (static_cast<long>(max_seq_len) > static_cast<long>(max_blocks_per_seq) * h->cfg.block_size)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_lat, 16) || !aligned(cache, 16) || !aligned(block_table, 4) ||
      !aligned(seq_lens, 4) || (cache_scale && !aligned(cache_scale, 16)))
    return MLA_ERR_ALIGNMENT;
  DecodeArgs a{};
  a.q_lat = q_lat;
  a.cache = cache;
  a.cache_scale = cache_scale;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  const size_t parts = static_cast<size_t>(batch) * S * h->cfg.num_heads;
  a.o_part = workspace;
  a.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + opart_bytes(h, parts));
  a.err = h->err;
  a.batch = batch;
  a.num_heads = h->cfg.num_heads;
  a.d_c = h->cfg.d_c;
  a.d_r = h->cfg.d_r;
  a.block_size = h->cfg.block_size;
  a.max_blocks = max_blocks_per_seq;
  a.num_splits = S;
  a.num_blocks = num_blocks;
  a.max_seq_len = max_seq_len;
  a.scale = h->cfg.softmax_scale;
  a.wait_limit = h->wait_limit;
  if (umma_decode_supported(h)) return map_cuda(launch_decode_umma(h, a, stream));
  return map_cuda(launch_decode_generic(a, h->cfg.act_dtype, h->cfg.cache_dtype, stream));
}

int mla_decode_combine(mla_handle_t h, int32_t batch, int32_t max_seq_len, int32_t num_splits,
                       const void* workspace, size_t workspace_bytes, void* o_lat, float* lse,
                       cudaStream_t stream) {
  int S = 0;
  int st = decode_check(h, batch, max_seq_len, num_splits, workspace, workspace_bytes, &S);
  if (st != MLA_OK || batch == 0) return st;
  if (o_lat == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned(o_lat, 16) || (lse && !aligned(lse, 4))) return MLA_ERR_ALIGNMENT;
  CombineArgs a{};
  const size_t parts = static_cast<size_t>(batch) * S * h->cfg.num_heads;
  a.o_part = workspace;
  a.lse_part = reinterpret_cast<const float*>(static_cast<const char*>(workspace) + opart_bytes(h, parts));
  a.o_lat = o_lat;
  a.lse = lse;
  a.batch = batch;
  a.num_heads = h->cfg.num_heads;
  a.d_c = h->cfg.d_c;
  a.num_splits = S;
  a.overlap = h->overlap;
  return map_cuda(launch_combine(a, h->cfg.act_dtype, h->num_sms, stream));
}

int mla_decode(mla_handle_t h, const void* q_lat, const void* cache, const float* cache_scale,
               int32_t num_blocks, const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
               int32_t batch, int32_t max_seq_len, int32_t num_splits, void* workspace,
               size_t workspace_bytes, void* o_lat, float* lse, cudaStream_t stream) {
  if (o_lat == nullptr && batch > 0) return MLA_ERR_INVALID_ARG;
  int st = mla_decode_partial(h, q_lat, cache, cache_scale, num_blocks, block_table,
                              max_blocks_per_seq,
                              seq_lens, batch, max_seq_len, num_splits, workspace,
                              workspace_bytes, stream);
  if (st != MLA_OK) return st;
  return mla_decode_combine(h, batch, max_seq_len, num_splits, workspace, workspace_bytes, o_lat,
                            lse, stream);
}

size_t mla_out_proj_workspace_bytes(mla_handle_t h, int32_t batch) {
  if (h == nullptr || batch <= 0) return 0;
  return round_up(static_cast<size_t>(batch) * h->cfg.num_heads * h->cfg.d_v *
                      act_bytes(h->cfg.act_dtype),
                  256) +
         umma_out_proj_extra_workspace(h, batch);
}

int mla_out_proj(mla_handle_t h, const void* o_lat, const void* w_uv, const void* w_o,
                 int32_t batch, void* workspace, size_t workspace_bytes, void* y, void* o_out,
                 cudaStream_t stream) {
  if (h == nullptr || o_lat == nullptr || w_uv == nullptr || w_o == nullptr || y == nullptr ||
      batch < 0)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (workspace == nullptr || workspace_bytes < mla_out_proj_workspace_bytes(h, batch))
    return MLA_ERR_WORKSPACE;
  if (!aligned(o_lat, 16) || !aligned(w_uv, 16) || !aligned(w_o, 16) || !aligned(y, 16) ||
      !aligned(workspace, 16) || (o_out && !aligned(o_out, 16)))
    return MLA_ERR_ALIGNMENT;
  if (!on_handle_device(h)) return MLA_ERR_INVALID_ARG;
  OutProjArgs a{};
  a.o_lat = o_lat;
  a.w_uv = w_uv;
  a.w_o = w_o;
  a.o = o_out ? o_out : workspace;
  a.y = y;
  a.batch = batch;
  a.num_heads = h->cfg.num_heads;
  a.d_c = h->cfg.d_c;
  a.d_v = h->cfg.d_v;
  a.d_model = h->cfg.d_model;
  a.w_o_tiled = h->w_o_tiled;
  if (umma_out_proj_supported(h, batch)) {
    void* extra = static_cast<char*>(workspace) +
                  round_up(static_cast<size_t>(batch) * h->cfg.num_heads * h->cfg.d_v *
                               act_bytes(h->cfg.act_dtype),
                           256);
    return map_cuda(launch_out_proj_umma(h, a, extra, stream));
  }
  return map_cuda(launch_out_proj_generic(a, h->cfg.act_dtype, stream));
}

int mla_combine_out_proj(mla_handle_t h, int32_t batch, int32_t max_seq_len, int32_t num_splits,
                         const void* workspace, size_t workspace_bytes, const void* w_uv,
                         const void* w_o, void* op_workspace, size_t op_workspace_bytes,
                         void* o_lat, float* lse, void* y, void* o_out, cudaStream_t stream) {
  int S = 0;
  int st = decode_check(h, batch, max_seq_len, num_splits, workspace, workspace_bytes, &S);
  if (st != MLA_OK || batch == 0) return st;
  if (o_lat == nullptr || w_uv == nullptr || w_o == nullptr || y == nullptr) return MLA_ERR_INVALID_ARG;
  if (op_workspace == nullptr || op_workspace_bytes < mla_out_proj_workspace_bytes(h, batch))
    return MLA_ERR_WORKSPACE;
  if (!aligned(o_lat, 16) || (lse && !aligned(lse, 4)) || !aligned(w_uv, 16) || !aligned(w_o, 16) ||
      !aligned(y, 16) || !aligned(op_workspace, 16) || (o_out && !aligned(o_out, 16)))
    return MLA_ERR_ALIGNMENT;
  if (!umma_combine_out_proj_supported(h, batch, S)) {
    // the merge and the output projection as two calls
    st = mla_decode_combine(h, batch, max_seq_len, num_splits, workspace, workspace_bytes, o_lat, lse, stream);
    if (st != MLA_OK) return st;
    return mla_out_proj(h, o_lat, w_uv, w_o, batch, op_workspace, op_workspace_bytes, y, o_out, stream);
  }
  const size_t parts = static_cast<size_t>(batch) * S * h->cfg.num_heads;
  OutProjArgs a{};
  a.o_lat = o_lat;
  a.w_uv = w_uv;
  a.w_o = w_o;
  a.o = o_out ? o_out : op_workspace;
  a.y = y;
  a.batch = batch;
  a.num_heads = h->cfg.num_heads;
  a.d_c = h->cfg.d_c;
  a.d_v = h->cfg.d_v;
  a.d_model = h->cfg.d_model;
  a.comb_opart = static_cast<const __half*>(workspace);
  a.comb_lse = reinterpret_cast<const float*>(static_cast<const char*>(workspace) + opart_bytes(h, parts));
  a.comb_splits = S;
  a.comb_lse_out = lse;
  a.w_o_tiled = h->w_o_tiled;
  void* extra = static_cast<char*>(op_workspace) +
                round_up(static_cast<size_t>(batch) * h->cfg.num_heads * h->cfg.d_v * act_bytes(h->cfg.act_dtype), 256);
  return map_cuda(launch_out_proj_umma(h, a, extra, stream));
}

int mla_last_device_error(mla_handle_t h, cudaStream_t stream) {
  if (h == nullptr) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (v != 0 && cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  return v;
}

int mla_set_wait_limit(mla_handle_t h, uint32_t limit) {
  if (h == nullptr) return MLA_ERR_INVALID_ARG;
  h->wait_limit = limit == 0 ? kDefaultWaitLimit : limit;
  return MLA_OK;
}

static bool w_o_tileable(const mla_ctx* h) {
  return h->cfg.d_model % 128 == 0 && (static_cast<long>(h->cfg.num_heads) * h->cfg.d_v) % 64 == 0;
}

int mla_pack_w_o(mla_handle_t h, const void* w_o, void* w_o_tiled, cudaStream_t stream) {
  if (h == nullptr || w_o == nullptr || w_o_tiled == nullptr || w_o == w_o_tiled) return MLA_ERR_INVALID_ARG;
  if (!w_o_tileable(h)) return MLA_ERR_UNSUPPORTED;
  if (!aligned(w_o, 16) || !aligned(w_o_tiled, 16)) return MLA_ERR_ALIGNMENT;
  if (!on_handle_device(h)) return MLA_ERR_INVALID_ARG;
  return map_cuda(launch_pack_tiles(w_o, w_o_tiled, h->cfg.d_model,
                                    static_cast<long>(h->cfg.num_heads) * h->cfg.d_v,
                                    static_cast<int>(act_bytes(h->cfg.act_dtype)), stream));
}

int mla_set_w_o_layout(mla_handle_t h, int tiled) {
  if (h == nullptr) return MLA_ERR_INVALID_ARG;
  if (tiled && !w_o_tileable(h)) return MLA_ERR_UNSUPPORTED;
  h->w_o_tiled = tiled ? 1 : 0;
  return MLA_OK;
}

int mla_set_launch_overlap(mla_handle_t h, int enable) {
  if (h == nullptr) return MLA_ERR_INVALID_ARG;
  h->overlap = enable != 0 ? 1 : 0;
  return MLA_OK;
}

}  // extern "C"
