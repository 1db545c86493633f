// Internal declarations of libmla shared by the host C-ABI layer and the
// kernel translation units.  Not part of the public interface (include/mla.h).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/mla.h"

struct mla_ctx {
  mla_config_t cfg;
  int device;
  int num_sms;
  int cc_major, cc_minor;
  float2* rope_cs;     // device [max_position][d_r/2] (cos, sin)
  int* err;            // device error word (0 = no error)
  uint32_t wait_limit; // bounded-wait iteration limit (0 = default)
  int overlap;         // launch kernels as programmatic dependents of the previous one
  int w_o_tiled;       // W_O arguments are tile-major (mla_pack_w_o)
};

namespace mla {

constexpr uint32_t kDefaultWaitLimit = 1u << 26;

// Counts kernel launches (host side); read through mla_launch_count().
void note_launches(int n);

// Launch `k`; with `overlap`, as a programmatic dependent launch: the kernel may
// begin while the previous kernel of the stream is still running, so it must
// call grid_dep_wait() before it touches anything that kernel reads or writes.
template <typename... P, typename... A>
cudaError_t launch_kernel(bool overlap, void (*k)(P...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, std::forward<A>(args)...);
}

// Work description shared by the append kernels.
struct AppendArgs {
  const void* c_kv;     // [T, d_c]   (append)
  const void* k_r;      // [T, d_r]   (append)
  const void* x;        // [T, d_model] (project-append)
  const void* w_dkv;    // [d_c, d_model]
  const void* w_kr;     // [d_r, d_model]
  const int32_t* seq_idx;
  const int32_t* pos;
  int32_t num_tokens;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t batch;
  void* cache;
  float* cache_scale;
  int32_t num_blocks;
  const float2* rope_cs;
  int* err;
  int32_t d_c, d_r, d_model, block_size, max_position;
  int32_t overlap;      // programmatic dependent launch
};

struct AbsorbArgs {
  const void* q_nope;   // [B, H, d_nope]
  const void* q_pe;     // [B, H, d_r]
  const int32_t* pos;   // [B]
  const void* w_uk;     // [H, d_nope, d_c]
  void* q_lat;          // [B, H, d_c + d_r]
  const float2* rope_cs;
  int* err;
  int32_t batch, num_heads, d_nope, d_c, d_r, max_position;
};

struct DecodeArgs {
  const void* q_lat;          // [B, H, D]
  const void* cache;          // [num_blocks, block_size, D]
  const float* cache_scale;   // [num_blocks, block_size] (fp8)
  const int32_t* block_table; // [B, max_blocks]
  const int32_t* seq_lens;    // [B]
  // split partials: bf16 activations: fp16 [B, S, d_c/8, H, 8]; fp32
  // activations: fp32 [B, S, d_c/4, H, 4] (16 bytes per head and column group)
  void* o_part;
  float* lse_part;            // [B, S, H]
  int* err;
  int32_t batch, num_heads, d_c, d_r, block_size, max_blocks, num_splits, num_blocks;
  int32_t max_seq_len;
  float scale;
  uint32_t wait_limit;
};

struct CombineArgs {
  const void* o_part;         // as DecodeArgs::o_part
  const float* lse_part;
  void* o_lat;                // [B, H, d_c] act dtype
  float* lse;                 // [B, H] or null
  int32_t batch, num_heads, d_c, num_splits;
  int32_t overlap;            // programmatic dependent launch
};

struct OutProjArgs {
  const void* o_lat;   // [B, H, d_c]
  const void* w_uv;    // [H, d_v, d_c]
  const void* w_o;     // [d_model, H*d_v]
  void* o;             // [B, H, d_v]
  void* y;             // [B, d_model]
  int32_t batch, num_heads, d_c, d_v, d_model;
  // merge fused into W_UV: o_lat (then an output) is built from the split-KV
  // partials; comb_splits = 0 turns this off
  const __half* comb_opart;  // fp16 [B, S, d_c/8, H, 8]
  const float* comb_lse;     // [B, S, H]
  int32_t comb_splits;
  float* comb_lse_out;       // [B, H] or null
  int32_t w_o_tiled;         // w_o is tile-major: [d_model/128][H*d_v/64][128][64]
};

// Launchers (return cudaGetLastError() of their launches).
cudaError_t launch_append(const AppendArgs& a, int act_dtype, int cache_dtype, bool project,
                          cudaStream_t s);
cudaError_t launch_absorb_generic(const AbsorbArgs& a, int act_dtype, cudaStream_t s);
cudaError_t launch_decode_generic(const DecodeArgs& a, int act_dtype, int cache_dtype,
                                  cudaStream_t s);
cudaError_t launch_combine(const CombineArgs& a, int act_dtype, int num_sms, cudaStream_t s);
cudaError_t launch_out_proj_generic(const OutProjArgs& a, int act_dtype, cudaStream_t s);
// dst[r/128][c/64][r%128][c%64] = src[r][c] for a rows x cols matrix of
// elem_bytes-wide elements (rows % 128 == 0, cols % 64 == 0).
cudaError_t launch_pack_tiles(const void* src, void* dst, long rows, long cols, int elem_bytes,
                              cudaStream_t s);

}  // namespace mla
