// CUDA-core kernels of libmla that serve every configuration:
//   * the paged row write (append and project-append), the split merge and
//     the RoPE of the query -- element-wise, HBM/latency bound at every size;
//   * dimension-generic absorb / decode / output projections, used for shapes
//     the tensor-core kernels are not specialised for (e.g. the tiny fp32
//     configuration with H=8, d_c=64, d_r=16).
//
// Method: DeepSeek V2 MLA page (snabindia.com), sections 2.1-2.3.
#include <algorithm>
#include <type_traits>

#include "device_common.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// paged row write (V2 page section 2.2 mla_rope, section 2.3 cache layout)
// ---------------------------------------------------------------------------

constexpr int kAppendWarps = 4;

// Stage n values of type T (a 16-byte-aligned row, n * sizeof(T) a multiple of
// 16) into shared memory as fp32, with 16-byte loads that are all issued
// before any is used (a row is one round trip, not one per element).
template <typename T>
__device__ __forceinline__ void stage_row(float* stage, const T* src, int n, int lane) {
  constexpr int kPer = 16 / static_cast<int>(sizeof(T));
  const int nv = n / kPer;
  const uint4* v = reinterpret_cast<const uint4*>(src);
  for (int j0 = lane; j0 < nv; j0 += 4 * 32) {
    uint4 buf[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j0 + 32 * u < nv) buf[u] = v[j0 + 32 * u];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (j0 + 32 * u < nv) {
        const T* e = reinterpret_cast<const T*>(&buf[u]);
#pragma unroll
        for (int q = 0; q < kPer; ++q) stage[(j0 + 32 * u) * kPer + q] = ld_f32(e, q);
      }
    }
  }
}

// Store n fp32 staged values as CT with 16-byte stores (n * sizeof(CT) a
// multiple of 16, dst 16-byte aligned).
template <typename CT>
__device__ __forceinline__ void store_row(CT* dst, const float* stage, int n, int lane) {
  constexpr int kPer = 16 / static_cast<int>(sizeof(CT));
  uint4* v = reinterpret_cast<uint4*>(dst);
  for (int j = lane; j < n / kPer; j += 32) {
    uint4 w;
    CT* e = reinterpret_cast<CT*>(&w);
#pragma unroll
    for (int q = 0; q < kPer; ++q) e[q] = cvt_out<CT>(stage[j * kPer + q]);
    v[j] = w;
  }
}

// Rotate the staged k_R (after c_KV in `stage`) in place at position p:
// pairs (i, i + d_r/2).  The first rotation factor of each lane comes in
// preloaded (r0, for i = lane).
__device__ __forceinline__ void rope_stage(const AppendArgs& a, float* stage, const float2* cs,
                                           float2 r0, int lane) {
  const int half = a.d_r / 2;
  for (int i = lane; i < half; i += 32) {
    const float x1 = stage[a.d_c + i], x2 = stage[a.d_c + half + i];
    const float2 r = i == lane ? r0 : cs[i];
    stage[a.d_c + i] = x1 * r.x - x2 * r.y;
    stage[a.d_c + half + i] = x2 * r.x + x1 * r.y;
  }
}

__device__ void write_row_warp_fp8(const AppendArgs& a, const float* stage, long slot, int lane) {
  const int D = a.d_c + a.d_r;
  float amax = 0.f;
  for (int i = lane; i < D; i += 32) amax = fmaxf(amax, fabsf(stage[i]));
  amax = warp_max(amax);
  uint8_t* row = reinterpret_cast<uint8_t*>(a.cache) + slot * D;
  if (amax == 0.f) {
    for (int i = lane; i < D; i += 32) row[i] = 0;
    if (lane == 0) a.cache_scale[slot] = 1.f;
    return;
  }
  const float inv = 448.f / amax;
  for (int i = lane; i < D; i += 32) row[i] = encode_e4m3(stage[i] * inv);
  if (lane == 0) a.cache_scale[slot] = amax / 448.f;
}

// One warp per token.  The first memory round trip loads the token's sequence,
// position and values together; the second the page-table entry and the RoPE
// factors, which depend on them; then the row is rotated, converted and written.  An out-of-range
// sequence, position or page is reported and the token skipped.
template <typename T, typename CT, bool kFp8, bool kProject>
__global__ void __launch_bounds__(kAppendWarps * 32) append_kernel(AppendArgs a) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.d_c + a.d_r;
  const int t = blockIdx.x * kAppendWarps + warp;
  grid_dep_wait();
  grid_dep_trigger();
  if (t >= a.num_tokens) return;
  const int b = a.seq_idx ? a.seq_idx[t] : t;
  const int p = a.pos[t];
  float* stage = smem + warp * D;
  if (kProject) {
    // c_kv = W_DKV x, k_raw = W_KR x: one output per warp iteration, lanes over d_model
    float* xs = smem + kAppendWarps * D + warp * a.d_model;
    const T* x = reinterpret_cast<const T*>(a.x) + static_cast<long>(t) * a.d_model;
    stage_row(xs, x, a.d_model, lane);
    __syncwarp();
    for (int j = 0; j < D; ++j) {
      const T* w = j < a.d_c ? reinterpret_cast<const T*>(a.w_dkv) + static_cast<long>(j) * a.d_model
                             : reinterpret_cast<const T*>(a.w_kr) +
                                   static_cast<long>(j - a.d_c) * a.d_model;
      float acc = 0.f;
      for (int i = lane; i < a.d_model; i += 32) acc += ld_f32(w, i) * xs[i];
      acc = warp_sum(acc);
      if (lane == 0) stage[j] = acc;
    }
  } else {
    stage_row(stage, reinterpret_cast<const T*>(a.c_kv) + static_cast<long>(t) * a.d_c, a.d_c, lane);
    stage_row(stage + a.d_c, reinterpret_cast<const T*>(a.k_r) + static_cast<long>(t) * a.d_r, a.d_r, lane);
  }
  const bool in_range = b >= 0 && b < a.batch && p >= 0 && p < a.max_position &&
                        p / a.block_size < a.max_blocks;
  const int page = in_range ? a.block_table[static_cast<long>(b) * a.max_blocks + p / a.block_size] : -1;
  const int half = a.d_r / 2;
  const float2* cs = a.rope_cs + static_cast<long>(in_range ? p : 0) * half;
  const float2 r0 = lane < half ? cs[lane] : make_float2(1.f, 0.f);
  if (page < 0 || page >= a.num_blocks) {
    if (lane == 0) report_error(a.err, MLA_ERR_BAD_INDEX);
    return;
  }
  const long slot = static_cast<long>(page) * a.block_size + p % a.block_size;
  __syncwarp();
  rope_stage(a, stage, cs, r0, lane);
  __syncwarp();
  if constexpr (kFp8) {
    write_row_warp_fp8(a, stage, slot, lane);
  } else {
    store_row(reinterpret_cast<CT*>(a.cache) + slot * D, stage, D, lane);
  }
}

cudaError_t launch_append(const AppendArgs& a, int act_dtype, int cache_dtype, bool project,
                          cudaStream_t s) {
  if (a.num_tokens == 0) return cudaSuccess;
  const int D = a.d_c + a.d_r;
  size_t smem = sizeof(float) * kAppendWarps * (D + (project ? a.d_model : 0));
  dim3 grid((a.num_tokens + kAppendWarps - 1) / kAppendWarps), block(kAppendWarps * 32);
  void (*k)(AppendArgs) = nullptr;
  if (act_dtype == MLA_FP32 && cache_dtype == MLA_FP32) {
    k = project ? append_kernel<float, float, false, true> : append_kernel<float, float, false, false>;
  } else if (act_dtype == MLA_BF16 && cache_dtype == MLA_BF16) {
    k = project ? append_kernel<__nv_bfloat16, __nv_bfloat16, false, true>
                : append_kernel<__nv_bfloat16, __nv_bfloat16, false, false>;
  } else if (act_dtype == MLA_BF16 && cache_dtype == MLA_FP8_E4M3) {
    k = project ? append_kernel<__nv_bfloat16, uint8_t, true, true>
                : append_kernel<__nv_bfloat16, uint8_t, true, false>;
  } else {
    return cudaErrorInvalidValue;
  }
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_kernel(a.overlap != 0, k, grid, block, smem, s, a);
  note_launches(1);
  return e;
}

// ---------------------------------------------------------------------------
// absorbed query, dimension-generic (V2 page section 2.3)
// ---------------------------------------------------------------------------

constexpr int kAbsorbThreads = 128;
constexpr int kAbsorbBatchChunk = 32;

// grid (H, ceil(d_c / 128) + 1): the last y-slice applies RoPE to q_pe.
template <typename T>
__global__ void __launch_bounds__(kAbsorbThreads) absorb_generic_kernel(AbsorbArgs a) {
  extern __shared__ float qs[];  // [kAbsorbBatchChunk][d_nope]
  const int h = blockIdx.x;
  const int D = a.d_c + a.d_r;
  const int nslices = (a.d_c + kAbsorbThreads - 1) / kAbsorbThreads;
  T* out = reinterpret_cast<T*>(a.q_lat);
  if (static_cast<int>(blockIdx.y) == nslices) {
    const int half = a.d_r / 2;
    const T* qpe = reinterpret_cast<const T*>(a.q_pe);
    for (int idx = threadIdx.x; idx < a.batch * half; idx += blockDim.x) {
      const int b = idx / half, i = idx % half;
      const int p = a.pos[b];
      if (p < 0 || p >= a.max_position) {
        report_error(a.err, MLA_ERR_BAD_INDEX);
        continue;
      }
      const float2 r = a.rope_cs[static_cast<long>(p) * half + i];
      const long base = (static_cast<long>(b) * a.num_heads + h) * a.d_r;
      const float x1 = ld_f32(qpe, base + i), x2 = ld_f32(qpe, base + half + i);
      const long ob = (static_cast<long>(b) * a.num_heads + h) * D + a.d_c;
      out[ob + i] = cvt_out<T>(x1 * r.x - x2 * r.y);
      out[ob + half + i] = cvt_out<T>(x2 * r.x + x1 * r.y);
    }
    return;
  }
  const int c = blockIdx.y * kAbsorbThreads + threadIdx.x;
  const T* qn = reinterpret_cast<const T*>(a.q_nope);
  const T* w = reinterpret_cast<const T*>(a.w_uk) + static_cast<long>(h) * a.d_nope * a.d_c;
  for (int b0 = 0; b0 < a.batch; b0 += kAbsorbBatchChunk) {
    const int nb = min(kAbsorbBatchChunk, a.batch - b0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nb * a.d_nope; idx += blockDim.x) {
      const int i = idx / a.d_nope, k = idx % a.d_nope;
      qs[i * a.d_nope + k] = ld_f32(qn, (static_cast<long>(b0 + i) * a.num_heads + h) * a.d_nope + k);
    }
    __syncthreads();
    if (c < a.d_c) {
      float acc[kAbsorbBatchChunk];
#pragma unroll
      for (int i = 0; i < kAbsorbBatchChunk; ++i) acc[i] = 0.f;
      for (int k = 0; k < a.d_nope; ++k) {
        const float wv = ld_f32(w, static_cast<long>(k) * a.d_c + c);
#pragma unroll
        for (int i = 0; i < kAbsorbBatchChunk; ++i) acc[i] += wv * qs[i * a.d_nope + k];
      }
      for (int i = 0; i < nb; ++i)
        out[(static_cast<long>(b0 + i) * a.num_heads + h) * D + c] = cvt_out<T>(acc[i]);
    }
  }
}

cudaError_t launch_absorb_generic(const AbsorbArgs& a, int act_dtype, cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  dim3 grid(a.num_heads, (a.d_c + kAbsorbThreads - 1) / kAbsorbThreads + 1);
  size_t smem = sizeof(float) * kAbsorbBatchChunk * a.d_nope;
  if (act_dtype == MLA_FP32) {
    absorb_generic_kernel<float><<<grid, kAbsorbThreads, smem, s>>>(a);
  } else {
    absorb_generic_kernel<__nv_bfloat16><<<grid, kAbsorbThreads, smem, s>>>(a);
  }
  note_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// split-KV decode, dimension-generic (CUDA cores)
// ---------------------------------------------------------------------------
// One CTA per (sequence b, split s, group of up to 16 heads).  Tiles of 32
// tokens are staged in shared memory as fp32 (fp8 rows are dequantised with
// their per-token scale); every warp owns two heads and runs the online
// softmax over the tile's 32 scores with warp-shuffle reductions.

constexpr int kGenThreads = 256;
constexpr int kGenTile = 32;
constexpr int kGenHeads = 16;
constexpr int kGenColsPerThread = 2;   // d_c <= 512

template <typename T, typename CT, bool kFp8>
__global__ void __launch_bounds__(kGenThreads) decode_generic_kernel(DecodeArgs a) {
  extern __shared__ float sm[];
  const int D = a.d_c + a.d_r;
  const int b = blockIdx.x, split = blockIdx.y, hg = blockIdx.z;
  const int h0 = hg * kGenHeads;
  const int nh = min(kGenHeads, a.num_heads - h0);
  float* qs = sm;                           // [kGenHeads][D]
  float* ks = qs + kGenHeads * D;           // [kGenTile][D]
  float* ps = ks + kGenTile * D;            // [kGenHeads][kGenTile]
  float* alpha_s = ps + kGenHeads * kGenTile;  // [kGenHeads]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int len = a.seq_lens[b];
  const int cap = a.max_blocks * a.block_size;
  if (len < 0 || len > cap) {          // never read past the page-table row
    if (tid == 0) report_error(a.err, MLA_ERR_BAD_INDEX);
    len = len < 0 ? 0 : cap;
  }
  // token range of this split: pages divided evenly over the splits
  const int pages = (len + a.block_size - 1) / a.block_size;
  const int pps = (pages + a.num_splits - 1) / a.num_splits;
  const int t_begin = min(len, split * pps * a.block_size);
  const int t_end = min(len, (split + 1) * pps * a.block_size);

  const T* q = reinterpret_cast<const T*>(a.q_lat);
  for (int idx = tid; idx < kGenHeads * D; idx += kGenThreads) {
    const int g = idx / D, d = idx % D;
    qs[idx] = g < nh ? ld_f32(q, (static_cast<long>(b) * a.num_heads + h0 + g) * D + d) : 0.f;
  }
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2*warp, 2*warp+1
  float acc[kGenHeads][kGenColsPerThread];
#pragma unroll
  for (int g = 0; g < kGenHeads; ++g)
#pragma unroll
    for (int j = 0; j < kGenColsPerThread; ++j) acc[g][j] = 0.f;

  const float sl2 = a.scale * 1.4426950408889634f;   // scores in log2 units
  for (int t0 = t_begin; t0 < t_end; t0 += kGenTile) {
    const int nt = min(kGenTile, t_end - t0);
    __syncthreads();
    // stage the tile
    for (int idx = tid; idx < kGenTile * D; idx += kGenThreads) {
      const int j = idx / D, d = idx % D;
      float v = 0.f;
      if (j < nt) {
        const int tok = t0 + j;
        const int page = a.block_table[static_cast<long>(b) * a.max_blocks + tok / a.block_size];
        if (page >= 0 && page < a.num_blocks) {
          const long slot = static_cast<long>(page) * a.block_size + tok % a.block_size;
          if constexpr (kFp8) {
            v = decode_e4m3(reinterpret_cast<const uint8_t*>(a.cache)[slot * D + d]) *
                a.cache_scale[slot];
          } else {
            v = ld_f32(reinterpret_cast<const CT*>(a.cache), slot * D + d);
          }
        } else if (d == 0) {
          report_error(a.err, MLA_ERR_BAD_INDEX);
        }
      }
      ks[idx] = v;
    }
    __syncthreads();
    // scores: warp w handles heads 2w, 2w+1; lane j handles token j
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int g = warp * 2 + hh;
      float s = -INFINITY;
      if (g < nh && lane < nt) {
        float dot = 0.f;
        const float* qg = qs + g * D;
        const float* kj = ks + lane * D;
        // lanes start at different columns so the 32 rows hit 32 banks
        for (int dd = 0; dd < D; ++dd) {
          int d = dd + lane;
          if (d >= D) d -= D;
          dot += qg[d] * kj[d];
        }
        s = dot * sl2;
      }
      const float m_tile = warp_max(s);
      const float m_new = fmaxf(m_run[hh], m_tile);
      const float p = (g < nh && lane < nt) ? exp2f(s - m_new) : 0.f;
      const float alpha = (m_run[hh] == -INFINITY) ? 0.f : exp2f(m_run[hh] - m_new);
      l_run[hh] = l_run[hh] * alpha + warp_sum(p);
      m_run[hh] = m_new;
      if (g < kGenHeads) {
        ps[g * kGenTile + lane] = p;
        if (lane == 0) alpha_s[g] = alpha;
      }
    }
    __syncthreads();
    // O[g][c] = alpha_g O[g][c] + sum_j p[g][j] row_j[c]
#pragma unroll
    for (int jc = 0; jc < kGenColsPerThread; ++jc) {
      const int c = tid + jc * kGenThreads;
      if (c < a.d_c) {
#pragma unroll
        for (int g = 0; g < kGenHeads; ++g) {
          float o = acc[g][jc] * alpha_s[g];
          for (int j = 0; j < nt; ++j) o += ps[g * kGenTile + j] * ks[j * D + c];
          acc[g][jc] = o;
        }
      }
    }
  }
  // write the normalised partial and its log-sum-exp
  __syncthreads();
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int g = warp * 2 + hh;
      if (g < kGenHeads) {
        ps[g] = l_run[hh];                       // reuse: l per head
        alpha_s[g] = m_run[hh];                  // reuse: m per head (log2 units)
      }
    }
  }
  __syncthreads();
  const long part = (static_cast<long>(b) * a.num_splits + split) * a.num_heads;
  // o_part[b][s][c/4][h][c%4] in fp32 (fp32 activations) or [c/8][h][c%8] in
  // fp16 (bf16 activations)
  const long obase = (static_cast<long>(b) * a.num_splits + split) * a.d_c * a.num_heads;
  float big = 0.f;
#pragma unroll
  for (int jc = 0; jc < kGenColsPerThread; ++jc) {
    const int c = tid + jc * kGenThreads;
    if (c < a.d_c) {
#pragma unroll
      for (int g = 0; g < kGenHeads; ++g) {
        if (g < nh) {
          const float l = ps[g];
          const float x = l > 0.f ? acc[g][jc] / l : 0.f;
          if constexpr (std::is_same<T, float>::value) {
            static_cast<float*>(a.o_part)[obase + ((c >> 2) * a.num_heads + h0 + g) * 4 + (c & 3)] = x;
          } else {
            big = fmaxf(big, fabsf(x));
            static_cast<__half*>(a.o_part)[obase + ((c >> 3) * a.num_heads + h0 + g) * 8 + (c & 7)] =
                __float2half_rn(x);
          }
        }
      }
    }
  }
  if (!(big <= 65504.f)) report_error(a.err, MLA_ERR_RANGE);
  if (tid < nh) {
    const float l = ps[tid];
    a.lse_part[part + h0 + tid] =
        l > 0.f ? (alpha_s[tid] + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
}

cudaError_t launch_decode_generic(const DecodeArgs& a, int act_dtype, int cache_dtype,
                                  cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  if (a.d_c > kGenThreads * kGenColsPerThread) return cudaErrorInvalidValue;
  const int D = a.d_c + a.d_r;
  dim3 grid(a.batch, a.num_splits, (a.num_heads + kGenHeads - 1) / kGenHeads);
  size_t smem = sizeof(float) * (kGenHeads * D + kGenTile * D + kGenHeads * kGenTile + kGenHeads);
  void (*k)(DecodeArgs) = nullptr;
  if (act_dtype == MLA_FP32 && cache_dtype == MLA_FP32) {
    k = decode_generic_kernel<float, float, false>;
  } else if (act_dtype == MLA_BF16 && cache_dtype == MLA_BF16) {
    k = decode_generic_kernel<__nv_bfloat16, __nv_bfloat16, false>;
  } else if (act_dtype == MLA_BF16 && cache_dtype == MLA_FP8_E4M3) {
    k = decode_generic_kernel<__nv_bfloat16, uint8_t, true>;
  } else {
    return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k<<<grid, kGenThreads, smem, s>>>(a);
  note_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// split merge by log-sum-exp
// ---------------------------------------------------------------------------

// One CTA per (sequence b, chunk of kCols latent columns); thread = head.
// Reads o_part[b][s][c/4][h][c%4] as float4 (coalesced over heads), merges the
// splits with weights exp(lse_s - lse), transposes through shared memory and
// writes o_lat[b][h][c] rows of kCols contiguous columns.  16 columns per CTA
// keep the register count low with many loads in flight; small batches take 4
// (four times the CTAs) so that the GPU stays full.
template <typename T, int kCols>
__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
  extern __shared__ float cw[];               // [num_splits][H] weights
  __shared__ float tile[kCols][129];          // [c][h], padded
  const int b = blockIdx.x, c0 = blockIdx.y * kCols;
  const int S = a.num_splits, H = a.num_heads;
  const int h = threadIdx.x;                  // blockDim.x == 128 >= H
  grid_dep_wait();
  grid_dep_trigger();
  if (h < H) {
    const float* lp = a.lse_part + static_cast<long>(b) * S * H + h;
    float m = -INFINITY;
#pragma unroll 4
    for (int s = 0; s < S; ++s) m = fmaxf(m, lp[static_cast<long>(s) * H]);
    float z = 0.f;
#pragma unroll 4
    for (int s = 0; s < S; ++s) {
      const float w = (m == -INFINITY) ? 0.f : __expf(lp[static_cast<long>(s) * H] - m);
      cw[s * H + h] = w;
      z += w;
    }
    const float inv_z = z > 0.f ? 1.f / z : 0.f;
    if (blockIdx.y == 0 && a.lse != nullptr)
      a.lse[static_cast<long>(b) * H + h] = z > 0.f ? m + __logf(z) : -INFINITY;
    // o_part: fp32 [b][s][c/4][h][4] with fp32 activations, fp16 [b][s][c/8][h][8]
    // with bf16 ones; a 4-column group c.. is then half (c/4) & 1 of 16 bytes
    constexpr bool kF32 = std::is_same<T, float>::value;
    const long obase = static_cast<long>(b) * S * a.d_c * H;
    float acc[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[c] = 0.f;
    const int nq = min(kCols, a.d_c - c0) / 4;        // d_c is a multiple of 4
#pragma unroll 2
    for (int s = 0; s < S; ++s) {
      const float w = cw[s * H + h];
      const long sbase = obase + static_cast<long>(s) * a.d_c * H;
#pragma unroll
      for (int g = 0; g < kCols / 4; ++g) {
        if (g < nq) {
          const int c = c0 + 4 * g;
          float4 v;
          if constexpr (kF32) {
            v = reinterpret_cast<const float4*>(static_cast<const float*>(a.o_part) + sbase)[(c >> 2) * H + h];
          } else {
            const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __half*>(a.o_part) + sbase +
                                                            ((c >> 3) * H + h) * 8 + (c & 7));
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
            v = make_float4(lo.x, lo.y, hi.x, hi.y);
          }
          acc[4 * g] += w * v.x;
          acc[4 * g + 1] += w * v.y;
          acc[4 * g + 2] += w * v.z;
          acc[4 * g + 3] += w * v.w;
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kCols; ++c) tile[c][h] = acc[c] * inv_z;
  }
  __syncthreads();
  // o_lat[b][hh][c0 + cc]: each group of kCols threads writes one head row
  T* out = reinterpret_cast<T*>(a.o_lat) + static_cast<long>(b) * H * a.d_c;
  const int cc = threadIdx.x % kCols;
  for (int hh = threadIdx.x / kCols; hh < H; hh += 128 / kCols)
    if (c0 + cc < a.d_c) out[static_cast<long>(hh) * a.d_c + c0 + cc] = cvt_out<T>(tile[cc][hh]);
}

template <int kCols>
cudaError_t launch_combine_cols(const CombineArgs& a, int act_dtype, cudaStream_t s) {
  dim3 grid(a.batch, (a.d_c + kCols - 1) / kCols);
  const size_t smem = sizeof(float) * a.num_splits * a.num_heads;
  void (*k)(CombineArgs) =
      act_dtype == MLA_FP32 ? combine_kernel<float, kCols> : combine_kernel<__nv_bfloat16, kCols>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_kernel(a.overlap != 0, k, grid, dim3(128), smem, s, a);
  note_launches(1);
  return e;
}

cudaError_t launch_combine(const CombineArgs& a, int act_dtype, int num_sms, cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  if (a.num_heads > 128) return cudaErrorInvalidValue;
  if (static_cast<long>(a.batch) * ((a.d_c + 15) / 16) >= 2L * num_sms)
    return launch_combine_cols<16>(a, act_dtype, s);
  return launch_combine_cols<4>(a, act_dtype, s);
}

// ---------------------------------------------------------------------------
// output side, dimension-generic: o = W_UV o_lat per head, y = W_O o
// ---------------------------------------------------------------------------

constexpr int kOpBatch = 32;

// grid (H, ceil(d_v / 8)); warp per output row v; lanes over d_c.
template <typename T>
__global__ void __launch_bounds__(256) uv_generic_kernel(OutProjArgs a) {
  extern __shared__ float ol[];   // [kOpBatch][d_c]
  const int h = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v = blockIdx.y * 8 + warp;
  const T* olat = reinterpret_cast<const T*>(a.o_lat);
  const T* w = reinterpret_cast<const T*>(a.w_uv) + (static_cast<long>(h) * a.d_v + v) * a.d_c;
  T* o = reinterpret_cast<T*>(a.o);
  for (int b0 = 0; b0 < a.batch; b0 += kOpBatch) {
    const int nb = min(kOpBatch, a.batch - b0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nb * a.d_c; idx += blockDim.x) {
      const int i = idx / a.d_c, c = idx % a.d_c;
      ol[idx] = ld_f32(olat, (static_cast<long>(b0 + i) * a.num_heads + h) * a.d_c + c);
    }
    __syncthreads();
    if (v < a.d_v) {
      float acc[kOpBatch];
#pragma unroll
      for (int i = 0; i < kOpBatch; ++i) acc[i] = 0.f;
      for (int c = lane; c < a.d_c; c += 32) {
        const float wv = ld_f32(w, c);
#pragma unroll
        for (int i = 0; i < kOpBatch; ++i) acc[i] += wv * ol[(i < nb ? i : 0) * a.d_c + c];
      }
#pragma unroll
      for (int i = 0; i < kOpBatch; ++i) {
        const float r = warp_sum(acc[i]);
        if (lane == 0 && i < nb)
          o[(static_cast<long>(b0 + i) * a.num_heads + h) * a.d_v + v] = cvt_out<T>(r);
      }
    }
  }
}

// Offset of W_O[m][k] (K columns) in the row-major or the tile-major layout.
__device__ __forceinline__ long w_o_offset(int m, int k, int K, bool tiled) {
  return tiled ? ((static_cast<long>(m >> 7) * (K >> 6) + (k >> 6)) << 13) + ((m & 127) << 6) + (k & 63)
               : static_cast<long>(m) * K + k;
}

// grid ceil(d_model / 8); warp per output row m; K = H*d_v streamed in chunks of 256.
template <typename T>
__global__ void __launch_bounds__(256) wo_generic_kernel(OutProjArgs a) {
  __shared__ float os[kOpBatch][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  const int K = a.num_heads * a.d_v;
  const T* o = reinterpret_cast<const T*>(a.o);
  const T* w = reinterpret_cast<const T*>(a.w_o);
  const bool tiled = a.w_o_tiled != 0;
  T* y = reinterpret_cast<T*>(a.y);
  for (int b0 = 0; b0 < a.batch; b0 += kOpBatch) {
    const int nb = min(kOpBatch, a.batch - b0);
    float acc[kOpBatch];
#pragma unroll
    for (int i = 0; i < kOpBatch; ++i) acc[i] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 256) {
      __syncthreads();
      // os[b][e*32 + l] = o[b][k0 + 8*l + e]
      for (int idx = threadIdx.x; idx < kOpBatch * 256; idx += blockDim.x) {
        const int i = idx / 256, r = idx % 256;
        const int kk = k0 + r;
        const int l = r / 8, e = r % 8;
        os[i][e * 32 + l] = (i < nb && kk < K) ? ld_f32(o, static_cast<long>(b0 + i) * K + kk) : 0.f;
      }
      __syncthreads();
      if (m < a.d_model) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int kk = k0 + 8 * lane + e;
          const float wv = kk < K ? ld_f32(w, w_o_offset(m, kk, K, tiled)) : 0.f;
#pragma unroll
          for (int i = 0; i < kOpBatch; ++i) acc[i] += wv * os[i][e * 32 + lane];
        }
      }
    }
    if (m < a.d_model) {
#pragma unroll
      for (int i = 0; i < kOpBatch; ++i) {
        const float r = warp_sum(acc[i]);
        if (lane == 0 && i < nb) y[static_cast<long>(b0 + i) * a.d_model + m] = cvt_out<T>(r);
      }
    }
  }
}

// One thread per 16-byte unit of the tile-major output, in its order (the
// reads are 16-byte pieces of 128-byte row segments).
template <int kElem>
__global__ void __launch_bounds__(256) pack_tiles_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         long rows, long cols) {
  constexpr int kPerUnit = 16 / kElem;                // elements per 16-byte unit
  constexpr int kUnitsPerRow = 64 / kPerUnit;         // units per 64-column tile row
  const long units = rows * cols / kPerUnit;
  const long ctiles = cols / 64;
  for (long u = blockIdx.x * 256L + threadIdx.x; u < units; u += gridDim.x * 256L) {
    const long e = u % kUnitsPerRow, r = (u / kUnitsPerRow) % 128, tile = u / (kUnitsPerRow * 128);
    const long rt = tile / ctiles, ct = tile % ctiles;
    dst[u] = src[((rt * 128 + r) * cols + ct * 64) / kPerUnit + e];
  }
}

cudaError_t launch_pack_tiles(const void* src, void* dst, long rows, long cols, int elem_bytes,
                              cudaStream_t s) {
  if (rows % 128 != 0 || cols % 64 != 0 || (elem_bytes != 2 && elem_bytes != 4)) return cudaErrorInvalidValue;
  if (rows == 0 || cols == 0) return cudaSuccess;
  const long units = rows * cols * elem_bytes / 16;
  const dim3 grid(static_cast<unsigned>(std::min<long>((units + 255) / 256, 4096)));
  if (elem_bytes == 2)
    pack_tiles_kernel<2><<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, cols);
  else
    pack_tiles_kernel<4><<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, cols);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_out_proj_generic(const OutProjArgs& a, int act_dtype, cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  dim3 g1(a.num_heads, (a.d_v + 7) / 8);
  size_t smem1 = sizeof(float) * kOpBatch * a.d_c;
  dim3 g2((a.d_model + 7) / 8);
  if (act_dtype == MLA_FP32) {
    cudaError_t e = cudaFuncSetAttribute(uv_generic_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    uv_generic_kernel<float><<<g1, 256, smem1, s>>>(a);
    wo_generic_kernel<float><<<g2, 256, 0, s>>>(a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(uv_generic_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    uv_generic_kernel<__nv_bfloat16><<<g1, 256, smem1, s>>>(a);
    wo_generic_kernel<__nv_bfloat16><<<g2, 256, 0, s>>>(a);
  }
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace mla
