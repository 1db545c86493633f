// tcgen05 / TMEM / TMA kernels of libmla (sm_100a) and their launchers.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>

#include "decode_umma.cuh"
#include "gemm_umma.cuh"
#include "umma_kernels.h"

namespace mla {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Rows of `chunks` x 64 bf16 columns read as a 3-D tensor (64 columns, rows,
// column chunk), so that one box of box_rows x chunks lands in shared memory
// chunk-major: [chunk][row][128 bytes], 128-byte swizzled -- the UMMA K-major
// (and, for V, MN-major) operand layout.
cudaError_t make_map_3d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t row_bytes,
                        uint64_t chunks, uint64_t chunk_bytes, uint32_t box_rows, uint32_t box_chunks) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {64, rows, chunks};
  const cuuint64_t strides[2] = {row_bytes, chunk_bytes};
  const cuuint32_t box[3] = {64, box_rows, box_chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_map_rows_chunked(CUtensorMap* map, const void* base, uint64_t rows,
                                  uint64_t row_bytes, uint32_t chunks, uint32_t box_rows,
                                  uint32_t box_chunks) {
  return make_map_3d(map, base, rows, row_bytes, chunks, 128, box_rows, box_chunks);
}

}  // namespace

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------

bool umma_decode_supported(const mla_ctx* h) {
  const mla_config_t& c = h->cfg;
  return h->cc_major == 10 && c.num_heads == dec::kH && c.d_c == dec::kDc &&
         c.d_c + c.d_r == dec::kD && c.block_size == dec::kTok && c.act_dtype == MLA_BF16 &&
         (c.cache_dtype == MLA_BF16 || c.cache_dtype == MLA_FP8_E4M3) && encode_fn() != nullptr;
}

namespace {

template <bool kFp8>
cudaError_t launch_decode_kernel(const CUtensorMap& kmap, const CUtensorMap& vmap, const CUtensorMap& qmap,
                                 const DecodeArgs& a, unsigned ctas, bool overlap, cudaStream_t s) {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dec::decode_umma_kernel<kFp8>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_kernel(overlap, dec::decode_umma_kernel<kFp8>, dim3(ctas), dim3(dec::threads<kFp8>()),
                       dec::kSmemBytes, s, kmap, vmap, qmap, a);
}

}  // namespace

cudaError_t launch_decode_umma(const mla_ctx* h, const DecodeArgs& a, cudaStream_t s) {
  const bool fp8 = h->cfg.cache_dtype == MLA_FP8_E4M3;
  CUtensorMap kmap, vmap, qmap;
  std::memset(&kmap, 0, sizeof(kmap));
  std::memset(&vmap, 0, sizeof(vmap));
  const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * dec::kTok;
  cudaError_t e = cudaSuccess;
  if (fp8) {
    // pages and their scales are fetched by untiled bulk copies: 16-byte aligned sources
    if ((reinterpret_cast<uintptr_t>(a.cache) | reinterpret_cast<uintptr_t>(a.cache_scale)) & 15)
      return cudaErrorMisalignedAddress;
  } else {
    e = make_map_rows_chunked(&kmap, a.cache, rows, dec::kD * 2, dec::kKBoxes, dec::kTok, dec::kKBoxes);
    if (e != cudaSuccess) return e;
    e = make_map_rows_chunked(&vmap, a.cache, rows, dec::kD * 2, dec::kKBoxes, dec::kTok, dec::kVBoxes);
    if (e != cudaSuccess) return e;
  }
  // absorbed queries as [B*H rows][576 columns], half of a sequence's heads per box
  e = make_map_rows_chunked(&qmap, a.q_lat, static_cast<uint64_t>(a.batch) * dec::kH, dec::kD * 2,
                            dec::kKBoxes, 64, dec::kKBoxes);
  if (e != cudaSuccess) return e;
  const long ctas = 2L * a.batch * a.num_splits;
  if (ctas > 0x7fffffffL) return cudaErrorInvalidValue;
  const bool ov = h->overlap != 0;
  e = fp8 ? launch_decode_kernel<true>(kmap, vmap, qmap, a, static_cast<unsigned>(ctas), ov, s)
          : launch_decode_kernel<false>(kmap, vmap, qmap, a, static_cast<unsigned>(ctas), ov, s);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

// ---------------------------------------------------------------------------
// projections: weight-streaming tcgen05 GEMM
// ---------------------------------------------------------------------------

namespace {

constexpr int kOProjSplits = 3;      // K split of W_O when stream-K does not apply

// How W_O is split over the GPU: stream-K, one CTA per SM, each CTA taking an
// equal run of the (M tile, box of kcs K chunks) stages.
struct WoPlan {
  int kcs;      // K chunks per stage (box depth)
  int stages;
  int box;      // stages per M tile
  int units;    // M tiles x box
  int g;        // CTAs
  int slots;    // partial tiles per CTA (M tiles one run can touch)
  bool stream_k;
};

int tmem_block_cols(int n) { return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : 256)); }

int padded_n(int batch) { return (batch + 15) / 16 * 16; }

size_t gemm_smem_bytes(const gemm::Params& p) {
  const size_t xres = p.x_chunks > 0 ? static_cast<size_t>(p.n) * gemm::kKc * 2 * p.x_chunks : 0;
  const size_t stage = gemm::kM * gemm::kKc * 2 * p.kcs + (p.x_chunks > 0 ? 0 : p.n * gemm::kKc * 2 * p.kcs);
  // merge weights [n][S] and 1/z [n] when the merge runs in the kernel
  const size_t wts = p.comb_splits > 0 ? static_cast<size_t>(p.n) * (p.comb_splits + 1) * 4 : 0;
  return xres + static_cast<size_t>(p.stages) * stage + 8 * (2 * p.stages + 4) + 16 + wts + 1024;
}

// Raise a kernel's dynamic shared-memory limit once (per process) to the
// largest size requested so far; launches then pay no driver call.
// (keyed by the kernel's address: every instantiation of a kernel template has
// the same function type).
template <typename K>
cudaError_t ensure_smem_limit(K kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<const void*, size_t> current;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = current[reinterpret_cast<const void*>(kernel)];
  if (bytes <= cur) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(bytes));
  if (e == cudaSuccess) cur = bytes;
  return e;
}

// TMEM columns a CTA of the GEMM allocates (the kernel's own rule): one block of
// 32/64/128/256 columns per M tile, rounded up to a power of two.
int gemm_tmem_cols(const gemm::Params& p) {
  const int ncpt = p.n <= 32 ? 32 : (p.n <= 64 ? 64 : (p.n <= 128 ? 128 : 256));
  int cols = 32;
  while (cols < ncpt * p.mt_per_cta) cols <<= 1;
  return cols;
}

template <bool kAMn, gemm::Epi kEpi>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tx, gemm::Params p, dim3 grid,
                        bool overlap, cudaStream_t s) {
  if (gemm_tmem_cols(p) > 512) return cudaErrorInvalidValue;     // TMEM holds 512 columns
  // as many stages as requested that fit in shared memory (larger batches: fewer)
  while (p.stages > 2 && gemm_smem_bytes(p) > 232448) --p.stages;
  const size_t smem = gemm_smem_bytes(p);
  if (smem > 232448) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(gemm::gemm_wt_kernel<kAMn, kEpi>, smem);
  if (e != cudaSuccess) return e;
  e = launch_kernel(overlap, gemm::gemm_wt_kernel<kAMn, kEpi>, grid, dim3(256), smem, s, ta, tx, p);
  note_launches(1);
  return e;
}

bool v2_bf16(const mla_ctx* h) {
  const mla_config_t& c = h->cfg;
  return h->cc_major == 10 && c.act_dtype == MLA_BF16 && c.num_heads == 128 && c.d_c == 512 &&
         c.d_r == 64 && c.d_nope == 128 && c.d_v == 128 && c.d_model % 128 == 0 &&
         encode_fn() != nullptr;
}

}  // namespace

bool umma_absorb_supported(const mla_ctx* h, int batch) {
  return v2_bf16(h) && batch >= 1 && batch <= 256;
}

cudaError_t launch_absorb_umma(const mla_ctx* h, const AbsorbArgs& a, cudaStream_t s) {
  const int H = a.num_heads, n = padded_n(a.batch);
  CUtensorMap ta, tx;
  // W_UK [H*d_nope rows (k)][d_c columns (c)], read MN-major: a box is 128 rows of K
  // by two 64-column slices of one 128-wide M tile
  cudaError_t e = make_map_rows_chunked(&ta, a.w_uk, static_cast<uint64_t>(H) * a.d_nope, a.d_c * 2,
                                        a.d_c / gemm::kKc, 2 * gemm::kKc, 2);
  if (e != cudaSuccess) return e;
  // q_nope as [B rows][H*d_nope columns]
  e = make_map_rows_chunked(&tx, a.q_nope, a.batch, static_cast<uint64_t>(H) * a.d_nope * 2,
                            H * a.d_nope / gemm::kKc, n, 2);
  if (e != cudaSuccess) return e;
  gemm::Params p{};
  p.n = n;
  p.batch = a.batch;
  p.k_chunks = a.d_nope / gemm::kKc;
  p.k_split = 1;
  p.m_per_group = a.d_c;
  // two M tiles per CTA, two CTAs per head: small CTAs (the head's q_nope slice
  // loaded once and kept, two 32 KB weight boxes) of which several share an SM
  p.mt_per_cta = 2;
  p.kcs = 2;
  p.x_chunks = a.d_nope / gemm::kKc;
  p.a_row_group = a.d_nope;
  p.x_col_group = a.d_nope;
  p.stages = 2;
  p.out = a.q_lat;
  p.out_ld = static_cast<long>(H) * (a.d_c + a.d_r);
  p.out_group = a.d_c + a.d_r;
  p.q_pe = static_cast<const __nv_bfloat16*>(a.q_pe);
  p.pos = a.pos;
  p.rope_cs = a.rope_cs;
  p.num_heads = H;
  p.d_c = a.d_c;
  p.d_r = a.d_r;
  p.max_position = a.max_position;
  p.err = a.err;
  p.wait_limit = h->wait_limit;
  const int ctas_per_head = (a.d_c / gemm::kM) / p.mt_per_cta;
  return launch_gemm<true, gemm::Epi::kAbsorb>(ta, tx, p, dim3(H * ctas_per_head, 1), h->overlap != 0, s);
}

bool umma_out_proj_supported(const mla_ctx* h, int batch) {
  return v2_bf16(h) && batch >= 1 && batch <= 256;
}

namespace {

WoPlan wo_plan(const mla_ctx* h, int batch) {
  const int n = padded_n(batch);
  WoPlan w{};
  auto fits = [&](int kcs, int stages) {
    return static_cast<long>(stages) * (gemm::kM + n) * gemm::kKc * 2 * kcs + 8 * (2 * stages + 4) + 16 + 1024 <=
           232448;
  };
  // (measured) the row-major weight streams fastest as 64 KB boxes in two stages,
  // the tile-major one as 48 KB boxes in three; larger batches fall back to 32 KB
  // boxes in as many stages as fit
  if (h->w_o_tiled && fits(3, 3)) {
    w.kcs = 3;
    w.stages = 3;
  } else if (fits(4, 2)) {
    w.kcs = 4;
    w.stages = 2;
  } else {
    w.kcs = 2;
    w.stages = 5;
  }
  const int k_chunks = h->cfg.num_heads * h->cfg.d_v / gemm::kKc;
  const int m_tiles = h->cfg.d_model / gemm::kM;
  w.box = (k_chunks + w.kcs - 1) / w.kcs;
  w.units = m_tiles * w.box;
  w.g = std::max(1, std::min(h->num_sms, w.units));
  const int run = (w.units + w.g - 1) / w.g;
  w.slots = std::min((run + w.box - 1) / w.box + 1, m_tiles);
  int cols = 32;
  while (cols < tmem_block_cols(n) * w.slots) cols <<= 1;
  // (the reduce kernel locates partials in 32-bit arithmetic)
  w.stream_k = cols <= 512 && static_cast<long>(w.units) * w.g < (1L << 31);
  return w;
}

}  // namespace

bool umma_combine_out_proj_supported(const mla_ctx* h, int batch, int num_splits) {
  if (!umma_out_proj_supported(h, batch) || num_splits < 1 || h->cfg.num_heads > 128) return false;
  // the W_UV kernel keeps the merged slice resident: X, two 64 KB weight boxes
  // and the merge weights must fit in shared memory
  const long n = padded_n(batch);
  const long bytes = n * h->cfg.d_c * 2 + 2L * gemm::kM * gemm::kKc * 2 * 4 + n * (num_splits + 1) * 4 + 4096;
  return bytes <= 232448;
}

size_t umma_out_proj_extra_workspace(const mla_ctx* h, int batch) {
  if (!umma_out_proj_supported(h, batch)) return 0;
  const WoPlan w = wo_plan(h, batch);
  const size_t ks = static_cast<size_t>(kOProjSplits) * batch * h->cfg.d_model * sizeof(float);
  const size_t sk = static_cast<size_t>(w.g) * w.slots * batch * gemm::kM * sizeof(float);
  return (w.stream_k ? sk : ks) + 256;
}

cudaError_t launch_out_proj_umma(const mla_ctx* h, const OutProjArgs& a, void* extra,
                                 cudaStream_t s) {
  const int H = a.num_heads, n = padded_n(a.batch);
  const long kdim = static_cast<long>(H) * a.d_v;
  // o[b][h][v] = W_UV[h] o_lat[b][h]: one CTA per head; while the head's o_lat
  // slice fits next to two 64 KB weight boxes it is loaded once and kept -- or,
  // with the merge fused, built in the kernel from the split partials
  {
    const bool xres = static_cast<long>(n) * a.d_c * 2 + 2L * gemm::kM * gemm::kKc * 2 * 4 + 4096 <= 232448;
    if (a.comb_splits > 0 && !umma_combine_out_proj_supported(h, a.batch, a.comb_splits))
      return cudaErrorNotSupported;
    const int kcs = xres ? 4 : 2;
    CUtensorMap ta, tx;
    cudaError_t e = make_map_rows_chunked(&ta, a.w_uv, static_cast<uint64_t>(H) * a.d_v, a.d_c * 2,
                                          a.d_c / gemm::kKc, gemm::kM, kcs);
    if (e != cudaSuccess) return e;
    e = make_map_rows_chunked(&tx, a.o_lat, a.batch, static_cast<uint64_t>(H) * a.d_c * 2,
                              H * a.d_c / gemm::kKc, n, xres ? a.d_c / gemm::kKc : kcs);
    if (e != cudaSuccess) return e;
    gemm::Params p{};
    p.n = n;
    p.batch = a.batch;
    p.k_chunks = a.d_c / gemm::kKc;
    p.k_split = 1;
    p.m_per_group = a.d_v;
    p.mt_per_cta = 1;
    p.kcs = kcs;
    p.x_chunks = xres ? a.d_c / gemm::kKc : 0;
    p.a_row_group = a.d_v;
    p.x_col_group = a.d_c;
    p.stages = xres ? 2 : 4;
    p.out = a.o;
    p.out_ld = kdim;
    p.out_group = a.d_v;
    p.num_heads = H;
    p.d_c = a.d_c;
    if (a.comb_splits > 0) {
      p.comb_opart = a.comb_opart;
      p.comb_lse = a.comb_lse;
      p.comb_splits = a.comb_splits;
      p.comb_olat = static_cast<__nv_bfloat16*>(const_cast<void*>(a.o_lat));
      p.comb_lse_out = a.comb_lse_out;
    }
    p.err = h->err;
    p.wait_limit = h->wait_limit;
    e = launch_gemm<false, gemm::Epi::kStoreBf16T>(ta, tx, p, dim3(H, 1), h->overlap != 0, s);
    if (e != cudaSuccess) return e;
  }
  // fp32 partials of y: stream-K slots, or one [b][m] block per K split
  float* part = static_cast<float*>(extra);
  const WoPlan w = wo_plan(h, a.batch);
  {
    CUtensorMap ta, tx;
    // row-major: (64 columns, row, chunk); tile-major: (64 columns, row of the
    // tile, tile * k_chunks + chunk), a 16 KB tile per 64-column chunk
    cudaError_t e =
        a.w_o_tiled ? make_map_3d(&ta, a.w_o, gemm::kM, 128, static_cast<uint64_t>(a.d_model / gemm::kM) * (kdim / gemm::kKc),
                                  gemm::kM * 128, gemm::kM, w.kcs)
                    : make_map_rows_chunked(&ta, a.w_o, a.d_model, kdim * 2, kdim / gemm::kKc, gemm::kM, w.kcs);
    if (e != cudaSuccess) return e;
    e = make_map_rows_chunked(&tx, a.o, a.batch, kdim * 2, kdim / gemm::kKc, n, w.kcs);
    if (e != cudaSuccess) return e;
    gemm::Params p{};
    p.n = n;
    p.batch = a.batch;
    p.k_chunks = static_cast<int>(kdim / gemm::kKc);
    p.m_per_group = a.d_model;
    p.kcs = w.kcs;
    p.a_row_group = 0;
    p.x_col_group = 0;
    p.stages = w.stages;
    p.a_tiled = a.w_o_tiled;
    p.out = part;
    p.out_group = 0;
    p.err = h->err;
    p.wait_limit = h->wait_limit;
    dim3 grid;
    if (w.stream_k) {
      // partial[c * slots + t][b][r] for the t-th M tile of CTA c
      p.k_split = 1;
      p.mt_per_cta = w.slots;
      p.sk_units = w.units;
      p.sk_box = w.box;
      p.out_ld = gemm::kM;
      p.out_split = static_cast<long>(a.batch) * gemm::kM;
      grid = dim3(w.g, 1);
    } else {
      // partial[s][b][m] = sum over split s's K of W_O[m][k] o[b][k]
      p.k_split = kOProjSplits;
      p.mt_per_cta = 1;
      p.out_ld = a.d_model;
      p.out_split = static_cast<long>(a.batch) * a.d_model;
      grid = dim3(a.d_model / gemm::kM, kOProjSplits);
    }
    e = launch_gemm<false, gemm::Epi::kPartialF32>(ta, tx, p, grid, h->overlap != 0, s);
    if (e != cudaSuccess) return e;
  }
  const long count = static_cast<long>(a.batch) * a.d_model;
  const dim3 rgrid(static_cast<unsigned>(std::min<long>((count + 255) / 256, 1184)));
  cudaError_t e;
  if (w.stream_k) {
    e = launch_kernel(h->overlap != 0, gemm::reduce_stream_k_kernel,
                      dim3(a.d_model / gemm::kM, (a.batch + 1) / 2), dim3(256), 0, s, part,
                      static_cast<__nv_bfloat16*>(a.y), a.batch, a.d_model, w.units, w.box, w.g, w.slots);
  } else {
    e = launch_kernel(h->overlap != 0, gemm::reduce_splits_kernel, rgrid, dim3(256), 0, s, part,
                      static_cast<__nv_bfloat16*>(a.y), kOProjSplits, count);
  }
  note_launches(1);
  return e;
}

}  // namespace mla
