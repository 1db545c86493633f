// tcgen05 / TMEM / TMA kernels of libmla (sm_100a) and their launchers.
#include <cudaTypedefs.h>

#include <mutex>

#include "decode_umma.cuh"
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

// 2-D bf16 tensor map, 128-byte swizzle, box = box_cols x box_rows.
cudaError_t make_map_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                          uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------

bool umma_decode_supported(const mla_ctx* h) {
  const mla_config_t& c = h->cfg;
  return h->cc_major == 10 && c.num_heads == dec::kH && c.d_c == dec::kDc &&
         c.d_c + c.d_r == dec::kD && c.block_size == dec::kTok && c.act_dtype == MLA_BF16 &&
         c.cache_dtype == MLA_BF16 && encode_fn() != nullptr;
}

cudaError_t launch_decode_umma(const mla_ctx* h, const DecodeArgs& a, cudaStream_t s) {
  CUtensorMap map;
  cudaError_t e = make_map_bf16(&map, a.cache, dec::kD, static_cast<uint64_t>(a.num_blocks) * dec::kTok,
                                dec::kD * 2, 64, 64);
  if (e != cudaSuccess) return e;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dec::decode_umma_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const long ctas = 2L * a.batch * a.num_splits;
  if (ctas > 0x7fffffffL) return cudaErrorInvalidValue;
  dec::decode_umma_kernel<<<dim3(static_cast<unsigned>(ctas)), 256, dec::kSmemBytes, s>>>(map, a);
  note_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// absorb and output projection: not yet on tensor cores
// ---------------------------------------------------------------------------

bool umma_absorb_supported(const mla_ctx*, int) { return false; }
cudaError_t launch_absorb_umma(const mla_ctx*, const AbsorbArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool umma_out_proj_supported(const mla_ctx*, int) { return false; }
size_t umma_out_proj_extra_workspace(const mla_ctx*, int) { return 0; }
cudaError_t launch_out_proj_umma(const mla_ctx*, const OutProjArgs&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace mla
