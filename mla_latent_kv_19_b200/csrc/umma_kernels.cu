// tcgen05 / TMEM / TMA kernels of libmla (sm_100a).
#include "umma_kernels.h"

namespace mla {

bool umma_decode_supported(const mla_ctx*) { return false; }
cudaError_t launch_decode_umma(const mla_ctx*, const DecodeArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}
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
