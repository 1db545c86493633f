// Dispatch hooks of the tcgen05 (5th-generation tensor core) kernels.  Each
// *_supported() says whether the tensor-core kernel covers the handle's
// configuration; the host falls back to nothing else than the
// dimension-generic CUDA-core kernels for shapes it does not cover.
#pragma once

#include "internal.h"

namespace mla {

bool umma_decode_supported(const mla_ctx* h);
cudaError_t launch_decode_umma(const mla_ctx* h, const DecodeArgs& a, cudaStream_t s);

bool umma_absorb_supported(const mla_ctx* h, int batch);
cudaError_t launch_absorb_umma(const mla_ctx* h, const AbsorbArgs& a, cudaStream_t s);

bool umma_out_proj_supported(const mla_ctx* h, int batch);
// Whether the split merge can run inside the W_UV kernel (launch_out_proj_umma
// with comb_splits > 0) for this batch and split count.
bool umma_combine_out_proj_supported(const mla_ctx* h, int batch, int num_splits);
size_t umma_out_proj_extra_workspace(const mla_ctx* h, int batch);
cudaError_t launch_out_proj_umma(const mla_ctx* h, const OutProjArgs& a, void* extra,
                                 cudaStream_t s);

}  // namespace mla
