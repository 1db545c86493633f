// mla_decode_noalloc: the split-KV decode for callers that cannot allocate
// device memory.
//
// mla_decode needs a caller-provided workspace for its split partials.  Some
// callers have no way to provide one: a plugin living inside a host framework
// that owns all device memory through its own pool and forbids side
// allocations, or a latency-critical loop in which a cudaMalloc would
// implicitly synchronise the device.  This entry point takes the partials from
// a fixed array compiled into the library instead, so it allocates nothing.
//
// The array lives in device memory for as long as the library is loaded, on
// every GPU that loads it (kScratchBytes each).  Host code only sees a
// stand-in for it, so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current.
#include <mutex>

#include "internal.h"

namespace {

// Largest workspace this entry point can serve: 32 MiB, enough for 128 heads x
// 512 latent columns x 127 (sequence, split) partials, e.g. batch 32 with 3
// splits, batch 4 with 31 splits or batch 2 with 63 splits.
constexpr size_t kScratchBytes = size_t{32} << 20;
constexpr int kMaxDevices = 64;

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

namespace {

// Device address of g_decode_scratch on the current device (looked up on the
// first call per device and cached).
int scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" MLA_API int mla_decode_noalloc(mla_handle_t h, const void* q_lat, const void* cache,
                                          const float* cache_scale, int32_t num_blocks,
                                          const int32_t* block_table, int32_t max_blocks_per_seq,
                                          const int32_t* seq_lens, int32_t batch,
                                          int32_t max_seq_len, int32_t num_splits, void* o_lat,
                                          float* lse, cudaStream_t stream) {
  if (h == nullptr || batch < 0 || num_splits < 0 || max_seq_len < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const size_t need = mla_decode_workspace_bytes(h, batch, num_splits, max_seq_len);
  if (need == 0 || need > kScratchBytes) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_on_current_device(&scratch);
  if (st != MLA_OK) return st;
  // The partial kernel writes every slot the merge kernel reads, so leftovers
  // of an earlier call need no clearing.
  return mla_decode(h, q_lat, cache, cache_scale, num_blocks, block_table, max_blocks_per_seq,
                    seq_lens, batch, max_seq_len, num_splits, scratch, kScratchBytes, o_lat, lse,
                    stream);
}
