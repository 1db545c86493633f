// Small device helpers shared by the kernel translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace mla {

__device__ __forceinline__ float ld_f32(const float* p, long i) { return p[i]; }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16* p, long i) {
  return __bfloat162float(p[i]);
}

template <typename T> __device__ __forceinline__ T cvt_out(float x);
template <> __device__ __forceinline__ float cvt_out<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt_out<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel issued before it on the stream is
// still running.  grid_dep_wait() returns once that kernel has completed and
// its writes are visible (a no-op for a normal launch); grid_dep_trigger()
// lets the kernel issued after this one begin its launch.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Record the first device-side error of a handle (later ones are dropped).
__device__ __forceinline__ void report_error(int* err, int code) {
  if (err != nullptr && *reinterpret_cast<volatile int*>(err) == 0) atomicCAS(err, 0, code);
}

// e4m3 encode: round to nearest even, saturate finite values to +-448.
__device__ __forceinline__ uint8_t encode_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float decode_e4m3(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace mla
