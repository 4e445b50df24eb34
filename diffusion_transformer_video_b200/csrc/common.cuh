// Shared device helpers of libdit3d: bf16 packing and the device error word.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace dit3d {

// Error bits a kernel raises instead of trapping; read and cleared by dit_check_device().
enum : uint32_t { kDevErrTimeout = 1u };
// Defined here: the library is one translation unit (dit3d_abi.cu includes every kernel).
__device__ uint32_t g_device_error = 0;

// bf16x2 word <-> two fp32 (element 0 in the low half, as in memory)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 128-bit global accesses: streaming (read once / write once) and read-only cached.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ uint4 ld_cached(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream(void* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}

}  // namespace dit3d
