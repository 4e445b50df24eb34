// FP8 E4M3 quantisation of bf16 activations.
//
// "DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA", section
// "Engenharia de inferencia e paralelismo de contexto: Ulysses, Ring Attention e
// FP8": activations quantised to FP8 E4M3. out = e4m3(x * inv_scale) with round to
// nearest even and saturation at +-448 (cvt.rn.satfinite), one byte per element.
// A grid-stride HBM stream: 16-byte loads of 8 bf16, 8-byte stores of 8 codes.
#pragma once
#include "common.cuh"

namespace dit3d {

// two floats -> two E4M3 codes, a in the low byte
__device__ __forceinline__ uint16_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

__device__ __forceinline__ uint32_t e4m3x4(uint32_t w0, uint32_t w1, float s) {
  const uint32_t lo = e4m3x2(bf16lo(w0) * s, bf16hi(w0) * s);
  const uint32_t hi = e4m3x2(bf16lo(w1) * s, bf16hi(w1) * s);
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(256)
quantize_e4m3_kernel(const uint4* __restrict__ x, uint2* __restrict__ out, int64_t n8, float inv_scale) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = ld_stream(x + i);
    out[i] = make_uint2(e4m3x4(v.x, v.y, inv_scale), e4m3x4(v.z, v.w, inv_scale));
  }
}

}  // namespace dit3d
