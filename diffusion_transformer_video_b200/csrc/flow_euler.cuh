// One explicit Euler step of the rectified-flow ODE with per-frame local times.
//
// "DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA", section "Flow
// Matching e Rectified Flow": the path from noise to data is the straight line
// x_t = (1 - t) x_0 + t x_1, the network predicts its velocity u, and frames come out
// of 10-25 steps of a standard ODE sampler such as Euler. "Flowception: Temporally
// Expansive Flow Matching for Video Generation", section "Metodologia", interleaved
// time schedule: every frame carries its own local time t_i, so each frame advances
// by its own step dt_i = t_i' - t_i.
//
//   out[r, :] = x[r, :] + dt[r / rows_per_group] * u[r, :]
//
// A CTA per token row streams x and u once and writes out once (6 bytes per
// element): an HBM stream. fp32 FMA, one bf16 rounding; a zero step returns x's
// bits unchanged (frames whose local time has reached 1 stay put exactly).
#pragma once
#include "adaln.cuh"
#include "common.cuh"

namespace dit3d {

__device__ __forceinline__ uint32_t euler_pair(uint32_t xw, uint32_t uw, float dt) {
  if (dt == 0.f) return xw;
  return pack_bf16x2(fmaf(dt, bf16lo(uw), bf16lo(xw)), fmaf(dt, bf16hi(uw), bf16hi(xw)));
}

template <int NV>
__global__ void __launch_bounds__(kRowThreads)
flow_euler_kernel(const __nv_bfloat16* x, const __nv_bfloat16* u, const float* __restrict__ dt,
                  __nv_bfloat16* out, int32_t D, int64_t rows_per_group) {
  const int64_t row = blockIdx.x;
  const int nchunk = D >> 3;
  const int64_t off = row * static_cast<int64_t>(D) * 2;
  const char* xr = reinterpret_cast<const char*>(x) + off;
  const char* ur = reinterpret_cast<const char*>(u) + off;
  char* orow = reinterpret_cast<char*>(out) + off;
  const float h = __ldg(dt + row / rows_per_group);
  uint4 xv[NV], uv[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nchunk) {
      xv[k] = ld_stream(xr + c * 16);
      uv[k] = ld_stream(ur + c * 16);
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nchunk)
      st_stream(orow + c * 16, make_uint4(euler_pair(xv[k].x, uv[k].x, h), euler_pair(xv[k].y, uv[k].y, h),
                                          euler_pair(xv[k].z, uv[k].z, h), euler_pair(xv[k].w, uv[k].w, h)));
  }
}

__global__ void __launch_bounds__(kRowThreads)
flow_euler_wide_kernel(const __nv_bfloat16* x, const __nv_bfloat16* u, const float* __restrict__ dt,
                       __nv_bfloat16* out, int32_t D, int64_t rows_per_group) {
  const int64_t row = blockIdx.x;
  const int nchunk = D >> 3;
  const int64_t off = row * static_cast<int64_t>(D) * 2;
  const float h = __ldg(dt + row / rows_per_group);
  for (int c = threadIdx.x; c < nchunk; c += kRowThreads) {
    const uint4 xv = ld_stream(reinterpret_cast<const char*>(x) + off + c * 16);
    const uint4 uv = ld_stream(reinterpret_cast<const char*>(u) + off + c * 16);
    st_stream(reinterpret_cast<char*>(out) + off + c * 16,
              make_uint4(euler_pair(xv.x, uv.x, h), euler_pair(xv.y, uv.y, h),
                         euler_pair(xv.z, uv.z, h), euler_pair(xv.w, uv.w, h)));
  }
}

}  // namespace dit3d
