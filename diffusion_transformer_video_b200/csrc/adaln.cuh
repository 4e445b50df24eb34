// adaLN-Zero memory-bound kernels: LayerNorm modulation and the gated residual.
//
// "DiT, Flow Matching e 3D Attention", section "A ruptura da U-Net":
//   x' = x + alpha * SelfAttn(gamma * LN(x) + beta); alpha starts at zero so the
//   block is the identity.
//
// One CTA of kRowThreads threads (64 for the modulation at d_model <= 3072) owns one
// token row. Each thread keeps its NV 16-byte chunks of the row in registers, so x is read from HBM exactly once and
// the output written once (4 bytes of traffic per element for the modulation,
// 6 for the residual). Mean and variance are two warp-shuffle + shared-memory
// reductions over the register-resident row (variance around the mean, fp32).
#pragma once
#include "common.cuh"

namespace dit3d {

constexpr int kRowThreads = 128;

// Sum over a block of WARPS warps (warp shuffles, then one shared-memory exchange).
template <int WARPS>
__device__ __forceinline__ float block_sum_w(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float t = red[0];
#pragma unroll
  for (int w = 1; w < WARPS; ++w) t += red[w];
  return t;
}
__device__ __forceinline__ float block_sum_128(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

// EARLY: gamma and beta are loaded with x, before the reductions (their latency hidden
// behind x's), at the price of registers. Measured on B200 at d_model 3072: with one
// parameter group per frame (1560 rows) the early form moves 5.3 TB/s against 4.3;
// with a few large groups (a group per sample) the late form is faster (5.5 against
// 5.2 TB/s), its parameter reads hitting in L1.
// TH threads per row (TH / 32 warps). The launch uses 64 for the late form at
// d_model <= 3072: the row's registers then limit an SM to 14 resident rows instead of
// 10 with 128 threads, measured +10 % inside the 720P step (4.99 against 4.49 TB/s).
// At d_model <= 3072 the early form is replaced by adaln_modulate_staged_kernel (with
// 64 threads its 119 registers would leave 8 rows per SM).
template <int NV, bool EARLY, int TH = kRowThreads>
__global__ void __launch_bounds__(TH)
adaln_modulate_kernel(const __nv_bfloat16* x, const __nv_bfloat16* __restrict__ gamma,
                      const __nv_bfloat16* __restrict__ beta, __nv_bfloat16* out, int32_t D,
                      int64_t rows_per_group, float eps, float scale_offset) {
  __shared__ float red[2][TH / 32];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nchunk = D >> 3;
  const char* xr = reinterpret_cast<const char*>(x) + row * static_cast<int64_t>(D) * 2;
  const int64_t g = row / rows_per_group;
  const char* gr = reinterpret_cast<const char*>(gamma) + g * static_cast<int64_t>(D) * 2;
  const char* br = reinterpret_cast<const char*>(beta) + g * static_cast<int64_t>(D) * 2;
  uint4 v[NV], gv_e[EARLY ? NV : 1], bv_e[EARLY ? NV : 1];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = tid + k * TH;
    v[k] = (c < nchunk) ? ld_stream(xr + c * 16) : make_uint4(0, 0, 0, 0);
    if constexpr (EARLY) {
      if (c < nchunk) {
        gv_e[k] = ld_cached(gr + c * 16);
        bv_e[k] = ld_cached(br + c * 16);
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) s += bf16lo(w[e]) + bf16hi(w[e]);
  }
  const float mean = block_sum_w<TH / 32>(s, red[0]) / static_cast<float>(D);
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    if (tid + k * TH < nchunk) {
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo(w[e]) - mean, b = bf16hi(w[e]) - mean;
        q = fmaf(a, a, q);
        q = fmaf(b, b, q);
      }
    }
  }
  const float var = block_sum_w<TH / 32>(q, red[1]) / static_cast<float>(D);
  const float rstd = rsqrtf(var + eps);
  char* orow = reinterpret_cast<char*>(out) + row * static_cast<int64_t>(D) * 2;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = tid + k * TH;
    if (c < nchunk) {
      uint4 gv, bv;
      if constexpr (EARLY) {
        gv = gv_e[k];
        bv = bv_e[k];
      } else {
        gv = ld_cached(gr + c * 16);
        bv = ld_cached(br + c * 16);
      }
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = fmaf((bf16lo(w[e]) - mean) * rstd, scale_offset + bf16lo(gw[e]), bf16lo(bw[e]));
        const float hi = fmaf((bf16hi(w[e]) - mean) * rstd, scale_offset + bf16hi(gw[e]), bf16hi(bw[e]));
        o[e] = pack_bf16x2(lo, hi);
      }
      st_stream(orow + c * 16, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// The early form with the parameters staged in shared memory instead of registers:
// gamma and beta are copied with cp.async (L1-allocating) when x is loaded, each thread
// reading back only its own chunks after its own copies completed, so the row needs the
// late form's registers (14 resident rows of 64 threads per SM at d_model 3072, against
// 8 rows for the register-held early form). Measured on B200 inside the packed-varlen
// step (one parameter group per frame): 5.06-5.10 against 4.71-4.75 TB/s; with the
// L2-only copy (cp.async.cg) it was twice as slow, every row then refetching its
// parameters from L2.
template <int NV, int TH>
__global__ void __launch_bounds__(TH)
adaln_modulate_staged_kernel(const __nv_bfloat16* x, const __nv_bfloat16* __restrict__ gamma,
                             const __nv_bfloat16* __restrict__ beta, __nv_bfloat16* out, int32_t D,
                             int64_t rows_per_group, float eps, float scale_offset) {
  __shared__ float red[2][TH / 32];
  __shared__ uint4 gb[2 * NV * TH];  // [gamma chunks | beta chunks], chunk k of thread t at k * TH + t
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nchunk = D >> 3;
  const char* xr = reinterpret_cast<const char*>(x) + row * static_cast<int64_t>(D) * 2;
  const int64_t g = row / rows_per_group;
  const char* gr = reinterpret_cast<const char*>(gamma) + g * static_cast<int64_t>(D) * 2;
  const char* br = reinterpret_cast<const char*>(beta) + g * static_cast<int64_t>(D) * 2;
  uint4 v[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = tid + k * TH;
    v[k] = (c < nchunk) ? ld_stream(xr + c * 16) : make_uint4(0, 0, 0, 0);
    if (c < nchunk) {
      cp_async16(&gb[k * TH + tid], gr + c * 16);
      cp_async16(&gb[(NV + k) * TH + tid], br + c * 16);
    }
  }
  cp_async_commit();
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) s += bf16lo(w[e]) + bf16hi(w[e]);
  }
  const float mean = block_sum_w<TH / 32>(s, red[0]) / static_cast<float>(D);
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    if (tid + k * TH < nchunk) {
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo(w[e]) - mean, b = bf16hi(w[e]) - mean;
        q = fmaf(a, a, q);
        q = fmaf(b, b, q);
      }
    }
  }
  const float var = block_sum_w<TH / 32>(q, red[1]) / static_cast<float>(D);
  const float rstd = rsqrtf(var + eps);
  cp_async_wait_all();
  char* orow = reinterpret_cast<char*>(out) + row * static_cast<int64_t>(D) * 2;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = tid + k * TH;
    if (c < nchunk) {
      const uint4 gv = gb[k * TH + tid], bv = gb[(NV + k) * TH + tid];
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = fmaf((bf16lo(w[e]) - mean) * rstd, scale_offset + bf16lo(gw[e]), bf16lo(bw[e]));
        const float hi = fmaf((bf16hi(w[e]) - mean) * rstd, scale_offset + bf16hi(gw[e]), bf16hi(bw[e]));
        o[e] = pack_bf16x2(lo, hi);
      }
      st_stream(orow + c * 16, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// Rows wider than the register-resident variant (D > 8192): three passes over the
// row, the second and third served from L1/L2.
__global__ void __launch_bounds__(kRowThreads)
adaln_modulate_wide_kernel(const __nv_bfloat16* x, const __nv_bfloat16* __restrict__ gamma,
                           const __nv_bfloat16* __restrict__ beta, __nv_bfloat16* out, int32_t D,
                           int64_t rows_per_group, float eps, float scale_offset) {
  __shared__ float red[2][4];
  const int64_t row = blockIdx.x;
  const int nchunk = D >> 3;
  const char* xr = reinterpret_cast<const char*>(x) + row * static_cast<int64_t>(D) * 2;
  float s = 0.f;
  for (int c = threadIdx.x; c < nchunk; c += kRowThreads) {
    const uint4 v = ld_cached(xr + c * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    for (int e = 0; e < 4; ++e) s += bf16lo(w[e]) + bf16hi(w[e]);
  }
  const float mean = block_sum_128(s, red[0]) / static_cast<float>(D);
  float q = 0.f;
  for (int c = threadIdx.x; c < nchunk; c += kRowThreads) {
    const uint4 v = ld_cached(xr + c * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    for (int e = 0; e < 4; ++e) {
      const float a = bf16lo(w[e]) - mean, b = bf16hi(w[e]) - mean;
      q = fmaf(a, a, fmaf(b, b, q));
    }
  }
  const float rstd = rsqrtf(block_sum_128(q, red[1]) / static_cast<float>(D) + eps);
  const int64_t g = row / rows_per_group;
  const char* gr = reinterpret_cast<const char*>(gamma) + g * static_cast<int64_t>(D) * 2;
  const char* br = reinterpret_cast<const char*>(beta) + g * static_cast<int64_t>(D) * 2;
  char* orow = reinterpret_cast<char*>(out) + row * static_cast<int64_t>(D) * 2;
  for (int c = threadIdx.x; c < nchunk; c += kRowThreads) {
    const uint4 v = ld_cached(xr + c * 16), gv = ld_cached(gr + c * 16), bv = ld_cached(br + c * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w},
                   bw[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t o[4];
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(
          fmaf((bf16lo(w[e]) - mean) * rstd, scale_offset + bf16lo(gw[e]), bf16lo(bw[e])),
          fmaf((bf16hi(w[e]) - mean) * rstd, scale_offset + bf16hi(gw[e]), bf16hi(bw[e])));
    // out may alias x: a thread only overwrites the chunks it has just read itself, and
    // every thread finished its statistics passes before the reductions' barriers.
    st_stream(orow + c * 16, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// x + a*y on a bf16 pair. A zero gate returns x's bits unchanged (the adaLN-Zero
// identity holds exactly, -0.0 included, whatever y holds).
__device__ __forceinline__ float gate1(float x, float y, float a) {
  return a == 0.f ? x : fmaf(a, y, x);
}
__device__ __forceinline__ uint32_t gate_pair(uint32_t xw, uint32_t yw, uint32_t aw) {
  // bf16 -> fp32 -> bf16 of an unchanged x is exact, so a zero gate keeps x's bits
  return pack_bf16x2(gate1(bf16lo(xw), bf16lo(yw), bf16lo(aw)),
                     gate1(bf16hi(xw), bf16hi(yw), bf16hi(aw)));
}

template <int NV>
__global__ void __launch_bounds__(kRowThreads)
gated_residual_kernel(const __nv_bfloat16* x, const __nv_bfloat16* y,
                      const __nv_bfloat16* __restrict__ alpha, __nv_bfloat16* out, int32_t D,
                      int64_t rows_per_group) {
  const int64_t row = blockIdx.x;
  const int nchunk = D >> 3;
  const int64_t off = row * static_cast<int64_t>(D) * 2;
  const char* xr = reinterpret_cast<const char*>(x) + off;
  const char* yr = reinterpret_cast<const char*>(y) + off;
  const char* ar = reinterpret_cast<const char*>(alpha) + (row / rows_per_group) * static_cast<int64_t>(D) * 2;
  char* orow = reinterpret_cast<char*>(out) + off;
  uint4 xv[NV], yv[NV], av[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nchunk) {
      xv[k] = ld_stream(xr + c * 16);
      yv[k] = ld_stream(yr + c * 16);
      av[k] = ld_cached(ar + c * 16);
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nchunk) {
      const uint32_t xw[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
      const uint32_t yw[4] = {yv[k].x, yv[k].y, yv[k].z, yv[k].w};
      const uint32_t aw[4] = {av[k].x, av[k].y, av[k].z, av[k].w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = gate_pair(xw[e], yw[e], aw[e]);
      st_stream(orow + c * 16, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

__global__ void __launch_bounds__(kRowThreads)
gated_residual_wide_kernel(const __nv_bfloat16* x, const __nv_bfloat16* y,
                           const __nv_bfloat16* __restrict__ alpha, __nv_bfloat16* out, int32_t D,
                           int64_t rows_per_group) {
  const int64_t row = blockIdx.x;
  const int nchunk = D >> 3;
  const int64_t off = row * static_cast<int64_t>(D) * 2;
  const char* ar = reinterpret_cast<const char*>(alpha) + (row / rows_per_group) * static_cast<int64_t>(D) * 2;
  for (int c = threadIdx.x; c < nchunk; c += kRowThreads) {
    const uint4 xv = ld_stream(reinterpret_cast<const char*>(x) + off + c * 16);
    const uint4 yv = ld_stream(reinterpret_cast<const char*>(y) + off + c * 16);
    const uint4 av = ld_cached(ar + c * 16);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, yw[4] = {yv.x, yv.y, yv.z, yv.w},
                   aw[4] = {av.x, av.y, av.z, av.w};
    uint32_t o[4];
    for (int e = 0; e < 4; ++e) o[e] = gate_pair(xw[e], yw[e], aw[e]);
    st_stream(reinterpret_cast<char*>(out) + off + c * 16, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

}  // namespace dit3d
