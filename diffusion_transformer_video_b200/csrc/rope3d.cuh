// 3D rotary position embedding.
//
// "DiT, Flow Matching e 3D Attention", section "3D-RoPE e atencao espaco-temporal":
// the head dimension is split into bands d_t + d_h + d_w; each band's pairs turn
// with frequencies tied to the latent frame index t, the row y and the column x,
// and q_rot = R3D(t, y, x) q, k_rot = R3D(t, y, x) k.
// Library reading: band order t|h|w, interleaved pairs (2i, 2i+1), angle
// pos * base^(-2i/d_a), rotation [[cos, -sin], [sin, cos]], positions counted from
// 0 at each sequence start plus a constant offset.
//
// The cos/sin values come from a table the host fills in fp64 and stores in fp32:
// three sections, [T_ext][d_t/2], [grid_h][d_h/2], [grid_w][d_w/2], of float2
// (cos, sin), with the position offsets already folded into the angles.
#pragma once
#include "common.cuh"

namespace dit3d {

struct RopeParams {
  const float2* table;
  int32_t n_entries;     // float2 entries in the table
  int32_t grid_h, grid_w;
  int32_t d_t, d_h, d_w;
  int32_t off_h, off_w;  // start (in float2) of the h and w sections; t starts at 0
};

// Table index, for position 0, and per-position stride of pair p (0 <= p < d/2).
struct PairRef {
  int32_t axis;    // 0 = t, 1 = h, 2 = w
  int32_t base;    // index of (pos = 0, this pair)
  int32_t stride;  // float2 entries per position step
};

__device__ __forceinline__ PairRef rope_pair_ref(const RopeParams& rp, int p) {
  const int ht = rp.d_t >> 1, hh = rp.d_h >> 1, hw = rp.d_w >> 1;
  PairRef r;
  if (p < ht) {
    r.axis = 0; r.base = p; r.stride = ht;
  } else if (p < ht + hh) {
    r.axis = 1; r.base = rp.off_h + (p - ht); r.stride = hh;
  } else {
    r.axis = 2; r.base = rp.off_w + (p - ht - hh); r.stride = hw;
  }
  return r;
}

__device__ __forceinline__ void token_pos(int64_t j, int gh, int gw, int& t, int& h, int& w) {
  const int64_t hw = static_cast<int64_t>(gh) * gw;
  t = static_cast<int>(j / hw);
  const int r = static_cast<int>(j - static_cast<int64_t>(t) * hw);
  h = r / gw;
  w = r - h * gw;
}

__device__ __forceinline__ float2 rope_cs(const RopeParams& rp, const PairRef& pr, int t, int h,
                                          int w) {
  const int pos = pr.axis == 0 ? t : (pr.axis == 1 ? h : w);
  return __ldg(rp.table + pr.base + pos * pr.stride);
}
// Same lookup in a copy of the table (shared memory or global, generic address).
__device__ __forceinline__ float2 rope_cs_at(const float2* tab, const PairRef& pr, int t, int h,
                                             int w) {
  const int pos = pr.axis == 0 ? t : (pr.axis == 1 ? h : w);
  return tab[pr.base + pos * pr.stride];
}

// Rotate the 4 pairs of one 16-byte chunk.
__device__ __forceinline__ uint4 rope_rotate_chunk(uint4 v, const float2 (&cs)[4]) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x0 = bf16lo(w[e]), x1 = bf16hi(w[e]);
    const float c = cs[e].x, s = cs[e].y;
    w[e] = pack_bf16x2(fmaf(x0, c, -x1 * s), fmaf(x0, s, x1 * c));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Sequence start of global row `row` (largest s with cu[s] <= row).
__device__ __forceinline__ int64_t seq_start_of_row(const int32_t* __restrict__ cu, int n_seq,
                                                    int64_t row, int64_t dense_len) {
  if (cu == nullptr) return (row / dense_len) * dense_len;
  int lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(__ldg(cu + mid)) <= row) lo = mid; else hi = mid - 1;
  }
  return __ldg(cu + lo);
}

// Standalone RoPE: one warp per token row. Lane l always handles column chunk
// l % (D_HEAD/8) of every head, so its four (cos, sin) pairs are fetched once per
// row and reused for all heads of q and of k.
template <int D_HEAD>
__global__ void __launch_bounds__(256)
rope3d_qk_kernel(const uint4* q_in, const uint4* k_in, uint4* q_out, uint4* k_out, int64_t rows,
                 int32_t H, const int32_t* __restrict__ cu, int32_t n_seq, int64_t dense_len,
                 RopeParams rp) {
  static_assert(32 % (D_HEAD / 8) == 0, "lane-fixed chunks need D_HEAD/8 to divide 32");
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t j = row - seq_start_of_row(cu, n_seq, row, dense_len);
  int t, h, w;
  token_pos(j, rp.grid_h, rp.grid_w, t, h, w);
  const int cc = lane % (D_HEAD / 8);
  float2 cs[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) cs[e] = rope_cs(rp, rope_pair_ref(rp, cc * 4 + e), t, h, w);
  const int nchunk = H * (D_HEAD / 8);
  const int64_t base = row * nchunk;
  for (int c = lane; c < nchunk; c += 32) {
    q_out[base + c] = rope_rotate_chunk(q_in[base + c], cs);
  }
  if (k_in != nullptr) {
    for (int c = lane; c < nchunk; c += 32) {
      k_out[base + c] = rope_rotate_chunk(k_in[base + c], cs);
    }
  }
}

}  // namespace dit3d
