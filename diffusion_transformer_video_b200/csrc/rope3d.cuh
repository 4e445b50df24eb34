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
// cos/sin come from a table computed in fp64 and stored in fp32, laid out so
// that one 16-byte data chunk (8 bf16 = 4 pairs) needs two 16-byte table reads.
// For band a (t, h, w) the table holds, per position pos, the values of every pair
// of the chunks the band touches -- chunk-aligned, pairs outside the band set to the
// identity (cos 1, sin 0) -- starting at float2 index  off_a + pos * stride_a +
// 4 * (c - cf_a) for chunk c, as (cos p0, cos p1, sin p0, sin p1, cos p2, cos p3,
// sin p2, sin p3): each pair couple's cosines and sines are adjacent, ready for
// packed f32x2 arithmetic. stride_a is an odd number of 16-byte units, so 32 lanes
// reading 32 different positions hit distinct bank groups. A chunk that straddles a
// band edge is rotated once per band it touches; the identity entries leave the
// other band's pairs exact in fp32, so the result equals a single rotation.
// The position offsets are folded into the angles.
#pragma once
#include "common.cuh"
#include "quant.cuh"

namespace dit3d {

struct RopeParams {
  const float2* table;
  int32_t n_entries;          // float2 entries in the table
  int32_t grid_h, grid_w;
  int32_t p1, p2;             // first pair of the h band and of the w band (t starts at 0)
  int32_t off0, off1, off2;   // first float2 of each band's section
  int32_t str0, str1, str2;   // float2 entries per position in each section
  int32_t cf0, cf1, cf2;      // first chunk each band touches
};

__device__ __forceinline__ int rope_band_of_pair(const RopeParams& rp, int p) {
  return p < rp.p1 ? 0 : (p < rp.p2 ? 1 : 2);
}

__device__ __forceinline__ void token_pos(int64_t j, int gh, int gw, int& t, int& h, int& w) {
  const int64_t hw = static_cast<int64_t>(gh) * gw;
  t = static_cast<int>(j / hw);
  const int r = static_cast<int>(j - static_cast<int64_t>(t) * hw);
  h = r / gw;
  w = r - h * gw;
}

// Float2 index, in band a's section, of the first pair of chunk c at position pos.
__device__ __forceinline__ int rope_entry(const RopeParams& rp, int a, int pos, int c) {
  const int off = a == 0 ? rp.off0 : (a == 1 ? rp.off1 : rp.off2);
  const int str = a == 0 ? rp.str0 : (a == 1 ? rp.str1 : rp.str2);
  const int cf = a == 0 ? rp.cf0 : (a == 1 ? rp.cf1 : rp.cf2);
  return off + pos * str + 4 * (c - cf);
}

// x0' = x0 cos - x1 sin, x1' = x0 sin + x1 cos for the two pairs (a0, a1), (b0, b1) of
// a couple, with f = (cos_a, cos_b, sin_a, sin_b), in packed f32x2 arithmetic (the
// same roundings as the scalar fmaf(x0, c, -(x1 s)) and fmaf(x0, s, x1 c)).
__device__ __forceinline__ void rope_rotate_couple(float& a0, float& a1, float& b0, float& b1,
                                                   float4 f) {
  const uint64_t X0 = f2_pack(a0, b0), X1 = f2_pack(a1, b1);
  const uint64_t C = f2_pack(f.x, f.y), S = f2_pack(f.z, f.w);
  const uint64_t o0 = f2_fma(X0, C, f2_mul(X1, f2_neg(S)));
  const uint64_t o1 = f2_fma(X0, S, f2_mul(X1, C));
  f2_unpack(o0, a0, b0);
  f2_unpack(o1, a1, b1);
}

// Rotate the four fp32 pairs of a chunk, (x[0], x[1]) .. (x[6], x[7]).
__device__ __forceinline__ void rope_rotate4(float (&x)[8], float4 f01, float4 f23) {
  rope_rotate_couple(x[0], x[1], x[2], x[3], f01);
  rope_rotate_couple(x[4], x[5], x[6], x[7], f23);
}

// Width (in float2 entries per position) of band a's table section; 0 for an empty band.
__device__ __forceinline__ int rope_band_stride(const RopeParams& rp, int a) {
  return a == 0 ? rp.str0 : (a == 1 ? rp.str1 : rp.str2);
}

// Rotate chunk c (pairs 4c .. 4c+3) of one row at position (t, h, w). `tab` is the
// table (in global or shared memory, generic address). The bands are applied in
// order; an empty band between two others (d_h = 0) has no section and is skipped.
__device__ __forceinline__ uint4 rope_chunk(const RopeParams& rp, const float2* tab, uint4 v, int c,
                                            int t, int h, int w) {
  float x[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
  const int a_lo = rope_band_of_pair(rp, 4 * c), a_hi = rope_band_of_pair(rp, 4 * c + 3);
  for (int a = a_lo; a <= a_hi; ++a) {
    if (rope_band_stride(rp, a) == 0) continue;
    const int pos = a == 0 ? t : (a == 1 ? h : w);
    const float4* e = reinterpret_cast<const float4*>(tab + rope_entry(rp, a, pos, c));
    rope_rotate4(x, e[0], e[1]);
  }
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

// What the table holds, per band a (t, h, w): its width d_a, its number of positions,
// its position offset and the head pair where it starts; the frequency base.
struct RopeTableSpec {
  float base;
  int32_t width[3], ext[3], offs[3], first_pair[3];
  int32_t n_fill;  // float2 entries to write (n_entries, at least 2)
};

// Writes the cos/sin table of the layout above, one float2 entry per thread: for pair
// i of band a at position pos, the angle (pos + offset_a) * base^(-2i/d_a) in fp64,
// its cosine and sine rounded to fp32. Entries outside every band, pairs of a chunk
// outside its band, and the two padding entries that end each position's row hold the
// identity (cos 1, sin 0): even entries are cosine couples, odd ones sine couples.
__global__ void __launch_bounds__(256)
rope_table_fill_kernel(float2* __restrict__ table, RopeParams rp, RopeTableSpec s) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= s.n_fill) return;
  const int off[3] = {rp.off0, rp.off1, rp.off2};
  const int str[3] = {rp.str0, rp.str1, rp.str2};
  const int cf[3] = {rp.cf0, rp.cf1, rp.cf2};
  const bool is_sin = (e & 1) != 0;
  float res[2] = {is_sin ? 0.f : 1.f, is_sin ? 0.f : 1.f};
  for (int a = 0; a < 3; ++a) {
    if (str[a] == 0) continue;  // empty band: no section
    const int r = e - off[a];
    if (r < 0 || r >= s.ext[a] * str[a]) continue;
    const int pos = r / str[a], k = r - pos * str[a];
    if (k < str[a] - 2) {
      const int u = (k & 3) >> 1;  // couple inside the chunk
      for (int w = 0; w < 2; ++w) {
        const int p = 4 * (cf[a] + (k >> 2)) + 2 * u + w;  // pair index in the head
        const int i = p - s.first_pair[a];
        if (i < 0 || 2 * i >= s.width[a]) continue;
        const double theta = pow(static_cast<double>(s.base), -2.0 * i / s.width[a]);
        const double phi = static_cast<double>(pos + s.offs[a]) * theta;
        res[w] = static_cast<float>(is_sin ? sin(phi) : cos(phi));
      }
    }
    break;
  }
  table[e] = make_float2(res[0], res[1]);
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

// The rotation of one chunk by up to three bands whose table entries are already in
// registers (nb of them, in band order): the arithmetic of rope_chunk.
__device__ __forceinline__ uint4 rope_chunk_reg(uint4 v, int nb, const float4 (&f)[3][2]) {
  float x[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
  rope_rotate4(x, f[0][0], f[0][1]);
  if (nb > 1) rope_rotate4(x, f[1][0], f[1][1]);
  if (nb > 2) rope_rotate4(x, f[2][0], f[2][1]);
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

// Standalone RoPE, an HBM stream: one warp per token row. Lane l always handles
// chunk l % (D_HEAD/8) of a head, so the row's table entries for that chunk are read
// once into registers and reused for every head of q and of k; the head loop keeps
// kUnroll 16-byte loads of q and of k in flight per lane before rotating and
// storing them. Same per-chunk arithmetic as rope_chunk (and the attention kernel),
// so all produce the same bits. In place (q_out == q_in) is safe: every element is
// read and written by the same thread.
// With E4M3 set the rotated chunk, rounded to bf16 as above, is scaled by q_inv (k_inv)
// and written as 8 E4M3 codes (8 bytes) with quantize_e4m3_kernel's conversion: the
// same bytes as the rotation followed by the separate quantisation pass, without
// writing and re-reading the rotated bf16 tensors. The outputs then hold half the
// bytes of the inputs, so they must not overlap them.
template <int D_HEAD, bool E4M3 = false>
__global__ void __launch_bounds__(256, 3)
rope3d_qk_kernel(const uint4* q_in, const uint4* k_in, void* q_out, void* k_out, int64_t rows,
                 int32_t H, const int32_t* __restrict__ cu, int32_t n_seq, int64_t dense_len,
                 RopeParams rp, float q_inv = 1.f, float k_inv = 1.f) {
  constexpr int kCpr = D_HEAD / 8;  // 16-byte chunks per head
  constexpr int kUnroll = 4;
  static_assert(32 % kCpr == 0, "lane-fixed chunks need D_HEAD/8 to divide 32");
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t j = row - seq_start_of_row(cu, n_seq, row, dense_len);
  int t, h, w;
  token_pos(j, rp.grid_h, rp.grid_w, t, h, w);
  const int cc = lane % kCpr;
  const float4 one = make_float4(1.f, 1.f, 0.f, 0.f);  // identity (cos 1, sin 0)
  float4 f[3][2] = {{one, one}, {one, one}, {one, one}};
  int nb = 0;
  const int a_lo = rope_band_of_pair(rp, 4 * cc), a_hi = rope_band_of_pair(rp, 4 * cc + 3);
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    if (a < a_lo || a > a_hi || rope_band_stride(rp, a) == 0) continue;
    const int pos = a == 0 ? t : (a == 1 ? h : w);
    const float4* e = reinterpret_cast<const float4*>(rp.table + rope_entry(rp, a, pos, cc));
    const float4 e0 = __ldg(e), e1 = __ldg(e + 1);
    // nb is 0, 1 or 2 here; selects keep f in registers
    f[0][0] = nb == 0 ? e0 : f[0][0];
    f[0][1] = nb == 0 ? e1 : f[0][1];
    f[1][0] = nb == 1 ? e0 : f[1][0];
    f[1][1] = nb == 1 ? e1 : f[1][1];
    f[2][0] = nb == 2 ? e0 : f[2][0];
    f[2][1] = nb == 2 ? e1 : f[2][1];
    ++nb;
  }
  const int nchunk = H * kCpr;
  const int64_t base = row * nchunk;
  const bool has_k = k_in != nullptr;
  for (int c0 = lane; c0 < nchunk; c0 += 32 * kUnroll) {
    uint4 vq[kUnroll], vk[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        vq[u] = q_in[base + c];
        if (has_k) vk[u] = k_in[base + c];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        const uint4 rq = rope_chunk_reg(vq[u], nb, f);
        if constexpr (E4M3)
          static_cast<uint2*>(q_out)[base + c] =
              make_uint2(e4m3x4(rq.x, rq.y, q_inv), e4m3x4(rq.z, rq.w, q_inv));
        else
          static_cast<uint4*>(q_out)[base + c] = rq;
        if (has_k) {
          const uint4 rk = rope_chunk_reg(vk[u], nb, f);
          if constexpr (E4M3)
            static_cast<uint2*>(k_out)[base + c] =
                make_uint2(e4m3x4(rk.x, rk.y, k_inv), e4m3x4(rk.z, rk.w, k_inv));
          else
            static_cast<uint4*>(k_out)[base + c] = rk;
        }
      }
    }
  }
}

}  // namespace dit3d
