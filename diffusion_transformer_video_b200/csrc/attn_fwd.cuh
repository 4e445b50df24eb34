// Flash-style forward attention for sm_100a, with optional in-kernel 3D-RoPE and
// optional FP8 (E4M3) operands (template mode F8, described at the kernel).
//
//   o = softmax(q_rot k_rot^T * scale) v     per (sequence, head), non-causal
//
// ("DiT, Flow Matching e 3D Attention", section "3D-RoPE e atencao
// espaco-temporal"; "Por que e absurdamente dificil gerar um filme inteiro usando
// IA", section "Matematica por tras". The N x N score matrix never leaves the SM:
// it lives in tensor memory one 128 x 128 tile at a time.)
//
// One CTA computes two 128-row query tiles (Q0, Q1) of one head of one sequence
// and streams the sequence's keys/values in 128-row tiles through shared-memory
// rings. 512 threads in four warpgroups:
//   WG0 (warps 0-3)  softmax of Q0: thread i owns query row i = TMEM lane i.
//   WG1 (warps 4-7)  softmax of Q1.
//   WG2 (warps 8-11) 3D-RoPE: rotate Q0/Q1 and every K_j in shared memory, in
//                    place, right after TMA lands them (fp32 math, bf16 result).
//   warp 12          TMA producer of Q0, Q1 (once) and of the 2-stage K ring.
//   warp 13          TMEM allocator and tcgen05.mma issuer (the whole warp runs the
//                    loop, one elected lane issues).
//   warp 14          TMA producer of the 2-stage V ring.
//   warp 15          idle (it only gives its registers away).
// A K stage is released right after both QK^T products read it, a V stage after
// both PV products, so K tiles (and their RoPE) run ahead of the V tiles. The
// RoPE cos/sin table (up to 32 KB) is copied into shared memory once per CTA.
// setmaxnreg moves registers to the softmax warpgroups (184 each; 80 for RoPE, 64 else)
// so a thread can hold its whole 128-column score row.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d),
// O1 [384,384+d). P_i (bf16, two per column) overwrites the first 64 columns of
// S_i once the softmax has read S_i into registers.
// MMA order (ping-pong, so one tile's softmax overlaps the other tile's MMAs):
//   S0=Q0K0, S1=Q1K0, then for each j: O0+=P0V_j, S0=Q0K_{j+1}, O1+=P1V_j, S1=Q1K_{j+1}.
// Tensor-core operations issued by one thread (the elected lane) run in order, and a
// commit arrives only when every earlier operation of that thread is complete, so when
// the softmax sees S_i(j+1) the product O_i += P_i(j)V_j has landed and O_i may be
// rescaled in place.
// Online softmax in base 2 with a lazily updated row maximum: the running max is
// only raised (and O, l rescaled) when a new score exceeds it by more than 2^8,
// which keeps every exponent <= 8 and skips most O rescales.
// Every mbarrier wait is bounded; on expiry the CTA sets an error bit, drains its
// in-flight copies and MMAs, frees its tensor memory and exits.
// Key-range split (Params::kv_split > 1, the last partial wave of a dense batch): the
// CTAs of a cluster share one unit's key tiles; each leaves its unnormalised O rows and
// (m, l) in its own shared memory, and after a cluster barrier merges a share of the
// unit's rows from every CTA's (merge_split_rows); a second barrier keeps each CTA's
// memory alive until its peers have read it. Every path, bounded-wait expiry included,
// reaches both barriers.
#pragma once
#include <type_traits>
#include "common.cuh"
#include "quant.cuh"
#include "rope3d.cuh"
#include "sm100_ptx.cuh"

namespace dit3d {
namespace attn {

constexpr int kThreads = 512;
constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kKStages = 2;  // K ring: released as soon as both Q tiles' QK^T read it
constexpr int kVStages = 2;  // V ring: released after both PV products
constexpr int kRopeThreads = 128;
constexpr int kWarpRope0 = 8, kWarpTma = 12, kWarpMma = 13, kWarpTmaV = 14;
// register split (setmaxnreg): 2*128*184 + 128*80 + 128*64 = 65536 = 512*128
constexpr int kSoftmaxRegs = 184, kRopeRegs = 80, kCtrlRegs = 64;
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int qi) { return qi ? 128u : 0u; }
__host__ __device__ constexpr uint32_t col_o(int qi) { return qi ? 384u : 256u; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Params {
  const int32_t* cu_seqlens;  // device, n_seq + 1 entries, or nullptr (dense)
  int32_t n_seq;
  int64_t dense_len;          // sequence length when cu_seqlens == nullptr
  int32_t pairs_per_dense_seq;
  int32_t H;
  float scale_log2;           // softmax scale * log2(e)
  __nv_bfloat16* o;
  float* lse;                 // nullable, [rows, H]
  int32_t use_rope;
  RopeParams rope;
  int32_t force_timeout;
  float o_scale;              // multiplies O in the epilogue (V's dequantisation scale; 1 else)
  uint64_t wait_limit_ns;     // bound of the waits that give up the CTA's work (2 s by default)
  // packed batches of up to kMaxOrder sequences: their order, longest first, on a 1-D
  // grid (n_order > 0); otherwise a (pairs, heads) grid in cu_seqlens order
  int32_t n_order;
  int32_t seq_order[64];
  // dense batches: work units (a pair of query tiles of one sequence and head) are
  // numbered head-major from unit0. kv_split > 1: a 1-D grid of clusters of kv_split
  // CTAs, one cluster per unit, CTA s of a cluster taking key tiles
  // [s * nk / kv_split, (s + 1) * nk / kv_split) and the cluster merging the partial
  // results through distributed shared memory (the launch's last partial wave)
  int32_t kv_split;
  int32_t unit0;
  // programmatic dependent launch of the split wave: 1 = let the next launch (the split
  // units) start as this grid's CTAs are all resident; 2 = wait, before exiting, for the
  // launch this one overlaps, so that later work on the stream still follows both
  int32_t pdl;
};
constexpr int kMaxOrder = 64;
constexpr int kMaxSplit = 8;  // portable cluster size

template <int D>
struct Smem {
  static constexpr uint32_t kTile = kTileM * D * 2;           // one Q, K or V tile
  static constexpr uint32_t kQ0 = 0, kQ1 = kTile;
  static constexpr uint32_t kK = 2 * kTile;                   // + stage * kTile
  static constexpr uint32_t kV = kK + kKStages * kTile;       // + stage * kTile
  static constexpr uint32_t kTab = kV + kVStages * kTile;     // RoPE cos/sin table copy
  static constexpr uint32_t kTabBytes = 32 * 1024;
  static constexpr uint32_t kBytes = kTab + kTabBytes;
  // key-range split: once every MMA has completed, the Q/K/V area holds the CTA's
  // partial O (fp32 rows of D + 4 floats: a row shift of 16 bytes keeps a warp's row
  // stores conflict-free) for its 2 * kTileM query rows, then (m, l) per row
  static constexpr uint32_t kPartStride = (D + 4) * 4;
  static constexpr uint32_t kPartMl = 2 * kTileM * kPartStride;
  static_assert(kPartMl + 2 * kTileM * 8 <= kTab, "partial results fit in the Q/K/V area");
  // dynamic smem request: forces one CTA per SM (the CTA takes all 512 TMEM columns)
  static constexpr uint32_t kRequest = (kBytes + 1024 > 120 * 1024) ? kBytes + 1024 : 120 * 1024;
};

struct Barriers {
  uint64_t q_full, q_ready;
  uint64_t k_full[kKStages], k_ready[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_half[2], p_full[2];  // P of keys 0-63 / all 128 keys in TMEM
  uint64_t o_final, drain;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^t of a pair of scores on the MUFU unit (ex2.approx; 16 results per clock per SM
// on B200, and the packed f16x2 / bf16x2 forms give no more). Moving a share of these
// to the FMA pipe (rounding by adding 1.5 * 2^23, degree-3 minimax polynomial for 2^f,
// 2^j added to the exponent field: no conversion instruction, which would issue to the
// MUFU pipe as well) was measured slower on B200 in the bf16 kernel: a quarter of the
// pairs -3 to -5 %, three eighths or half -12 to -17 %. In the E4M3 modes, whose MMAs
// take half the time, the MUFU pipe does set the pace: there three pairs in sixteen run
// on the FMA pipe (exp2_pair_fma; measured 2-4 % faster in both E4M3 modes, while one in
// four or more slowed the E4M3 Q K^T mode).
__device__ __forceinline__ void exp2_pair(uint64_t t2, float& e0, float& e1) {
  float t0, t1;
  f2_unpack(t2, t0, t1);
  e0 = ex2(t0);
  e1 = ex2(t1);
}

// 2^t of a pair of scores on the FMA and integer pipes:
//  - t = j + f with j = round(t): adding 1.5 * 2^23 (round to nearest) leaves j in the
//    low mantissa bits, with no conversion instruction (those share the MUFU pipe);
//  - 2^f for f in [-1/2, 1/2] by a degree-3 polynomial fitted by the Remez exchange for
//    relative error (7.5e-5 in fp32 Horner form; P is then rounded to bf16 or E4M3);
//  - 2^j enters as j << 23 added to the exponent field.
// t is clamped to >= -126 so the exponent field cannot wrap: a score more than 126
// below the running maximum then weighs about 2^-126 instead of 0. Masked (-inf) keys
// never take this path (a ragged last tile keeps every exponential on the MUFU unit).
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
constexpr float kP0 = 0.9999280571937561f, kP1 = 0.6932609677314758f;
constexpr float kP2 = 0.2426111251115799f, kP3 = 0.0551716685295105f;
__device__ __forceinline__ void exp2_pair_fma(uint64_t t2, float& e0, float& e1) {
  float t0, t1;
  f2_unpack(t2, t0, t1);
  const uint64_t tc = f2_pack(fmaxf(t0, -126.f), fmaxf(t1, -126.f));
  const uint64_t r = f2_add(tc, f2_pack(kRound, kRound));    // j in the low bits
  const uint64_t jf = f2_add(r, f2_pack(-kRound, -kRound));  // j, exact
  const uint64_t f = f2_fma(jf, f2_pack(-1.f, -1.f), tc);    // t - j, exact
  uint64_t q = f2_fma(f2_pack(kP3, kP3), f, f2_pack(kP2, kP2));
  q = f2_fma(q, f, f2_pack(kP1, kP1));
  q = f2_fma(q, f, f2_pack(kP0, kP0));
  float q0, q1, r0, r1;
  f2_unpack(q, q0, q1);
  f2_unpack(r, r0, r1);
  e0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(r0) << 23));
  e1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(r1) << 23));
}
// Pairs c of each 32-key chunk (bit c, c = 0..15) whose exponential runs on the FMA
// pipe in the E4M3 modes: 3, 8 and 13.
constexpr uint32_t kExpFmaMaskF8 = 0x2108u;

// Byte offset of the 16-byte chunk `cc` (8 bf16) of row r inside a 128-row tile
// stored as d/64 column blocks of [128 rows x 128 B] with the 128-byte TMA swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int cc) {
  return static_cast<uint32_t>((cc >> 3) * 16384 + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}
// Same for a tile whose 64-column blocks are `block` bytes apart.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int cc, uint32_t block) {
  return static_cast<uint32_t>((cc >> 3) * block + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

// 16-byte shared-memory load / store. The loads carry no memory clobber, so the
// compiler may hoist the next chunks' loads above this chunk's store (the table and
// the chunks a thread touches never overlap).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
  float4 v;
  asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
// Ordered 16-byte load: after every earlier store and never merged with another load
// of the same address (a chunk re-read after its own rotation was written back).
__device__ __forceinline__ uint4 lds128_ordered(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 rope_apply(uint4 v, float4 e0, float4 e1) {
  float x[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
  rope_rotate4(x, e0, e1);
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

// Rotate rows [0, n_valid) of one tile in shared memory, in place. Row r of the tile
// is token (row0 + r) of its sequence; RoPE thread r owns row r: it decodes the
// row's (t, h, w) once and walks the row's d/8 chunks (a warp then covers 32 rows
// of one chunk column: no divergence, conflict-free swizzled accesses).
// Pass 1 rotates every chunk by the band of its first pair, four chunks at a time
// with all their loads issued first; pass 2 applies the other band(s) to the few
// chunks that straddle a band edge. Every pair is turned exactly once (identity
// entries elsewhere, and the bf16 round trip of an untouched value is exact), so the
// result equals the standalone kernel's single rotation bit for bit.
template <int D>
__device__ __forceinline__ void rope_tile_smem(uint32_t tile, int64_t row0, int n_valid,
                                               const RopeParams& rp, uint32_t tab, int rt) {
  static_assert(kRopeThreads == kTileM, "one tile row per RoPE thread");
  if (rt >= n_valid) return;
  const int j = static_cast<int>(row0) + rt;  // positions inside a sequence fit in 32 bits
  const int hw = rp.grid_h * rp.grid_w;
  const int t = j / hw, rr = j - t * hw, h = rr / rp.grid_w, w = rr - h * rp.grid_w;
  const uint32_t row_t = tab + 8u * static_cast<uint32_t>(rp.off0 + t * rp.str0 - 4 * rp.cf0);
  const uint32_t row_h = tab + 8u * static_cast<uint32_t>(rp.off1 + h * rp.str1 - 4 * rp.cf1);
  const uint32_t row_w = tab + 8u * static_cast<uint32_t>(rp.off2 + w * rp.str2 - 4 * rp.cf2);
#pragma unroll
  for (int c0 = 0; c0 < D / 8; c0 += 4) {
    uint4 v[4];
    float4 e0[4], e1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u;
      const int a = rope_band_of_pair(rp, 4 * c);
      const uint32_t e = (a == 0 ? row_t : (a == 1 ? row_h : row_w)) + 32u * c;
      v[u] = lds128(tile + sw128_chunk(rt, c));
      e0[u] = lds128f(e);
      e1[u] = lds128f(e + 16u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) sts128(tile + sw128_chunk(rt, c0 + u), rope_apply(v[u], e0[u], e1[u]));
  }
  // pass 2: chunks across a band edge get the rotation of their later band(s)
  const int cs1 = (rp.p1 & 3) ? (rp.p1 >> 2) : -1;   // chunk holding the t/h edge
  const int cs2 = (rp.p2 & 3) ? (rp.p2 >> 2) : -1;   // chunk holding the h/w edge
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {
    const int c = k ? cs2 : cs1;
    if (c < 0 || (k && c == cs1)) continue;
    const int a_lo = rope_band_of_pair(rp, 4 * c), a_hi = rope_band_of_pair(rp, 4 * c + 3);
    for (int a = a_lo + 1; a <= a_hi; ++a) {
      if (rope_band_stride(rp, a) == 0) continue;  // an empty middle band
      const uint32_t e = (a == 1 ? row_h : row_w) + 32u * c;
      const uint32_t ad = tile + sw128_chunk(rt, c);
      sts128(ad, rope_apply(lds128_ordered(ad), lds128f(e), lds128f(e + 16u)));
    }
  }
}

// Same rotation with the table in global memory (tables larger than the shared copy).
template <int D>
__device__ __forceinline__ void rope_tile_global(uint8_t* tile, int64_t row0, int n_valid,
                                                 const RopeParams& rp, int rt) {
  if (rt >= n_valid) return;
  const int j = static_cast<int>(row0) + rt;
  const int hw = rp.grid_h * rp.grid_w;
  const int t = j / hw, rr = j - t * hw, h = rr / rp.grid_w, w = rr - h * rp.grid_w;
#pragma unroll 1
  for (int c = 0; c < D / 8; ++c) {
    uint4* p = reinterpret_cast<uint4*>(tile + sw128_chunk(rt, c));
    *p = rope_chunk(rp, rp.table, *p, c, t, h, w);
  }
}

// Merge of a key-range split (Params::kv_split): CTA `split` of the cluster combines
// rows [split * 256 / n_split, (split + 1) * 256 / n_split) of the unit's 256 query rows
// from every CTA's partial (O_s, m_s, l_s), read from their shared memory:
//   M = max_s m_s,  w_s = 2^(m_s - M),  o = sum_s w_s O_s / sum_s w_s l_s,
// the same rescaling the online softmax applies between key tiles, in a fixed order
// of s. Thread t (of the 256 softmax threads) takes 16-byte output chunks t, t + 256, ...
template <int D>
__device__ __forceinline__ void merge_split_rows(uint8_t* smem, const Params& p, int split,
                                                 int n_split, int64_t q_row0, int64_t seq_len,
                                                 int64_t seq_start, int head, int t) {
  using L = Smem<D>;
  constexpr int kCh = D / 8;  // 16-byte output chunks (8 bf16) per row
  constexpr int kRows = 2 * kTileM;
  const int g0 = split * kRows / n_split, g1 = (split + 1) * kRows / n_split;
  const uint32_t part = ptx::smem_u32(smem);
#pragma unroll 1
  for (int idx = t; idx < (g1 - g0) * kCh; idx += kRows) {
    const int g = g0 + idx / kCh, c = idx % kCh;
    const int64_t row_in_seq = q_row0 + g;
    if (row_in_seq >= seq_len) continue;
    float mt[kMaxSplit], lt[kMaxSplit];
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) {
      if (s < n_split) {
        const float2 v = ptx::ld_cluster_f2(ptx::mapa_shared(part + L::kPartMl + g * 8, s));
        mt[s] = v.x;
        lt[s] = v.y;
        M = fmaxf(M, v.x);
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lsum = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) {
      if (s < n_split) {
        const float w = ex2(mt[s] - M);
        lsum = fmaf(w, lt[s], lsum);
        const uint32_t a = ptx::mapa_shared(part + g * L::kPartStride + c * 32, s);
        const float4 u0 = ptx::ld_cluster_f4(a), u1 = ptx::ld_cluster_f4(a + 16);
        acc[0] = fmaf(w, u0.x, acc[0]);
        acc[1] = fmaf(w, u0.y, acc[1]);
        acc[2] = fmaf(w, u0.z, acc[2]);
        acc[3] = fmaf(w, u0.w, acc[3]);
        acc[4] = fmaf(w, u1.x, acc[4]);
        acc[5] = fmaf(w, u1.y, acc[5]);
        acc[6] = fmaf(w, u1.z, acc[6]);
        acc[7] = fmaf(w, u1.w, acc[7]);
      }
    }
    const float inv = p.o_scale / lsum;
    uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) +
                    ((seq_start + row_in_seq) * p.H + head) * static_cast<int64_t>(D) * 2;
    *reinterpret_cast<uint4*>(orow + c * 16) =
        make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                   pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
    if (c == 0 && p.lse != nullptr)
      p.lse[(seq_start + row_in_seq) * p.H + head] = (M + __log2f(lsum)) * 0.69314718055994531f;
  }
}

// F8 = 1: q and k arrive as FP8 E4M3 codes (one byte per element, d = 128: one
// 128-byte swizzle row per token) and S = Q K^T runs as kind::f8f6f4 MMAs (K = 32
// each); the host folds the two dequantisation scales into the softmax scale; P and V
// stay bf16. F8 = 2: v is E4M3 too (an MN-major B operand) and P is packed as E4M3
// (4 per TMEM column; P <= 2^8 under the lazy maximum, inside E4M3's range), so
// O += P V also runs on kind::f8f6f4; V's scale multiplies O in the epilogue. The
// tiles keep the bf16 layout's shared-memory slots (half of each is used).
template <int D, int F8 = 0>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Smem<D>;
  constexpr bool QK8 = F8 >= 1, PV8 = F8 == 2;
  static_assert(!QK8 || D == 128, "E4M3 tiles use 128-byte rows (head_dim 128)");
  constexpr int kQKBoxes = QK8 ? 1 : D / 64;                       // TMA boxes per Q/K tile
  constexpr uint32_t kQKBytes = QK8 ? kTileM * D : L::kTile;       // bytes per Q/K tile
  constexpr int kVBoxes = PV8 ? 1 : D / 64;
  constexpr uint32_t kVBytes = PV8 ? kTileN * D : L::kTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ Barriers bars;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  int head = blockIdx.y;
  if (p.pdl & 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // key-range split (dense batches only): this CTA's share, = its rank in the cluster
  const int n_split = p.kv_split > 1 ? p.kv_split : 1;
  const int split = n_split > 1 ? static_cast<int>(blockIdx.x % n_split) : 0;

  // ---- work decode: which sequence, head and pair of query tiles
  int64_t seq_start, seq_len;
  int pair;
  if (p.n_order > 0) {
    // packed batch, longest sequence first (1-D grid): every head of a sequence, then the
    // next sequence, so the CTAs that finish last are those of the shortest sequences
    int rem = blockIdx.x;
    head = 0;
    pair = 0;
    seq_start = 0;
    seq_len = 0;
    for (int i = 0; i < p.n_order; ++i) {
      const int s = p.seq_order[i];
      const int64_t a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
      const int np = static_cast<int>((b - a + 2 * kTileM - 1) / (2 * kTileM));
      if (rem < np * p.H) {
        head = rem / np;
        pair = rem - head * np;
        seq_start = a;
        seq_len = b - a;
        break;
      }
      rem -= np * p.H;
    }
  } else if (p.cu_seqlens == nullptr) {
    // head-major unit numbering: the (pairs, heads) grid's own block order
    const int64_t per_head = static_cast<int64_t>(p.pairs_per_dense_seq) * p.n_seq;
    const int64_t unit =
        p.unit0 + (n_split > 1 ? static_cast<int64_t>(blockIdx.x / n_split)
                               : static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x);
    head = static_cast<int>(unit / per_head);
    const int x = static_cast<int>(unit - static_cast<int64_t>(head) * per_head);
    const int seq = x / p.pairs_per_dense_seq;
    pair = x - seq * p.pairs_per_dense_seq;
    seq_len = p.dense_len;
    seq_start = static_cast<int64_t>(seq) * p.dense_len;
  } else {
    int acc = 0, s = 0;
    pair = 0;
    seq_start = 0;
    seq_len = 0;
    for (; s < p.n_seq; ++s) {
      const int64_t a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
      const int np = static_cast<int>((b - a + 2 * kTileM - 1) / (2 * kTileM));
      if (static_cast<int>(blockIdx.x) < acc + np) {
        pair = blockIdx.x - acc;
        seq_start = a;
        seq_len = b - a;
        break;
      }
      acc += np;
    }
  }
  const int64_t q_row0 = static_cast<int64_t>(pair) * 2 * kTileM;  // within the sequence
  const int nk = static_cast<int>((seq_len + kTileN - 1) / kTileN);
  const int last_valid = static_cast<int>(seq_len - static_cast<int64_t>(nk - 1) * kTileN);
  // key tiles [kb0, kb0 + nkl) of the nk (nk < 2^24, split < 8: int products); the
  // loops below count j from 0 within them
  const int kb0 = split * nk / n_split;
  const int nkl = (split + 1) * nk / n_split - kb0;
  // the last tile of the range is the sequence's ragged one
  const bool ragged_last = kb0 + nkl == nk && last_valid < kTileN;

  Barriers* b = &bars;
  volatile int* abort = &s_abort;
  if (tid == 0) {
    s_abort = p.force_timeout ? 1 : 0;
    ptx::mbar_init(ptx::smem_u32(&b->q_full), 1);
    ptx::mbar_init(ptx::smem_u32(&b->q_ready), kRopeThreads);
    for (int s = 0; s < kKStages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&b->k_full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&b->k_ready[s]), kRopeThreads);
      ptx::mbar_init(ptx::smem_u32(&b->k_empty[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&b->v_full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&b->v_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(ptx::smem_u32(&b->s_full[i]), 1);
      // one arrival per softmax warp: measured 4 % faster at 480P than one per thread
      ptx::mbar_init(ptx::smem_u32(&b->p_half[i]), kTileM / 32);
      ptx::mbar_init(ptx::smem_u32(&b->p_full[i]), kTileM / 32);
    }
    ptx::mbar_init(ptx::smem_u32(&b->o_final), 1);
    ptx::mbar_init(ptx::smem_u32(&b->drain), 1);
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_u32(&s_tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem_base;

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
  } else if (warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRopeRegs));
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
  }

  if (warp < 8) {
    // =========================================================== softmax warpgroups
    const int qi = warp >> 2;
    const int r = tid & 127;  // query row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(qi);
    const uint32_t tO = tmem + lane_base + col_o(qi);
    const uint32_t bar_s = ptx::smem_u32(&b->s_full[qi]);
    const uint32_t bar_p = ptx::smem_u32(&b->p_full[qi]);
    const uint32_t bar_ph = ptx::smem_u32(&b->p_half[qi]);
    float m = -INFINITY;  // running max of scale*log2(e)*score (lazily updated)
    uint64_t l2 = f2_pack(0.f, 0.f);  // running row sum, two partial sums
    bool ok = true;
    for (int j = 0; j < nkl; ++j) {
      // warp-uniform decision: tcgen05.ld/st below are warp-collective
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_s, j & 1, abort, p.wait_limit_ns))) { ok = false; break; }
      ptx::tc_fence_after();
      uint32_t sr[128];
      ptx::tmem_ld64(tS, sr);
      ptx::tmem_ld64(tS + 64, sr + 64);
      ptx::tmem_wait_ld();
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      const bool ragged = ragged_last && j == nkl - 1;
      if (ragged) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= last_valid) s[c] = -INFINITY;
      }
      // row max: 3-input max in four independent chains
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c + 8 <= 128; c += 8) {
        mx0 = max3f(mx0, s[c], s[c + 1]);
        mx1 = max3f(mx1, s[c + 2], s[c + 3]);
        mx2 = max3f(mx2, s[c + 4], s[c + 5]);
        mx3 = max3f(mx3, s[c + 6], s[c + 7]);
      }
      mx0 = max3f(mx0, s[124], s[125]);
      mx1 = max3f(mx1, s[126], s[127]);
      const float mcand = max3f(mx0, mx1, fmaxf(mx2, mx3)) * p.scale_log2;
      const bool raise = mcand > m + kRescaleThreshold;
      if (__any_sync(0xffffffffu, raise && j > 0)) {
        // warp-collective O rescale (lanes that keep their max use factor 1)
        const float f = raise ? ex2(m - mcand) : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t ov[16];
          ptx::tmem_ld16(tO + c * 16, ov);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          ptx::tmem_st16(tO + c * 16, ov);
        }
        l2 = f2_mul(l2, f2_pack(f, f));
      }
      if (raise) m = mcand;
      // p = 2^(s * scale * log2(e) - m): packed FFMA2 for the affine part, MUFU ex2,
      // packed FADD2 for the row sum
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m, -m);
      // FMA_MASK: the pairs whose exponential runs on the FMA pipe (compile-time)
      auto store_p = [&](auto fma_mask) {
        constexpr uint32_t FMA_MASK = decltype(fma_mask)::value;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          // P for 32 keys -> 16 packed bf16 columns (8 E4M3 columns), stored as soon as
          // they are ready
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t t2 = f2_fma(f2_pack(s[32 * q4 + 2 * c], s[32 * q4 + 2 * c + 1]), sc2, nm2);
            float e0, e1;
            if ((FMA_MASK >> c) & 1u) exp2_pair_fma(t2, e0, e1);
            else exp2_pair(t2, e0, e1);
            l2 = f2_add(l2, f2_pack(e0, e1));
            if constexpr (PV8) {
              const uint32_t h = e4m3x2(e0, e1);
              pw[c >> 1] = (c & 1) ? (pw[c >> 1] | (h << 16)) : h;
            } else {
              pw[c] = pack_bf16x2(e0, e1);
            }
          }
          if constexpr (PV8) ptx::tmem_st8(tS + 8 * q4, pw);
          else ptx::tmem_st16(tS + 16 * q4, pw);
          if (q4 == 1) {
            // keys 0-63 are in TMEM: the MMA warp may start O += P V on them
            // (every lane's stores complete and fenced, then one arrival for the warp)
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_ph);
          }
        }
      };
      if constexpr (QK8) {
        if (ragged) store_p(std::integral_constant<uint32_t, 0u>{});
        else store_p(std::integral_constant<uint32_t, kExpFmaMaskF8>{});
      } else {
        store_p(std::integral_constant<uint32_t, 0u>{});
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_p);
    }
    // ---- epilogue: O / l -> bf16 -> global, plus the log-sum-exp
    if (__all_sync(0xffffffffu, ok && ptx::mbar_wait(ptx::smem_u32(&b->o_final), 0, abort, p.wait_limit_ns))) {
      ptx::tc_fence_after();
      const int64_t row_in_seq = q_row0 + qi * kTileM + r;
      const bool valid = row_in_seq < seq_len;
      float l_lo, l_hi;
      f2_unpack(l2, l_lo, l_hi);
      const float l = l_lo + l_hi;
      const float inv_l = p.o_scale / l;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) +
                      ((seq_start + row_in_seq) * p.H + head) * static_cast<int64_t>(D) * 2;
      if (n_split > 1) {
        // a share of the keys: publish the unnormalised O row and (m, l) for the merge
        const int g = qi * kTileM + r;
        uint8_t* prow = smem + g * L::kPartStride;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          ptx::tmem_ld32(tO + c * 32, ov);
          ptx::tmem_wait_ld();
          uint4* dst = reinterpret_cast<uint4*>(prow + c * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_uint4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
        }
        reinterpret_cast<float2*>(smem + L::kPartMl)[g] = make_float2(m, l);
      }
#pragma unroll 1
      for (int c = 0; c < (n_split > 1 ? 0 : D / 32); ++c) {
        uint32_t ov[32];
        ptx::tmem_ld32(tO + c * 32, ov);
        ptx::tmem_wait_ld();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l,
                                __uint_as_float(ov[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (valid && n_split == 1 && p.lse != nullptr)
        p.lse[(seq_start + row_in_seq) * p.H + head] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    if (n_split > 1) {
      ptx::cluster_sync_all();  // every CTA of the cluster has published its partial rows
      merge_split_rows<D>(smem, p, split, n_split, q_row0, seq_len, seq_start, head, tid);
      ptx::cluster_sync_all();  // no CTA leaves while another may still read its memory
    }
  } else if (warp == kWarpTma || warp == kWarpTmaV) {
    // =========================================================== TMA producers
    // warp 12 loads Q once and then the K ring; warp 14 loads the V ring.
    if (lane == 0) {
      const bool is_k = warp == kWarpTma;
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      const int stages = is_k ? kKStages : kVStages;
      const uint32_t ring = is_k ? L::kK : L::kV;
      uint64_t* full = is_k ? b->k_full : b->v_full;
      uint64_t* empty = is_k ? b->k_empty : b->v_empty;
      ptx::prefetch_tmap(tm);
      const int x0 = head * D;
      const uint32_t q_full = ptx::smem_u32(&b->q_full);
      int issued = 0;  // tiles issued into this ring
      if (!*abort) {
        if (is_k) {
          ptx::prefetch_tmap(&tm_q);
          ptx::mbar_arrive_expect_tx(q_full, 2 * kQKBytes);
          for (int qi = 0; qi < 2; ++qi)
            for (int blk = 0; blk < kQKBoxes; ++blk)
              ptx::tma_load_2d(ptx::smem_u32(smem + (qi ? L::kQ1 : L::kQ0) + blk * 16384), &tm_q,
                               x0 + blk * 64, static_cast<int>(seq_start + q_row0 + qi * kTileM),
                               q_full);
        }
        for (int j = 0; j < nkl; ++j) {
          const int st = j % stages;
          if (j >= stages &&
              !ptx::mbar_wait(ptx::smem_u32(&empty[st]), ((j / stages) - 1) & 1, abort, p.wait_limit_ns))
            break;
          const int y = static_cast<int>(seq_start + static_cast<int64_t>(kb0 + j) * kTileN);
          const uint32_t f = ptx::smem_u32(&full[st]);
          ptx::mbar_arrive_expect_tx(f, is_k ? kQKBytes : kVBytes);
          const int boxes = is_k ? kQKBoxes : kVBoxes;
          for (int blk = 0; blk < boxes; ++blk)
            ptx::tma_load_2d(ptx::smem_u32(smem + ring + st * L::kTile + blk * 16384), tm,
                             x0 + blk * 64, y, f);
          ++issued;
        }
        // drain: no copy may still be in flight into shared memory when the CTA exits
        // (normally these phases completed long ago and the waits return at once)
        volatile int never = 0;
        if (is_k) ptx::mbar_wait(q_full, 0, &never);
        for (int j = (issued > stages ? issued - stages : 0); j < issued; ++j)
          ptx::mbar_wait(ptx::smem_u32(&full[j % stages]), (j / stages) & 1, &never);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // =========================================================== MMA issuer
    // The whole warp runs the issue loop, so control flow and every operand are
    // warp-uniform, and one elected lane issues each tcgen05 instruction. Measured on
    // B200: with a single lane running the loop, a key step (32 MMAs of 64 clocks) took
    // ~3,600 clocks while no wait found its barrier incomplete, i.e. issue, not data,
    // set the pace; the whole-warp form is 6-12 % faster on every workload, same bits.
    {
      const bool leader = ptx::elect_one();
      // every lane waits; the result is made warp-uniform
      auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, p.wait_limit_ns));
      };
      constexpr uint32_t idesc_qk = ptx::make_idesc_bf16_f32(kTileM, kTileN, false);
      constexpr uint32_t idesc_pv = ptx::make_idesc_bf16_f32(kTileM, D, true);
      const uint32_t sbase = ptx::smem_u32(smem);
      bool issued_any = false;
      auto qk = [&](int qi, int st) {
        const uint32_t qa = sbase + (qi ? L::kQ1 : L::kQ0);
        const uint32_t ka = sbase + L::kK + st * L::kTile;
        if constexpr (QK8) {
          constexpr uint32_t idesc_qk8 = ptx::make_idesc_e4m3_f32(kTileM, kTileN);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)  // 32 bytes = 32 E4M3 elements per MMA
            if (leader) ptx::umma_ss_f8(tmem + col_s(qi),
                            ptx::make_smem_desc(qa + kk * 32, 16, 1024, ptx::kSwizzle128B),
                            ptx::make_smem_desc(ka + kk * 32, 16, 1024, ptx::kSwizzle128B),
                            idesc_qk8, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            if (leader) ptx::umma_ss(tmem + col_s(qi), ptx::make_smem_desc(qa + off, 16, 1024, ptx::kSwizzle128B),
                         ptx::make_smem_desc(ka + off, 16, 1024, ptx::kSwizzle128B), idesc_qk,
                         kk > 0);
          }
        }
        if (leader) ptx::umma_commit(ptx::smem_u32(&b->s_full[qi]));
      };
      // O_qi (+)= P_qi V over keys [64 * half, 64 * half + 64)
      auto pv = [&](int qi, int st, bool acc, int half) {
        const uint32_t va = sbase + L::kV + st * L::kTile;
        if constexpr (PV8) {
          // 32 keys per MMA: 8 TMEM columns of E4M3 P, 32 V rows of 128 bytes
          constexpr uint32_t idesc_pv8 = ptx::make_idesc_e4m3_f32_bmn(kTileM, D);
#pragma unroll
          for (int k2 = 0; k2 < kTileN / 64; ++k2) {
            const int kk = half * (kTileN / 64) + k2;
            if (leader) ptx::umma_ts_f8(tmem + col_o(qi), tmem + col_s(qi) + kk * 8,
                            ptx::make_smem_desc(va + kk * 4096, 16384, 1024, ptx::kSwizzle128B),
                            idesc_pv8, (acc || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int k4 = 0; k4 < kTileN / 32; ++k4) {
            const int kk = half * (kTileN / 32) + k4;
            if (leader) ptx::umma_ts(tmem + col_o(qi), tmem + col_s(qi) + kk * 8,
                         ptx::make_smem_desc(va + kk * 2048, 16384, 1024, ptx::kSwizzle128B),
                         idesc_pv, (acc || kk > 0) ? 1u : 0u);
          }
        }
      };
      // both halves, the second once the softmax has stored all of P
      auto pv_tile = [&](int qi, int st, bool acc, int j) -> bool {
        if (!wait(ptx::smem_u32(&b->p_half[qi]), j & 1)) return false;
        ptx::tc_fence_after();
        pv(qi, st, acc, 0);
        if (!wait(ptx::smem_u32(&b->p_full[qi]), j & 1)) return false;
        ptx::tc_fence_after();
        pv(qi, st, acc, 1);
        return true;
      };
      const uint32_t q_wait = ptx::smem_u32(p.use_rope ? &b->q_ready : &b->q_full);
      bool ok = wait(q_wait, 0);
      if (ok) ok = wait(ptx::smem_u32(p.use_rope ? &b->k_ready[0] : &b->k_full[0]), 0);
      if (ok) {
        ptx::tc_fence_after();
        qk(0, 0);
        qk(1, 0);
        if (leader) ptx::umma_commit(ptx::smem_u32(&b->k_empty[0]));
        issued_any = true;
      }
      for (int j = 0; ok && j < nkl; ++j) {
        const int vs = j % kVStages, vph = (j / kVStages) & 1;
        const int ks1 = (j + 1) % kKStages, kph1 = ((j + 1) / kKStages) & 1;
        const bool more = j + 1 < nkl;
        if (!(ok = wait(ptx::smem_u32(&b->v_full[vs]), vph))) break;
        if (!(ok = pv_tile(0, vs, j > 0, j))) break;
        if (more) {
          if (!(ok = wait(ptx::smem_u32(p.use_rope ? &b->k_ready[ks1] : &b->k_full[ks1]), kph1))) break;
          ptx::tc_fence_after();
          qk(0, ks1);
        }
        if (!(ok = pv_tile(1, vs, j > 0, j))) break;
        if (leader) ptx::umma_commit(ptx::smem_u32(&b->v_empty[vs]));
        if (more) {
          qk(1, ks1);
          if (leader) ptx::umma_commit(ptx::smem_u32(&b->k_empty[ks1]));
        }
      }
      if (ok && leader) ptx::umma_commit(ptx::smem_u32(&b->o_final));
      if (issued_any) {
        // all MMAs of this CTA complete before tensor memory is released
        volatile int never = 0;
        if (leader) ptx::umma_commit(ptx::smem_u32(&b->drain));
        ptx::mbar_wait(ptx::smem_u32(&b->drain), 0, &never);
      }
    }
    __syncwarp();
  } else if (warp >= kWarpRope0 && warp < kWarpRope0 + 4) {
    // =========================================================== 3D-RoPE warps
    if (p.use_rope) {
      const int rt = tid - kWarpRope0 * 32;
      // the cos/sin table is read for every K tile: keep a copy in shared memory when it
      // fits (L1 is small next to this kernel's shared-memory footprint)
      const bool tab_in_smem = p.rope.n_entries * 8 <= static_cast<int>(L::kTabBytes);
      if (tab_in_smem) {
        float4* st = reinterpret_cast<float4*>(smem + L::kTab);
        const float4* src = reinterpret_cast<const float4*>(p.rope.table);
        for (int i = rt; i < p.rope.n_entries / 2; i += kRopeThreads) st[i] = __ldg(src + i);
        asm volatile("bar.sync 1, %0;" ::"n"(kRopeThreads) : "memory");
      }
      const uint32_t tab = ptx::smem_u32(smem + L::kTab);
      auto rope_tile = [&](uint8_t* tile, int64_t row0, int nv) {
        if (tab_in_smem) rope_tile_smem<D>(ptx::smem_u32(tile), row0, nv, p.rope, tab, rt);
        else rope_tile_global<D>(tile, row0, nv, p.rope, rt);
      };
      if (ptx::mbar_wait(ptx::smem_u32(&b->q_full), 0, abort, p.wait_limit_ns)) {
        for (int qi = 0; qi < 2; ++qi) {
          const int64_t r0 = q_row0 + qi * kTileM;
          const int64_t rem = seq_len - r0;
          const int nv = rem <= 0 ? 0 : (rem >= kTileM ? kTileM : static_cast<int>(rem));
          rope_tile(smem + (qi ? L::kQ1 : L::kQ0), r0, nv);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_u32(&b->q_ready));
        for (int j = 0; j < nkl; ++j) {
          const int st = j % kKStages, ph = (j / kKStages) & 1;
          if (!ptx::mbar_wait(ptx::smem_u32(&b->k_full[st]), ph, abort, p.wait_limit_ns)) break;
          const int nv = (kb0 + j == nk - 1) ? last_valid : kTileN;
          rope_tile(smem + L::kK + st * L::kTile, static_cast<int64_t>(kb0 + j) * kTileN, nv);
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(ptx::smem_u32(&b->k_ready[st]));
        }
      }
    }
  }

  if (n_split > 1 && warp >= 8) {
    // the two cluster barriers of the softmax warps' merge
    ptx::cluster_sync_all();
    ptx::cluster_sync_all();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) atomicOr(&g_device_error, kDevErrTimeout);
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if ((p.pdl & 2) && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace attn
}  // namespace dit3d
