// Flash-style forward attention with fused 3D-RoPE on a CTA pair (sm_100a
// cta_group::2), head_dim 128.
//
//   o = softmax(q_rot k_rot^T * scale) v     per (sequence, head), non-causal
//
// ("DiT, Flow Matching e 3D Attention", section "3D-RoPE e atencao
// espaco-temporal"; "Por que e absurdamente dificil gerar um filme inteiro usando
// IA", section "Matematica por tras".)
//
// The two CTAs of a cluster run on two SMs and share every tensor-core instruction:
// one MMA of M = 256 rows takes its first 128 rows (and writes its accumulator) in the
// even CTA and the other 128 in the odd CTA, and splits its N extent between them.
// So for a 128-key tile each CTA loads only half of K (its 64 keys: the N of QK^T) and
// half of V (its 64 of the 128 output columns: the N of P V), and rotates only its 64
// K rows -- half the shared-memory operand traffic and half the RoPE work per SM of
// the single-CTA kernel, for the same tensor work.
//
// A pair covers 512 query rows of one head: CTA r holds rows [128 r, 128 r + 128) of
// query tile A (pair rows 0-255) and of query tile B (pair rows 256-511) -- its Q0 and
// Q1 -- and the pair ping-pongs A and B as the single-CTA kernel does Q0 and Q1.
// Per CTA, 512 threads:
//   WG0, WG1  softmax of this CTA's Q0 / Q1 rows (thread = row = TMEM lane).
//   WG2       3D-RoPE of this CTA's Q rows and K halves; it also tells the even CTA
//             when this CTA's K and V halves are ready.
//   warp 12   TMA: Q0, Q1 once, then the K ring (4 slots of 64 rows).
//   warp 13   TMEM allocation (both CTAs) and, in the even CTA only, the MMA issuer.
//   warp 14   TMA: the V ring (4 slots of 128 rows x 64 columns).
// Tensor memory (512 columns per CTA, same map as the single-CTA kernel): S0, S1
// (128 fp32 columns), O0, O1 (128); P overwrites the first 64 columns of its S.
// Cross-CTA signals: the MMA warp's commits arrive on both CTAs' barriers (multicast
// commit); readiness of the odd CTA's Q, K, V halves and P goes to the even CTA's
// barriers by remote mbarrier arrives (release / acquire at cluster scope), one per
// CTA per event after a named barrier of the producing warpgroup.
// Every mbarrier wait is bounded; on expiry the CTA raises an error bit, drains its
// copies and MMAs, meets its peer at the final cluster barrier, frees its tensor
// memory and exits.
#pragma once
#include "attn_fwd.cuh"

namespace dit3d {
namespace attn2 {

using attn::ex2;
using attn::exp2_pair;
using attn::lds128;
using attn::lds128f;
using attn::lds128_ordered;
using attn::Params;
using attn::rope_apply;
using attn::sts128;
using attn::sw128_chunk;

constexpr int kThreads = 512;
constexpr int kD = 128;
constexpr int kTileM = 128;   // rows of one CTA's query tile
constexpr int kPairRows = 512;  // query rows of a pair (two M = 256 MMA tiles)
constexpr int kTileN = 128;   // keys per step (pair total)
constexpr int kHalfN = 64;    // keys per step held by one CTA
constexpr int kSlots = 4;     // K ring and V ring depth
constexpr int kRopeThreads = 128;
constexpr int kWarpRope0 = 8, kWarpTma = 12, kWarpMma = 13, kWarpTmaV = 14;
constexpr int kSoftmaxRegs = 184, kRopeRegs = 80, kCtrlRegs = 64;
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int qi) { return qi ? 128u : 0u; }
__host__ __device__ constexpr uint32_t col_o(int qi) { return qi ? 384u : 256u; }
constexpr float kRescaleThreshold = 8.0f;

struct Smem {
  static constexpr uint32_t kQTile = kTileM * kD * 2;     // 32 KB: 2 blocks of 128 rows
  static constexpr uint32_t kQBlock = kTileM * 128;
  static constexpr uint32_t kKSlot = kHalfN * kD * 2;     // 16 KB: 2 blocks of 64 rows
  static constexpr uint32_t kKBlock = kHalfN * 128;
  static constexpr uint32_t kVSlot = kTileN * 64 * 2;     // 16 KB: 1 block of 128 rows
  static constexpr uint32_t kQ0 = 0, kQ1 = kQTile;
  static constexpr uint32_t kK = 2 * kQTile;
  static constexpr uint32_t kV = kK + kSlots * kKSlot;
  static constexpr uint32_t kTab = kV + kSlots * kVSlot;
  static constexpr uint32_t kTabBytes = 32 * 1024;
  static constexpr uint32_t kBytes = kTab + kTabBytes;
  static constexpr uint32_t kRequest = kBytes + 1024;
};

// Identical layout in both CTAs (multicast commits and remote arrives address the
// same offsets). The "ready" and P barriers are only waited on in the even CTA.
struct Barriers {
  uint64_t q_full, k_full[kSlots], v_full[kSlots];         // local TMA completion
  uint64_t q_ready, k_ready[kSlots], v_ready[kSlots];      // even CTA: both halves ready
  uint64_t p_half[2], p_full[2];                           // even CTA: P of both CTAs
  uint64_t k_empty[kSlots], v_empty[kSlots];               // both: slot free in both CTAs
  uint64_t s_full[2], o_final, drain;                      // both: MMA results
};

// Rotate chunks [c_lo, c_lo + NCH) of row r of a tile in shared memory (token j of its
// sequence): same procedure and bits as attn::rope_tile_smem, restricted to a range.
template <int NCH>
__device__ __forceinline__ void rope_row_range(uint32_t tile, uint32_t block, int r, int j, int c_lo,
                                               const RopeParams& rp, uint32_t tab) {
  const int hw = rp.grid_h * rp.grid_w;
  const int t = j / hw, rr = j - t * hw, h = rr / rp.grid_w, w = rr - h * rp.grid_w;
  const uint32_t row_t = tab + 8u * static_cast<uint32_t>(rp.off0 + t * rp.str0 - 4 * rp.cf0);
  const uint32_t row_h = tab + 8u * static_cast<uint32_t>(rp.off1 + h * rp.str1 - 4 * rp.cf1);
  const uint32_t row_w = tab + 8u * static_cast<uint32_t>(rp.off2 + w * rp.str2 - 4 * rp.cf2);
#pragma unroll
  for (int c0 = 0; c0 < NCH; c0 += 4) {
    uint4 v[4];
    float4 e0[4], e1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c_lo + c0 + u;
      const int a = rope_band_of_pair(rp, 4 * c);
      const uint32_t e = (a == 0 ? row_t : (a == 1 ? row_h : row_w)) + 32u * c;
      v[u] = lds128(tile + sw128_chunk(r, c, block));
      e0[u] = lds128f(e);
      e1[u] = lds128f(e + 16u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      sts128(tile + sw128_chunk(r, c_lo + c0 + u, block), rope_apply(v[u], e0[u], e1[u]));
  }
  const int cs1 = (rp.p1 & 3) ? (rp.p1 >> 2) : -1;
  const int cs2 = (rp.p2 & 3) ? (rp.p2 >> 2) : -1;
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {
    const int c = k ? cs2 : cs1;
    if (c < c_lo || c >= c_lo + NCH || (k && c == cs1)) continue;
    const int a_lo = rope_band_of_pair(rp, 4 * c), a_hi = rope_band_of_pair(rp, 4 * c + 3);
    for (int a = a_lo + 1; a <= a_hi; ++a) {
      if (rope_band_stride(rp, a) == 0) continue;  // an empty middle band
      const uint32_t e = (a == 1 ? row_h : row_w) + 32u * c;
      const uint32_t ad = tile + sw128_chunk(r, c, block);
      sts128(ad, rope_apply(lds128_ordered(ad), lds128f(e), lds128f(e + 16u)));
    }
  }
}

// Generic-table fallback (tables larger than the shared copy).
__device__ __forceinline__ void rope_row_range_global(uint8_t* tile, uint32_t block, int r, int j,
                                                      int c_lo, int n_ch, const RopeParams& rp) {
  const int hw = rp.grid_h * rp.grid_w;
  const int t = j / hw, rr = j - t * hw, h = rr / rp.grid_w, w = rr - h * rp.grid_w;
#pragma unroll 1
  for (int c = c_lo; c < c_lo + n_ch; ++c) {
    uint4* ptr = reinterpret_cast<uint4*>(tile + sw128_chunk(r, c, block));
    *ptr = rope_chunk(rp, rp.table, *ptr, c, t, h, w);
  }
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// true on every participating thread iff it is true on all of them (named barrier id)
__device__ __forceinline__ bool group_all(bool ok, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, %3, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(ok)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_fwd_2sm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ Barriers bars;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int head = blockIdx.y;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;

  // ---- work decode: which sequence and which 512-row unit of it (both CTAs agree)
  const int unit_id = blockIdx.x >> 1;
  int64_t seq_start, seq_len;
  int unit;
  if (p.cu_seqlens == nullptr) {
    const int seq = unit_id / p.pairs_per_dense_seq;
    unit = unit_id - seq * p.pairs_per_dense_seq;
    seq_len = p.dense_len;
    seq_start = static_cast<int64_t>(seq) * p.dense_len;
  } else {
    int acc = 0;
    unit = 0;
    seq_start = 0;
    seq_len = 0;
    for (int s = 0; s < p.n_seq; ++s) {
      const int64_t a = __ldg(p.cu_seqlens + s), e = __ldg(p.cu_seqlens + s + 1);
      const int nu = static_cast<int>((e - a + kPairRows - 1) / kPairRows);
      if (unit_id < acc + nu) {
        unit = unit_id - acc;
        seq_start = a;
        seq_len = e - a;
        break;
      }
      acc += nu;
    }
  }
  // this CTA's two query tiles, within the sequence
  const int64_t q_row0 = static_cast<int64_t>(unit) * kPairRows + rank * kTileM;
  auto q_row = [&](int qi) { return q_row0 + (qi ? 256 : 0); };
  const int nk = static_cast<int>((seq_len + kTileN - 1) / kTileN);
  const int last_valid = static_cast<int>(seq_len - static_cast<int64_t>(nk - 1) * kTileN);

  Barriers* b = &bars;
  volatile int* abort = &s_abort;
  if (tid == 0) {
    s_abort = p.force_timeout ? 1 : 0;
    ptx::mbar_init(ptx::smem_u32(&b->q_full), 1);
    ptx::mbar_init(ptx::smem_u32(&b->q_ready), 2);
    for (int s = 0; s < kSlots; ++s) {
      ptx::mbar_init(ptx::smem_u32(&b->k_full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&b->v_full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&b->k_ready[s]), 2);
      ptx::mbar_init(ptx::smem_u32(&b->v_ready[s]), 2);
      ptx::mbar_init(ptx::smem_u32(&b->k_empty[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&b->v_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(ptx::smem_u32(&b->p_half[i]), 2);
      ptx::mbar_init(ptx::smem_u32(&b->p_full[i]), 2);
      ptx::mbar_init(ptx::smem_u32(&b->s_full[i]), 1);
    }
    ptx::mbar_init(ptx::smem_u32(&b->o_final), 1);
    ptx::mbar_init(ptx::smem_u32(&b->drain), 1);
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) ptx::tmem_alloc_pair(ptx::smem_u32(&s_tmem_base), kTmemCols);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // both CTAs' barriers and tensor memory exist from here on
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem_base;

  // one arrival on the even CTA's copy of barrier `bar`
  auto arrive_leader = [&](uint64_t* bar) {
    const uint32_t a = ptx::smem_u32(bar);
    if (leader) ptx::mbar_arrive(a);
    else ptx::mbar_arrive_cluster(ptx::mapa_shared(a, 0));
  };

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
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(qi);
    const uint32_t tO = tmem + lane_base + col_o(qi);
    const uint32_t bar_s = ptx::smem_u32(&b->s_full[qi]);
    float m = -INFINITY;
    uint64_t l2 = f2_pack(0.f, 0.f);
    bool ok = true;
    // P stored (this CTA's rows) -> one arrival on the even CTA's barrier
    auto signal_p = [&](uint64_t* bar) {
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      named_sync(2 + qi, kTileM);
      if (r == 0) arrive_leader(bar);
    };
    for (int j = 0; j < nk; ++j) {
      // warpgroup-uniform decision: named barriers and warp-collective tcgen05 ops follow
      if (!group_all(ptx::mbar_wait_cluster(bar_s, j & 1, abort), 6 + qi, kTileM)) { ok = false; break; }
      ptx::tc_fence_after();
      uint32_t sr[128];
      ptx::tmem_ld64(tS, sr);
      ptx::tmem_ld64(tS + 64, sr + 64);
      ptx::tmem_wait_ld();
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      if (j == nk - 1 && last_valid < kTileN) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= last_valid) s[c] = -INFINITY;
      }
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
        const float f = raise ? ex2(m - mcand) : 1.f;
#pragma unroll 1
        for (int c = 0; c < kD / 16; ++c) {
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
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m, -m);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pw[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint64_t t2 = f2_fma(f2_pack(s[32 * q4 + 2 * c], s[32 * q4 + 2 * c + 1]), sc2, nm2);
          float e0, e1;
          exp2_pair(t2, e0, e1);
          l2 = f2_add(l2, f2_pack(e0, e1));
          pw[c] = pack_bf16x2(e0, e1);
        }
        ptx::tmem_st16(tS + 16 * q4, pw);
        if (q4 == 1) signal_p(&b->p_half[qi]);
      }
      signal_p(&b->p_full[qi]);
    }
    // ---- epilogue
    if (group_all(ok && ptx::mbar_wait_cluster(ptx::smem_u32(&b->o_final), 0, abort), 6 + qi, kTileM)) {
      ptx::tc_fence_after();
      const int64_t row_in_seq = q_row(qi) + r;
      const bool valid = row_in_seq < seq_len;
      float l_lo, l_hi;
      f2_unpack(l2, l_lo, l_hi);
      const float l = l_lo + l_hi;
      const float inv_l = 1.f / l;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) +
                      ((seq_start + row_in_seq) * p.H + head) * static_cast<int64_t>(kD) * 2;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
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
      if (valid && p.lse != nullptr)
        p.lse[(seq_start + row_in_seq) * p.H + head] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  } else if (warp == kWarpTma || warp == kWarpTmaV) {
    // =========================================================== TMA producers
    if (lane == 0) {
      const bool is_k = warp == kWarpTma;
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      const uint32_t ring = is_k ? L::kK : L::kV;
      const uint32_t slot_bytes = is_k ? L::kKSlot : L::kVSlot;
      uint64_t* full = is_k ? b->k_full : b->v_full;
      uint64_t* empty = is_k ? b->k_empty : b->v_empty;
      ptx::prefetch_tmap(tm);
      const uint32_t q_full = ptx::smem_u32(&b->q_full);
      int issued = 0;
      if (!*abort) {
        if (is_k) {
          ptx::prefetch_tmap(&tm_q);
          ptx::mbar_arrive_expect_tx(q_full, 2 * L::kQTile);
          for (int qi = 0; qi < 2; ++qi)
            for (int blk = 0; blk < kD / 64; ++blk)
              ptx::tma_load_2d(ptx::smem_u32(smem + (qi ? L::kQ1 : L::kQ0) + blk * L::kQBlock),
                               &tm_q, head * kD + blk * 64, static_cast<int>(seq_start + q_row(qi)),
                               q_full);
        }
        for (int j = 0; j < nk; ++j) {
          const int sl = j % kSlots;
          if (j >= kSlots &&
              !ptx::mbar_wait_cluster(ptx::smem_u32(&empty[sl]), ((j / kSlots) - 1) & 1, abort))
            break;
          const uint32_t f = ptx::smem_u32(&full[sl]);
          ptx::mbar_arrive_expect_tx(f, slot_bytes);
          const uint32_t dst = ptx::smem_u32(smem + ring + sl * slot_bytes);
          if (is_k) {
            // this CTA's 64 keys of tile j, all 128 columns
            const int y = static_cast<int>(seq_start + static_cast<int64_t>(j) * kTileN + rank * kHalfN);
            for (int blk = 0; blk < kD / 64; ++blk)
              ptx::tma_load_2d(dst + blk * L::kKBlock, tm, head * kD + blk * 64, y, f);
          } else {
            // all 128 keys of tile j, this CTA's 64 of the 128 value columns
            const int y = static_cast<int>(seq_start + static_cast<int64_t>(j) * kTileN);
            ptx::tma_load_2d(dst, tm, head * kD + static_cast<int>(rank) * 64, y, f);
          }
          ++issued;
        }
        volatile int never = 0;
        if (is_k) ptx::mbar_wait(q_full, 0, &never);
        for (int j = (issued > kSlots ? issued - kSlots : 0); j < issued; ++j)
          ptx::mbar_wait(ptx::smem_u32(&full[j % kSlots]), (j / kSlots) & 1, &never);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // =========================================================== MMA issuer (even CTA)
    // whole warp, one elected lane issuing (warp-uniform control flow and operands)
    if (leader) {
      const bool issuer = ptx::elect_one();
      auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait_cluster(bar, parity, abort));
      };
      constexpr uint32_t idesc_qk = ptx::make_idesc_bf16_f32(256, kTileN, false);
      constexpr uint32_t idesc_pv = ptx::make_idesc_bf16_f32(256, kD, true);
      const uint32_t sbase = ptx::smem_u32(smem);
      bool issued_any = false;
      auto qk = [&](int qi, int sl) {
        const uint32_t qa = sbase + (qi ? L::kQ1 : L::kQ0);
        const uint32_t ka = sbase + L::kK + sl * L::kKSlot;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          if (issuer) ptx::umma_ss_pair(tmem + col_s(qi),
                            ptx::make_smem_desc(qa + (kk >> 2) * L::kQBlock + (kk & 3) * 32, 16,
                                                1024, ptx::kSwizzle128B),
                            ptx::make_smem_desc(ka + (kk >> 2) * L::kKBlock + (kk & 3) * 32, 16,
                                                1024, ptx::kSwizzle128B),
                            idesc_qk, kk > 0);
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->s_full[qi]));
      };
      auto pv = [&](int qi, int sl, bool acc, int half) {
        const uint32_t va = sbase + L::kV + sl * L::kVSlot;
#pragma unroll
        for (int k4 = 0; k4 < kTileN / 32; ++k4) {
          const int kk = half * (kTileN / 32) + k4;
          if (issuer) ptx::umma_ts_pair(tmem + col_o(qi), tmem + col_s(qi) + kk * 8,
                            ptx::make_smem_desc(va + kk * 2048, L::kVSlot, 1024, ptx::kSwizzle128B),
                            idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto pv_tile = [&](int qi, int sl, bool acc, int j) -> bool {
        if (!wait(ptx::smem_u32(&b->p_half[qi]), j & 1)) return false;
        ptx::tc_fence_after();
        pv(qi, sl, acc, 0);
        if (!wait(ptx::smem_u32(&b->p_full[qi]), j & 1)) return false;
        ptx::tc_fence_after();
        pv(qi, sl, acc, 1);
        return true;
      };
      bool ok = wait(ptx::smem_u32(&b->q_ready), 0);
      if (ok) ok = wait(ptx::smem_u32(&b->k_ready[0]), 0);
      if (ok) {
        ptx::tc_fence_after();
        qk(0, 0);
        qk(1, 0);
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->k_empty[0]));
        issued_any = true;
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int sl = j % kSlots, ph = (j / kSlots) & 1;
        const int sl1 = (j + 1) % kSlots, ph1 = ((j + 1) / kSlots) & 1;
        const bool more = j + 1 < nk;
        if (!(ok = wait(ptx::smem_u32(&b->v_ready[sl]), ph))) break;
        if (!(ok = pv_tile(0, sl, j > 0, j))) break;
        if (more) {
          if (!(ok = wait(ptx::smem_u32(&b->k_ready[sl1]), ph1))) break;
          ptx::tc_fence_after();
          qk(0, sl1);
        }
        if (!(ok = pv_tile(1, sl, j > 0, j))) break;
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->v_empty[sl]));
        if (more) {
          qk(1, sl1);
          if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->k_empty[sl1]));
        }
      }
      if (ok && issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->o_final));
      if (issued_any) {
        volatile int never = 0;
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&b->drain));
        ptx::mbar_wait_cluster(ptx::smem_u32(&b->drain), 0, &never);
      }
    }
    __syncwarp();
  } else if (warp >= kWarpRope0 && warp < kWarpRope0 + 4) {
    // =========================================================== RoPE + readiness
    const int rt = tid - kWarpRope0 * 32;
    const bool rope = p.use_rope != 0;
    const bool tab_in_smem = rope && p.rope.n_entries * 8 <= static_cast<int>(L::kTabBytes);
    if (tab_in_smem) {
      float4* st = reinterpret_cast<float4*>(smem + L::kTab);
      const float4* src = reinterpret_cast<const float4*>(p.rope.table);
      for (int i = rt; i < p.rope.n_entries / 2; i += kRopeThreads) st[i] = __ldg(src + i);
      named_sync(1, kRopeThreads);
    }
    const uint32_t tab = ptx::smem_u32(smem + L::kTab);
    // this warpgroup's part of an event is done -> one arrival on the even CTA's barrier
    auto signal = [&](uint64_t* bar) {
      ptx::fence_proxy_async_smem();
      named_sync(4, kRopeThreads);
      if (rt == 0) arrive_leader(bar);
    };
    if (group_all(ptx::mbar_wait(ptx::smem_u32(&b->q_full), 0, abort), 5, kRopeThreads)) {
      if (rope) {
        for (int qi = 0; qi < 2; ++qi) {
          const int64_t row = q_row(qi) + rt;
          if (row < seq_len) {
            uint8_t* tile = smem + (qi ? L::kQ1 : L::kQ0);
            if (tab_in_smem)
              rope_row_range<kD / 8>(ptx::smem_u32(tile), L::kQBlock, rt, static_cast<int>(row), 0,
                                     p.rope, tab);
            else
              rope_row_range_global(tile, L::kQBlock, rt, static_cast<int>(row), 0, kD / 8, p.rope);
          }
        }
      }
      signal(&b->q_ready);
      // K halves (64 rows): two threads per row, each half of the row's 16 chunks
      const int kr = rt & (kHalfN - 1), part = rt / kHalfN;
      for (int j = 0; j < nk; ++j) {
        const int sl = j % kSlots, ph = (j / kSlots) & 1;
        if (!group_all(ptx::mbar_wait(ptx::smem_u32(&b->k_full[sl]), ph, abort), 5, kRopeThreads))
          break;
        const int64_t row = static_cast<int64_t>(j) * kTileN + rank * kHalfN + kr;
        if (rope && row < seq_len) {
          uint8_t* tile = smem + L::kK + sl * L::kKSlot;
          if (tab_in_smem)
            rope_row_range<kD / 16>(ptx::smem_u32(tile), L::kKBlock, kr, static_cast<int>(row),
                                    part * (kD / 16), p.rope, tab);
          else
            rope_row_range_global(tile, L::kKBlock, kr, static_cast<int>(row), part * (kD / 16),
                                  kD / 16, p.rope);
        }
        signal(&b->k_ready[sl]);
        // the V half of this tile: tell the even CTA once it has landed here
        if (rt == 0) {
          if (ptx::mbar_wait(ptx::smem_u32(&b->v_full[sl]), ph, abort)) arrive_leader(&b->v_ready[sl]);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) atomicOr(&g_device_error, kDevErrTimeout);
  ptx::cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace attn2
}  // namespace dit3d
