// Linear layers of the DiT block on tcgen05, with fused epilogues.
//
//   y = x w^T (+ bias)            "Por que e absurdamente dificil gerar um filme inteiro
//                                 usando IA", section "Matematica por tras": Y = X W
//   y = gelu(y)    (optional)     the MLP of "DiT, Flow Matching e 3D Attention",
//                                 section "A ruptura da U-Net" (tanh form: a reading)
//   out = res + alpha_g * y       the adaLN-Zero gate of the same section (optional)
//
// x [M, K] and w [N, K] bf16 (w in the [out, in] layout of a linear layer), fp32
// accumulation in tensor memory, bf16 out. The gate fuses the block's residual update
// into the projection's epilogue, so the attention output projection and the second
// MLP layer write the block output directly.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles in grouped order (16
// M-tiles share each sweep over N, so the A rows and B columns of one wave stay in
// L2). 256 threads:
//   warp 0     TMA producer: A (128 x 64) and B (256 x 64) boxes with the 128-byte
//              swizzle into a 4-stage ring (48 KB per stage)
//   warp 1     TMEM allocator and MMA issuer (whole warp, one elected lane):
//              4 x tcgen05.mma M128 N256 K16 per stage into one of two 256-column
//              accumulators
//   warps 4-7  epilogue: thread = output row = TMEM lane; tcgen05.ld 32 columns at a
//              time, bias / GELU / gate in fp32, one bf16 rounding, 16-byte stores
// The two accumulators let the epilogue of tile i overlap the main loop of tile i+1.
// Every mbarrier wait is bounded; on expiry the CTA drains its copies and MMAs, frees
// its tensor memory and reports DIT_ERR_TIMEOUT through the device error word.
#pragma once
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace dit3d {
namespace lin {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kThreads = 256;
constexpr int kGroupM = 16;
constexpr uint32_t kABytes = kBM * kBK * 2;            // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;            // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;    // 48 KB
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024;
constexpr uint32_t kTmemCols = 2 * kBN;

struct Params {
  const __nv_bfloat16* bias;   // [N] or null
  const __nv_bfloat16* res;    // [M, N] or null (then out = y)
  const __nv_bfloat16* alpha;  // [M / rows_per_group, N] when res is given
  __nv_bfloat16* out;          // [M, N]
  int64_t M;
  int32_t N, K;
  int32_t act;                 // 0: none, 1: GELU (tanh form)
  int64_t rows_per_group;
  int32_t tiles_m, tiles_n, k_blocks;
  int32_t force_timeout;
  float acc_scale;             // multiplies the accumulator (x_scale * w_scale for E4M3; 1 else)
  uint64_t wait_limit_ns;      // bound of the waits that give up the CTA's work (2 s by default)
};

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& tm, int& tn) {
  const int per_group = kGroupM * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * kGroupM;
  const int gm = min(kGroupM, p.tiles_m - first_m);
  const int r = t - g * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float gelu_tanh(float y) {
  const float c = 0.7978845608028654f;  // sqrt(2 / pi)
  const float u = c * fmaf(0.044715f * y, y * y, y);
  return 0.5f * y * (1.f + tanh_approx(u));
}

// Epilogue of 8 consecutive columns (one 16-byte store) of one row.
__device__ __forceinline__ uint4 epilogue8(const float* acc, const Params& p, int64_t row, int col) {
  float y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = acc[e] * p.acc_scale;
  if (p.bias != nullptr) {
    const uint4 bv = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      y[2 * e] += bf16lo(bw[e]);
      y[2 * e + 1] += bf16hi(bw[e]);
    }
  }
  if (p.act == 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = gelu_tanh(y[e]);
  }
  uint32_t o[4];
  if (p.res != nullptr) {
    const uint4 rv = *reinterpret_cast<const uint4*>(p.res + row * p.N + col);
    const uint4 av = __ldg(reinterpret_cast<const uint4*>(p.alpha + (row / p.rows_per_group) * p.N + col));
    const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w}, aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // a zero gate returns the residual's bits (the adaLN-Zero identity)
      const float a0 = bf16lo(aw[e]), a1 = bf16hi(aw[e]);
      const float r0 = bf16lo(rw[e]), r1 = bf16hi(rw[e]);
      const float o0 = a0 == 0.f ? r0 : fmaf(a0, y[2 * e], r0);
      const float o1 = a1 == 0.f ? r1 : fmaf(a1, y[2 * e + 1], r1);
      o[e] = pack_bf16x2(o0, o1);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// F8: x and w arrive as FP8 E4M3 codes; a stage then holds 128 elements of K per row
// (the same 128 bytes) and each MMA is kind::f8f6f4 with K = 32; the epilogue applies
// x_scale * w_scale before the bias.
template <bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
              const Params p) {
  constexpr int kKPerStage = F8 ? 128 : kBK;  // elements of K per 128-byte row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles = p.tiles_m * p.tiles_n;
  volatile int* abort = &s_abort;

  if (tid == 0) {
    s_abort = p.force_timeout ? 1 : 0;
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&acc_full[b]), 1);
      ptx::mbar_init(ptx::smem_u32(&acc_empty[b]), kBM);
    }
    ptx::mbar_init(ptx::smem_u32(&drain), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&s_tmem), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_a);
      ptx::prefetch_tmap(&tm_b);
      int it = 0;
      bool ok = !*abort;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, p, tm, tn);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages &&
              !ptx::mbar_wait(ptx::smem_u32(&empty[s]), ((it / kStages) - 1) & 1, abort, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t f = ptx::smem_u32(&full[s]);
          const uint32_t dst = ptx::smem_u32(smem + s * kStageBytes);
          ptx::mbar_arrive_expect_tx(f, kStageBytes);
          ptx::tma_load_2d(dst, &tm_a, kb * kKPerStage, tm * kBM, f);
          ptx::tma_load_2d(dst + kABytes, &tm_b, kb * kKPerStage, tn * kBN, f);
        }
      }
      // no copy may still be in flight into shared memory when the CTA exits
      volatile int never = 0;
      for (int j = (it > kStages ? it - kStages : 0); j < it; ++j)
        ptx::mbar_wait(ptx::smem_u32(&full[j % kStages]), (j / kStages) & 1, &never);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The whole warp runs the loop (warp-uniform control flow and operands); one
    // elected lane issues each tcgen05 instruction.
    {
      const bool leader = ptx::elect_one();
      auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, p.wait_limit_ns));
      };
      constexpr uint32_t idesc = ptx::make_idesc_bf16_f32(kBM, kBN, false);
      int it = 0, local = 0;
      bool ok = true, issued = false;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++local) {
        const int b = local & 1;
        const uint32_t acc = tmem + static_cast<uint32_t>(b * kBN);
        if (local >= 2 && !wait(ptx::smem_u32(&acc_empty[b]), ((local / 2) - 1) & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!wait(ptx::smem_u32(&full[s]), (it / kStages) & 1)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(smem + s * kStageBytes), b0 = a0 + kABytes;
          // four MMAs of 32 bytes of K each (16 bf16 or 32 E4M3 elements)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = ptx::make_smem_desc(a0 + kk * 32, 16, 1024, ptx::kSwizzle128B);
            const uint64_t db = ptx::make_smem_desc(b0 + kk * 32, 16, 1024, ptx::kSwizzle128B);
            if (!leader) continue;
            if constexpr (F8)
              ptx::umma_ss_f8(acc, da, db, ptx::make_idesc_e4m3_f32(kBM, kBN),
                              (kb > 0 || kk > 0) ? 1u : 0u);
            else
              ptx::umma_ss(acc, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          if (leader) ptx::umma_commit(ptx::smem_u32(&empty[s]));
          issued = true;
        }
        if (!ok) break;
        if (leader) ptx::umma_commit(ptx::smem_u32(&acc_full[b]));
      }
      if (issued) {
        // every MMA of this CTA completes before tensor memory is released
        volatile int never = 0;
        if (leader) ptx::umma_commit(ptx::smem_u32(&drain));
        ptx::mbar_wait(ptx::smem_u32(&drain), 0, &never);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ epilogue
    const int r = tid - 128;  // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int b = local & 1;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&acc_full[b]), (local / 2) & 1, abort, p.wait_limit_ns)))
        break;
      ptx::tc_fence_after();
      int tm, tn;
      tile_coords(t, p, tm, tn);
      const int64_t row = static_cast<int64_t>(tm) * kBM + r;
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + static_cast<uint32_t>(b * kBN + c * 32) + lane_base, v);
        ptx::tmem_wait_ld();
        const int col0 = tn * kBN + c * 32;
        if (row_ok) {
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            const int col = col0 + g8 * 8;
            if (col < p.N) {
              float acc8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) acc8[e] = __uint_as_float(v[g8 * 8 + e]);
              *reinterpret_cast<uint4*>(p.out + row * p.N + col) = epilogue8(acc8, p, row, col);
            }
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(ptx::smem_u32(&acc_empty[b]));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) atomicOr(&g_device_error, kDevErrTimeout);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------
// CTA-pair form (cta_group::2): a cluster of two CTAs computes a 256 x 256 output
// tile with M = 256 MMAs issued by the even CTA. Each CTA loads its own 128 rows of A
// and one half (128 rows) of the B tile, so a k-block costs each SM 32 KB of loads
// instead of 48 KB, and the 6-stage ring holds more k-blocks in flight. Each CTA's
// TMEM holds its 128 rows x 256 columns (two buffers). Both CTAs' loads complete on
// the even CTA's full[s] (cta_group::2 tensor loads; the even CTA's producer expects
// both CTAs' bytes), which is all the MMA thread waits for; the MMA commits arrive on
// both CTAs' barriers (multicast commit), so each producer waits for its own empty[s];
// the epilogue of each CTA signals the even CTA's acc_empty[b] once its 128 threads
// have drained buffer b. No load is multicast.
constexpr int kStages2 = 6;
constexpr int kGroupM2 = 8;                            // pair tiles (256 rows) per group
constexpr uint32_t kHalfBytes = kBM * kBK * 2;         // 16 KB: A half or B half
constexpr uint32_t kStageBytes2 = 2 * kHalfBytes;      // 32 KB per CTA per stage
constexpr uint32_t kSmemBytes2 = kStages2 * kStageBytes2 + 1024;

__device__ __forceinline__ void pair_tile_coords(int t, const Params& p, int& tp, int& tn) {
  const int tiles_p = (p.tiles_m + 1) / 2;
  const int per_group = kGroupM2 * p.tiles_n;
  const int g = t / per_group;
  const int first = g * kGroupM2;
  const int gm = min(kGroupM2, tiles_p - first);
  const int r = t - g * per_group;
  tp = first + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// F8: E4M3 x and w, 128 elements of K per 128-byte stage row, kind::f8f6f4 MMAs (as in
// the single-CTA kernel).
template <bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
linear_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const Params p) {
  constexpr int kKPerStage = F8 ? 128 : kBK;  // elements of K per 128-byte row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full[kStages2], empty[kStages2], acc_full[2], acc_empty[2],
      drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int n_tiles = ((p.tiles_m + 1) / 2) * p.tiles_n;
  volatile int* abort = &s_abort;

  if (tid == 0) {
    s_abort = p.force_timeout ? 1 : 0;
    for (int s = 0; s < kStages2; ++s) {
      ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&acc_full[b]), 1);
      ptx::mbar_init(ptx::smem_u32(&acc_empty[b]), 2);
    }
    ptx::mbar_init(ptx::smem_u32(&drain), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) ptx::tmem_alloc_pair(ptx::smem_u32(&s_tmem), kTmemCols);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // both CTAs' barriers and tensor memory exist from here on
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  // one arrival on the even CTA's copy of barrier `bar`
  auto arrive_leader = [&](uint64_t* bar) {
    const uint32_t a = ptx::smem_u32(bar);
    if (leader) ptx::mbar_arrive(a);
    else ptx::mbar_arrive_cluster(ptx::mapa_shared(a, 0));
  };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_a);
      ptx::prefetch_tmap(&tm_b);
      int it = 0;
      bool ok = !*abort;
      for (int t = cluster; ok && t < n_tiles; t += n_clusters) {
        int tp, tn;
        pair_tile_coords(t, p, tp, tn);
        const int ya = tp * 2 * kBM + static_cast<int>(rank) * kBM;
        const int yb = tn * kBN + static_cast<int>(rank) * kBM;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages2;
          if (it >= kStages2 &&
              !ptx::mbar_wait_cluster(ptx::smem_u32(&empty[s]), ((it / kStages2) - 1) & 1, abort)) {
            ok = false;
            break;
          }
          // both CTAs' bytes land on the even CTA's full[s]
          const uint32_t f_even = ptx::mapa_shared(ptx::smem_u32(&full[s]), 0);
          const uint32_t dst = ptx::smem_u32(smem + s * kStageBytes2);
          if (leader) ptx::mbar_arrive_expect_tx(ptx::smem_u32(&full[s]), 2 * kStageBytes2);
          ptx::tma_load_2d_pair(dst, &tm_a, kb * kKPerStage, ya, f_even);
          ptx::tma_load_2d_pair(dst + kHalfBytes, &tm_b, kb * kKPerStage, yb, f_even);
        }
      }
      // no copy may still be in flight into either CTA's shared memory when the pair
      // exits: the even CTA's full[s] counts both CTAs' bytes, and both producers issue
      // the same stages (each waits for the same multicast commits), so the even CTA
      // waits for them and the cluster barrier at the end holds the odd CTA until then
      if (leader) {
        volatile int never = 0;
        for (int j = (it > kStages2 ? it - kStages2 : 0); j < it; ++j)
          ptx::mbar_wait(ptx::smem_u32(&full[j % kStages2]), (j / kStages2) & 1, &never);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer (even CTA)
    // whole warp, one elected lane issuing (as in the single-CTA kernel)
    if (leader) {
      const bool issuer = ptx::elect_one();
      constexpr uint32_t idesc = F8 ? ptx::make_idesc_e4m3_f32(2 * kBM, kBN)
                                    : ptx::make_idesc_bf16_f32(2 * kBM, kBN, false);
      int it = 0, local = 0;
      bool ok = true, issued = false;
      for (int t = cluster; ok && t < n_tiles; t += n_clusters, ++local) {
        const int b = local & 1;
        const uint32_t acc = tmem + static_cast<uint32_t>(b * kBN);
        if (local >= 2 &&
            !__all_sync(0xffffffffu, ptx::mbar_wait_cluster(ptx::smem_u32(&acc_empty[b]),
                                                            ((local / 2) - 1) & 1, abort))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages2;
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&full[s]), (it / kStages2) & 1, abort))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(smem + s * kStageBytes2), b0 = a0 + kHalfBytes;
          // four MMAs of 32 bytes of K each (16 bf16 or 32 E4M3 elements)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = ptx::make_smem_desc(a0 + kk * 32, 16, 1024, ptx::kSwizzle128B);
            const uint64_t db = ptx::make_smem_desc(b0 + kk * 32, 16, 1024, ptx::kSwizzle128B);
            if (!issuer) continue;
            if constexpr (F8) ptx::umma_ss_pair_f8(acc, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            else ptx::umma_ss_pair(acc, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&empty[s]));
          issued = true;
        }
        if (!ok) break;
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&acc_full[b]));
      }
      if (issued) {
        volatile int never = 0;
        if (issuer) ptx::umma_commit_pair(ptx::smem_u32(&drain));
        ptx::mbar_wait_cluster(ptx::smem_u32(&drain), 0, &never);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ epilogue
    const int r = tid - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    int local = 0;
    for (int t = cluster; t < n_tiles; t += n_clusters, ++local) {
      const int b = local & 1;
      if (!__all_sync(0xffffffffu,
                      ptx::mbar_wait_cluster(ptx::smem_u32(&acc_full[b]), (local / 2) & 1, abort)))
        break;
      ptx::tc_fence_after();
      int tp, tn;
      pair_tile_coords(t, p, tp, tn);
      const int64_t row = static_cast<int64_t>(tp) * 2 * kBM + rank * kBM + r;
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + static_cast<uint32_t>(b * kBN + c * 32) + lane_base, v);
        ptx::tmem_wait_ld();
        const int col0 = tn * kBN + c * 32;
        if (row_ok) {
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            const int col = col0 + g8 * 8;
            if (col < p.N) {
              float acc8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) acc8[e] = __uint_as_float(v[g8 * 8 + e]);
              *reinterpret_cast<uint4*>(p.out + row * p.N + col) = epilogue8(acc8, p, row, col);
            }
          }
        }
      }
      ptx::tc_fence_before();
      named_sync(1, 128);
      if (r == 0) arrive_leader(&acc_empty[b]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  if (tid == 0 && *abort) atomicOr(&g_device_error, kDevErrTimeout);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace lin
}  // namespace dit3d
