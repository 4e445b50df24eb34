// C ABI of libdit3d (declared in include/dit3d.h): argument validation, tensor
// maps, the RoPE cos/sin table cache and kernel launches. All device work is in
// the kernels of adaln.cuh, rope3d.cuh and attn_fwd.cuh.
#include <algorithm>
#include <type_traits>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <thread>
#include <tuple>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/dit3d.h"
#include "adaln.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_2sm.cuh"
#include "common.cuh"
#include "flow_euler.cuh"
#include "linear.cuh"
#include "quant.cuh"
#include "rope3d.cuh"

using namespace dit3d;

namespace {

std::mutex g_mu;
int g_force_timeout = 0;
uint64_t g_wait_limit_ns = 2000000000ull;  // bound of the single-CTA kernels' waits
int g_linear_variant = 1;  // 1 (default): CTA pairs per 256x256 tile; 0: one CTA per 128x256 tile
int g_attn_variant = 0;  // 0: one CTA per query-tile pair; 1: CTA pairs (head_dim 128)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 check, cached per device.
int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_DEVICE;
  static std::map<int, int> ok_cache;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = ok_cache.find(dev);
  if (it == ok_cache.end()) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return DIT_ERR_DEVICE;
    it = ok_cache.emplace(dev, major == 10 ? DIT_OK : DIT_ERR_DEVICE).first;
  }
  return it->second;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_LAUNCH; }

int check_rows_groups(int64_t rows, int32_t D, int64_t rows_per_group) {
  if (rows < 0 || D <= 0 || (D % 8) != 0 || rows_per_group <= 0 || (rows % rows_per_group) != 0)
    return DIT_ERR_SHAPE;
  if (rows > INT32_MAX) return DIT_ERR_SHAPE;  // one CTA per row
  return DIT_OK;
}

// Sequence layout shared by RoPE and attention: fills the host copy of the lengths.
int check_seqs(int64_t rows, int32_t n_seq, const int32_t* cu_dev, const int32_t* cu_host,
               std::vector<int64_t>* lens) {
  if (n_seq <= 0) return DIT_ERR_SHAPE;
  lens->clear();
  if (cu_dev == nullptr && cu_host == nullptr) {
    if (rows % n_seq != 0) return DIT_ERR_SHAPE;
    lens->assign(n_seq, rows / n_seq);
    return DIT_OK;
  }
  if (cu_dev == nullptr || cu_host == nullptr) return DIT_ERR_NULL;
  if (cu_host[0] != 0 || cu_host[n_seq] != rows) return DIT_ERR_SEQLENS;
  for (int s = 0; s < n_seq; ++s) {
    if (cu_host[s + 1] < cu_host[s]) return DIT_ERR_SEQLENS;
    lens->push_back(static_cast<int64_t>(cu_host[s + 1]) - cu_host[s]);
  }
  return DIT_OK;
}

// ---------------------------------------------------------------- RoPE tables
struct TableKey {
  int dev, gh, gw, dt, dh, dw, t_ext, t0, h0, w0;
  uint32_t base_bits;
  bool operator<(const TableKey& o) const {
    return std::tie(dev, gh, gw, dt, dh, dw, t_ext, t0, h0, w0, base_bits) <
           std::tie(o.dev, o.gh, o.gw, o.dt, o.dh, o.dw, o.t_ext, o.t0, o.h0, o.w0, o.base_bits);
  }
};
std::map<TableKey, float2*> g_tables;

int validate_rope(const dit_rope3d_desc* r, int32_t d, const std::vector<int64_t>& lens,
                  int* t_ext) {
  if (r->grid_h < 1 || r->grid_w < 1 || r->grid_h > 2047 || r->grid_w > 1023) return DIT_ERR_SHAPE;
  if (r->d_t < 0 || r->d_h < 0 || r->d_w < 0 || (r->d_t | r->d_h | r->d_w) & 1) return DIT_ERR_SHAPE;
  if (r->d_t + r->d_h + r->d_w != d) return DIT_ERR_SHAPE;
  if (!(r->base > 1.0f) || !std::isfinite(r->base)) return DIT_ERR_SHAPE;
  if (r->t0 < 0 || r->h0 < 0 || r->w0 < 0) return DIT_ERR_SHAPE;
  const int64_t fr = static_cast<int64_t>(r->grid_h) * r->grid_w;
  int64_t tmax = 1;
  for (int64_t L : lens) {
    if (L % fr != 0) return DIT_ERR_SHAPE;
    tmax = std::max<int64_t>(tmax, L / fr);
  }
  if (tmax > 2047) return DIT_ERR_SHAPE;
  *t_ext = static_cast<int>((tmax + 31) / 32 * 32);  // round up: fewer distinct tables
  return DIT_OK;
}

// Section parameters of the RoPE table (layout described in rope3d.cuh).
void rope_table_layout(const dit_rope3d_desc* r, int t_ext, RopeParams* rp) {
  const int width[3] = {r->d_t, r->d_h, r->d_w};
  const int ext[3] = {t_ext, r->grid_h, r->grid_w};
  const int first_pair[3] = {0, r->d_t / 2, (r->d_t + r->d_h) / 2};
  int off[3], str[3], cf[3], n = 0;
  for (int a = 0; a < 3; ++a) {
    const int np = width[a] / 2;
    off[a] = n;
    str[a] = 0;
    cf[a] = 0;
    if (np == 0) continue;
    cf[a] = first_pair[a] / 4;
    const int nchunks = (first_pair[a] + np - 1) / 4 - cf[a] + 1;
    str[a] = 4 * nchunks + 2;  // an odd number of 16-byte units per position
    n += ext[a] * str[a];
  }
  rp->grid_h = r->grid_h;
  rp->grid_w = r->grid_w;
  rp->p1 = first_pair[1];
  rp->p2 = first_pair[2];
  rp->off0 = off[0]; rp->off1 = off[1]; rp->off2 = off[2];
  rp->str0 = str[0]; rp->str1 = str[1]; rp->str2 = str[2];
  rp->cf0 = cf[0]; rp->cf1 = cf[1]; rp->cf2 = cf[2];
  rp->n_entries = n;
}

// What the fill kernel needs besides the layout: band widths, extents, offsets,
// first pairs and the base.
RopeTableSpec rope_table_spec(const dit_rope3d_desc* r, int t_ext, const RopeParams& rp) {
  RopeTableSpec s{};
  s.base = r->base;
  const int width[3] = {r->d_t, r->d_h, r->d_w};
  const int ext[3] = {t_ext, r->grid_h, r->grid_w};
  const int offs[3] = {r->t0, r->h0, r->w0};
  const int first_pair[3] = {0, r->d_t / 2, (r->d_t + r->d_h) / 2};
  for (int a = 0; a < 3; ++a) {
    s.width[a] = width[a];
    s.ext[a] = ext[a];
    s.offs[a] = offs[a];
    s.first_pair[a] = first_pair[a];
  }
  s.n_fill = std::max(rp.n_entries, 2);
  return s;
}

// Writes the table of descriptor `r` into `dst` (at least max(n_entries, 2) float2) with
// one kernel on `stream`: no host buffer, no copy.
int fill_table(float2* dst, const dit_rope3d_desc* r, int t_ext, const RopeParams& rp,
               cudaStream_t stream) {
  const RopeTableSpec spec = rope_table_spec(r, t_ext, rp);
  rope_table_fill_kernel<<<(spec.n_fill + 255) / 256, 256, 0, stream>>>(dst, rp, spec);
  return launch_status();
}

// Cached device copy of the table for a descriptor (allocated once per device).
int get_table(const dit_rope3d_desc* r, int t_ext, cudaStream_t stream, RopeParams* rp) {
  int dev = 0;
  cudaGetDevice(&dev);
  uint32_t bb;
  std::memcpy(&bb, &r->base, 4);
  TableKey key{dev, r->grid_h, r->grid_w, r->d_t, r->d_h, r->d_w, t_ext, r->t0, r->h0, r->w0, bb};
  rope_table_layout(r, t_ext, rp);
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_tables.find(key);
  if (it != g_tables.end()) {
    rp->table = it->second;
    return DIT_OK;
  }
  float2* dptr = nullptr;
  if (cudaMalloc(&dptr, sizeof(float2) * std::max(rp->n_entries, 2)) != cudaSuccess)
    return DIT_ERR_ALLOC;
  // the table is shared by later calls on any stream: let its fill finish first
  int s = fill_table(dptr, r, t_ext, *rp, stream);
  if (s == DIT_OK && cudaStreamSynchronize(stream) != cudaSuccess) s = DIT_ERR_LAUNCH;
  if (s != DIT_OK) {
    cudaFree(dptr);
    return s;
  }
  g_tables.emplace(key, dptr);
  rp->table = dptr;
  return DIT_OK;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// [rows, H*d] bf16, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols,
               uint32_t box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, cols] bytes (E4M3 codes), boxes of 128 columns x box_rows rows, 128-byte swizzle.
bool make_tmap8(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols,
                uint32_t box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Longest-first order of a packed batch for the single-CTA attention kernel (fills
// prm->seq_order; stable for equal lengths). Left empty (natural order on a 2-D grid)
// for dense batches, more than attn::kMaxOrder sequences, or a grid too large for 1-D.
void set_seq_order(attn::Params* prm, const std::vector<int64_t>& lens, int64_t n_work, int32_t H,
                   bool packed) {
  prm->n_order = 0;
  if (!packed || lens.size() > static_cast<size_t>(attn::kMaxOrder) ||
      n_work * H >= (int64_t(1) << 31))
    return;
  std::vector<int32_t> order(lens.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int32_t>(i);
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return lens[a] > lens[b]; });
  for (size_t i = 0; i < order.size(); ++i) prm->seq_order[i] = order[i];
  prm->n_order = static_cast<int32_t>(order.size());
}

int dev_index() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev >= 0 && dev < 64 ? dev : 0;
}
int g_sm_count[64] = {};
int g_last_attn_split = 0;  // key-range split of the last single-CTA attention launch

// Key-range split of a dense attention launch's last partial wave. `units` work units
// of one CTA each run in waves of one per SM; when the last wave holds
// tail = units % sms units, the SMs it leaves idle can share their work instead: every
// tail unit becomes a cluster of S CTAs, each over nk / S of the key tiles, which merge
// their partial results (attn_fwd_kernel, Params::kv_split). Returns the largest S in
// [2, kMaxSplit] with tail * S CTAs within one wave, at least two key tiles per CTA, and
// tail clusters of S resident at once (resident(S): the occupancy calculator's count,
// asked only for the S values that pass the first two tests); 1 (no split) when none
// qualifies.
template <typename Resident>
int tail_split_choice(int64_t units, int64_t sms, int64_t nk, Resident resident) {
  if (sms <= 0 || units <= 0) return 1;
  const int64_t tail = units % sms;
  if (tail == 0) return 1;
  for (int S = attn::kMaxSplit; S >= 2; --S) {
    if (tail * S > sms || 2 * S > nk) continue;
    const int mc = resident(S);
    if (mc > 0 && tail <= mc) return S;
  }
  return 1;
}

// tail_split_choice for a launch of this kernel (whose residency depends on D only) on
// the current device.
template <int D, typename Kernel>
int attn_tail_split(Kernel kernel, uint32_t smem, const attn::Params& prm, int n_work, int32_t H) {
  const int dev = dev_index();
  if (g_sm_count[dev] == 0) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g_sm_count[dev] = sms > 0 ? sms : 148;
  }
  const int64_t units = static_cast<int64_t>(n_work) * H;
  const int64_t nk = (prm.dense_len + attn::kTileN - 1) / attn::kTileN;
  // clusters of S resident at once, per S (0: not yet asked; -1: the query failed)
  static int max_clusters[64][attn::kMaxSplit + 1] = {};
  return tail_split_choice(units, g_sm_count[dev], nk, [&](int S) {
    int& mc = max_clusters[dev][S];
    if (mc == 0) {
      cudaLaunchConfig_t cfg{};
      cudaLaunchAttribute attr[1];
      cfg.gridDim = dim3(static_cast<unsigned>(S));
      cfg.blockDim = dim3(attn::kThreads);
      cfg.dynamicSmemBytes = smem;
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(S);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // clear the query's error; the split is simply not used
        n = -1;
      }
      mc = n;
    }
    return mc;
  });
}

// F8: 0 all bf16; 1 E4M3 q and k; 2 E4M3 q, k and v (see attn_fwd_kernel)
template <int D, int F8 = 0>
int launch_attn(const void* q, const void* k, const void* v, int64_t rows, int32_t H,
                const attn::Params& prm, int n_work, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  const int64_t cols = static_cast<int64_t>(H) * D;
  const bool ok_qk = F8 >= 1 ? (make_tmap8(&tq, q, rows, cols) && make_tmap8(&tk, k, rows, cols))
                             : (make_tmap(&tq, q, rows, cols) && make_tmap(&tk, k, rows, cols));
  const bool ok_v = F8 == 2 ? make_tmap8(&tv, v, rows, cols) : make_tmap(&tv, v, rows, cols);
  if (!ok_qk || !ok_v) return DIT_ERR_LAUNCH;
  constexpr uint32_t smem = attn::Smem<D>::kRequest;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn::attn_fwd_kernel<D, F8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DIT_ERR_LAUNCH;
    attr_set[dev] = true;
  }
  attn::Params base = prm;
  base.kv_split = 1;
  base.unit0 = 0;
  base.pdl = 0;
  const int split = prm.cu_seqlens == nullptr && prm.n_order == 0
                        ? attn_tail_split<D>(attn::attn_fwd_kernel<D, F8>, smem, prm, n_work, H)
                        : 1;
  g_last_attn_split = split;
  if (split <= 1) {
    // packed: 1-D grid over (sequence in prm.seq_order, head, pair); else (pairs, heads)
    const dim3 grid = prm.n_order > 0 ? dim3(static_cast<unsigned>(n_work) * H) : dim3(n_work, H);
    attn::attn_fwd_kernel<D, F8><<<grid, attn::kThreads, smem, stream>>>(tq, tk, tv, base);
    return launch_status();
  }
  // dense batch whose last wave would run a few units on a mostly idle GPU: the whole
  // waves as usual (1-D grid, head-major units), then the rest with each unit split
  // over a cluster of `split` CTAs by key range
  const int64_t units = static_cast<int64_t>(n_work) * H;
  const int64_t tail = units % g_sm_count[dev_index()];
  const int64_t full = units - tail;
  if (full > 0) {
    // the split units may start on SMs as the whole waves drain (they read only q, k, v)
    attn::Params mp = base;
    mp.pdl = 1;
    attn::attn_fwd_kernel<D, F8><<<static_cast<unsigned>(full), attn::kThreads, smem, stream>>>(
        tq, tk, tv, mp);
    if (int s = launch_status()) return s;
  }
  attn::Params tp = base;
  tp.kv_split = split;
  tp.unit0 = static_cast<int32_t>(full);
  tp.pdl = full > 0 ? 2 : 0;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(tail * split));
  cfg.blockDim = dim3(attn::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // overlap only the launch just made above: with no whole waves before it, the split
  // launch follows the stream's previous work in the usual order
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = full > 0 ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, attn::attn_fwd_kernel<D, F8>, tq, tk, tv, tp) != cudaSuccess)
    return DIT_ERR_LAUNCH;
  return launch_status();
}

// head_dim 128 on CTA pairs (cta_group::2): 512 query rows per pair.
int launch_attn_2sm(const void* q, const void* k, const void* v, int64_t rows, int32_t H,
                    attn::Params prm, const std::vector<int64_t>& lens, bool dense,
                    cudaStream_t stream) {
  constexpr int D = attn2::kD;
  prm.n_order = 0;  // the pair kernel walks packed sequences in cu_seqlens order
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, rows, static_cast<int64_t>(H) * D, 128) ||
      !make_tmap(&tk, k, rows, static_cast<int64_t>(H) * D, attn2::kHalfN) ||
      !make_tmap(&tv, v, rows, static_cast<int64_t>(H) * D, attn2::kTileN))
    return DIT_ERR_LAUNCH;
  int64_t units = 0;
  if (dense) {
    prm.pairs_per_dense_seq =
        static_cast<int32_t>((prm.dense_len + attn2::kPairRows - 1) / attn2::kPairRows);
    units = static_cast<int64_t>(prm.pairs_per_dense_seq) * prm.n_seq;
  } else {
    for (int64_t L : lens) units += (L + attn2::kPairRows - 1) / attn2::kPairRows;
  }
  if (units == 0) return DIT_OK;
  if (2 * units > INT32_MAX) return DIT_ERR_SHAPE;
  constexpr uint32_t smem = attn2::Smem::kRequest;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn2::attn_fwd_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DIT_ERR_LAUNCH;
    attr_set[dev] = true;
  }
  dim3 grid(static_cast<unsigned>(2 * units), H);
  attn2::attn_fwd_2sm_kernel<<<grid, attn2::kThreads, smem, stream>>>(tq, tk, tv, prm);
  return launch_status();
}

// Parameter groups shorter than this many rows (a group per frame) take the form that
// loads gamma and beta with x (see adaln_modulate_kernel).
constexpr int64_t kEarlyParamRows = 8192;

template <int NV>
void launch_modulate(const void* x, const void* g, const void* b, void* o, int64_t rows, int32_t D,
                     int64_t rpg, float eps, float s0, cudaStream_t st) {
  // d_model <= 3072: 64 threads per row, NV64 = ceil(D / 512) chunks each; large parameter
  // groups take the late form, small ones the form with parameters staged in shared memory
  if (D <= 3072) {
    const int nv64 = (D + 511) / 512;
    auto run = [&](auto nv_tag) {
      constexpr int NV64 = decltype(nv_tag)::value;
      if (rpg >= kEarlyParamRows)
        adaln_modulate_kernel<NV64, false, 64><<<static_cast<unsigned>(rows), 64, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(g),
            static_cast<const __nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(o), D, rpg, eps, s0);
      else
        adaln_modulate_staged_kernel<NV64, 64><<<static_cast<unsigned>(rows), 64, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(g),
            static_cast<const __nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(o), D, rpg, eps, s0);
    };
    switch (nv64) {
      case 1: run(std::integral_constant<int, 1>{}); return;
      case 2: run(std::integral_constant<int, 2>{}); return;
      case 3: run(std::integral_constant<int, 3>{}); return;
      case 4: run(std::integral_constant<int, 4>{}); return;
      case 5: run(std::integral_constant<int, 5>{}); return;
      default: run(std::integral_constant<int, 6>{}); return;
    }
  }
  if (rpg < kEarlyParamRows) {
    adaln_modulate_kernel<NV, true><<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(g),
        static_cast<const __nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(o), D, rpg, eps, s0);
    return;
  }
  adaln_modulate_kernel<NV, false><<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(g),
      static_cast<const __nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(o), D, rpg, eps, s0);
}

template <int NV>
void launch_residual(const void* x, const void* y, const void* a, void* o, int64_t rows, int32_t D,
                     int64_t rpg, cudaStream_t st) {
  gated_residual_kernel<NV><<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y),
      static_cast<const __nv_bfloat16*>(a), static_cast<__nv_bfloat16*>(o), D, rpg);
}

template <int NV>
void launch_euler(const void* x, const void* u, const float* dt, void* o, int64_t rows, int32_t D,
                  int64_t rpg, cudaStream_t st) {
  flow_euler_kernel<NV><<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(u), dt,
      static_cast<__nv_bfloat16*>(o), D, rpg);
}

}  // namespace

extern "C" {

const char* dit_status_string(int status) {
  switch (status) {
    case DIT_OK: return "DIT_OK";
    case DIT_ERR_NULL: return "DIT_ERR_NULL: a required pointer is NULL";
    case DIT_ERR_SHAPE: return "DIT_ERR_SHAPE: unsupported or inconsistent sizes";
    case DIT_ERR_ALIGN: return "DIT_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case DIT_ERR_SEQLENS: return "DIT_ERR_SEQLENS: invalid cu_seqlens";
    case DIT_ERR_DEVICE: return "DIT_ERR_DEVICE: current device is not sm_100";
    case DIT_ERR_LAUNCH: return "DIT_ERR_LAUNCH: a CUDA call or kernel launch failed";
    case DIT_ERR_TIMEOUT: return "DIT_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case DIT_ERR_ALLOC: return "DIT_ERR_ALLOC: device allocation for the RoPE table failed";
    case DIT_ERR_SCRATCH:
      return "DIT_ERR_SCRATCH: the RoPE table is larger than the fixed array of the "
             "allocation-free call (65536 entries)";
    default: return "unknown dit_status";
  }
}

int dit_adaln_modulate(const void* x, const void* gamma, const void* beta, void* out, int64_t rows,
                       int32_t D, int64_t rows_per_group, float eps, float scale_offset,
                       void* stream) {
  if (!x || !gamma || !beta || !out) return DIT_ERR_NULL;
  if (int s = check_rows_groups(rows, D, rows_per_group)) return s;
  if (!(eps >= 0.f) || !std::isfinite(scale_offset)) return DIT_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(out)) return DIT_ERR_ALIGN;
  if (int s = check_device()) return s;
  if (rows == 0) return DIT_OK;
  auto st = static_cast<cudaStream_t>(stream);
  const int nv = (D / 8 + kRowThreads - 1) / kRowThreads;
  switch (nv) {
    case 1: launch_modulate<1>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 2: launch_modulate<2>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 3: launch_modulate<3>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 4: launch_modulate<4>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 5: launch_modulate<5>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 6: launch_modulate<6>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 7: launch_modulate<7>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    case 8: launch_modulate<8>(x, gamma, beta, out, rows, D, rows_per_group, eps, scale_offset, st); break;
    default:
      adaln_modulate_wide_kernel<<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(gamma),
          static_cast<const __nv_bfloat16*>(beta), static_cast<__nv_bfloat16*>(out), D,
          rows_per_group, eps, scale_offset);
  }
  return launch_status();
}

int dit_gated_residual(const void* x, const void* y, const void* alpha, void* out, int64_t rows,
                       int32_t D, int64_t rows_per_group, void* stream) {
  if (!x || !y || !alpha || !out) return DIT_ERR_NULL;
  if (int s = check_rows_groups(rows, D, rows_per_group)) return s;
  if (!aligned16(x) || !aligned16(y) || !aligned16(alpha) || !aligned16(out)) return DIT_ERR_ALIGN;
  if (int s = check_device()) return s;
  if (rows == 0) return DIT_OK;
  auto st = static_cast<cudaStream_t>(stream);
  const int nv = (D / 8 + kRowThreads - 1) / kRowThreads;
  switch (nv) {
    case 1: launch_residual<1>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 2: launch_residual<2>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 3: launch_residual<3>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 4: launch_residual<4>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 5: launch_residual<5>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 6: launch_residual<6>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 7: launch_residual<7>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    case 8: launch_residual<8>(x, y, alpha, out, rows, D, rows_per_group, st); break;
    default:
      gated_residual_wide_kernel<<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y),
          static_cast<const __nv_bfloat16*>(alpha), static_cast<__nv_bfloat16*>(out), D,
          rows_per_group);
  }
  return launch_status();
}

int dit_flow_euler_step(const void* x, const void* u, const float* dt, void* out, int64_t rows,
                        int32_t D, int64_t rows_per_group, void* stream) {
  if (!x || !u || !dt || !out) return DIT_ERR_NULL;
  if (int s = check_rows_groups(rows, D, rows_per_group)) return s;
  if (!aligned16(x) || !aligned16(u) || !aligned16(out) || (reinterpret_cast<uintptr_t>(dt) & 3u))
    return DIT_ERR_ALIGN;
  if (int s = check_device()) return s;
  if (rows == 0) return DIT_OK;
  auto st = static_cast<cudaStream_t>(stream);
  const int nv = (D / 8 + kRowThreads - 1) / kRowThreads;
  switch (nv) {
    case 1: launch_euler<1>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 2: launch_euler<2>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 3: launch_euler<3>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 4: launch_euler<4>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 5: launch_euler<5>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 6: launch_euler<6>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 7: launch_euler<7>(x, u, dt, out, rows, D, rows_per_group, st); break;
    case 8: launch_euler<8>(x, u, dt, out, rows, D, rows_per_group, st); break;
    default:
      flow_euler_wide_kernel<<<static_cast<unsigned>(rows), kRowThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(u), dt,
          static_cast<__nv_bfloat16*>(out), D, rows_per_group);
  }
  return launch_status();
}

}  // extern "C"

static int linear_impl(const void* x, const void* w, const void* bias, void* out, int64_t M, int32_t N,
                       int32_t K, int32_t activation, const void* residual, const void* alpha,
                       int64_t rows_per_group, bool f8, float acc_scale, void* stream) {
  if (!x || !w || !out || (residual && !alpha)) return DIT_ERR_NULL;
  if (M < 0 || M >= (int64_t(1) << 31) || N <= 0 || K <= 0 || (N % 8) || (K % (f8 ? 16 : 8)) ||
      (activation != 0 && activation != 1))
    return DIT_ERR_SHAPE;
  if (residual && (rows_per_group <= 0 || (M % rows_per_group) != 0)) return DIT_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (bias && !aligned16(bias)) ||
      (residual && (!aligned16(residual) || !aligned16(alpha))))
    return DIT_ERR_ALIGN;
  if (int s = check_device()) return s;
  if (M == 0) return DIT_OK;
  auto st = static_cast<cudaStream_t>(stream);
  CUtensorMap ta, tb;
  const bool maps = f8 ? (make_tmap8(&ta, x, M, K, lin::kBM) && make_tmap8(&tb, w, N, K, lin::kBN))
                       : (make_tmap(&ta, x, M, K, lin::kBM) && make_tmap(&tb, w, N, K, lin::kBN));
  if (!maps) return DIT_ERR_LAUNCH;
  lin::Params prm{};
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.res = static_cast<const __nv_bfloat16*>(residual);
  prm.alpha = static_cast<const __nv_bfloat16*>(alpha);
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.act = activation;
  prm.rows_per_group = residual ? rows_per_group : 1;
  prm.tiles_m = static_cast<int32_t>((M + lin::kBM - 1) / lin::kBM);
  prm.tiles_n = (N + lin::kBN - 1) / lin::kBN;
  const int k_per_stage = f8 ? 128 : lin::kBK;
  prm.k_blocks = (K + k_per_stage - 1) / k_per_stage;
  prm.acc_scale = acc_scale;
  prm.force_timeout = g_force_timeout;
  prm.wait_limit_ns = g_wait_limit_ns;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static bool attr_set[2][64] = {};
  if (dev < 64 && !attr_set[f8][dev]) {
    const cudaError_t e =
        f8 ? cudaFuncSetAttribute(lin::linear_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(lin::kSmemBytes))
           : cudaFuncSetAttribute(lin::linear_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(lin::kSmemBytes));
    if (e != cudaSuccess) return DIT_ERR_LAUNCH;
    attr_set[f8][dev] = true;
  }
  const int64_t tiles = static_cast<int64_t>(prm.tiles_m) * prm.tiles_n;
  if (tiles >= (int64_t(1) << 31)) return DIT_ERR_SHAPE;
  if (sms <= 0) sms = 148;
  if (g_linear_variant == 1) {
    // CTA pairs: 256 x 256 tiles, each CTA loads 128 rows of A and of B
    CUtensorMap tb2;
    if (!(f8 ? make_tmap8(&tb2, w, N, K, lin::kBM) : make_tmap(&tb2, w, N, K, lin::kBM)))
      return DIT_ERR_LAUNCH;
    static bool attr2_set[2][64] = {};
    if (dev < 64 && !attr2_set[f8][dev]) {
      const cudaError_t e =
          f8 ? cudaFuncSetAttribute(lin::linear_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(lin::kSmemBytes2))
             : cudaFuncSetAttribute(lin::linear_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(lin::kSmemBytes2));
      if (e != cudaSuccess) return DIT_ERR_LAUNCH;
      attr2_set[f8][dev] = true;
    }
    const int64_t pair_tiles = static_cast<int64_t>((prm.tiles_m + 1) / 2) * prm.tiles_n;
    const unsigned grid = 2u * static_cast<unsigned>(std::min<int64_t>(pair_tiles, sms / 2));
    if (f8) lin::linear_pair_kernel<true><<<grid, lin::kThreads, lin::kSmemBytes2, st>>>(ta, tb2, prm);
    else lin::linear_pair_kernel<false><<<grid, lin::kThreads, lin::kSmemBytes2, st>>>(ta, tb2, prm);
    return launch_status();
  }
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, sms));
  if (f8) lin::linear_kernel<true><<<grid, lin::kThreads, lin::kSmemBytes, st>>>(ta, tb, prm);
  else lin::linear_kernel<false><<<grid, lin::kThreads, lin::kSmemBytes, st>>>(ta, tb, prm);
  return launch_status();
}


// bf16 attention behind dit_attn_fwd and dit_attn_fwd_noalloc: argument checks, work
// count, launch. `table` provides the RoPE cos/sin table (cached, or the fixed array).
template <typename TableFn>
int attn_bf16_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t rows,
                   int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                   const int32_t* cu_seqlens_host, float softmax_scale,
                   const dit_rope3d_desc* rope, void* stream, TableFn table) {
  if (!q || !k || !v || !o) return DIT_ERR_NULL;
  if (rows <= 0 || H <= 0 || H > 65535 || (d != 64 && d != 128)) return DIT_ERR_SHAPE;
  if (rows >= (int64_t(1) << 31)) return DIT_ERR_SHAPE;  // TMA row coordinates are int32
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return DIT_ERR_ALIGN;
  std::vector<int64_t> lens;
  if (int s = check_seqs(rows, n_seq, cu_seqlens_dev, cu_seqlens_host, &lens)) return s;
  int t_ext = 0;
  if (rope)
    if (int s = validate_rope(rope, d, lens, &t_ext)) return s;
  if (int s = check_device()) return s;
  auto st = static_cast<cudaStream_t>(stream);

  attn::Params prm{};
  prm.cu_seqlens = cu_seqlens_dev;
  prm.n_seq = n_seq;
  prm.H = H;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.force_timeout = g_force_timeout;
  prm.wait_limit_ns = g_wait_limit_ns;
  prm.o_scale = 1.f;
  int64_t n_work = 0;
  if (cu_seqlens_dev == nullptr) {
    prm.dense_len = rows / n_seq;
    prm.pairs_per_dense_seq = static_cast<int32_t>((prm.dense_len + 2 * attn::kTileM - 1) / (2 * attn::kTileM));
    n_work = static_cast<int64_t>(prm.pairs_per_dense_seq) * n_seq;
  } else {
    for (int64_t L : lens) n_work += (L + 2 * attn::kTileM - 1) / (2 * attn::kTileM);
  }
  if (n_work == 0) return DIT_OK;
  if (n_work > INT32_MAX) return DIT_ERR_SHAPE;
  if (rope) {
    prm.use_rope = 1;
    if (int s = table(rope, t_ext, st, &prm.rope)) return s;
  }
  set_seq_order(&prm, lens, n_work, H, cu_seqlens_dev != nullptr);
  if (d == 128 && g_attn_variant == 1)
    return launch_attn_2sm(q, k, v, rows, H, prm, lens, cu_seqlens_dev == nullptr, st);
  if (d == 128) return launch_attn<128>(q, k, v, rows, H, prm, static_cast<int>(n_work), st);
  return launch_attn<64>(q, k, v, rows, H, prm, static_cast<int>(n_work), st);
}

extern "C" {

int dit_linear(const void* x, const void* w, const void* bias, void* out, int64_t M, int32_t N,
               int32_t K, int32_t activation, const void* residual, const void* alpha,
               int64_t rows_per_group, void* stream) {
  return linear_impl(x, w, bias, out, M, N, K, activation, residual, alpha, rows_per_group, false,
                     1.f, stream);
}

int dit_linear_fp8(const void* x8, const void* w8, const void* bias, void* out, int64_t M,
                   int32_t N, int32_t K, int32_t activation, const void* residual,
                   const void* alpha, int64_t rows_per_group, float x_scale, float w_scale,
                   void* stream) {
  if (!(x_scale > 0.f) || !(w_scale > 0.f) || !std::isfinite(x_scale) || !std::isfinite(w_scale))
    return DIT_ERR_SHAPE;
  return linear_impl(x8, w8, bias, out, M, N, K, activation, residual, alpha, rows_per_group, true,
                     x_scale * w_scale, stream);
}

int dit_set_linear_variant(int variant) {
  if (variant != 0 && variant != 1) return DIT_ERR_SHAPE;
  g_linear_variant = variant;
  return DIT_OK;
}

}  // extern "C"

namespace {
// [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
  const auto pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + static_cast<uintptr_t>(nb) && pb < pa + static_cast<uintptr_t>(na);
}

// Shared body of dit_rope3d_qk (bf16 out) and dit_rope3d_qk_e4m3 (E4M3 codes out).
int rope3d_qk_impl(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t rows,
                   int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                   const int32_t* cu_seqlens_host, const dit_rope3d_desc* rope, bool e4m3,
                   float q_inv, float k_inv, void* stream) {
  if (!q_in || !q_out || !rope || (k_in && !k_out)) return DIT_ERR_NULL;
  if (rows < 0 || H <= 0 || (d != 64 && d != 128)) return DIT_ERR_SHAPE;
  if (e4m3 && (!std::isfinite(q_inv) || (k_in && !std::isfinite(k_inv)))) return DIT_ERR_SHAPE;
  if (!aligned16(q_in) || !aligned16(k_in)) return DIT_ERR_ALIGN;
  const uintptr_t out_mask = e4m3 ? 7u : 15u;
  if ((reinterpret_cast<uintptr_t>(q_out) & out_mask) ||
      (k_in && (reinterpret_cast<uintptr_t>(k_out) & out_mask)))
    return DIT_ERR_ALIGN;
  if (e4m3) {
    // codes are half the size of their sources: a chunk written by one thread could
    // land on a source chunk another thread has yet to read
    const int64_t n = rows * H * d;
    const void* ins[2] = {q_in, k_in};
    void* outs[2] = {q_out, k_in ? k_out : nullptr};
    for (void* o : outs) {
      if (!o) continue;
      for (const void* i : ins)
        if (i && overlaps(o, n, i, 2 * n)) return DIT_ERR_SHAPE;
    }
    if (outs[1] && overlaps(outs[0], n, outs[1], n)) return DIT_ERR_SHAPE;
  }
  std::vector<int64_t> lens;
  if (int s = check_seqs(rows, n_seq, cu_seqlens_dev, cu_seqlens_host, &lens)) return s;
  int t_ext = 0;
  if (int s = validate_rope(rope, d, lens, &t_ext)) return s;
  if (int s = check_device()) return s;
  if (rows == 0) return DIT_OK;
  auto st = static_cast<cudaStream_t>(stream);
  RopeParams rp;
  if (int s = get_table(rope, t_ext, st, &rp)) return s;
  const int64_t dense_len = cu_seqlens_dev ? 0 : rows / n_seq;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  const auto* qi = static_cast<const uint4*>(q_in);
  const auto* ki = static_cast<const uint4*>(k_in);
  auto launch = [&](auto d_head, auto quant) {
    rope3d_qk_kernel<decltype(d_head)::value, decltype(quant)::value><<<grid, 256, 0, st>>>(
        qi, ki, q_out, k_out, rows, H, cu_seqlens_dev, n_seq, dense_len, rp, q_inv, k_inv);
  };
  using D128 = std::integral_constant<int, 128>;
  using D64 = std::integral_constant<int, 64>;
  if (e4m3) {
    if (d == 128) launch(D128{}, std::true_type{}); else launch(D64{}, std::true_type{});
  } else {
    if (d == 128) launch(D128{}, std::false_type{}); else launch(D64{}, std::false_type{});
  }
  return launch_status();
}
}  // namespace

extern "C" {

int dit_rope3d_qk(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t rows,
                  int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                  const int32_t* cu_seqlens_host, const dit_rope3d_desc* rope, void* stream) {
  return rope3d_qk_impl(q_in, k_in, q_out, k_out, rows, H, d, n_seq, cu_seqlens_dev,
                        cu_seqlens_host, rope, false, 1.f, 1.f, stream);
}

int dit_rope3d_qk_e4m3(const void* q_in, const void* k_in, void* q8_out, void* k8_out,
                       int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                       const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                       const dit_rope3d_desc* rope, float q_inv_scale, float k_inv_scale,
                       void* stream) {
  return rope3d_qk_impl(q_in, k_in, q8_out, k8_out, rows, H, d, n_seq, cu_seqlens_dev,
                        cu_seqlens_host, rope, true, q_inv_scale, k_inv_scale, stream);
}

int dit_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t rows,
                 int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                 const int32_t* cu_seqlens_host, float softmax_scale, const dit_rope3d_desc* rope,
                 void* stream) {
  return attn_bf16_impl(q, k, v, o, lse, rows, H, d, n_seq, cu_seqlens_dev, cu_seqlens_host,
                        softmax_scale, rope, stream, get_table);
}

}  // extern "C"

namespace {
int attn_fp8_impl(const void* q8, const void* k8, const void* v, void* o, float* lse, int64_t rows,
                  int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                  const int32_t* cu_seqlens_host, float softmax_scale, float q_scale,
                  float k_scale, float v_scale, bool v8, void* stream) {
  if (!q8 || !k8 || !v || !o) return DIT_ERR_NULL;
  if (rows <= 0 || H <= 0 || H > 65535 || d != 128) return DIT_ERR_SHAPE;
  if (rows >= (int64_t(1) << 31)) return DIT_ERR_SHAPE;
  for (float sc : {q_scale, k_scale, v_scale})
    if (!(sc > 0.f) || !std::isfinite(sc)) return DIT_ERR_SHAPE;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return DIT_ERR_ALIGN;
  std::vector<int64_t> lens;
  if (int s = check_seqs(rows, n_seq, cu_seqlens_dev, cu_seqlens_host, &lens)) return s;
  if (int s = check_device()) return s;
  auto st = static_cast<cudaStream_t>(stream);
  attn::Params prm{};
  prm.cu_seqlens = cu_seqlens_dev;
  prm.n_seq = n_seq;
  prm.H = H;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  prm.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.force_timeout = g_force_timeout;
  prm.wait_limit_ns = g_wait_limit_ns;
  prm.o_scale = v8 ? v_scale : 1.f;
  int64_t n_work = 0;
  if (cu_seqlens_dev == nullptr) {
    prm.dense_len = rows / n_seq;
    prm.pairs_per_dense_seq =
        static_cast<int32_t>((prm.dense_len + 2 * attn::kTileM - 1) / (2 * attn::kTileM));
    n_work = static_cast<int64_t>(prm.pairs_per_dense_seq) * n_seq;
  } else {
    for (int64_t L : lens) n_work += (L + 2 * attn::kTileM - 1) / (2 * attn::kTileM);
  }
  if (n_work == 0) return DIT_OK;
  if (n_work > INT32_MAX) return DIT_ERR_SHAPE;
  set_seq_order(&prm, lens, n_work, H, cu_seqlens_dev != nullptr);
  return v8 ? launch_attn<128, 2>(q8, k8, v, rows, H, prm, static_cast<int>(n_work), st)
            : launch_attn<128, 1>(q8, k8, v, rows, H, prm, static_cast<int>(n_work), st);
}
}  // namespace

extern "C" {

int dit_attn_fwd_qk8(const void* q8, const void* k8, const void* v, void* o, float* lse,
                     int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                     const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                     float softmax_scale, float q_scale, float k_scale, void* stream) {
  return attn_fp8_impl(q8, k8, v, o, lse, rows, H, d, n_seq, cu_seqlens_dev, cu_seqlens_host,
                       softmax_scale, q_scale, k_scale, 1.f, false, stream);
}

int dit_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse,
                     int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                     const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                     float softmax_scale, float q_scale, float k_scale, float v_scale,
                     void* stream) {
  return attn_fp8_impl(q8, k8, v8, o, lse, rows, H, d, n_seq, cu_seqlens_dev, cu_seqlens_host,
                       softmax_scale, q_scale, k_scale, v_scale, true, stream);
}

int dit_quantize_e4m3(const void* x, void* out8, int64_t n, float inv_scale, void* stream) {
  if (!x || !out8) return DIT_ERR_NULL;
  if (n < 0 || (n % 8) != 0 || !std::isfinite(inv_scale)) return DIT_ERR_SHAPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(out8) & 7u)) return DIT_ERR_ALIGN;
  if (int s = check_device()) return s;
  if (n == 0) return DIT_OK;
  const int64_t n8 = n / 8;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, static_cast<int64_t>(sms > 0 ? sms : 148) * 8);
  quantize_e4m3_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(x), static_cast<uint2*>(out8), n8, inv_scale);
  return launch_status();
}

}  // extern "C"

namespace {
// Host watchdog loop: polls ready() (1 done, 0 not yet, -1 failed) until it is done or
// fails, or until timeout_us of wall time have passed since the first poll; sleeps
// between polls, from 1 us doubling up to 100 us.
template <typename Ready>
int poll_until(Ready ready, int64_t timeout_us) {
  const auto t0 = std::chrono::steady_clock::now();
  int64_t nap = 1;
  for (;;) {
    const int r = ready();
    if (r > 0) return DIT_OK;
    if (r < 0) return DIT_ERR_LAUNCH;
    const int64_t waited = std::chrono::duration_cast<std::chrono::microseconds>(
                               std::chrono::steady_clock::now() - t0).count();
    if (waited >= timeout_us) return DIT_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(std::min(nap, timeout_us - waited)));
    nap = std::min<int64_t>(2 * nap, 100);
  }
}
}  // namespace

extern "C" {

int dit_wait_device(void* stream, int64_t timeout_us) {
  if (timeout_us < 0) return DIT_ERR_SHAPE;
  auto st = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return DIT_ERR_LAUNCH;
  if (cudaEventRecord(ev, st) != cudaSuccess) {
    cudaEventDestroy(ev);
    return DIT_ERR_LAUNCH;
  }
  const int s = poll_until(
      [&] {
        const cudaError_t e = cudaEventQuery(ev);
        return e == cudaSuccess ? 1 : (e == cudaErrorNotReady ? 0 : -1);
      },
      timeout_us);
  cudaEventDestroy(ev);  // released once the recorded work completes
  if (s != DIT_OK) return s;
  // the stream has finished: read and clear the error word on it (no device-wide wait)
  uint32_t err = 0;
  const uint32_t zero = 0;
  if (cudaMemcpyFromSymbolAsync(&err, g_device_error, sizeof(err), 0, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return DIT_ERR_LAUNCH;
  if (err != 0 && (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0,
                                           cudaMemcpyHostToDevice, st) != cudaSuccess ||
                   cudaStreamSynchronize(st) != cudaSuccess))
    return DIT_ERR_LAUNCH;
  return (err & kDevErrTimeout) ? DIT_ERR_TIMEOUT : DIT_OK;
}

namespace {
// exp2_pair_fma on pairs of an fp32 array (a lone last element is paired with itself)
__global__ void exp2_fma_probe_kernel(const float* t, float* e, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float t0 = t[i], t1 = i + 1 < n ? t[i + 1] : t0;
  float e0, e1;
  attn::exp2_pair_fma(f2_pack(t0, t1), e0, e1);
  e[i] = e0;
  if (i + 1 < n) e[i + 1] = e1;
}
}  // namespace

int dit_debug_exp2_fma(const float* t, float* out, int64_t n, void* stream) {
  if (n < 0) return DIT_ERR_SHAPE;
  if (n == 0) return DIT_OK;
  if (t == nullptr || out == nullptr) return DIT_ERR_NULL;
  const int64_t pairs = (n + 1) / 2;
  if ((pairs + 255) / 256 >= (int64_t(1) << 31)) return DIT_ERR_SHAPE;
  exp2_fma_probe_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0,
                          static_cast<cudaStream_t>(stream)>>>(t, out, n);
  return launch_status();
}

int dit_debug_poll_fake(int64_t busy_polls, int fail, int64_t timeout_us, int64_t* polls) {
  int64_t n = 0;
  const int s = poll_until(
      [&] {
        ++n;
        if (n > busy_polls) return fail ? -1 : 1;
        return 0;
      },
      timeout_us);
  if (polls) *polls = n;
  return s;
}

int dit_check_device(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DIT_ERR_LAUNCH;
  uint32_t err = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&err, g_device_error, sizeof(err)) != cudaSuccess) return DIT_ERR_LAUNCH;
  if (err != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return DIT_ERR_LAUNCH;
  return (err & kDevErrTimeout) ? DIT_ERR_TIMEOUT : DIT_OK;
}

void dit_debug_force_timeout(int enable) { g_force_timeout = enable ? 1 : 0; }

void dit_debug_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns ? ns : 2000000000ull; }

int dit_debug_last_attn_split(void) { return g_last_attn_split; }

int dit_debug_tail_split(int64_t units, int64_t sms, int64_t nk, const int32_t* resident,
                         int32_t* split) {
  if (resident == nullptr || split == nullptr) return DIT_ERR_NULL;
  *split = tail_split_choice(units, sms, nk, [&](int S) { return static_cast<int>(resident[S]); });
  return DIT_OK;
}

int dit_set_attn_variant(int variant) {
  if (variant != 0 && variant != 1) return DIT_ERR_SHAPE;
  g_attn_variant = variant;
  return DIT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free attention
// dit_attn_fwd_noalloc: the same attention, but the 3D-RoPE cos/sin table lives in a
// fixed array of device memory that is part of the loaded library, so the call never
// allocates. The array is shared by every call on a device and holds the last call's
// table; every call rewrites the whole range it uses, with a kernel on its stream.
namespace {

constexpr int kNoAllocTableEntries = 65536;  // float2 entries: 512 KiB per device
static __device__ __align__(256) float2 g_noalloc_rope_table[kNoAllocTableEntries];

std::mutex g_noalloc_mu;
std::map<int, float2*> g_noalloc_addr;  // per device: the array's device address

// Device address of the array on the current device. The array's name in host code
// is only a stand-in, so the address is asked from the runtime once per device.
int noalloc_table_address(float2** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  auto it = g_noalloc_addr.find(dev);
  if (it == g_noalloc_addr.end()) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_rope_table);
    if (e == cudaErrorMemoryAllocation) {
      cudaGetLastError();  // not sticky: clear it
      return DIT_ERR_ALLOC;  // loading the library's module onto the device needs memory
    }
    if (e != cudaSuccess || ptr == nullptr) return DIT_ERR_LAUNCH;
    it = g_noalloc_addr.emplace(dev, static_cast<float2*>(ptr)).first;
  }
  *out = it->second;
  return DIT_OK;
}

}  // namespace

extern "C" int dit_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int64_t rows, int32_t H, int32_t d,
                                    int32_t n_seq, const int32_t* cu_seqlens_dev,
                                    const int32_t* cu_seqlens_host, float softmax_scale,
                                    const dit_rope3d_desc* rope, void* stream) {
  // the table is written into the fixed array by a kernel on `stream`, ahead of the
  // attention on the same stream
  auto fixed_table = [](const dit_rope3d_desc* r, int t_ext, cudaStream_t st, RopeParams* rp) {
    rope_table_layout(r, t_ext, rp);
    if (std::max(rp->n_entries, 2) > kNoAllocTableEntries) return static_cast<int>(DIT_ERR_SCRATCH);
    float2* table = nullptr;
    if (int s = noalloc_table_address(&table)) return s;
    rp->table = table;
    return fill_table(table, r, t_ext, *rp, st);
  };
  return attn_bf16_impl(q, k, v, o, lse, rows, H, d, n_seq, cu_seqlens_dev, cu_seqlens_host,
                        softmax_scale, rope, stream, fixed_table);
}

extern "C" void dit_shutdown(void) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto& kv : g_tables) {
      cudaSetDevice(kv.first.dev);
      cudaFree(kv.second);
    }
    g_tables.clear();
    cudaSetDevice(cur);
  }
  // the fixed array's addresses are looked up again on next use (a device reset
  // between two uses would leave them stale)
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  g_noalloc_addr.clear();
}
