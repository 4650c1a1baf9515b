// bca.cu -- host side of libbca.so: argument validation, TMA descriptors, launches.
//
// The three calls of the method (see include/bca.h for the contract of each):
//   bca_prefill      step-1 block-causal attention (+ prefix K/V into a slot)
//   bca_kv_store     prefix K/V cache layout, bf16 or OFP8 E4M3 with per-head scales
//   bca_step_attend  cached-step target attention for a ragged same-phase batch
// and around them: bca_step_attend_q8 (the cached step with e4m3 Q against e4m3
// cached keys), bca_qk_norm_rope (Q/K RMS norm + rotary embedding of the rows
// entering attention), bca_step_graph_* (all layers' cached steps as one graph) and
// bca_ulysses_pack/unpack (layouts around the all-to-all of head-sharded
// sequence parallelism).
// Every step of the path runs in the kernels of attn_kernel.cuh, kv_store_kernel.cuh
// (also the Q quantisation of the e4m3-Q step), qk_norm_rope_kernel.cuh and
// ulysses_kernel.cuh; this file only checks arguments and enqueues them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <numeric>
#include <type_traits>
#include <vector>

#include "../../include/bca.h"
#include "attn_kernel.cuh"
#include "kv_expand_kernel.cuh"
#include "kv_store_kernel.cuh"
#include "qk_norm_rope_kernel.cuh"
#include "qkv_proj_kernel.cuh"
#include "ulysses_kernel.cuh"

namespace {

using bca::AttnParams;

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<unsigned long long*> g_trace{nullptr};
std::atomic<int> g_trace_cta{0};

// ---------------------------------------------------------------------------
// Driver entry point for cuTensorMapEncodeTiled (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode != nullptr;
}

// 3-D tiled map over a row-major tensor whose innermost dimension is the 128-wide
// head dimension.  dims/strides as the driver expects (dims[0] innermost, strides
// in bytes for dims 1..2).
bool make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0,
                 uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                 uint32_t b1, uint32_t b2) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1, stride2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, H, 128] bf16 activations: box = 64 head-dim elements x 1 head x 128 rows.
bool map_thd(CUtensorMap* m, const void* base, int64_t rows, int heads) {
  return make_map_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, heads,
                     static_cast<uint64_t>(rows), 128 * 2, static_cast<uint64_t>(heads) * 128 * 2,
                     64, 1, 128);
}

// [H, cap, 128] bf16 cache, exposing only the first n_tokens rows of each head
// (rows beyond read as zero and are masked by the kernel).
bool map_cache_bf16(CUtensorMap* m, const void* base, int n_tokens, int cap, int heads) {
  return make_map_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128,
                     static_cast<uint64_t>(std::max(n_tokens, 1)), static_cast<uint64_t>(heads),
                     128 * 2, static_cast<uint64_t>(cap) * 128 * 2, 64, 128, 1);
}

// [H, cap, 128] e4m3 cache: one 128-byte box row per token, 128 rows per box.
bool map_cache_e4m3(CUtensorMap* m, const void* base, int n_tokens, int cap, int heads) {
  return make_map_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128,
                     static_cast<uint64_t>(std::max(n_tokens, 1)), static_cast<uint64_t>(heads),
                     128, static_cast<uint64_t>(cap) * 128, 128, 128, 1);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device one-time kernel attribute setup.
template <typename K>
bool ensure_smem_attr(K kernel, int bytes, std::vector<char>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (done.size() <= static_cast<size_t>(dev)) done.resize(dev + 1, 0);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

bool dtype_valid(int32_t dt) { return dt == BCA_KV_BF16 || dt == BCA_KV_FP8_V || dt == BCA_KV_FP8_KV; }
bool k_is_fp8(int32_t dt) { return dt == BCA_KV_FP8_KV; }
bool v_is_fp8(int32_t dt) { return dt == BCA_KV_FP8_V || dt == BCA_KV_FP8_KV; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <typename T>
struct MaxRequests;
template <int MAXR>
struct MaxRequests<AttnParams<MAXR>> {
  static constexpr int value = MAXR;
};

// e4m3-Q scratch: codes [H, rows, 128], then scales [n_req][H] fp32.
size_t q8_codes_bytes(int64_t rows, int heads) {
  return round256(static_cast<size_t>(rows) * static_cast<size_t>(heads) * 128);
}
size_t q8_table_bytes(int n_req, int heads) {
  return round256(static_cast<size_t>(n_req) * static_cast<size_t>(heads) * 4);
}

struct SlotLayout {
  size_t k_off, v_off, ks_off, vs_off, total;
};

SlotLayout slot_layout(int32_t cap, int32_t heads, int32_t hd, int32_t dt) {
  SlotLayout L{};
  const size_t elems = static_cast<size_t>(cap) * heads * hd;
  const size_t kb = elems * (k_is_fp8(dt) ? 1 : 2);
  const size_t vb = elems * (v_is_fp8(dt) ? 1 : 2);
  L.k_off = 0;
  L.v_off = round256(kb);
  L.ks_off = L.v_off + round256(vb);
  L.vs_off = L.ks_off + round256(static_cast<size_t>(heads) * 4);
  L.total = L.vs_off + round256(static_cast<size_t>(heads) * 4);
  return L;
}

bca_status check_slot_shape(const bca_kv_slot* s, int heads, int hd) {
  if (!s || !s->k || !s->v) return BCA_ERR_INVALID_ARG;
  if (!dtype_valid(s->dtype) || s->cap_tokens < 0 || s->num_heads != heads ||
      s->head_dim != hd)
    return BCA_ERR_INVALID_ARG;
  if (!aligned16(s->k) || !aligned16(s->v)) return BCA_ERR_INVALID_ARG;
  if ((k_is_fp8(s->dtype) && (!s->k_scale || !aligned16(s->k_scale))) ||
      (v_is_fp8(s->dtype) && (!s->v_scale || !aligned16(s->v_scale))))
    return BCA_ERR_INVALID_ARG;
  return BCA_OK;
}

template <int MAXR, bool kQ8>
std::vector<char>& attr_flags() {
  static std::vector<char> done;  // per device: attributes set
  return done;
}

int sm_count() {
  static std::mutex mu;
  static std::vector<int> counts;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (counts.size() <= static_cast<size_t>(dev)) counts.resize(dev + 1, 0);
  if (!counts[dev] &&
      cudaDeviceGetAttribute(&counts[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    counts[dev] = 0;
  return counts[dev];
}

// Work-item schedule of the persistent kernel.  `unit_tiles(u)` gives the KV tiles
// of unit u (units are in scheduling order, heaviest first).  With a workspace, the
// units of the last partial round are split along the keys into k chunks so that
// all CTAs finish together: k = grid / leftover units, limited by the workspace,
// kMaxSplit and the smallest split unit's tile count.
template <int MAXR, typename TilesFn>
int plan_items(AttnParams<MAXR>& p, int units, int grid, size_t ws_chunks, TilesFn unit_tiles) {
  p.full_items = units;
  p.n_items = units;
  p.split_k = 1;
  p.split_units = 0;
  if (ws_chunks == 0 || units <= grid) return 0;
  const int rounds = units / grid, rem = units - rounds * grid;
  if (rem == 0) return 0;
  int k = std::min<int>(grid / rem, bca::kMaxSplit);
  k = std::min<int>(k, static_cast<int>(ws_chunks / static_cast<size_t>(rem)));
  for (int u = rounds * grid; u < units && k >= 2; ++u) k = std::min(k, unit_tiles(u));
  if (k < 2) return 0;
  p.full_items = rounds * grid;
  p.split_k = k;
  p.split_units = rem;
  p.n_items = rounds * grid + rem * k;
  return rem;
}

// Prefill schedule.  Units are in decreasing order of work (KV tiles).  The heavy
// units (at least half the heaviest) fill whole rounds; those of their last partial
// round are split along the keys (as in plan_items); the lighter units follow, whole,
// and fill the gaps the split chunks leave.  E.g. the T2I prefill (512 units of 36
// tiles, 64 of 4, 148 SMs): 3 whole rounds, 68 units in 2 chunks, then the 64 light
// units -- 130 tiles on the busiest SM instead of 144.
template <int MAXR, typename TilesFn>
int plan_items_weighted(AttnParams<MAXR>& p, int units, int grid, size_t ws_chunks,
                        TilesFn unit_tiles) {
  p.full_items = units;
  p.n_items = units;
  p.split_k = 1;
  p.split_units = 0;
  if (ws_chunks == 0 || units <= 1) return 0;
  const int wmax = unit_tiles(0);
  int heavy = 0;
  while (heavy < units && 2 * unit_tiles(heavy) >= wmax) ++heavy;
  const int rounds = heavy / grid, rem = heavy - rounds * grid;
  if (rem == 0) return 0;
  int k = std::min<int>(grid / rem, bca::kMaxSplit);
  k = std::min<int>(k, static_cast<int>(ws_chunks / static_cast<size_t>(rem)));
  for (int u = rounds * grid; u < heavy && k >= 2; ++u) k = std::min(k, unit_tiles(u));
  if (k < 2) return 0;
  p.full_items = rounds * grid;
  p.split_k = k;
  p.split_units = rem;
  p.n_items = units - rem + rem * k;
  return rem;
}

// One-time (per device) kernel attributes; also run before a stream capture so that
// no attribute call happens inside it.
template <int MAXR, bool kQ8 = false>
bool prepare_attn() {
  if (!ensure_smem_attr(bca::attn_fwd_kernel<MAXR, kQ8>, bca::Smem::kDynamicBytes,
                        attr_flags<MAXR, kQ8>()))
    return false;
  // The kernel re-splits its launch registers between warpgroups (setmaxnreg); that
  // only works if the compiled register count provides the pool the split assumes.
  static std::once_flag regs_once;
  static bool regs_ok = false;
  std::call_once(regs_once, [] {
    cudaFuncAttributes a{};
    regs_ok = cudaFuncGetAttributes(&a, bca::attn_fwd_kernel<MAXR, kQ8>) == cudaSuccess &&
              static_cast<uint32_t>(a.numRegs) * bca::kAttnThreads >=
                  128u * (2u * bca::kSoftmaxRegs + bca::kOtherRegs);
  });
  return regs_ok;
}

template <int MAXR, bool kQ8 = false>
bca_status launch_attn(const AttnParams<MAXR>& p, int n_split_units, cudaStream_t stream) {
  if (p.n_items <= 0) return BCA_OK;
  if (!prepare_attn<MAXR, kQ8>()) return BCA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  const int grid = std::min(sms, p.n_items);
  bca::attn_fwd_kernel<MAXR, kQ8>
      <<<grid, bca::kAttnThreads, bca::Smem::kDynamicBytes, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return BCA_ERR_CUDA;
  if (n_split_units > 0) {
    const int rows = n_split_units * bca::kChunkRows;
    const int blocks = (rows + bca::kCombineRowsPerBlock - 1) / bca::kCombineRowsPerBlock;
    bca::attn_combine_kernel<MAXR><<<blocks, 32 * bca::kCombineRowsPerBlock, 0, stream>>>(
        p, n_split_units);
    if (cudaGetLastError() != cudaSuccess) return BCA_ERR_CUDA;
  }
  return BCA_OK;
}

// One tensor (K or V of a request, or a request's Q) for the store kernel.
struct StoreJob {
  const void* src;
  void* dst;
  float* scale;
  int64_t row_stride;
  int64_t head_stride;
  int32_t rows;
  int32_t heads;
  bool quant;
};

// Clusters of the store kernel that can be resident at once on the current device
// (cached per device; the GPCs' sizes decide how many clusters of bca::kStoreCluster
// CTAs fit).  0: the kernel attribute could not be set.
int store_max_clusters() {
  static std::mutex mu;
  static std::vector<int> n;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (n.size() <= static_cast<size_t>(dev)) n.resize(dev + 1, 0);
  if (!n[dev]) {
    if (cudaFuncSetAttribute(bca::kv_store_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bca::kStoreRingBytes) != cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(bca::kStoreCluster));
    cfg.blockDim = dim3(bca::kStoreThreads);
    cfg.dynamicSmemBytes = bca::kStoreRingBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = bca::kStoreCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, bca::kv_store_kernel, &cfg) != cudaSuccess || c < 1)
      c = std::max(1, sm_count() / bca::kStoreCluster);
    n[dev] = c;
  }
  return n[dev];
}

// Source map of one store job: {128 channels, heads, rows} bf16 bits with the
// caller's row stride, box {128, 1, kStoreTileRows}, no swizzle.
bool map_store_src(CUtensorMap* m, const StoreJob& j) {
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(j.heads), static_cast<cuuint64_t>(j.rows)};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(j.row_stride) * 2};
  const cuuint32_t box[3] = {128, 1, static_cast<cuuint32_t>(bca::kStoreTileRows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(j.src), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One launch of bca::kv_store_kernel over every job, in clusters of
// bca::kStoreCluster CTAs, as many as are resident at once (so that few columns are
// in flight and the encode pass re-reads them from L2).  bf16 heads are cut into row
// pieces when there are too few of them to keep every cluster busy (about 8 columns
// per cluster); e4m3 heads stay whole.  Tensors with the longest columns go first.
bca_status launch_store(std::vector<StoreJob> jobs, int32_t* dev_status, cudaStream_t stream) {
  jobs.erase(std::remove_if(jobs.begin(), jobs.end(), [](const StoreJob& j) { return j.rows == 0; }),
             jobs.end());
  if (jobs.empty()) return BCA_OK;
  if (jobs.size() > static_cast<size_t>(bca::kMaxStoreTensors)) return BCA_ERR_INVALID_ARG;
  if (!get_encode()) return BCA_ERR_CUDA;
  const int max_clusters = store_max_clusters();
  if (max_clusters < 1) return BCA_ERR_CUDA;
  constexpr int csize = bca::kStoreCluster;
  int64_t quant_cols = 0, copy_cols = 0;
  for (const StoreJob& j : jobs) (j.quant ? quant_cols : copy_cols) += j.heads;
  std::vector<int> pieces(jobs.size(), 1);
  const int64_t want = 8LL * max_clusters;
  if (copy_cols > 0 && quant_cols + copy_cols < want) {
    const int64_t per = (want - quant_cols + copy_cols - 1) / copy_cols;
    for (size_t i = 0; i < jobs.size(); ++i) {
      if (jobs[i].quant) continue;
      // at least 2 tiles per CTA of the cluster in every piece
      const int64_t tiles = (jobs[i].rows + bca::kStoreTileRows - 1) / bca::kStoreTileRows;
      pieces[i] = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(per, tiles / (2 * csize))));
    }
  }
  std::vector<size_t> order(jobs.size());
  std::iota(order.begin(), order.end(), size_t{0});
  std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) {
    return static_cast<int64_t>(jobs[a].rows) * pieces[b] > static_cast<int64_t>(jobs[b].rows) * pieces[a];
  });
  static_assert(sizeof(bca::StoreParams) <= 32764, "kernel parameter limit");
  bca::StoreParams p;
  std::memset(&p, 0, sizeof(p));
  int cols = 0;
  for (size_t k = 0; k < order.size(); ++k) {
    const StoreJob& j = jobs[order[k]];
    if (!map_store_src(&p.map[k], j)) return BCA_ERR_INVALID_ARG;
    bca::StoreTensor& t = p.t[k];
    t.dst = j.dst;
    t.scale = j.scale;
    t.head_stride = j.head_stride;
    t.rows = j.rows;
    t.heads = j.heads;
    t.quant = j.quant ? 1 : 0;
    t.col0 = cols;
    t.pieces = pieces[order[k]];
    cols += j.heads * t.pieces;
  }
  p.n_tensors = static_cast<int32_t>(jobs.size());
  p.n_cols = cols;
  p.dev_status = dev_status;
  p.timeout_ns = g_timeout_ns.load();
  const int clusters = std::max(1, std::min(cols, max_clusters));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize));
  cfg.blockDim = dim3(bca::kStoreThreads);
  cfg.dynamicSmemBytes = bca::kStoreRingBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, bca::kv_store_kernel, p) != cudaSuccess) return BCA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

// The K and V jobs of one slot's store (no host-side slot updates).
void store_jobs(const void* k, const void* v, int32_t n_prefix, int64_t row_stride,
                const bca_kv_slot* slot, std::vector<StoreJob>& jobs) {
  const void* src[2] = {k, v};
  void* dst[2] = {slot->k, slot->v};
  float* sc[2] = {slot->k_scale, slot->v_scale};
  const bool q[2] = {k_is_fp8(slot->dtype), v_is_fp8(slot->dtype)};
  for (int t = 0; t < 2; ++t)
    jobs.push_back(StoreJob{src[t], dst[t], sc[t], row_stride, slot->cap_tokens, n_prefix,
                            slot->num_heads, q[t]});
}

bca_status validate_store(const void* k, const void* v, int32_t n_prefix, int64_t row_stride,
                          const bca_kv_slot* slot, uint32_t epoch) {
  if (!slot) return BCA_ERR_INVALID_ARG;
  if (slot->head_dim != 128) return BCA_ERR_UNSUPPORTED;
  if (slot->num_heads < 1 || slot->num_heads > 256) return BCA_ERR_INVALID_ARG;
  bca_status st = check_slot_shape(slot, slot->num_heads, 128);
  if (st != BCA_OK) return st;
  if (epoch == 0 || n_prefix < 0) return BCA_ERR_INVALID_ARG;
  if (n_prefix > slot->cap_tokens) return BCA_ERR_CAPACITY;
  if (n_prefix > 0) {
    if (!k || !v || !aligned16(k) || !aligned16(v)) return BCA_ERR_INVALID_ARG;
    if (row_stride < static_cast<int64_t>(slot->num_heads) * 128 || row_stride % 8 != 0)
      return BCA_ERR_INVALID_ARG;
  }
  return BCA_OK;
}

}  // namespace

extern "C" {

const char* bca_status_string(bca_status s) {
  switch (s) {
    case BCA_OK: return "BCA_OK";
    case BCA_ERR_INVALID_ARG: return "BCA_ERR_INVALID_ARG";
    case BCA_ERR_UNSUPPORTED: return "BCA_ERR_UNSUPPORTED";
    case BCA_ERR_CAPACITY: return "BCA_ERR_CAPACITY";
    case BCA_ERR_STATE: return "BCA_ERR_STATE";
    case BCA_ERR_CUDA: return "BCA_ERR_CUDA";
    case BCA_ERR_DEVICE_TIMEOUT: return "BCA_ERR_DEVICE_TIMEOUT";
    case BCA_ERR_NONFINITE: return "BCA_ERR_NONFINITE";
  }
  return "BCA_UNKNOWN_STATUS";
}

const char* bca_version(void) { return "bca 0.1.0 (sm_100a)"; }

void bca_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(std::max<uint64_t>(ns, 1000000ull));
}

bca_status bca_debug_set_trace(unsigned long long* dev_buffer, int32_t cta) {
#ifdef BCA_TRACE
  g_trace.store(dev_buffer);
  g_trace_cta.store(cta);
  return BCA_OK;
#else
  (void)dev_buffer;
  (void)cta;
  return BCA_ERR_UNSUPPORTED;
#endif
}

size_t bca_kv_slot_bytes(int32_t cap, int32_t heads, int32_t hd, bca_kv_dtype dt) {
  if (cap < 0 || heads < 1 || hd < 1 || !dtype_valid(dt)) return 0;
  return slot_layout(cap, heads, hd, dt).total;
}

bca_status bca_kv_slot_init(bca_kv_slot* slot, void* base, int32_t cap, int32_t heads,
                            int32_t hd, bca_kv_dtype dt) {
  if (!slot || !base || (reinterpret_cast<uintptr_t>(base) & 255u) != 0) return BCA_ERR_INVALID_ARG;
  if (cap < 0 || heads < 1 || hd < 1 || !dtype_valid(dt)) return BCA_ERR_INVALID_ARG;
  const SlotLayout L = slot_layout(cap, heads, hd, dt);
  char* b = static_cast<char*>(base);
  slot->k = b + L.k_off;
  slot->v = b + L.v_off;
  slot->k_scale = reinterpret_cast<float*>(b + L.ks_off);
  slot->v_scale = reinterpret_cast<float*>(b + L.vs_off);
  slot->cap_tokens = cap;
  slot->n_tokens = 0;
  slot->num_heads = heads;
  slot->head_dim = hd;
  slot->dtype = dt;
  slot->epoch = 0;
  return BCA_OK;
}

bca_status bca_kv_store(const void* k, const void* v, int32_t n_prefix, int32_t row_stride_elems,
                        bca_kv_slot* slot, uint32_t epoch, int32_t* dev_status, void* stream) {
  bca_status st = validate_store(k, v, n_prefix, row_stride_elems, slot, epoch);
  if (st != BCA_OK) return st;
  std::vector<StoreJob> jobs;
  store_jobs(k, v, n_prefix, row_stride_elems, slot, jobs);
  st = launch_store(std::move(jobs), dev_status, static_cast<cudaStream_t>(stream));
  if (st != BCA_OK) return st;
  slot->n_tokens = n_prefix;
  slot->epoch = epoch;
  return BCA_OK;
}

bca_status bca_kv_store_batch(const bca_kv_store_item* items, int32_t n_items, uint32_t epoch,
                              int32_t* dev_status, void* stream) {
  if (!items || n_items < 1 || n_items > BCA_MAX_BATCH) return BCA_ERR_INVALID_ARG;
  for (int i = 0; i < n_items; ++i) {
    bca_status st = validate_store(items[i].k, items[i].v, items[i].n_prefix,
                                   items[i].row_stride_elems, items[i].slot, epoch);
    if (st != BCA_OK) return st;
    for (int j = 0; j < i; ++j)
      if (items[j].slot == items[i].slot) return BCA_ERR_INVALID_ARG;
  }
  std::vector<StoreJob> jobs;
  for (int i = 0; i < n_items; ++i)
    store_jobs(items[i].k, items[i].v, items[i].n_prefix, items[i].row_stride_elems,
               items[i].slot, jobs);
  bca_status st = launch_store(std::move(jobs), dev_status, static_cast<cudaStream_t>(stream));
  if (st != BCA_OK) return st;
  for (int i = 0; i < n_items; ++i) {
    items[i].slot->n_tokens = items[i].n_prefix;
    items[i].slot->epoch = epoch;
  }
  return BCA_OK;
}

bca_status bca_prefill(const void* q, const void* k, const void* v, void* o, int32_t seq_len,
                       const int32_t* off, int32_t n_blocks, int32_t heads, int32_t head_dim,
                       float scale, bca_kv_slot* slot, uint32_t epoch, int32_t* dev_status,
                       void* stream) {
  return bca_prefill_ws(q, k, v, o, seq_len, off, n_blocks, heads, head_dim, scale, slot, epoch,
                        nullptr, 0, dev_status, stream);
}

bca_status bca_prefill_ws(const void* q, const void* k, const void* v, void* o, int32_t seq_len,
                          const int32_t* off, int32_t n_blocks, int32_t heads, int32_t head_dim,
                          float scale, bca_kv_slot* slot, uint32_t epoch, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BCA_ERR_INVALID_ARG;
  const size_t ws_chunks = workspace ? workspace_bytes / bca::kChunkBytes : 0;
  if (!q || !k || !v || !o || !off) return BCA_ERR_INVALID_ARG;
  if (head_dim != 128) return BCA_ERR_UNSUPPORTED;
  if (heads < 1 || heads > 256 || seq_len < 1) return BCA_ERR_INVALID_ARG;
  if (n_blocks < 1 || n_blocks > BCA_MAX_BLOCKS) return BCA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return BCA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return BCA_ERR_INVALID_ARG;
  if (off[0] != 0 || off[n_blocks] != seq_len) return BCA_ERR_INVALID_ARG;
  for (int b = 0; b < n_blocks; ++b)
    if (off[b + 1] <= off[b]) return BCA_ERR_INVALID_ARG;
  const int32_t n_prefix = off[n_blocks - 1];
  if (slot) {
    if (slot->num_heads != heads) return BCA_ERR_INVALID_ARG;
    bca_status st = validate_store(k, v, n_prefix, static_cast<int64_t>(heads) * 128, slot, epoch);
    if (st != BCA_OK) return st;
  }
  if (!get_encode()) return BCA_ERR_CUDA;
  AttnParams<1> p;
  std::memset(&p, 0, sizeof(p));
  if (!map_thd(&p.tm_q, q, seq_len, heads) || !map_thd(&p.tm_k, k, seq_len, heads) ||
      !map_thd(&p.tm_o, o, seq_len, heads) ||
      !map_thd(&p.tm_v, v, seq_len, heads))
    return BCA_ERR_CUDA;
  p.tm_kc[0] = p.tm_k;  // unused in prefill mode
  p.tm_vc[0] = p.tm_v;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_rows = seq_len;
  p.dev_status = dev_status;
  p.trace = g_trace.load();
  p.trace_cta = g_trace_cta.load();
  p.timeout_ns = g_timeout_ns.load();
  p.heads = heads;
  p.mode = bca::kModePrefill;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.seq_len = seq_len;
  p.n_blocks = n_blocks;
  for (int b = 0; b <= n_blocks; ++b) p.block_off[b] = off[b];
  const int nqp = (seq_len + 2 * bca::kBM - 1) / (2 * bca::kBM);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  p.workspace = static_cast<float*>(workspace);
  // Unit u: Q-tile pair nqp - 1 - u / heads (its last row's block end sets its tiles).
  const int n_split = plan_items_weighted(p, nqp * heads, sms, ws_chunks, [&](int u) {
    const int qp = nqp - 1 - u / heads;
    const int last = std::min(seq_len, (qp + 1) * 2 * bca::kBM) - 1;
    int lim = seq_len;
    for (int b = 1; b <= n_blocks; ++b)
      if (last < off[b]) {
        lim = off[b];
        break;
      }
    return (lim + bca::kBN - 1) / bca::kBN;
  });
  bca_status st = launch_attn(p, n_split, s);
  if (st != BCA_OK) return st;
  if (slot) {
    std::vector<StoreJob> jobs;
    store_jobs(k, v, n_prefix, static_cast<int64_t>(heads) * 128, slot, jobs);
    st = launch_store(std::move(jobs), dev_status, s);
    if (st != BCA_OK) return st;
    slot->n_tokens = n_prefix;
    slot->epoch = epoch;
  }
  return BCA_OK;
}

size_t bca_step_workspace_bytes(void) {
  const int sms = sm_count();
  return sms > 0 ? static_cast<size_t>(sms) * bca::kChunkBytes : 0;
}

size_t bca_step_q8_scratch_bytes(int64_t rows, int32_t n_req, int32_t heads) {
  if (rows < 0 || n_req < 1 || n_req > BCA_MAX_BATCH || heads < 1 || heads > 256) return 0;
  return q8_codes_bytes(rows, heads) + q8_table_bytes(n_req, heads);
}

// Bytes of the bf16 expansion of one e4m3 cache tensor (rows x heads x 128).
static size_t dq_tensor_bytes(int32_t rows, int32_t heads) {
  return round256(static_cast<size_t>(rows) * static_cast<size_t>(heads) * 128 * 2);
}

size_t bca_step_dq_scratch_bytes(const bca_kv_slot* slots, int32_t n_req) {
  if (!slots || n_req < 1 || n_req > BCA_MAX_BATCH) return 0;
  size_t n = 0;
  for (int r = 0; r < n_req; ++r) {
    const bca_kv_slot& s = slots[r];
    if (s.n_tokens < 0 || s.num_heads < 1 || !dtype_valid(s.dtype)) return 0;
    if (k_is_fp8(s.dtype)) n += dq_tensor_bytes(s.n_tokens, s.num_heads);
    if (v_is_fp8(s.dtype)) n += dq_tensor_bytes(s.n_tokens, s.num_heads);
  }
  return n;
}

// The cached step; with q8_scratch, in e4m3-Q mode (bca_step_attend_q8); with dq, the
// e4m3 cache tensors are first expanded to bf16 in dq_scratch (bca_step_attend_dq).
static bca_status step_attend_impl(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                                   const int32_t* cu, const bca_kv_slot* slots, int32_t n_req,
                                   int32_t heads, int32_t head_dim, float scale, void* workspace,
                                   size_t workspace_bytes, bool q8, void* q8_scratch,
                                   size_t q8_bytes, int32_t* dev_status, void* stream,
                                   bool dq = false, void* dq_scratch = nullptr,
                                   size_t dq_bytes = 0) {
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BCA_ERR_INVALID_ARG;
  const size_t ws_chunks = workspace ? workspace_bytes / bca::kChunkBytes : 0;
  if (!cu || !slots) return BCA_ERR_INVALID_ARG;
  if (head_dim != 128) return BCA_ERR_UNSUPPORTED;
  if (heads < 1 || heads > 256 || n_req < 1 || n_req > BCA_MAX_BATCH) return BCA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return BCA_ERR_INVALID_ARG;
  if (cu[0] != 0) return BCA_ERR_INVALID_ARG;
  for (int r = 0; r < n_req; ++r)
    if (cu[r + 1] < cu[r]) return BCA_ERR_INVALID_ARG;
  const int32_t total = cu[n_req];
  if (total > 0) {
    if (!q_t || !k_t || !v_t || !o_t) return BCA_ERR_INVALID_ARG;
    if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(o_t))
      return BCA_ERR_INVALID_ARG;
  }
  for (int r = 0; r < n_req; ++r) {
    bca_status st = check_slot_shape(&slots[r], heads, 128);
    if (st != BCA_OK) return st;
    if (slots[r].epoch == 0) return BCA_ERR_STATE;
    if (slots[r].n_tokens < 0 || slots[r].n_tokens > slots[r].cap_tokens)
      return BCA_ERR_INVALID_ARG;
    if (slots[r].dtype != slots[0].dtype) return BCA_ERR_UNSUPPORTED;
  }
  if (q8) {
    if (slots[0].dtype != BCA_KV_FP8_KV) return BCA_ERR_UNSUPPORTED;
    if (!q8_scratch || (reinterpret_cast<uintptr_t>(q8_scratch) & 255u) != 0)
      return BCA_ERR_INVALID_ARG;
    if (q8_bytes < bca_step_q8_scratch_bytes(total, n_req, heads)) return BCA_ERR_CAPACITY;
  }
  std::vector<void*> dq_k(n_req, nullptr), dq_v(n_req, nullptr);
  if (dq) {
    if (slots[0].dtype == BCA_KV_BF16) return BCA_ERR_UNSUPPORTED;
    if (!dq_scratch || (reinterpret_cast<uintptr_t>(dq_scratch) & 255u) != 0)
      return BCA_ERR_INVALID_ARG;
    for (int r = 0; r < n_req; ++r)  // 32-bit chunk indices in the expansion kernel
      if (static_cast<int64_t>(slots[r].n_tokens) * heads * 8 >= (int64_t{1} << 32))
        return BCA_ERR_UNSUPPORTED;
    if (dq_bytes < bca_step_dq_scratch_bytes(slots, n_req)) return BCA_ERR_CAPACITY;
    char* b = static_cast<char*>(dq_scratch);
    for (int r = 0; r < n_req; ++r) {
      if (k_is_fp8(slots[r].dtype)) {
        dq_k[r] = b;
        b += dq_tensor_bytes(slots[r].n_tokens, heads);
      }
      if (v_is_fp8(slots[r].dtype)) {
        dq_v[r] = b;
        b += dq_tensor_bytes(slots[r].n_tokens, heads);
      }
    }
  }
  if (total == 0) return BCA_OK;
  const int32_t dt = slots[0].dtype;
  if (dq) {
    // Expand every e4m3 cache tensor that a request with target rows reads.
    bca::ExpandParams ep;
    std::memset(&ep, 0, sizeof(ep));
    int n = 0, max_chunks = 0;
    for (int r = 0; r < n_req; ++r) {
      if (cu[r + 1] == cu[r] || slots[r].n_tokens == 0) continue;
      for (int kv = 0; kv < 2; ++kv) {
        void* d = kv ? dq_v[r] : dq_k[r];
        if (!d) continue;
        bca::ExpandTensor& t = ep.t[n++];
        t.src = static_cast<const uint8_t*>(kv ? slots[r].v : slots[r].k);
        t.dst = static_cast<uint16_t*>(d);
        t.cap = slots[r].cap_tokens;
        t.rows = slots[r].n_tokens;
        t.heads = heads;
        max_chunks = std::max(max_chunks, slots[r].n_tokens * heads * 8);
      }
    }
    ep.n_tensors = n;
    if (n > 0) {
      const int sms = std::max(sm_count(), 1);
      const int bx = std::max(1, std::min((max_chunks + bca::kExpandThreads - 1) / bca::kExpandThreads,
                                          std::max(1, 8 * sms / n)));
      bca::kv_expand_kernel<<<dim3(bx, n), bca::kExpandThreads, 0,
                              static_cast<cudaStream_t>(stream)>>>(ep);
      if (cudaGetLastError() != cudaSuccess) return BCA_ERR_CUDA;
    }
  }
  if (!get_encode()) return BCA_ERR_CUDA;
  uint8_t* q8_codes = static_cast<uint8_t*>(q8_scratch);
  float* q8_scale = q8 ? reinterpret_cast<float*>(q8_codes + q8_codes_bytes(total, heads)) : nullptr;
  if (q8) {
    // Q codes and scales of every request, before the attention reads them: each
    // request's Q is stored like an e4m3 cache tensor into [H, total, 128].
    std::vector<StoreJob> jobs;
    const int64_t row_elems = static_cast<int64_t>(heads) * 128;
    for (int r = 0; r < n_req; ++r)
      jobs.push_back(StoreJob{static_cast<const uint16_t*>(q_t) + cu[r] * row_elems,
                              q8_codes + static_cast<int64_t>(cu[r]) * 128,
                              q8_scale + static_cast<size_t>(r) * heads, row_elems, total,
                              cu[r + 1] - cu[r], heads, true});
    bca_status st = launch_store(std::move(jobs), dev_status, static_cast<cudaStream_t>(stream));
    if (st != BCA_OK) return st;
  }

  // Longest key sequence first (largest per-unit work scheduled first).
  std::vector<int> order;
  for (int r = 0; r < n_req; ++r)
    if (cu[r + 1] > cu[r]) order.push_back(r);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return slots[a].n_tokens + (cu[a + 1] - cu[a]) > slots[b].n_tokens + (cu[b + 1] - cu[b]);
  });
  const int nr = static_cast<int>(order.size());
  auto fill = [&](auto& p) -> bca_status {
    std::memset(&p, 0, sizeof(p));
    if (!map_thd(&p.tm_q, q_t, total, heads) || !map_thd(&p.tm_k, k_t, total, heads) ||
        !map_thd(&p.tm_o, o_t, total, heads) ||
        !map_thd(&p.tm_v, v_t, total, heads))
      return BCA_ERR_CUDA;
    p.o = static_cast<__nv_bfloat16*>(o_t);
    p.o_rows = total;
    p.dev_status = dev_status;
    p.trace = g_trace.load();
    p.trace_cta = g_trace_cta.load();
    p.timeout_ns = g_timeout_ns.load();
    p.heads = heads;
    p.mode = bca::kModeStep;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_req = nr;
    p.k_fp8 = k_is_fp8(dt) && !dq ? 1 : 0;
    p.v_fp8 = v_is_fp8(dt) && !dq ? 1 : 0;
    p.k_scaled = k_is_fp8(dt) ? 1 : 0;
    p.v_scaled = v_is_fp8(dt) ? 1 : 0;
    int units = 0;
    for (int i = 0; i < nr; ++i) {
      const int r = order[i];
      const bca_kv_slot& sl = slots[r];
      // dq: the expanded tensors, [H, n_tokens, 128] bf16
      const bool kok =
          p.k_fp8 ? map_cache_e4m3(&p.tm_kc[i], sl.k, sl.n_tokens, sl.cap_tokens, heads)
          : dq_k[r] && sl.n_tokens > 0
              ? map_cache_bf16(&p.tm_kc[i], dq_k[r], sl.n_tokens, sl.n_tokens, heads)
                    : map_cache_bf16(&p.tm_kc[i], sl.k, sl.n_tokens, sl.cap_tokens, heads);
      const bool vok =
          p.v_fp8 ? map_cache_e4m3(&p.tm_vc[i], sl.v, sl.n_tokens, sl.cap_tokens, heads)
          : dq_v[r] && sl.n_tokens > 0
              ? map_cache_bf16(&p.tm_vc[i], dq_v[r], sl.n_tokens, sl.n_tokens, heads)
                    : map_cache_bf16(&p.tm_vc[i], sl.v, sl.n_tokens, sl.cap_tokens, heads);
      if (!kok || !vok) return BCA_ERR_CUDA;
      p.k_scale[i] = sl.k_scale;
      p.v_scale[i] = sl.v_scale;
      p.q_scale[i] = q8 ? q8_scale + static_cast<size_t>(r) * heads : nullptr;
      p.q_start[i] = cu[r];
      p.q_len[i] = cu[r + 1] - cu[r];
      p.n_cache[i] = sl.n_tokens;
      p.unit_start[i] = units;
      units += heads * ((p.q_len[i] + 2 * bca::kBM - 1) / (2 * bca::kBM));
    }
    p.unit_start[nr] = units;
    // e4m3-Q codes [H, total, 128]: one 128-byte box row per (head, row).
    if (q8 && !make_map_3d(&p.tm_q8, q8_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128,
                           static_cast<uint64_t>(total), static_cast<uint64_t>(heads), 128,
                           static_cast<uint64_t>(total) * 128, 128, 128, 1))
      return BCA_ERR_CUDA;
    p.workspace = static_cast<float*>(workspace);
    const int sms = sm_count();
    if (sms <= 0) return BCA_ERR_CUDA;
    const int n_split = plan_items(p, units, sms, ws_chunks, [&](int unit) {
      int i = 0;
      while (i + 1 < nr && unit >= p.unit_start[i + 1]) ++i;
      return (p.n_cache[i] + bca::kBN - 1) / bca::kBN + (p.q_len[i] + bca::kBN - 1) / bca::kBN;
    });
    constexpr int kMaxR = MaxRequests<std::remove_reference_t<decltype(p)>>::value;
    return q8 ? launch_attn<kMaxR, true>(p, n_split, static_cast<cudaStream_t>(stream))
              : launch_attn<kMaxR, false>(p, n_split, static_cast<cudaStream_t>(stream));
  };
  if (nr <= 1) {
    AttnParams<1> p;
    return fill(p);
  } else if (nr <= 8) {
    AttnParams<8> p;
    return fill(p);
  }
  AttnParams<64> p;
  return fill(p);
}

bca_status bca_step_attend(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                           const int32_t* cu, const bca_kv_slot* slots, int32_t n_req,
                           int32_t heads, int32_t head_dim, float scale, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return step_attend_impl(q_t, k_t, v_t, o_t, cu, slots, n_req, heads, head_dim, scale, workspace,
                          workspace_bytes, false, nullptr, 0, dev_status, stream);
}

bca_status bca_step_attend_dq(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                              const int32_t* cu, const bca_kv_slot* slots, int32_t n_req,
                              int32_t heads, int32_t head_dim, float scale, void* workspace,
                              size_t workspace_bytes, void* dq_scratch, size_t dq_scratch_bytes,
                              int32_t* dev_status, void* stream) {
  return step_attend_impl(q_t, k_t, v_t, o_t, cu, slots, n_req, heads, head_dim, scale, workspace,
                          workspace_bytes, false, nullptr, 0, dev_status, stream, true, dq_scratch,
                          dq_scratch_bytes);
}

bca_status bca_step_attend_q8(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                              const int32_t* cu, const bca_kv_slot* slots, int32_t n_req,
                              int32_t heads, int32_t head_dim, float scale, void* workspace,
                              size_t workspace_bytes, void* q8_scratch, size_t q8_scratch_bytes,
                              int32_t* dev_status, void* stream) {
  return step_attend_impl(q_t, k_t, v_t, o_t, cu, slots, n_req, heads, head_dim, scale, workspace,
                          workspace_bytes, true, q8_scratch, q8_scratch_bytes, dev_status, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Bounded-wait self-check
// ---------------------------------------------------------------------------
namespace {
__global__ void selftest_wait_kernel(int32_t* dev_status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort;
  const uint32_t b = bca::smem_u32(&bar);
  if (threadIdx.x == 0) {
    bca::mbar_init(b, 1);  // nothing ever arrives
    abort = 0;
    bca::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = bca::mbar_wait_bounded(b, 0, &abort, timeout_ns);
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0)
    bca::raise_abort(reinterpret_cast<volatile int*>(&abort), dev_status);
}
}  // namespace

extern "C" bca_status bca_selftest_wait_timeout(int32_t* dev_status, uint64_t timeout_ns,
                                                void* stream) {
  if (!dev_status) return BCA_ERR_INVALID_ARG;
  if (timeout_ns < 1000000ull || timeout_ns > 10000000000ull) return BCA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

extern "C" bca_status bca_selftest_e4m3_division(unsigned long long* mismatches, void* stream) {
  if (!mismatches) return BCA_ERR_INVALID_ARG;
  bca::e4m3_division_selftest_kernel<<<0x7F7F, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      mismatches);
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// bca_step_attend_noalloc: the cached step for callers that cannot allocate device
// memory.  Its split-chunk scratch is a file-scope device array instead of a
// caller-provided workspace; the GPU holds the array for as long as the library is
// loaded.
// ---------------------------------------------------------------------------
namespace {
// Capacity in split chunks (256 rows x (128 + 2) fp32 each): 160 x 133,120 B
// = 21.3 MB.  A split schedule uses at most one chunk per SM.
constexpr size_t kNoAllocChunks = 160;
constexpr size_t kNoAllocBytes = kNoAllocChunks * bca::kChunkBytes;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocBytes / sizeof(float)];

// Device address of g_noalloc_scratch on the current device.  Host code must not
// use the symbol itself (that is a host-side stand-in, not a device address); the
// address is looked up once per device, with that device current, and cached.
bool noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static std::vector<void*> ptrs;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(mu);
  if (ptrs.size() <= static_cast<size_t>(dev)) ptrs.resize(dev + 1, nullptr);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return false;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return true;
}
}  // namespace

extern "C" bca_status bca_step_attend_noalloc(const void* q_t, const void* k_t, const void* v_t,
                                              void* o_t, const int32_t* cu_target,
                                              const bca_kv_slot* slots, int32_t n_req,
                                              int32_t heads, int32_t head_dim, float scale,
                                              int32_t* dev_status, void* stream) {
  // The largest split schedule needs one chunk per SM.
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  if (static_cast<size_t>(sms) > kNoAllocChunks) return BCA_ERR_CAPACITY;
  void* scratch = nullptr;
  if (!noalloc_scratch_ptr(&scratch)) return BCA_ERR_CUDA;
  return bca_step_attend(q_t, k_t, v_t, o_t, cu_target, slots, n_req, heads, head_dim, scale,
                         scratch, kNoAllocBytes, dev_status, stream);
}

// ---------------------------------------------------------------------------
// Cached-step graphs: the launches of bca_step_attend for every layer of a fixed
// layout, recorded once by stream capture and replayed with one graph launch.
// ---------------------------------------------------------------------------
struct bca_step_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int device = -1;
  int32_t kernel_nodes = 0;
};

extern "C" bca_status bca_step_graph_create(const bca_step_graph_desc* d, bca_step_graph** out) {
  if (!d || !out) return BCA_ERR_INVALID_ARG;
  *out = nullptr;
  if (d->n_layers < 1 || d->n_layers > 4096 || !d->q_t || !d->k_t || !d->v_t || !d->o_t ||
      !d->slots || !d->cu_target || d->n_req < 1 || d->n_req > BCA_MAX_BATCH)
    return BCA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BCA_ERR_CUDA;
  if (!prepare_attn<1>() || !prepare_attn<8>() || !prepare_attn<64>() || sm_count() <= 0 ||
      !get_encode())
    return BCA_ERR_CUDA;
  const bool q8 = d->q8_scratch != nullptr;
  const bool dq = d->dq_scratch != nullptr;
  if (q8 && dq) return BCA_ERR_INVALID_ARG;
  if (q8 && (!prepare_attn<1, true>() || !prepare_attn<8, true>() || !prepare_attn<64, true>()))
    return BCA_ERR_CUDA;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return BCA_ERR_CUDA;
  // Each layer's call checks its arguments before it records anything; the first
  // failing layer ends the capture and its status is returned.
  bca_status st = BCA_OK;
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    st = BCA_ERR_CUDA;
  } else {
    for (int l = 0; l < d->n_layers && st == BCA_OK; ++l)
      st = step_attend_impl(d->q_t[l], d->k_t[l], d->v_t[l], d->o_t[l], d->cu_target,
                            d->slots + static_cast<size_t>(l) * d->n_req, d->n_req, d->heads,
                            d->head_dim, d->scale, d->workspace, d->workspace_bytes, q8,
                            d->q8_scratch, d->q8_scratch_bytes, d->dev_status, cs, dq,
                            d->dq_scratch, d->dq_scratch_bytes);
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess && st == BCA_OK) st = BCA_ERR_CUDA;
  }
  cudaStreamDestroy(cs);
  auto* g = new bca_step_graph();
  g->graph = graph;
  g->device = dev;
  if (st == BCA_OK && graph) {
    size_t n = 0;
    if (cudaGraphGetNodes(graph, nullptr, &n) != cudaSuccess) st = BCA_ERR_CUDA;
    std::vector<cudaGraphNode_t> nodes(n);
    if (st == BCA_OK && n > 0 && cudaGraphGetNodes(graph, nodes.data(), &n) != cudaSuccess)
      st = BCA_ERR_CUDA;
    for (size_t i = 0; st == BCA_OK && i < n; ++i) {
      cudaGraphNodeType t;
      if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) st = BCA_ERR_CUDA;
      else if (t == cudaGraphNodeTypeKernel) ++g->kernel_nodes;
    }
    if (st == BCA_OK && n > 0 && cudaGraphInstantiate(&g->exec, graph, 0) != cudaSuccess)
      st = BCA_ERR_CUDA;
  } else if (st == BCA_OK) {
    st = BCA_ERR_CUDA;
  }
  if (st != BCA_OK) {
    bca_step_graph_destroy(g);
    cudaGetLastError();  // clear a capture error so later calls see a clean state
    return st;
  }
  *out = g;
  return BCA_OK;
}

extern "C" bca_status bca_step_graph_launch(const bca_step_graph* g, void* stream) {
  if (!g) return BCA_ERR_INVALID_ARG;
  if (!g->exec) return BCA_OK;  // a layout without target rows records nothing
  return cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BCA_OK
             : BCA_ERR_CUDA;
}

extern "C" int32_t bca_step_graph_kernel_nodes(const bca_step_graph* g) {
  return g ? g->kernel_nodes : 0;
}

extern "C" void bca_step_graph_destroy(bca_step_graph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

// ---------------------------------------------------------------------------
// Q/K RMS norm + rotary embedding (in place)
// ---------------------------------------------------------------------------
extern "C" bca_status bca_qk_norm_rope(void* q, void* k, int64_t rows, int32_t heads,
                                       int32_t head_dim, const float* gamma_q,
                                       const float* gamma_k, const float* cos_t,
                                       const float* sin_t, float eps, void* stream) {
  if (head_dim != 128) return BCA_ERR_UNSUPPORTED;
  if (rows < 0 || heads < 1 || heads > 256 || !(eps > 0.0f) || !std::isfinite(eps))
    return BCA_ERR_INVALID_ARG;
  if (rows == 0) return BCA_OK;
  if (!q && !k) return BCA_ERR_INVALID_ARG;
  if ((q && (!aligned16(q) || !gamma_q || !aligned16(gamma_q))) ||
      (k && (!aligned16(k) || !gamma_k || !aligned16(gamma_k))) || !cos_t || !sin_t ||
      !aligned16(cos_t) || !aligned16(sin_t))
    return BCA_ERR_INVALID_ARG;
  bca::QkNormRopeParams p{};
  p.x[0] = static_cast<uint16_t*>(q);
  p.x[1] = static_cast<uint16_t*>(k);
  p.gamma[0] = gamma_q;
  p.gamma[1] = gamma_k;
  p.cos_t = cos_t;
  p.sin_t = sin_t;
  p.rows = rows;
  p.heads = heads;
  p.eps = eps;
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  const int64_t want = (2 * rows + bca::kNormWarpsPerBlock - 1) / bca::kNormWarpsPerBlock;
  const int blocks = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  bca::qk_norm_rope_kernel<<<blocks, bca::kNormThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Q/K/V projection with the Q/K norm and rotary embedding in the epilogue
// ---------------------------------------------------------------------------
namespace {
// 2-D tiled map, 128-byte swizzle: dims (d0 inner, d1), row stride in bytes.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1,
                 uint32_t b0, uint32_t b1) {
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride1};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
std::vector<char>& proj_attr_flags() {
  static std::vector<char> done;
  return done;
}
}  // namespace

extern "C" bca_status bca_qkv_project(const void* x, const void* w, void* q, void* k, void* v,
                                      int32_t rows, int32_t d_model, int32_t heads,
                                      int32_t head_dim, const float* gamma_q,
                                      const float* gamma_k, const float* cos_t,
                                      const float* sin_t, float eps, int32_t* dev_status,
                                      void* stream) {
  if (head_dim != 128) return BCA_ERR_UNSUPPORTED;
  if (d_model < 64 || d_model % 64 != 0) return BCA_ERR_UNSUPPORTED;
  if (rows < 0 || heads < 1 || heads > 256 || !(eps > 0.0f) || !std::isfinite(eps))
    return BCA_ERR_INVALID_ARG;
  if (rows == 0) return BCA_OK;
  for (const void* ptr : {x, w, static_cast<const void*>(q), static_cast<const void*>(k),
                          static_cast<const void*>(v), static_cast<const void*>(gamma_q),
                          static_cast<const void*>(gamma_k), static_cast<const void*>(cos_t),
                          static_cast<const void*>(sin_t)})
    if (!ptr || !aligned16(ptr)) return BCA_ERR_INVALID_ARG;
  if (!get_encode()) return BCA_ERR_CUDA;
  const int64_t feats = 3ll * heads * 128;
  bca::ProjParams p;
  std::memset(&p, 0, sizeof(p));
  if (!make_map_2d(&p.tm_x, x, d_model, rows, static_cast<uint64_t>(d_model) * 2, bca::kPBK,
                   bca::kPBM) ||
      !make_map_2d(&p.tm_w, w, d_model, feats, static_cast<uint64_t>(d_model) * 2, bca::kPBK,
                   bca::kPBN) ||
      !map_thd(&p.tm_out[0], q, rows, heads) || !map_thd(&p.tm_out[1], k, rows, heads) ||
      !map_thd(&p.tm_out[2], v, rows, heads))
    return BCA_ERR_CUDA;
  p.gamma_q = gamma_q;
  p.gamma_k = gamma_k;
  p.cos_t = cos_t;
  p.sin_t = sin_t;
  p.rows = rows;
  p.heads = heads;
  p.m_tiles = (rows + bca::kPBM - 1) / bca::kPBM;
  p.n_tiles = static_cast<int32_t>((feats + bca::kPBN - 1) / bca::kPBN);
  p.k_steps = d_model / bca::kPBK;
  p.eps = eps;
  p.dev_status = dev_status;
  p.timeout_ns = g_timeout_ns.load();
  if (!ensure_smem_attr(bca::qkv_proj_kernel, bca::ProjSmem::kDynamicBytes, proj_attr_flags()))
    return BCA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  const int grid = std::min(sms, p.m_tiles * p.n_tiles);
  bca::qkv_proj_kernel<<<grid, bca::kPThreads, bca::ProjSmem::kDynamicBytes,
                         static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Ulysses re-sharding copies
// ---------------------------------------------------------------------------
namespace {
template <bool kPack>
bca_status ulysses_copy(const void* src, void* dst, int64_t rows, int32_t heads, int32_t hd,
                        int32_t n_ranks, void* stream) {
  if (hd != 128) return BCA_ERR_UNSUPPORTED;
  if (rows < 0 || n_ranks < 1 || heads < 1 || heads > 256 || heads % n_ranks != 0)
    return BCA_ERR_INVALID_ARG;
  if (rows == 0) return BCA_OK;
  if (!src || !dst || !aligned16(src) || !aligned16(dst)) return BCA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return BCA_ERR_CUDA;
  const int64_t n = rows * heads * 16;
  const int blocks = static_cast<int>(
      std::min<int64_t>((n + bca::kUlyssesThreads - 1) / bca::kUlyssesThreads,
                        static_cast<int64_t>(sms) * 8));
  bca::ulysses_copy_kernel<kPack><<<blocks, bca::kUlyssesThreads, 0,
                                    static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, heads, n_ranks);
  return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}
}  // namespace

extern "C" bca_status bca_ulysses_pack(const void* x, void* send, int64_t rows_local,
                                       int32_t heads, int32_t head_dim, int32_t n_ranks,
                                       void* stream) {
  return ulysses_copy<true>(x, send, rows_local, heads, head_dim, n_ranks, stream);
}

extern "C" bca_status bca_ulysses_unpack(const void* recv, void* x, int64_t rows_local,
                                         int32_t heads, int32_t head_dim, int32_t n_ranks,
                                         void* stream) {
  return ulysses_copy<false>(recv, x, rows_local, heads, head_dim, n_ranks, stream);
}
