// kv_store_kernel.cuh -- prefix K/V cache writes, optionally OFP8 E4M3.
//
// What it computes ("Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV cache": the
// prompt and reference-image K/V from the first denoising step are kept for the
// rest of the generation, in the native dtype or in FP8 -- "fp8_v" quantises V
// only, "fp8" K and V):
//   bf16 tensor : cache[h, t, :] = x[t, h, :]                     for t < P
//   e4m3 tensor : amax_h = max_{t<P, c} |x[t, h, c]|
//                 s_h    = fp32(amax_h) / 448 (correctly rounded; 1 if amax_h = 0)
//                 cache[h, t, c] = e4m3_rn_satfinite(x[t, h, c] / s_h)   (fp32 quotient,
//                                  correctly rounded), scale[h] = s_h
// HBM-bound; one kernel (kv_store_kernel below) per store call, whatever the
// number of requests, with no scratch memory.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "../../include/bca.h"
#include "ptx.cuh"

namespace bca {

// Lane-wise unsigned 16-bit maximum of two packed pairs (sm_90+).
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float scale_from_amax_bits(unsigned bits) {
  const float amax = __uint_as_float(bits << 16);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// x / s for the encoder, from y = RN(1/s): q = RN(x y), then one correction with the
// exact residual x - q s (an FMA):  RN(q + (x - q s) y) -- the division scheme of
// P. Markstein, "IA-64 and Elementary Functions: Speed and Precision" (2000), ch. 8.
// The encoder runs it on two lanes at once (packed fp32x2 multiply and FMAs).  Its
// result has x's sign for every x except -0 (which comes out +0); the encoder
// therefore ORs each value's sign bit into its code afterwards.  For heads whose
// amax is below 2^-95 (bf16 bits < kFastDivMinBits) the reciprocal and the residual
// leave the normal range, so those take the correctly rounded division.
// bca_selftest_e4m3_division runs encode_chunk itself for every bf16 amax and every
// bf16 |x| <= amax and compares its codes with those of the correctly rounded
// quotient.
constexpr unsigned kFastDivMinBits = 0x1000u;

// Two fp32 -> packed e4m3x2, round to nearest even, saturate to +-448;
// `lo` lands in bits [0, 8).
__device__ __forceinline__ uint16_t e4m3x2_rn_satfinite(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Codes of one bf16 pair (channel 2i in the low half): a 16-bit e4m3 pair.
__device__ __forceinline__ uint32_t encode_word(uint32_t w, float s, uint64_t yy, uint64_t nss,
                                                bool fast) {
  float lo, hi;
  if (fast) {
    const uint64_t x = f2_pack(bf16_lo(w), bf16_hi(w));
    const uint64_t q = f2_mul(x, yy);
    const uint64_t r = f2_fma(q, nss, x);
    f2_unpack(f2_fma(r, yy, q), lo, hi);
  } else {
    lo = __fdiv_rn(bf16_lo(w), s);
    hi = __fdiv_rn(bf16_hi(w), s);
  }
  return e4m3x2_rn_satfinite(lo, hi);
}

// Codes of one 16-byte source chunk (8 channels) as 8 bytes, channel order kept.
__device__ __forceinline__ uint2 encode_chunk(const uint4 v, float s, uint64_t yy, uint64_t nss,
                                              bool fast) {
  uint2 out;
  out.x = encode_word(v.x, s, yy, nss, fast) | (encode_word(v.y, s, yy, nss, fast) << 16);
  out.y = encode_word(v.z, s, yy, nss, fast) | (encode_word(v.w, s, yy, nss, fast) << 16);
  // Sign bits of channels 0..3 (bit 15 and bit 31 of each source word) into bit 7
  // of code bytes 0..3: byte permute of the words' odd bytes, then a masked OR.
  out.x |= __byte_perm(v.x, v.y, 0x7531) & 0x80808080u;
  out.y |= __byte_perm(v.z, v.w, 0x7531) & 0x80808080u;
  return out;
}

// ---------------------------------------------------------------------------
// The store kernel.  A launch stores a list of tensors; tensor i has heads_i x
// pieces_i columns (one per head and row piece: e4m3 tensors are never split,
// pieces_i = 1, since a head's scale needs all its rows), numbered from col0_i.  A
// cluster takes
// whole columns (cluster c: columns c, c + #clusters, ...; the host lists the
// tensors with the longest columns first and launches only as many clusters as are
// resident at once), and its kStoreCluster CTAs split a column's tiles evenly.
//
// Warp specialisation (one CTA per SM):
//  * producer warp (one lane) schedules the CTA's work as a sequence of items, each
//    in one slot of a kStoreStages-deep ring: tiles, each one TMA load of
//    {128 channels, 1 head, kStoreTileRows rows} -- a copy tile of a bf16 column, an
//    absmax tile or an encode tile of an e4m3 column -- and two markers per e4m3
//    column, "absmax pass done" and "encode pass begins".  An e4m3 column's encode
//    tiles (descending, so that the most recently read rows come first) are
//    interleaved one for one with the first-pass tiles of the next column, after a
//    lead of kStoreLead of the latter: the DRAM-bound absmax pass of one column
//    overlaps the instruction-bound encode pass of the previous one, and the rank
//    exchange has those lead tiles' time to complete.  The slot's item descriptor
//    is written before the slot's barrier is armed.
//    Measured on the 8-request serving store (e4m3 K and V, 2.13 GB): this shape
//    0.588 ms; clusters of 8 0.647 ms and of 16 0.75 ms (fewer columns in flight, so
//    more of the encode pass hits L2, but fewer SMs and more per-column exchanges
//    per CTA); each column's encode pass a whole step later 0.632 ms; the encode
//    pass after the lead instead of interleaved 0.652 ms; 2 chunks per thread
//    0.780 ms.
//  * kStoreConsumerWarps consumer warps read every item (a tile: kStoreChunks
//    16-byte chunks per thread, kStoreStepRows rows apart, independent of one
//    another) and each warp releases the slot on its own:
//      copy tile    : the chunk goes straight to the cache row (streaming store);
//      absmax tile  : packed 16-bit max of the magnitudes;
//      absmax done  : every warp leaves its maximum in shared memory and arrives
//                     on the CTA's reduction mbarrier; warp 0 waits for all of them
//                     and sends the CTA's maximum to every CTA of the cluster
//                     (asynchronous distributed shared-memory stores, one lane per
//                     rank, each completing 4 transaction bytes on that CTA's
//                     exchange mbarrier, which its own CTA arms for the column);
//      encode begins: every warp waits on its CTA's exchange mbarrier for all the
//                     cluster's maxima, so it knows amax_h; rank 0 writes s_h;
//      encode tile  : codes with streaming stores (8 bytes per chunk).
//    The reduction and exchange buffers rotate over kStoreXBufs columns: a peer
//    sends column x's maximum only after it has the amax of column x - 2, which
//    needs this CTA's maximum of x - 2, sent after this CTA read the amax of
//    x - 4 -- so a buffer is never overwritten before it has been read.
// Rows past the tensor's end in its last tile read as zeros (TMA bounds) and are
// not written.  Every wait is bounded: a wait that runs out marks the CTA aborted
// (BCA_ERR_DEVICE_TIMEOUT in *dev_status); the producer then stops and waits
// (bounded) for its copies in flight, the consumer warps leave their loops (no
// consumer waits on a barrier that a warp which left would have to reach), and all
// threads meet at the final cluster barrier, after which an aborted CTA lets its
// peers' last asynchronous stores land before it leaves.
// A non-finite value in an e4m3 column makes its amax Inf or NaN: the column's codes
// and scale are then meaningless and BCA_ERR_NONFINITE is written to *dev_status
// (the inputs must be finite).
// ---------------------------------------------------------------------------
struct StoreTensor {
  void* dst;            // row t, head h at element (h * head_stride + t) * 128 (bf16 or e4m3)
  float* scale;         // [heads] fp32, e4m3 tensors only
  int64_t head_stride;  // destination rows between consecutive heads
  int32_t rows;
  int32_t heads;
  int32_t quant;        // 1: e4m3 with a per-head absmax scale, 0: bf16 copy
  int32_t col0;         // first column of this tensor
  int32_t pieces;       // row pieces per head (1 for e4m3)
};

constexpr int kMaxStoreTensors = 2 * BCA_MAX_BATCH;
constexpr int kStoreConsumerWarps = 16;
constexpr int kStoreConsumers = 32 * kStoreConsumerWarps;
constexpr int kStoreThreads = kStoreConsumers + 32;  // + the producer warp
constexpr int kStoreCluster = 4;
constexpr int kStoreChunks = 4;  // 16-byte chunks per consumer thread per tile
constexpr int kStoreStepRows = kStoreConsumers / 16;  // rows covered by one chunk of every thread
constexpr int kStoreTileRows = kStoreStepRows * kStoreChunks;
constexpr int kStoreTileBytes = kStoreTileRows * 256;
constexpr int kStoreRingBytes = 128 * 1024;
constexpr int kStoreStages = kStoreRingBytes / kStoreTileBytes;
constexpr int kStoreLead = kStoreStages / 2;  // first-pass tiles ahead of an encode pass
constexpr int kStoreXBufs = 4;
static_assert(kStoreConsumers * kStoreChunks * 16 == kStoreTileBytes, "tile split");
static_assert(kStoreConsumerWarps <= 32, "one warp maximum per lane in the reduction");
static_assert(kStoreTileRows <= 256, "TMA box rows");

struct StoreParams {
  // Source of tensor i (bf16 bits; row t, head h at src + t * row_stride + h * 128):
  // {128 channels, heads, rows}, box {128, 1, kStoreTileRows}, no swizzle (a tile is
  // kStoreTileRows rows of 256 bytes in shared memory).
  CUtensorMap map[kMaxStoreTensors];
  StoreTensor t[kMaxStoreTensors];
  int32_t n_tensors;
  int32_t n_cols;
  int32_t* dev_status;
  uint64_t timeout_ns;
};

// Work items of the ring.
enum : uint32_t {
  kItemCopy = 0,      // tile of a bf16 column
  kItemAbs = 1,       // absmax-pass tile of an e4m3 column
  kItemEnc = 2,       // encode-pass tile of an e4m3 column
  kItemAbsDone = 3,   // marker: the column's absmax pass is complete on this CTA
  kItemEncBegin = 4,  // marker: the column's encode pass begins
  kItemEnd = 5,       // marker: no more items
};
struct __align__(16) StoreItem {
  uint32_t kind;
  uint32_t ti;   // tensor
  int32_t h;     // head
  int32_t tile;  // kStoreTileRows-row tile (tiles only)
};
// What the consumers read of an item (the producer resolves the tensor's fields,
// so that the consumers index no parameter array).
struct __align__(16) StoreSlot {
  uint32_t kind;
  int32_t row0;   // first row of the tile
  int32_t rows;   // rows of the tensor (rows at or past it are not written)
  uint32_t pad;
  uint64_t dst;   // tiles: address of row 0 of the head in the cache; kItemEncBegin:
                  // address of the head's scale
  uint64_t unused;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; orders shared-memory writes (local and
// distributed) before the reads that follow it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t a, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  return ra;
}
// Asynchronous 32-bit store into CTA `rank`'s copy of the shared variable at local
// address `a`, completing 4 transaction bytes on that CTA's copy of the mbarrier at
// `bar` (no fence: the barrier's phase completion publishes the value).
__device__ __forceinline__ void st_async_cluster(uint32_t a, uint32_t bar, uint32_t rank,
                                                 uint32_t v) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(
          map_to_rank(a, rank)),
      "r"(v), "r"(map_to_rank(bar, rank))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity,
                                                          const volatile int* abort,
                                                          uint64_t timeout_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
  }
}

// Column `col` for this CTA: its tensor (ti advances monotonically over the sorted
// list), head, and this rank's tiles [t0, t1) of the head's rows.
struct StoreCol {
  int ti, h, t0, t1;
  bool quant, valid;
};
__device__ __forceinline__ StoreCol store_col(const StoreParams& p, int col, int& ti,
                                              uint32_t crank, uint32_t csize) {
  StoreCol c;
  c.valid = col < p.n_cols;
  if (!c.valid) return c;
  while (ti + 1 < p.n_tensors && col >= p.t[ti + 1].col0) ++ti;
  const StoreTensor& T = p.t[ti];
  const int local = col - T.col0;
  c.ti = ti;
  c.quant = T.quant != 0;
  c.h = local / T.pieces;
  const int piece = local - c.h * T.pieces;
  const int64_t ntiles = (T.rows + kStoreTileRows - 1) / kStoreTileRows;
  const int p0 = static_cast<int>(ntiles * piece / T.pieces);
  const int64_t n = ntiles * (piece + 1) / T.pieces - p0;
  c.t0 = p0 + static_cast<int>(n * crank / csize);
  c.t1 = p0 + static_cast<int>(n * (crank + 1) / csize);
  return c;
}

__device__ __forceinline__ void store_abort(volatile int* abort, int32_t* dev_status) {
  *abort = 1;
  if (dev_status) atomicExch(dev_status, static_cast<int32_t>(BCA_ERR_DEVICE_TIMEOUT));
}

// The producer's schedule over the CTA's columns (see above): step i interleaves the
// first-pass tiles of column i with the encode tiles of column i - 1 (if e4m3).
// next() returns the next item; `load` says whether it is a tile to fetch.
struct StoreSchedule {
  const StoreParams& p;
  uint32_t crank, csize;
  int col, col_step, ti_scan = 0;
  StoreCol cur;   // first pass in progress
  StoreCol prev;  // e4m3 column being encoded
  int a_done = 0, b_done = 0;
  bool abs_done_sent = false, enc_begun = false, toggle = false;

  __device__ StoreSchedule(const StoreParams& p_, uint32_t r, uint32_t n, int c0, int step)
      : p(p_), crank(r), csize(n), col(c0), col_step(step) {
    prev.valid = false;
    cur = store_col(p, col, ti_scan, crank, csize);
    col += col_step;
  }
  __device__ StoreItem next(bool& load) {
    load = false;
    for (;;) {
      const int a_total = cur.valid ? cur.t1 - cur.t0 : 0;
      const int b_total = prev.valid ? prev.t1 - prev.t0 : 0;
      const bool a_left = cur.valid && a_done < a_total;
      if (a_left && a_done < kStoreLead) return first_pass_tile(load);
      if (cur.valid && !a_left && cur.quant && !abs_done_sent) {
        abs_done_sent = true;
        return StoreItem{kItemAbsDone, static_cast<uint32_t>(cur.ti), cur.h, 0};
      }
      // After the lead: "encode begins" of prev, so a column's "absmax done" always
      // follows the "encode begins" of the e4m3 column two before it, which the
      // kStoreXBufs = 4 exchange buffers rely on.
      if (prev.valid && !enc_begun) {
        enc_begun = true;
        return StoreItem{kItemEncBegin, static_cast<uint32_t>(prev.ti), prev.h, 0};
      }
      if (prev.valid && b_done < b_total && (toggle || !a_left)) {
        toggle = false;
        load = true;
        const int tile = prev.t1 - 1 - b_done++;
        return StoreItem{kItemEnc, static_cast<uint32_t>(prev.ti), prev.h, tile};
      }
      if (a_left) {
        toggle = true;
        return first_pass_tile(load);
      }
      // The step is complete: cur's first pass and prev's encode pass are done.
      if (!cur.valid) return StoreItem{kItemEnd, 0, 0, 0};
      prev = cur;
      prev.valid = cur.quant;
      b_done = 0;
      enc_begun = false;
      cur = store_col(p, col, ti_scan, crank, csize);
      col += col_step;
      a_done = 0;
      abs_done_sent = false;
      toggle = false;
    }
  }
  __device__ StoreItem first_pass_tile(bool& load) {
    load = true;
    return StoreItem{cur.quant ? kItemAbs : kItemCopy, static_cast<uint32_t>(cur.ti), cur.h,
                     cur.t0 + a_done++};
  }
};

__global__ void __launch_bounds__(kStoreThreads, 1)
    kv_store_kernel(const __grid_constant__ StoreParams p) {
  extern __shared__ __align__(128) uint8_t store_ring[];
  __shared__ __align__(8) uint64_t s_full[kStoreStages], s_empty[kStoreStages];
  __shared__ __align__(8) uint64_t s_xbar[kStoreXBufs], s_rbar[kStoreXBufs];
  __shared__ StoreSlot s_item[kStoreStages];
  __shared__ uint32_t s_part[kStoreXBufs][kStoreCluster];        // CTA maxima by rank
  __shared__ uint32_t s_red[kStoreXBufs][kStoreConsumerWarps];  // warp maxima
  __shared__ int s_abort;
  const uint32_t ring = smem_u32(store_ring);
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kStoreStages; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_empty[i]), kStoreConsumerWarps);
    }
    for (int i = 0; i < kStoreXBufs; ++i) {
      mbar_init(smem_u32(&s_xbar[i]), 1);  // the CTA's own arm + csize x 4 bytes
      mbar_init(smem_u32(&s_rbar[i]), kStoreConsumerWarps);
    }
    s_abort = 0;
    fence_barrier_init();
  }
  cluster_sync();  // barriers initialised before any peer can arrive on them
  volatile int* abort = &s_abort;

  if (warp == kStoreConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      StoreSchedule sch(p, crank, csize, static_cast<int>(cluster_index()),
                        static_cast<int>(cluster_count()));
      uint32_t it = 0;
      for (;; ++it) {
        bool load;
        const StoreItem itm = sch.next(load);
        const uint32_t st = it % kStoreStages, ph = (it / kStoreStages) & 1u;
        if (!mbar_wait_bounded(smem_u32(&s_empty[st]), ph ^ 1u, abort, p.timeout_ns)) {
          store_abort(abort, p.dev_status);
          break;
        }
        {
          const StoreTensor& T = p.t[itm.ti];
          StoreSlot sl;
          sl.kind = itm.kind;
          sl.row0 = itm.tile * kStoreTileRows;
          sl.rows = T.rows;
          sl.pad = 0;
          sl.unused = 0;
          if (itm.kind == kItemEncBegin)
            sl.dst = reinterpret_cast<uint64_t>(T.scale + itm.h);
          else
            sl.dst = reinterpret_cast<uint64_t>(static_cast<uint8_t*>(T.dst)) +
                     static_cast<uint64_t>(itm.h) * static_cast<uint64_t>(T.head_stride) *
                         (T.quant ? 128u : 256u);
          s_item[st] = sl;
        }
        if (load) {
          mbar_arrive_expect_tx(smem_u32(&s_full[st]), kStoreTileBytes);
          tma_load_3d(ring + st * kStoreTileBytes, &p.map[itm.ti], smem_u32(&s_full[st]), 0,
                      itm.h, itm.tile * kStoreTileRows);
        } else {
          mbar_arrive(smem_u32(&s_full[st]));
        }
        if (itm.kind == kItemEnd) {
          ++it;
          break;
        }
      }
      if (*abort) {  // copies still in flight land before the CTA may leave
        const uint32_t n = it < kStoreStages ? it : kStoreStages;
        for (uint32_t j = it - n; j < it; ++j)
          mbar_wait_bounded(smem_u32(&s_full[j % kStoreStages]), (j / kStoreStages) & 1u,
                            nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    const int row = warp * 2 + (lane >> 4), chunk = lane & 15;  // rows row + kStoreStepRows k
    const uint32_t my_off = static_cast<uint32_t>(row * 256 + chunk * 16);
    uint32_t it = 0, n_abs = 0, n_enc = 0;
    uint32_t m = 0;  // running packed absmax of the column in its absmax pass
    float s = 1.0f;  // the encoded column's scale and its reciprocal pair
    uint64_t yy = 0, nss = 0;
    bool fast = true;
    for (;; ++it) {
      const uint32_t st = it % kStoreStages, ph = (it / kStoreStages) & 1u;
      const bool got =
          !*abort && mbar_wait_bounded(smem_u32(&s_full[st]), ph, abort, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) store_abort(abort, p.dev_status);
        break;
      }
      StoreSlot itm;
      uint4 v[kStoreChunks];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(itm.kind), "=r"(itm.row0), "=r"(itm.rows), "=r"(itm.pad)
                   : "r"(smem_u32(&s_item[st]))
                   : "memory");
      asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];"
                   : "=l"(itm.dst), "=l"(itm.unused)
                   : "r"(smem_u32(&s_item[st]) + 16)
                   : "memory");
      if (itm.kind <= kItemEnc) {
#pragma unroll
        for (int k = 0; k < kStoreChunks; ++k)
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w)
                       : "r"(ring + st * kStoreTileBytes + my_off + k * kStoreStepRows * 256)
                       : "memory");
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_empty[st]));
      if (itm.kind == kItemEnd) break;
      const int t = itm.row0 + row;  // row of chunk 0; chunk k: t + kStoreStepRows k
      if (itm.kind == kItemAbs) {
#pragma unroll
        for (int k = 0; k < kStoreChunks; ++k) {
          m = max_u16x2(m, v[k].x & 0x7FFF7FFFu);
          m = max_u16x2(m, v[k].y & 0x7FFF7FFFu);
          m = max_u16x2(m, v[k].z & 0x7FFF7FFFu);
          m = max_u16x2(m, v[k].w & 0x7FFF7FFFu);
        }
      } else if (itm.kind == kItemEnc) {
        uint2* dst = reinterpret_cast<uint2*>(itm.dst + static_cast<uint64_t>(t) * 128) + chunk;
        uint2 c[kStoreChunks];
#pragma unroll
        for (int k = 0; k < kStoreChunks; ++k) c[k] = encode_chunk(v[k], s, yy, nss, fast);
#pragma unroll
        for (int k = 0; k < kStoreChunks; ++k)
          if (t + kStoreStepRows * k < itm.rows) __stcs(dst + kStoreStepRows * 16 * k, c[k]);
      } else if (itm.kind == kItemCopy) {
        uint4* dst = reinterpret_cast<uint4*>(itm.dst + static_cast<uint64_t>(t) * 256) + chunk;
#pragma unroll
        for (int k = 0; k < kStoreChunks; ++k)
          if (t + kStoreStepRows * k < itm.rows) __stcs(dst + kStoreStepRows * 16 * k, v[k]);
      } else if (itm.kind == kItemAbsDone) {
        const uint32_t b = n_abs % kStoreXBufs, rph = (n_abs / kStoreXBufs) & 1u;
        ++n_abs;
        const uint32_t wm = __reduce_max_sync(0xffffffffu, max(m & 0xFFFFu, m >> 16));
        m = 0;
        if (lane == 0) {
          s_red[b][warp] = wm;
          mbar_arrive(smem_u32(&s_rbar[b]));  // release: the store above comes first
        }
        if (warp == 0) {
          const bool red = mbar_wait_bounded(smem_u32(&s_rbar[b]), rph, abort, p.timeout_ns);
          if (!__all_sync(0xffffffffu, red)) {
            if (lane == 0) store_abort(abort, p.dev_status);
            break;
          }
          uint32_t x = lane < kStoreConsumerWarps ? s_red[b][lane] : 0u;
          x = __reduce_max_sync(0xffffffffu, x);
          // Arm this CTA's exchange barrier for the column (its peers' values may
          // already have landed: the transaction count then runs negative for a
          // while, and the phase cannot complete before this arrive), then lane q
          // sends the CTA's maximum to rank q.
          if (lane == 0) mbar_arrive_expect_tx(smem_u32(&s_xbar[b]), 4u * csize);
          __syncwarp();
          if (static_cast<uint32_t>(lane) < csize)
            st_async_cluster(smem_u32(&s_part[b][crank]), smem_u32(&s_xbar[b]),
                             static_cast<uint32_t>(lane), x);
        }
      } else {  // kItemEncBegin
        const uint32_t b = n_enc % kStoreXBufs, xph = (n_enc / kStoreXBufs) & 1u;
        ++n_enc;
        const bool x_ok = mbar_wait_cluster_bounded(smem_u32(&s_xbar[b]), xph, abort, p.timeout_ns);
        if (!__all_sync(0xffffffffu, x_ok)) {
          if (lane == 0) store_abort(abort, p.dev_status);
          break;
        }
        uint32_t amax_bits = 0;
        for (uint32_t q = 0; q < csize; ++q) amax_bits = max(amax_bits, s_part[b][q]);
        s = scale_from_amax_bits(amax_bits);
        if (crank == 0 && tid == 0) {
          *reinterpret_cast<float*>(itm.dst) = s;
          if (amax_bits >= 0x7F80u && p.dev_status)
            atomicExch(p.dev_status, static_cast<int32_t>(BCA_ERR_NONFINITE));
        }
        const float y = __frcp_rn(s);
        yy = f2_pack(y, y);
        nss = f2_pack(-s, -s);
        fast = amax_bits >= kFastDivMinBits;
      }
    }
  }
  // No CTA leaves while a peer may still store into its shared memory: every peer's
  // sends precede its arrival here.  In a normal run each CTA has also waited for
  // every value sent to it; after an abort it may not have, so it gives sends issued
  // before the barrier (asynchronous stores land within microseconds) 100 us more.
  cluster_sync();
  if (*abort) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000u) {
    }
  }
}

// Self-check of encode_chunk as the store kernel runs it: for every positive finite
// bf16 amax (blockIdx.x + 1 as magnitude bits) and every bf16 x with |x| <= amax (and
// -x, and +-0), the e4m3 codes of encode_chunk(x, s, RN(1/s), amax >= 2^-95) must
// equal those of the correctly rounded x / s.
__global__ void __launch_bounds__(256) e4m3_division_selftest_kernel(unsigned long long* mismatch) {
  const unsigned amax_bits = blockIdx.x + 1;  // 0x0001 .. 0x7F7F
  const float s = scale_from_amax_bits(amax_bits);
  const float y = __frcp_rn(s);
  const uint64_t yy = f2_pack(y, y), nss = f2_pack(-s, -s);
  const bool fast = amax_bits >= kFastDivMinBits;
  const float amax = __uint_as_float(amax_bits << 16);
  unsigned long long bad = 0;
  for (unsigned m = threadIdx.x; m <= amax_bits; m += blockDim.x) {
    const float xp = __uint_as_float(m << 16);
    if (!(xp <= amax)) continue;
    const uint32_t w = m | ((m | 0x8000u) << 16);  // (+x, -x): +-0 for m = 0
    const uint16_t want = e4m3x2_rn_satfinite(__fdiv_rn(xp, s), __fdiv_rn(-xp, s));
    const uint2 got = encode_chunk(make_uint4(w, w, w, w), s, yy, nss, fast);
    const uint32_t want2 = want | (static_cast<uint32_t>(want) << 16);
    bad += (got.x != want2) + (got.y != want2);
  }
  if (bad) atomicAdd(mismatch, bad);
}

}  // namespace bca
