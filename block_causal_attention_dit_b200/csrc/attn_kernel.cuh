// attn_kernel.cuh -- block-causal / cached-step attention forward for sm_100a.
//
// What it computes (cited by page title and section):
//  * "Qwen-Image-2.1 + vLLM-Omni day-0", "What is Qwen-Image-2.1" and "Serving
//    architecture: the cross-step prefix KV cache": ordered blocks (text, refs,
//    target); row i of block b attends to every key of blocks 0..b.  Prefill
//    mode computes this over the whole sequence (denoising step 1).
//  * same section + "Qwen/Qwen-Image-2.1" (vLLM recipe), "Prefix KV cache": in
//    later steps only the target rows are recomputed; they attend to the cached
//    prefix K/V followed by their own K/V.  Step mode computes this for a ragged
//    batch of requests at the same phase ("Online serving": step-level batching).
//
// Design (B200).  A unit is (request, head, pair of 128-row Q tiles).  The kernel
// is persistent: one CTA per SM walks a static list of work items (item = CTA
// index + k * grid).  Items of the first rounds are whole units; the units of the
// last, partial round are split along the key dimension into `split_k` chunks so
// that every SM ends at about the same time -- a chunk writes its unnormalised O,
// row max and row sum to a workspace and attn_combine_kernel merges the chunks.
//  * warp 8      : TMA producer -- Q tiles of each item, then K_j, V_j tiles into a
//                  4-stage ring of 32 KiB bf16 tiles (128-byte swizzle).
//  * warp 9      : tcgen05 issuer (whole warp, one elected lane issues) --
//                  S_w = Q_w K_j^T (both operands in smem) and O_w += P_w V_j (P from
//                  TMEM, V in smem, MN-major), fp32 accumulators in TMEM.
//  * warps 10-11 : e4m3 cache tiles -> bf16 in shared memory (FP8 cache only).
//  * e4m3-Q mode (kQ8, bca_step_attend_q8): Q quantised per (request, head) like a
//    cache tensor; S of cached keys = Q8 K8^T by tcgen05.mma kind::f8f6f4 with both
//    operands as stored (Q8 tiles in the staging buffers, K8 tiles straight into
//    the ring); only V tiles are expanded, in place in their ring slot.
//  * warps 0..3  : softmax of Q tile 0, warps 4..7: Q tile 1.  One thread per row:
//                  load S from TMEM, mask ragged / block-causal keys, online softmax
//                  in the exp2 domain, write P (bf16) back over S in TMEM.  O is
//                  only rescaled when the running max grows by more than 2^8
//                  (exact: numerator and denominator use the same stale max).
//  * TMEM (512 columns): S0 | S1 | O0 | O1, 128 columns each; P_w aliases S_w.
//  * Block-mask tile skipping: a Q tile only visits KV tiles below the largest key
//    limit of its rows; masks are applied only inside the boundary tile.
// Every mbarrier wait is bounded (see ptx.cuh); on expiry the CTA raises an abort
// flag, reports BCA_ERR_DEVICE_TIMEOUT, drains and frees TMEM.
#pragma once
#include <cuda_bf16.h>

#include "../../include/bca.h"
#include "ptx.cuh"

namespace bca {

constexpr int kHeadDim = 128;
constexpr int kBM = 128;  // Q rows per tile
constexpr int kBN = 128;  // keys per KV tile
constexpr int kStages = 4;
constexpr int kTileBytes = kBM * kHeadDim * 2;  // 32 KiB bf16 tile
constexpr int kHalfBytes = kTileBytes / 2;      // one 64-column swizzled box
constexpr int kTile8Bytes = kBN * kHeadDim;     // 16 KiB e4m3 tile
constexpr int kAttnThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpConv0 = 10;  // warps 10 and 11 convert e4m3 cache tiles
constexpr int kConvThreads = 64;
// Register split: launched at kLaunchRegs per thread (384 x 168 = 64512), the two
// softmax warpgroups take kSoftmaxRegs and warpgroup 2 (producer, MMA, converter)
// keeps kOtherRegs: 128 * (2 * 200 + 104) = 64512.  The host checks the compiled
// register count against this before launching.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 200;
constexpr uint32_t kOtherRegs = 104;
static_assert(128 * (2 * kSoftmaxRegs + kOtherRegs) <= kAttnThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kNoLimit = 1 << 30;
// Split-chunk workspace: per chunk, O [256 rows][128] fp32, then m[256], l[256].
constexpr int kChunkRows = 2 * kBM;
constexpr size_t kChunkBytes = static_cast<size_t>(kChunkRows) * (kHeadDim + 2) * 4;

enum : int { kModePrefill = 0, kModeStep = 1 };

// Pipeline trace of one CTA (builds with BCA_TRACE only): clock64() stamps of the
// roles' events per KV tile t, counted over all items of the CTA,
// trace[t * kTraceEvents + ev].
constexpr int kTraceEvents = 32;
constexpr int kTraceTiles = 192;
#ifdef BCA_TRACE
#define BCA_TRACE_AT(p, t, ev)                                                          \
  do {                                                                                  \
    if ((p).trace && static_cast<int>(blockIdx.x) == (p).trace_cta && (t) < kTraceTiles && \
        (t) >= 0)                                                                       \
      (p).trace[(t) * kTraceEvents + (ev)] = clock64();                                 \
  } while (0)
#else
#define BCA_TRACE_AT(p, t, ev) \
  do {                         \
  } while (0)
#endif

template <int MAXR>
struct AttnParams {
  CUtensorMap tm_q;  // [rows, H, 128] bf16, dims (128, H, rows), box (64, 1, 128)
  CUtensorMap tm_k;  // own keys, same geometry
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // output, same geometry (bf16 mode: whole Q tiles stored by TMA)
  CUtensorMap tm_q8;  // e4m3-Q mode: codes [H, rows, 128], dims (128, rows, H), box (128, 128, 1)
  CUtensorMap tm_kc[MAXR];  // cache K of request r: dims (128, n_tokens, H), box (64, 128, 1)
                            // (e4m3: box (128, 128, 1) into the staging buffers)
  CUtensorMap tm_vc[MAXR];
  __nv_bfloat16* o;
  int32_t o_rows;  // rows of the Q/O tensors (bounds of the epilogue stores)
  int32_t* dev_status;
  unsigned long long* trace;  // BCA_TRACE builds: [kTraceTiles][kTraceEvents] cycle stamps
  int32_t trace_cta;
  unsigned long long timeout_ns;
  int32_t heads;
  int32_t mode;
  float scale_log2;  // softmax scale * log2(e)
  // work items: [0, full_items) are whole units; the next split_units units are
  // split into split_k chunks each (chunk c of a unit with n tiles covers tiles
  // [c*n/k, (c+1)*n/k)), written to `workspace` and merged by attn_combine_kernel;
  // the units after them (prefill: the light ones) are whole again.
  int32_t n_items;
  int32_t full_items;
  int32_t split_k;
  int32_t split_units;
  float* workspace;
  // prefill
  int32_t seq_len;
  int32_t n_blocks;
  int32_t block_off[BCA_MAX_BLOCKS + 1];
  // step: requests in scheduling order
  int32_t n_req;
  int32_t unit_start[MAXR + 1];
  int32_t q_start[MAXR];
  int32_t q_len[MAXR];
  int32_t n_cache[MAXR];
  // e4m3 cache tensors (step mode): codes are converted to bf16 in shared memory;
  // the K scale multiplies the scores of cache keys, the V scale their P.
  int32_t k_fp8;
  int32_t v_fp8;
  // The per-head scales apply to the cache tensor (e4m3 values): 1 for an e4m3
  // tensor, whether its tiles arrive as codes (k_fp8 / v_fp8) or were expanded to
  // bf16 beforehand (bca_step_attend_dq).
  int32_t k_scaled;
  int32_t v_scaled;
  const float* k_scale[MAXR];
  const float* v_scale[MAXR];
  const float* q_scale[MAXR];  // e4m3-Q mode: [H] scales of request i's Q codes
};

// Shared memory map (offsets from a 1024-byte aligned base).
struct Smem {
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kRing = 2 * kTileBytes;
  static constexpr int kStage8 = kRing + kStages * kTileBytes;  // 2 x 16 KiB e4m3 tiles
  static constexpr int kBars = kStage8 + 2 * kTile8Bytes;
  // barrier indices
  static constexpr int bQFull = 0;                     // 2
  static constexpr int bKvFull = 2;                    // kStages
  static constexpr int bKvEmpty = 2 + kStages;         // kStages
  static constexpr int bSFull = 2 + 2 * kStages;       // 2
  static constexpr int bPFull = 4 + 2 * kStages;       // 2 (128 arrivals each)
  static constexpr int bOFull = 6 + 2 * kStages;       // 2
  static constexpr int bDone = 8 + 2 * kStages;        // 1
  static constexpr int bStgFull = 9 + 2 * kStages;     // 2
  static constexpr int bStgEmpty = 11 + 2 * kStages;   // 2
  static constexpr int bConv = 13 + 2 * kStages;       // 1 (64 converter arrivals per tile)
  static constexpr int bQEmpty = 14 + 2 * kStages;     // 2 (Q tile w of an item consumed)
  static constexpr int bEpiFull = 16 + 2 * kStages;    // 2 (O box of tile w in smem: 128)
  static constexpr int bEpiFree = 18 + 2 * kStages;    // 2 (its TMA store has read it)
  static constexpr int kNumBars = 20 + 2 * kStages;
  static constexpr int kTmemSlot = kBars + 8 * kNumBars;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kDynamicBytes = kBytes + 1024;  // + alignment slack
};

// TMEM column bases: S0 | S1 | O0 | O1.
__host__ __device__ constexpr uint32_t col_s(int w) { return w == 0 ? 0u : 128u; }
__host__ __device__ constexpr uint32_t col_o(int w) { return w == 0 ? 256u : 384u; }

// One work item with every per-unit value it needs held in registers.
struct Item {
  int req;        // request slot in the params arrays (step mode)
  int h;          // head
  int q_row0;     // row of Q tile 0 in the Q/O tensors
  int rows[2];    // valid rows of each Q tile (<= 0: tile absent)
  int jend[2];    // Q tile w visits KV tiles [j0, jend[w]) (jend <= j0: inactive)
  int j0, j1;     // KV tile range of the item (j1 = max(jend))
  int n_cache;    // cached keys (step mode)
  int n_cache_tiles;
  int q_start;    // first packed row of the request (step mode)
  int q_len;      // target rows of the request (step mode)
  int partial;    // -1: whole unit; else workspace chunk index
};

template <int MAXR>
__device__ __forceinline__ int block_end(const AttnParams<MAXR>& p, int row) {
  for (int b = 1; b <= p.n_blocks; ++b)
    if (row < p.block_off[b]) return p.block_off[b];
  return p.seq_len;
}

template <int MAXR>
__device__ __forceinline__ Item decode_item(const AttnParams<MAXR>& p, int item) {
  Item it;
  int unit = item, chunk = 0, k = 1;
  it.partial = -1;
  if (item >= p.full_items) {
    const int q = item - p.full_items;
    if (q < p.split_units * p.split_k) {
      k = p.split_k;
      unit = p.full_items + q / k;
      chunk = q % k;
      it.partial = q;
    } else {
      unit = p.full_items + p.split_units + (q - p.split_units * p.split_k);
    }
  }
  int ntiles[2];
  if (p.mode == kModePrefill) {
    const int S = p.seq_len;
    const int nqp = (S + 2 * kBM - 1) / (2 * kBM);
    it.req = 0;
    // Heaviest (latest) Q-tile pairs of every head first: a pair's key limit, and
    // so its work, never decreases with its rows.
    it.h = unit % p.heads;
    const int qp = nqp - 1 - unit / p.heads;
    it.q_row0 = qp * 2 * kBM;
    it.n_cache = 0;
    it.n_cache_tiles = 0;
    it.q_start = 0;
    it.q_len = S;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      it.rows[w] = min(kBM, S - it.q_row0 - w * kBM);
      ntiles[w] = 0;
      if (it.rows[w] > 0) {
        const int lim = block_end(p, it.q_row0 + w * kBM + it.rows[w] - 1);
        ntiles[w] = (lim + kBN - 1) / kBN;
      }
    }
  } else {
    int r = 0;
    while (r + 1 < p.n_req && unit >= p.unit_start[r + 1]) ++r;
    const int T = p.q_len[r];
    const int nqp = (T + 2 * kBM - 1) / (2 * kBM);
    const int local = unit - p.unit_start[r];
    it.req = r;
    it.h = local / nqp;
    const int qp = local % nqp;
    it.q_start = p.q_start[r];
    it.q_len = T;
    it.q_row0 = it.q_start + qp * 2 * kBM;
    it.n_cache = p.n_cache[r];
    it.n_cache_tiles = (it.n_cache + kBN - 1) / kBN;
    const int nt = it.n_cache_tiles + (T + kBN - 1) / kBN;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      it.rows[w] = min(kBM, T - qp * 2 * kBM - w * kBM);
      ntiles[w] = it.rows[w] > 0 ? nt : 0;
    }
  }
  const int n = max(ntiles[0], ntiles[1]);
  it.j0 = chunk * n / k;
  it.j1 = (chunk + 1) * n / k;
#pragma unroll
  for (int w = 0; w < 2; ++w) it.jend[w] = min(it.j1, ntiles[w]);
  return it;
}

__device__ __forceinline__ bool tile_active(const Item& it, int w) {
  return (w ? it.rows[1] : it.rows[0]) > 0 && it.j0 < (w ? it.jend[1] : it.jend[0]);
}

// Geometry of KV tile j: number of valid keys and index of its first key in the
// row's key sequence (for the block-causal limit).  Registers only.
__device__ __forceinline__ void kv_tile_extent(bool prefill, const Item& it, int seq_len, int j,
                                               int& valid, int& key_base) {
  if (prefill) {
    key_base = j * kBN;
    valid = min(kBN, seq_len - key_base);
  } else if (j < it.n_cache_tiles) {
    key_base = j * kBN;
    valid = min(kBN, it.n_cache - key_base);
  } else {
    const int jj = j - it.n_cache_tiles;
    key_base = it.n_cache + jj * kBN;
    valid = min(kBN, it.q_len - jj * kBN);
  }
}

// On a failed wait: raise the CTA's abort flag and report the timeout.  Builds with
// BCA_DEVICE_CHECKS report 1000 + `site` instead (first report wins) so that the
// wait that gave up can be identified.
__device__ __forceinline__ void raise_abort(volatile int* abort, int32_t* dev_status,
                                            int site = 0) {
  *abort = 1;
#ifdef BCA_DEVICE_CHECKS
  if (dev_status) atomicCAS(dev_status, 0, 1000 + site);
#else
  (void)site;
  if (dev_status) atomicExch(dev_status, static_cast<int32_t>(BCA_ERR_DEVICE_TIMEOUT));
#endif
}

// Self-checks of checked builds: a failed check records 2000 + code and the caller
// skips the access.  Compiled out otherwise.
#ifdef BCA_DEVICE_CHECKS
#define BCA_CHECK(dev_status, cond, code) \
  ((cond) ? true : ((dev_status) ? (atomicCAS((dev_status), 0, 2000 + (code)), false) : false))
#else
#define BCA_CHECK(dev_status, cond, code) true
#endif

template <int MAXR>
__device__ __forceinline__ bool tile_is_fp8(const AttnParams<MAXR>& p, const Item& it, int j,
                                            int kv) {
  return p.mode == kModeStep && j < it.n_cache_tiles && (kv ? p.v_fp8 : p.k_fp8) != 0;
}

// e4m3 cache tiles the converter warps expand to bf16: all of them, except in
// e4m3-Q mode, where K tiles go to the MMA as stored and only V tiles are expanded.
template <int MAXR, bool kQ8>
__device__ __forceinline__ bool tile_is_converted(const AttnParams<MAXR>& p, const Item& it,
                                                  int j, int kv) {
  return tile_is_fp8(p, it, j, kv) && (!kQ8 || kv == 1);
}

// ---------------------------------------------------------------------------
// Producer: one thread.
// ---------------------------------------------------------------------------
template <int MAXR, bool kQ8>
__device__ void producer_role(const AttnParams<MAXR>& p, uint32_t sbase, uint32_t bars,
                              volatile int* abort) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  int it = 0, fi = 0, nq = 0;  // ring items, e4m3 items, items (Q loads) so far
  bool ok = true;
  for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++nq) {
    const Item c = decode_item(p, item);
    // Both Q tiles are always loaded (rows past the tensor read as zero), so every
    // item completes one phase of each Q barrier.  Tile w is reloaded as soon as
    // the previous item's last S_w MMA is done with it.
    BCA_TRACE_AT(p, it / 2, 27);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      if (!mbar_wait_bounded(bar(Smem::bQEmpty + w), (static_cast<uint32_t>(nq) & 1u) ^ 1u, abort,
                             p.timeout_ns)) {
        raise_abort(abort, p.dev_status, 10);
        ok = false;
        break;
      }
      const uint32_t dst = sbase + (w == 0 ? Smem::kQ0 : Smem::kQ1);
      const int z = c.q_row0 + w * kBM;
      mbar_arrive_expect_tx(bar(Smem::bQFull + w), kTileBytes + (kQ8 ? kTile8Bytes : 0));
      tma_load_3d(dst, &p.tm_q, bar(Smem::bQFull + w), 0, c.h, z);
      tma_load_3d(dst + kHalfBytes, &p.tm_q, bar(Smem::bQFull + w), 64, c.h, z);
      // e4m3-Q mode: the tile's Q codes go to staging buffer w (unused otherwise).
      if (kQ8)
        tma_load_3d(sbase + Smem::kStage8 + w * kTile8Bytes, &p.tm_q8, bar(Smem::bQFull + w), 0,
                    z, c.h);
    }
    if (!ok) break;
    if (item + static_cast<int>(gridDim.x) < p.n_items) {
      // Warm L2 with the next item's Q while this item runs.
      const Item nx = decode_item(p, item + gridDim.x);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        tma_prefetch_l2_3d(&p.tm_q, 0, nx.h, nx.q_row0 + w * kBM);
        tma_prefetch_l2_3d(&p.tm_q, 64, nx.h, nx.q_row0 + w * kBM);
      }
    }
    for (int j = c.j0; j < c.j1 && ok; ++j) {
      for (int kv = 0; kv < 2; ++kv, ++it) {
        if (tile_is_converted<MAXR, kQ8>(p, c, j, kv)) {
          // e4m3 cache tile -> staging buffer; the converter warps fill the ring slot.
          // e4m3-Q mode: the staging buffers hold Q codes, so the (V) tile lands in
          // the upper half of its own ring slot and is expanded in place.
          const int ss = fi & 1;
          const uint32_t ph = static_cast<uint32_t>(fi >> 1) & 1u;
          if (!mbar_wait_bounded(bar(Smem::bStgEmpty + ss), ph ^ 1u, abort, p.timeout_ns)) {
            raise_abort(abort, p.dev_status, 11);
            ok = false;
            break;
          }
          uint32_t dst8 = sbase + Smem::kStage8 + ss * kTile8Bytes;
          if (kQ8) {
            const int st = it % kStages;
            if (!mbar_wait_bounded(bar(Smem::bKvEmpty + st),
                                   (static_cast<uint32_t>(it / kStages) & 1u) ^ 1u, abort,
                                   p.timeout_ns)) {
              raise_abort(abort, p.dev_status, 13);
              ok = false;
              break;
            }
            dst8 = sbase + Smem::kRing + st * kTileBytes + kTile8Bytes;
          }
          const uint32_t fb = bar(Smem::bStgFull + ss);
          mbar_arrive_expect_tx(fb, kTile8Bytes);
          if (BCA_CHECK(p.dev_status, c.req < p.n_req && j * kBN < c.n_cache && c.h < p.heads, 1))
            tma_load_3d(dst8, kv ? &p.tm_vc[c.req] : &p.tm_kc[c.req], fb, 0, j * kBN, c.h);
          ++fi;
          continue;
        }
        const int st = it % kStages;
        const uint32_t ph = static_cast<uint32_t>(it / kStages) & 1u;
        if (!mbar_wait_bounded(bar(Smem::bKvEmpty + st), ph ^ 1u, abort, p.timeout_ns)) {
          raise_abort(abort, p.dev_status, 12);
          ok = false;
          break;
        }
        const uint32_t dst = sbase + Smem::kRing + st * kTileBytes;
        const uint32_t fb = bar(Smem::bKvFull + st);
        BCA_TRACE_AT(p, it / 2, 23 + kv);
        if (kQ8 && tile_is_fp8(p, c, j, kv)) {
          // e4m3-Q mode, K cache tile: read by the MMA as stored (16 KiB).
          mbar_arrive_expect_tx(fb, kTile8Bytes);
          if (BCA_CHECK(p.dev_status, c.req < p.n_req && j * kBN < c.n_cache && c.h < p.heads, 6))
            tma_load_3d(dst, &p.tm_kc[c.req], fb, 0, j * kBN, c.h);
          continue;
        }
        mbar_arrive_expect_tx(fb, kTileBytes);
        if (p.mode == kModeStep && j < c.n_cache_tiles) {
          const CUtensorMap* m = kv ? &p.tm_vc[c.req] : &p.tm_kc[c.req];
          tma_load_3d(dst, m, fb, 0, j * kBN, c.h);
          tma_load_3d(dst + kHalfBytes, m, fb, 64, j * kBN, c.h);
        } else {
          const CUtensorMap* m = kv ? &p.tm_v : &p.tm_k;
          const int z = p.mode == kModePrefill ? j * kBN
                                               : c.q_start + (j - c.n_cache_tiles) * kBN;
          tma_load_3d(dst, m, fb, 0, c.h, z);
          tma_load_3d(dst + kHalfBytes, m, fb, 64, c.h, z);
        }
      }
    }
  }
  if (!ok || *abort) {
    // Drain: wait (time-bounded only) for copies this thread may still have in flight.
    constexpr unsigned long long kDrainNs = 20000000ull;
    for (int i = max(0, it - kStages); i < it; ++i)
      mbar_wait_bounded(bar(Smem::bKvFull + i % kStages), static_cast<uint32_t>(i / kStages) & 1u,
                        nullptr, kDrainNs);
    for (int i = max(0, fi - 2); i < fi; ++i)
      mbar_wait_bounded(bar(Smem::bStgFull + (i & 1)), static_cast<uint32_t>(i >> 1) & 1u, nullptr,
                        kDrainNs);
    if (nq > 0)
      for (int w = 0; w < 2; ++w)
        mbar_wait_bounded(bar(Smem::bQFull + w), static_cast<uint32_t>(nq - 1) & 1u, nullptr,
                          kDrainNs);
  }
}

// ---------------------------------------------------------------------------
// Converter: warps 10-11 (64 threads) turn staged e4m3 cache tiles into the bf16
// 128-byte-swizzled layout the MMA reads (e4m3 -> f16 -> bf16 is exact).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(two & 0xFFFFu)));
  float lo, hi;
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(static_cast<uint16_t>(h & 0xFFFFu)));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(static_cast<uint16_t>(h >> 16)));
  return pack_bf16x2(lo, hi);
}

template <int MAXR, bool kQ8>
__device__ void converter_role(const AttnParams<MAXR>& p, uint32_t sbase, uint32_t bars,
                               volatile int* abort) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const int c = threadIdx.x - kWarpConv0 * 32;  // 0..63
  int it = 0, fi = 0;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    const Item ci = decode_item(p, item);
    for (int j = ci.j0; j < ci.j1; ++j) {
      for (int kv = 0; kv < 2; ++kv, ++it) {
        if (!tile_is_converted<MAXR, kQ8>(p, ci, j, kv)) continue;
        const int ss = fi & 1;
        const int st = it % kStages;
        // (e4m3-Q mode: the producer waited for the ring slot before loading into it.)
        const bool got =
            mbar_wait_bounded(bar(Smem::bStgFull + ss), static_cast<uint32_t>(fi >> 1) & 1u,
                              abort, p.timeout_ns) &&
            (kQ8 || mbar_wait_bounded(bar(Smem::bKvEmpty + st),
                                      (static_cast<uint32_t>(it / kStages) & 1u) ^ 1u, abort,
                                      p.timeout_ns));
        if (!got) {
          raise_abort(abort, p.dev_status, 21);
          return;
        }
        const uint32_t dst = sbase + Smem::kRing + st * kTileBytes;
        const uint32_t src = kQ8 ? dst + kTile8Bytes : sbase + Smem::kStage8 + ss * kTile8Bytes;
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
          const int gid = k * kConvThreads + c;
          const int row = gid >> 3, ch = gid & 7;
          const bool in_bounds =
              BCA_CHECK(p.dev_status, row < kBN && src + row * 128 + 128 <= sbase + Smem::kBars &&
                                          dst + kTileBytes <= sbase + Smem::kStage8, 2);
          uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;
          if (in_bounds)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                         : "r"(src + row * 128 + ((ch ^ (row & 7)) << 4)));
          // In place (e4m3-Q mode), the upper half of row `row`'s output overwrites
          // the row's own source bytes, which the row's 8 threads (8 lanes of one
          // warp) read above: every lane's load comes before any lane's store.
          if (kQ8) __syncwarp();
          if (!in_bounds) continue;
          const uint32_t o0 = e4m3x2_to_bf16x2(w0), o1 = e4m3x2_to_bf16x2(w0 >> 16);
          const uint32_t o2 = e4m3x2_to_bf16x2(w1), o3 = e4m3x2_to_bf16x2(w1 >> 16);
          const uint32_t o4 = e4m3x2_to_bf16x2(w2), o5 = e4m3x2_to_bf16x2(w2 >> 16);
          const uint32_t o6 = e4m3x2_to_bf16x2(w3), o7 = e4m3x2_to_bf16x2(w3 >> 16);
          const int k0 = 2 * (ch & 3);
          const uint32_t base = dst + (ch >> 2) * kHalfBytes + row * 128;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                           base + ((k0 ^ (row & 7)) << 4)),
                       "r"(o0), "r"(o1), "r"(o2), "r"(o3)
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                           base + (((k0 + 1) ^ (row & 7)) << 4)),
                       "r"(o4), "r"(o5), "r"(o6), "r"(o7)
                       : "memory");
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(Smem::bConv));
        // Every converter thread waits for the whole tile: none may run ahead and
        // arrive for the next tile while this phase is still open.
        if (!mbar_wait_bounded(bar(Smem::bConv), static_cast<uint32_t>(fi) & 1u, abort,
                               p.timeout_ns)) {
          raise_abort(abort, p.dev_status, 22);
          return;
        }
        if (c == 0) {
          mbar_arrive(bar(Smem::bKvFull + st));
          mbar_arrive(bar(Smem::bStgEmpty + ss));
        }
        ++fi;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// MMA issuer: the whole warp (values stay warp-uniform); one elected lane issues.
// ---------------------------------------------------------------------------
template <int MAXR, bool kQ8>
__device__ void mma_role(const AttnParams<MAXR>& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                         volatile int* abort) {
  // The items of this CTA are one stream of KV tiles.  Iteration t issues, per Q tile
  // w, O_w += P_w(t-1) V(t-1) and then S_w(t) = Q_w K(t)^T -- also across item
  // boundaries, so the last tile of an item overlaps the first tile of the next.
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);      // Q K^T: K-major B
  constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, kHeadDim, true);  // P V: MN-major B
  constexpr uint32_t kIdescS8 = idesc_e4m3_f32(kBM, kBN);            // Q8 K8^T (e4m3-Q mode)
  bool ok = true;
  auto wait = [&](int b, uint32_t parity) {
    if (ok) {
      const bool got = mbar_wait_bounded(bar(b), parity, abort, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (elect_one()) raise_abort(abort, p.dev_status, 30 + b);
        ok = false;
      }
    }
    return ok;
  };
  const uint64_t dq[2] = {sdesc_sw128(sbase + Smem::kQ0, 16, 1024),
                          sdesc_sw128(sbase + Smem::kQ1, 16, 1024)};
  int npv[2] = {0, 0};  // P tiles consumed per Q tile (P barrier phases)
  int nq = 0;           // items started (Q barrier phases)
  // The previous tile (its P V is issued in the next iteration).
  bool has_prev = false, prev_pv[2] = {false, false}, prev_last[2] = {false, false};
  bool prev_first[2] = {false, false};
  int prev_stV = 0;
  int t = 0;  // tiles of this CTA so far (ring items 2t, 2t+1)
  auto issue_pv = [&](int w, int stV, bool first_of_item, bool last_of_item) {
    const uint64_t dv = sdesc_sw128(sbase + Smem::kRing + stV * kTileBytes, kHalfBytes, 1024);
    if (!wait(Smem::bPFull + w, static_cast<uint32_t>(npv[w]) & 1u)) return;
    tc_fence_after();
    if (elect_one()) {
#pragma unroll
      for (int s = 0; s < kBN / 16; ++s)  // K = 16 keys per MMA
        mma_bf16_ts(tmem + col_o(w), tmem + col_s(w) + s * 8, dv + ((s * 2048) >> 4), kIdescO,
                    (!first_of_item || s > 0) ? 1u : 0u);
      if (last_of_item) mma_commit(bar(Smem::bOFull + w));
    }
    __syncwarp();
    ++npv[w];
  };
  for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++nq) {
    const Item c = decode_item(p, item);
    const bool act[2] = {tile_active(c, 0), tile_active(c, 1)};
    for (int j = c.j0; j < c.j1 && ok; ++j, ++t) {
      const int itK = 2 * t, itV = 2 * t - 1;
      const int stK = itK % kStages;
      BCA_TRACE_AT(p, t, 21);
      if (has_prev) wait(Smem::bKvFull + prev_stV, static_cast<uint32_t>(itV / kStages) & 1u);
      // At an item boundary the previous item's last P V does not need this item's Q
      // or K: issue it first, so that its O (and the epilogue) is not held up by the
      // new item's loads.
      bool pv_issued[2] = {false, false};
      if (j == c.j0 && has_prev && ok) {
        tc_fence_after();
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (prev_pv[w] && ok) {
            issue_pv(w, prev_stV, prev_first[w], prev_last[w]);
            pv_issued[w] = true;
          }
        }
      }
      wait(Smem::bKvFull + stK, static_cast<uint32_t>(itK / kStages) & 1u);
      BCA_TRACE_AT(p, t, 22);
      if (j == c.j0) {
        wait(Smem::bQFull + 0, static_cast<uint32_t>(nq) & 1u);
        wait(Smem::bQFull + 1, static_cast<uint32_t>(nq) & 1u);
        BCA_TRACE_AT(p, t, 26);
      }
      if (!ok) break;
      BCA_TRACE_AT(p, t, 0);
      tc_fence_after();
      const uint64_t dk = sdesc_sw128(sbase + Smem::kRing + stK * kTileBytes, 16, 1024);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        if (has_prev && prev_pv[w] && !pv_issued[w]) {
          issue_pv(w, prev_stV, prev_first[w], prev_last[w]);
          if (!ok) break;
          BCA_TRACE_AT(p, t, 1 + 2 * w);
        }
        const int jend = w ? c.jend[1] : c.jend[0];
        if (act[w] && j < jend) {
          if (elect_one()) {
            if (kQ8 && j < c.n_cache_tiles) {
              // Q codes of tile w in staging buffer w, K codes in the ring slot: one
              // 128-byte swizzle atom per row; the 4 MMAs of K = 32 step 32 bytes.
              // (Not unrolled: the unrolled descriptors spill the 104-register
              // warpgroup.)
              const uint64_t dq8 =
                  sdesc_sw128(sbase + Smem::kStage8 + w * kTile8Bytes, 16, 1024);
#pragma unroll 1
              for (int s = 0; s < kHeadDim / 32; ++s)
                mma_e4m3_ss(tmem + col_s(w), dq8 + ((s * 32) >> 4), dk + ((s * 32) >> 4),
                            kIdescS8, s > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int s = 0; s < kHeadDim / 16; ++s) {
                const uint32_t koff = ((s / 4) * kHalfBytes + (s % 4) * 32) >> 4;
                mma_bf16_ss(tmem + col_s(w), dq[w] + koff, dk + koff, kIdescS, s > 0 ? 1u : 0u);
              }
            }
            mma_commit(bar(Smem::bSFull + w));
            // Last S_w of the item: Q tile w may be reloaded once this MMA is done.
            if (j == jend - 1) mma_commit(bar(Smem::bQEmpty + w));
          }
          __syncwarp();
          BCA_TRACE_AT(p, t, 2 + 2 * w);
        }
      }
      if (!ok) break;
      if (elect_one()) {
        mma_commit(bar(Smem::bKvEmpty + stK));
        if (has_prev) mma_commit(bar(Smem::bKvEmpty + prev_stV));
        // A Q tile without rows in this item was loaded but is never read: release
        // it at once (the producer reloads every Q tile for every item).
        if (j == c.j0) {
          if (!act[0]) mma_commit(bar(Smem::bQEmpty + 0));
          if (!act[1]) mma_commit(bar(Smem::bQEmpty + 1));
        }
      }
      __syncwarp();
      has_prev = true;
      prev_stV = (2 * t + 1) % kStages;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int jend = w ? c.jend[1] : c.jend[0];
        prev_pv[w] = act[w] && j < jend;
        prev_first[w] = j == c.j0;
        prev_last[w] = j == jend - 1;
      }
    }
  }
  if (ok && has_prev) {
    // The last tile's P V.
    wait(Smem::bKvFull + prev_stV, static_cast<uint32_t>(2 * t - 1) / kStages & 1u);
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int w = 0; w < 2; ++w)
        if (prev_pv[w] && ok) issue_pv(w, prev_stV, prev_first[w], prev_last[w]);
      if (ok && elect_one()) mma_commit(bar(Smem::bKvEmpty + prev_stV));
      __syncwarp();
    }
  }
  // Everything issued must be complete before TMEM is released.  If that wait runs
  // out, the timeout is reported and the CTA waits once more (bounded) before the
  // kernel frees TMEM.
  if (elect_one()) mma_commit(bar(Smem::bDone));
  __syncwarp();
  const bool done = mbar_wait_bounded(bar(Smem::bDone), 0, nullptr, p.timeout_ns);
  if (!__all_sync(0xffffffffu, done)) {
    if (elect_one()) raise_abort(abort, p.dev_status, 30 + Smem::bDone);
    mbar_wait_bounded(bar(Smem::bDone), 0, nullptr, p.timeout_ns);
  }
}

// ---------------------------------------------------------------------------
// Softmax + epilogue: 128 threads (one warpgroup) per Q tile, one row each.
// ---------------------------------------------------------------------------
template <int MAXR, bool kQ8>
__device__ void softmax_role(const AttnParams<MAXR>& p, int w, uint32_t sbase, uint32_t bars,
                             uint32_t tmem, volatile int* abort) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const int warp = (threadIdx.x / 32) % 4;
  const int lane = threadIdx.x % 32;
  const int row = warp * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_off + col_s(w);
  const uint32_t tO = tmem + lane_off + col_o(w);
  const bool prefill = p.mode == kModePrefill;
  const int seq_len = p.seq_len;
  const uint32_t b_s = bar(Smem::bSFull + w);
  const uint32_t b_o = bar(Smem::bOFull + w);
  int ns = 0, no = 0;  // S tiles and O results consumed (barrier phases)
  int nep = 0;         // O boxes stored through shared memory (epilogue barrier phases)
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    const Item c = decode_item(p, item);
    if (!tile_active(c, w)) continue;
    const int rows_w = w ? c.rows[1] : c.rows[0];
    const int jend = w ? c.jend[1] : c.jend[0];
    const int grow = c.q_row0 + w * kBM + row;
    int lim = kNoLimit;
    if (prefill) lim = row < rows_w ? block_end(p, grow) : seq_len;
    // e4m3 cache tiles: scores scale by k_scale (folded into the exp2 scale) and P
    // by v_scale (folded into the exp2 bias; the row sum keeps the unscaled P).
    float sl2_cache = p.scale_log2, lg_vs = 0.f, inv_vs = 1.f;
    if (!prefill) {
      if (!BCA_CHECK(p.dev_status, c.req < p.n_req && (!p.k_scaled || p.k_scale[c.req]) &&
                                       (!p.v_scaled || p.v_scale[c.req]), 4))
        return;
      if (p.k_scaled) sl2_cache *= __ldg(p.k_scale[c.req] + c.h);
      // e4m3-Q mode: cached keys' scores are Q8 K8^T, so Q's scale joins K's.
      if (kQ8 && BCA_CHECK(p.dev_status, p.q_scale[c.req] != nullptr, 7))
        sl2_cache *= __ldg(p.q_scale[c.req] + c.h);
      if (p.v_scaled) {
        const float vs = __ldg(p.v_scale[c.req] + c.h);
        lg_vs = __log2f(vs);
        inv_vs = 1.0f / vs;
      }
    }
    const float sl2_base = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = c.j0; j < jend; ++j, ++ns) {
      const bool got = mbar_wait_bounded(b_s, static_cast<uint32_t>(ns) & 1u, abort, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        raise_abort(abort, p.dev_status, 61);
        return;
      }
      tc_fence_after();
      const bool tr = row == 0;
      const bool trw = lane == 0 && warp > 0;
      if (tr) BCA_TRACE_AT(p, ns, 5 + 5 * w);
      uint32_t r[128];
      tmem_ld_32x32b_x128(tS, r);
      tmem_wait_ld();
      if (tr) BCA_TRACE_AT(p, ns, 6 + 5 * w);
      int valid, key_base;
      kv_tile_extent(prefill, c, seq_len, j, valid, key_base);
      const bool cache_tile = !prefill && j < c.n_cache_tiles;
      const float sl2 = cache_tile ? sl2_cache : sl2_base;
      const int nv = min(valid, lim - key_base);
      if (nv < kBN) {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          if (cc >= nv) r[cc] = __float_as_uint(-INFINITY);
      }
      if (tr && w == 0) BCA_TRACE_AT(p, ns, 25);
      // Row max: 8 independent chains of three-input max, then a short tree.
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float* x = reinterpret_cast<const float*>(&r[16 * i]);
        float a = fmax3(x[0], x[1], x[2]);
#pragma unroll
        for (int e = 3; e < 15; e += 2) a = fmax3(a, x[e], x[e + 1]);
        t[i] = fmaxf(a, x[15]);
      }
      const float mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]), fmaxf(t[6], t[7]));
      const float m_new = mx * sl2;
      if (tr) BCA_TRACE_AT(p, ns, 7 + 5 * w);
      const bool need = m_new > m_run + kRescaleThreshold;
      float f = 1.0f;
      if (need) {
        f = ex2_approx(m_run - m_new);  // 0 on the first tile (m_run = -inf)
        l_run *= f;
        m_run = m_new;
      }
      // A row with no allowed key so far (only in a split chunk of a prefill unit
      // whose rows straddle a block end) keeps m = -inf: its p are exactly 0.
      const float neg_m = (cache_tile ? lg_vs : 0.f) - (m_run == -INFINITY ? 0.f : m_run);
      // O was last written by P(j-1) V(j-1), complete before S(j) was signalled; it
      // is rescaled before the first half of P(j) is handed over (P(j) V(j) waits).
      if (j > c.j0 && __any_sync(0xffffffffu, need)) {
        const uint64_t f2 = f2_pack(f, f);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[16];
          tmem_ld_32x32b_x16(tO + 16 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float y0, y1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), f2), y0,
                      y1);
            o[e] = __float_as_uint(y0);
            o[e + 1] = __float_as_uint(y1);
          }
          tmem_st_32x32b_x16(tO + 16 * cc, o);
        }
      }
      // p = 2^(s * sl2 - m) on column pairs: packed fp32x2 FMA for the exponent, MUFU
      // ex2 for the power; P is packed to bf16 in place over S (64 columns) and
      // handed to the MMA as a whole tile.
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int cc = 32 * half; cc < 32 * half + 32; ++cc) {
          const uint64_t x =
              f2_fma(f2_pack(__uint_as_float(r[2 * cc]), __uint_as_float(r[2 * cc + 1])), sl2x2,
                     negm2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
          acc[cc & 3] = f2_add(acc[cc & 3], pp);
          float p0, p1;
          f2_unpack(pp, p0, p1);
          r[cc] = pack_bf16x2(p0, p1);
        }
        tmem_st_32x32b_x32(tS + 32 * half, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * half]));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(Smem::bPFull + w));
      float a0, a1, b0, b1;
      f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
      f2_unpack(f2_add(acc[2], acc[3]), b0, b1);
      const float tile_sum = (a0 + a1) + (b0 + b1);
      l_run += cache_tile ? tile_sum * inv_vs : tile_sum;
      if (tr) BCA_TRACE_AT(p, ns, 8 + 5 * w);
      if (tr) BCA_TRACE_AT(p, ns, 9 + 5 * w);
      if (trw) BCA_TRACE_AT(p, ns, 14 + 3 * w + warp);
    }
    // Epilogue: O of this item is complete once its last P V is.
    {
      const bool got = mbar_wait_bounded(b_o, static_cast<uint32_t>(no) & 1u, abort, p.timeout_ns);
      ++no;
      if (!__all_sync(0xffffffffu, got)) {
        raise_abort(abort, p.dev_status, 62);
        return;
      }
    }
    tc_fence_after();
    const bool tma_epilogue = c.partial < 0 && rows_w == kBM && !p.k_fp8 && !p.v_fp8;
    if (tma_epilogue) {
      // Whole bf16 Q tile: normalise into a 64-column box in shared memory (the e4m3
      // staging buffer of tile w, unused with a bf16 cache) and store it with one TMA
      // copy per box -- full 128-byte rows instead of 16-byte pieces 8 KiB apart.
      const float inv = 1.0f / l_run;
      const uint32_t stg = sbase + Smem::kStage8 + w * kTile8Bytes;
#pragma unroll
      for (int half = 0; half < 2; ++half, ++nep) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(bar(Smem::bEpiFree + w),
                                          (static_cast<uint32_t>(nep) & 1u) ^ 1u, abort,
                                          p.timeout_ns))) {
          raise_abort(abort, p.dev_status, 66);
          return;
        }
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // 32 columns = chunks 4 part .. 4 part + 3
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + 64 * half + 32 * part, o);
          tmem_wait_ld();
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {  // 16-byte chunk q of the row, 128-byte swizzle
            const int q = 4 * part + qq;
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(o[8 * qq + 2 * e]) * inv,
                                  __uint_as_float(o[8 * qq + 2 * e + 1]) * inv);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             stg + row * 128 + ((q ^ (row & 7)) << 4)),
                         "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(Smem::bEpiFull + w));
        if (row == 0) {
          if (!mbar_wait_bounded(bar(Smem::bEpiFull + w), static_cast<uint32_t>(nep) & 1u, abort,
                                 p.timeout_ns)) {
            raise_abort(abort, p.dev_status, 67);
          } else {
            tma_store_3d(&p.tm_o, stg, 64 * half, c.h, c.q_row0 + w * kBM);
            bulk_commit();
            bulk_wait_read();
          }
          mbar_arrive(bar(Smem::bEpiFree + w));
        }
      }
    } else if (c.partial < 0) {
      const float inv = 1.0f / l_run;
      const bool store = row < rows_w &&
                         BCA_CHECK(p.dev_status, grow < p.o_rows && c.h < p.heads, 3);
      uint4* dst =
          reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(grow) * p.heads + c.h) * kHeadDim);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + 32 * cc, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (store) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[4 * cc + e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    } else {
      // Split chunk: unnormalised O (with this chunk's running max) plus m and l.
      float* ws = p.workspace + static_cast<size_t>(c.partial) * (kChunkBytes / 4);
      const int r2 = w * kBM + row;
      float4* od = reinterpret_cast<float4*>(ws + static_cast<size_t>(r2) * kHeadDim);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + 32 * cc, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          od[8 * cc + e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                       __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      }
      ws[kChunkRows * kHeadDim + r2] = m_run;
      ws[kChunkRows * kHeadDim + kChunkRows + r2] = l_run;
    }
    // O of this item has been read: the next item's first P V (accumulate = 0) only
    // runs after our next P arrival, which follows these TMEM loads in program order.
  }
  if (row == 0) bulk_wait_all();  // this thread's TMA stores of O are in global memory
}

// ---------------------------------------------------------------------------
// The kernel (persistent: one CTA per SM, static round-robin over work items)
// ---------------------------------------------------------------------------
template <int MAXR, bool kQ8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnParams<MAXR> p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + Smem::kBars;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Smem::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::kTmemSlot);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
#ifdef BCA_TRACE
  const long long t_start = clock64();
#endif

  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Smem::bQFull + i), 1);
      mbar_init(bar(Smem::bQEmpty + i), 1);
      mbar_init(bar(Smem::bSFull + i), 1);
      mbar_init(bar(Smem::bPFull + i), 128);
      mbar_init(bar(Smem::bOFull + i), 1);
      mbar_init(bar(Smem::bEpiFull + i), 128);
      mbar_init(bar(Smem::bEpiFree + i), 1);
      mbar_init(bar(Smem::bStgFull + i), 1);
      mbar_init(bar(Smem::bStgEmpty + i), 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(Smem::bKvFull + i), 1);
      mbar_init(bar(Smem::bKvEmpty + i), 1);
    }
    mbar_init(bar(Smem::bDone), 1);
    mbar_init(bar(Smem::bConv), kConvThreads);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (kQ8) tma_prefetch_desc(&p.tm_q8);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8) {
    regs_increase<kSoftmaxRegs>();
    softmax_role<MAXR, kQ8>(p, warp / 4, sbase, bars, tmem, abort);
  } else {
    regs_decrease<kOtherRegs>();
    if (warp == kWarpProducer) {
      if (lane == 0) producer_role<MAXR, kQ8>(p, sbase, bars, abort);
    } else if (warp == kWarpMma) {
      mma_role<MAXR, kQ8>(p, sbase, bars, tmem, abort);
      __syncwarp();
    } else if (p.mode == kModeStep && (p.k_fp8 || p.v_fp8)) {
      converter_role<MAXR, kQ8>(p, sbase, bars, abort);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#ifdef BCA_TRACE
  // Whole-CTA cycle count (cheap; independent of the per-tile trace).
  if (threadIdx.x == 0 && p.trace && blockIdx.x < 1024)
    p.trace[kTraceTiles * kTraceEvents + blockIdx.x] = clock64() - t_start;
#endif
}

// ---------------------------------------------------------------------------
// Merge the split chunks of a unit: O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c.
// One warp per (split unit, row), one float4 of the row per lane: every chunk row is
// read as one coalesced 512-byte segment.  8 rows per 256-thread block.
// ---------------------------------------------------------------------------
constexpr int kMaxSplit = 8;
constexpr int kCombineRowsPerBlock = 8;

template <int MAXR>
__global__ void __launch_bounds__(256)
    attn_combine_kernel(const __grid_constant__ AttnParams<MAXR> p, int n_split_units) {
  const int gw = blockIdx.x * kCombineRowsPerBlock + static_cast<int>(threadIdx.x / 32);
  const int lane = threadIdx.x % 32;
  const int su = gw / kChunkRows, r2 = gw % kChunkRows;
  if (su >= n_split_units) return;
  const int k = p.split_k;
  const Item c = decode_item(p, p.full_items + su * k);  // chunk 0 of the unit
  const int w = r2 / kBM, row = r2 % kBM;
  const int rows_w = w ? c.rows[1] : c.rows[0];
  if (row >= rows_w || k < 1 || k > kMaxSplit) return;
  const int grow = c.q_row0 + w * kBM + row;
  if (!BCA_CHECK(p.dev_status, grow < p.o_rows && c.h < p.heads, 5)) return;
  constexpr size_t kStride = kChunkBytes / 4;
  const float* ws0 = p.workspace + static_cast<size_t>(su) * k * kStride;
  // Every load of every chunk is issued before any of them is used.
  float m[kMaxSplit], l[kMaxSplit];
  float4 a[kMaxSplit];
#pragma unroll
  for (int ci = 0; ci < kMaxSplit; ++ci) {
    // A chunk whose key range lies wholly past Q tile w's key limit (prefill units
    // straddling a block end) wrote nothing for these rows.
    if (ci < k && (ci == 0 || tile_active(decode_item(p, p.full_items + su * k + ci), w))) {
      const float* chunk = ws0 + ci * kStride;
      m[ci] = chunk[kChunkRows * kHeadDim + r2];
      l[ci] = chunk[kChunkRows * kHeadDim + kChunkRows + r2];
      a[ci] = reinterpret_cast<const float4*>(chunk + static_cast<size_t>(r2) * kHeadDim)[lane];
    } else {
      m[ci] = -INFINITY;
      l[ci] = 0.f;
      a[ci] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int ci = 0; ci < kMaxSplit; ++ci) M = fmaxf(M, m[ci]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
#pragma unroll
  for (int ci = 0; ci < kMaxSplit; ++ci) {
    if (ci >= k) break;
    const float wgt = ex2_approx(m[ci] - M);
    L += wgt * l[ci];
    acc.x += wgt * a[ci].x;
    acc.y += wgt * a[ci].y;
    acc.z += wgt * a[ci].z;
    acc.w += wgt * a[ci].w;
  }
  const float inv = 1.0f / L;
  uint2* dst = reinterpret_cast<uint2*>(p.o + (static_cast<size_t>(grow) * p.heads + c.h) * kHeadDim);
  dst[lane] = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
}

}  // namespace bca
