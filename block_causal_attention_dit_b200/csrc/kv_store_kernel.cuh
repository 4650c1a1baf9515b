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
#include <cuda_bf16.h>

#include <cstdint>

#include "../../include/bca.h"

namespace bca {

__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t m, uint32_t w) {
  return max(m, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
}

__device__ __forceinline__ float scale_from_amax_bits(unsigned bits) {
  const float amax = __uint_as_float(bits << 16);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// x / s for the encoder, from y = RN(1/s): q = RN(x y), then one correction with the
// exact residual x - q s (an FMA):  RN(q + (x - q s) y) -- the division scheme of
// P. Markstein, "IA-64 and Elementary Functions: Speed and Precision" (2000), ch. 8.
// For heads whose amax is below 2^-95 (bf16 bits < kFastDivMinBits) the reciprocal
// and the residual leave the normal range, so those take the correctly rounded
// division.  bca_selftest_e4m3_division checks that the resulting codes equal those
// of the correctly rounded quotient for every bf16 amax and every bf16 |x| <= amax.
constexpr unsigned kFastDivMinBits = 0x1000u;
__device__ __forceinline__ float div_by_scale(float x, float s, float y, bool fast) {
  if (!fast) return __fdiv_rn(x, s);
  const float q = x * y;
  const float r = fmaf(-q, s, x);
  return copysignf(fmaf(r, y, q), x);  // s > 0: the quotient has x's sign (also for -0)
}

// Two fp32 -> packed e4m3x2, round to nearest even, saturate to +-448;
// `lo` lands in bits [0, 8).
__device__ __forceinline__ uint16_t e4m3x2_rn_satfinite(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// The store kernel.  A launch stores a list of tensors; tensor i has heads_i
// columns (one per head: rows [0, rows_i) of that head), numbered from col0_i.  A
// cluster of kStoreCluster CTAs takes whole columns (cluster c: columns c, c +
// #clusters, ...; the host lists tensors with the most rows first), and its CTAs
// split the column's rows evenly.  Only as many clusters are launched as can be
// resident at once (the cluster loop is persistent; a cluster that had to wait for
// another to finish would run its whole share of columns after it).
//  * bf16 column: a copy.
//  * e4m3 column: pass 1 reads the CTA's rows for the absmax; the CTAs' partial
//    maxima meet in every CTA's shared memory (distributed shared memory stores,
//    then a cluster barrier), so each CTA knows amax_h; rank 0 writes s_h.  Pass 2
//    reads the same rows again, last-read first, so that most of them still come
//    from L2 (a column is at most ~4.4 MB and only as many columns are in flight as
//    there are resident clusters), and writes the codes with streaming stores.
//    Measured on the 8-request serving store: clusters of 4 (all SMs busy) beat
//    clusters of 8 (15 resident, 120 SMs), 0.67 vs 0.72 ms.
// Every thread owns one 16-byte chunk (8 channels) of a row; 16 threads cover a
// 256-byte head row.  A thread streams its rows through its own ring of
// kStoreRing 16-byte slots in shared memory filled by cp.async (128 KiB per CTA in
// flight without holding registers).
// A non-finite value in an e4m3 column makes its amax Inf or NaN: the column's
// codes and scale are then meaningless and BCA_ERR_NONFINITE is written to
// *dev_status (the inputs must be finite).
// ---------------------------------------------------------------------------
struct StoreTensor {
  const uint16_t* src;  // bf16 bits; row t, head h at src + t * row_stride + h * 128
  void* dst;            // row t, head h at element (h * head_stride + t) * 128 (bf16 or e4m3)
  float* scale;         // [heads] fp32, e4m3 tensors only
  int64_t row_stride;   // source elements between consecutive rows
  int64_t head_stride;  // destination rows between consecutive heads
  int32_t rows;
  int32_t heads;
  int32_t quant;        // 1: e4m3 with a per-head absmax scale, 0: bf16 copy
  int32_t col0;         // first column of this tensor
};

constexpr int kMaxStoreTensors = 2 * BCA_MAX_BATCH;
constexpr int kStoreThreads = 512;
constexpr int kStoreCluster = 4;
constexpr int kStoreRing = 16;  // 16-byte copies in flight per thread
constexpr int kStoreRingBytes = kStoreRing * kStoreThreads * 16;
constexpr int kStoreRowsPerSweep = kStoreThreads / 16;

struct StoreParams {
  StoreTensor t[kMaxStoreTensors];
  int32_t n_tensors;
  int32_t n_cols;
  int32_t* dev_status;
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
// 32-bit store into CTA `rank`'s copy of the shared variable at local address `a`.
__device__ __forceinline__ void st_shared_cluster(uint32_t a, uint32_t rank, uint32_t v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}

__device__ __forceinline__ uint2 encode_chunk(const uint4 v, float s, float y, bool fast) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint16_t a = e4m3x2_rn_satfinite(div_by_scale(bf16_lo(w[2 * k]), s, y, fast),
                                           div_by_scale(bf16_hi(w[2 * k]), s, y, fast));
    const uint16_t b = e4m3x2_rn_satfinite(div_by_scale(bf16_lo(w[2 * k + 1]), s, y, fast),
                                           div_by_scale(bf16_hi(w[2 * k + 1]), s, y, fast));
    out[k] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
  }
  return make_uint2(out[0], out[1]);
}

// 16-byte asynchronous copy global -> shared (no register staging, L1 bypassed);
// one commit group per call site.
__device__ __forceinline__ void cp_async16(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The rows of one thread, k = 0..n-1 (row first + k * step), streamed through the
// thread's own ring of kStoreRing 16-byte slots in shared memory: the copy of row
// k + kStoreRing is issued as soon as row k has been used, so kStoreRing copies per
// thread (128 KiB per CTA) stay in flight without holding registers.
template <typename Fn>
__device__ __forceinline__ void stream_rows(uint32_t ring, const uint16_t* src, int64_t rs,
                                            int first, int step, int n, Fn&& use) {
  const uint32_t slot0 = ring + threadIdx.x * 16u;
#pragma unroll
  for (int i = 0; i < kStoreRing; ++i) {
    if (i < n) cp_async16(slot0 + i * (kStoreThreads * 16u), src + (first + i * step) * rs);
    cp_async_commit();
  }
  for (int k = 0; k < n; ++k) {
    cp_async_wait<kStoreRing - 1>();
    const uint32_t slot = slot0 + (k % kStoreRing) * (kStoreThreads * 16u);
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(slot)
                 : "memory");
    use(v, first + k * step);
    if (k + kStoreRing < n) cp_async16(slot, src + (first + (k + kStoreRing) * step) * rs);
    cp_async_commit();
  }
  cp_async_wait<0>();
}

__global__ void __launch_bounds__(kStoreThreads, 1)
    kv_store_kernel(const __grid_constant__ StoreParams p) {
  extern __shared__ __align__(16) uint8_t store_ring[];
  __shared__ unsigned s_part[2][kStoreCluster];  // partial maxima by rank, double-buffered
  __shared__ unsigned s_warp[kStoreThreads / 32];
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(store_ring));
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int tid = threadIdx.x, lane16 = tid & 15, rslot = tid >> 4;
  int ti = 0, nq = 0;
  for (int col = static_cast<int>(cluster_index()); col < p.n_cols;
       col += static_cast<int>(cluster_count())) {
    while (ti + 1 < p.n_tensors && col >= p.t[ti + 1].col0) ++ti;
    const StoreTensor& T = p.t[ti];
    const int h = col - T.col0;
    const int r0 = static_cast<int>(static_cast<int64_t>(T.rows) * crank / csize);
    const int r1 = static_cast<int>(static_cast<int64_t>(T.rows) * (crank + 1) / csize);
    const uint16_t* src = T.src + static_cast<int64_t>(h) * 128 + lane16 * 8;
    const int64_t rs = T.row_stride;
    const int64_t drow0 = static_cast<int64_t>(h) * T.head_stride;
    // This thread's rows: r0 + rslot + k * kStoreRowsPerSweep, k < n.
    const int n = r1 - r0 > rslot ? (r1 - r0 - rslot + kStoreRowsPerSweep - 1) / kStoreRowsPerSweep : 0;
    if (!T.quant) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(T.dst) + drow0 * 128) + lane16;
      stream_rows(ring, src, rs, r0 + rslot, kStoreRowsPerSweep, n,
                  [&](const uint4& v, int t) { __stcs(dst + static_cast<int64_t>(t) * 16, v); });
      continue;
    }
    // Pass 1: absmax of this CTA's rows, as bf16 magnitude bits.
    uint32_t m = 0;
    stream_rows(ring, src, rs, r0 + rslot, kStoreRowsPerSweep, n, [&](const uint4& v, int) {
      m = max_abs_bf16x2(m, v.x);
      m = max_abs_bf16x2(m, v.y);
      m = max_abs_bf16x2(m, v.z);
      m = max_abs_bf16x2(m, v.w);
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) s_warp[tid >> 5] = m;
    __syncthreads();
    if (tid < 32) {
      uint32_t x = tid < kStoreThreads / 32 ? s_warp[tid] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, o));
      if (tid == 0) {
        const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&s_part[nq & 1][crank]));
        for (uint32_t q = 0; q < csize; ++q) st_shared_cluster(a, q, x);
      }
    }
    cluster_sync();
    uint32_t amax_bits = 0;
    for (uint32_t q = 0; q < csize; ++q) amax_bits = max(amax_bits, s_part[nq & 1][q]);
    ++nq;
    const float s = scale_from_amax_bits(amax_bits);
    if (crank == 0 && tid == 0) {
      T.scale[h] = s;
      if (amax_bits >= 0x7F80u && p.dev_status)
        atomicExch(p.dev_status, static_cast<int32_t>(BCA_ERR_NONFINITE));
    }
    const float y = __frcp_rn(s);
    const bool fast = amax_bits >= kFastDivMinBits;
    // Pass 2: the same rows, last-read first (still in L2); codes with streaming
    // stores.
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(T.dst) + drow0 * 128) + lane16;
    if (n > 0)
      stream_rows(ring, src, rs, r0 + rslot + (n - 1) * kStoreRowsPerSweep, -kStoreRowsPerSweep,
                  n, [&](const uint4& v, int t) {
                    __stcs(dst + static_cast<int64_t>(t) * 16, encode_chunk(v, s, y, fast));
                  });
  }
  // No CTA leaves while a peer may still store into its shared memory.
  cluster_sync();
}

// Self-check of div_by_scale as the encoder uses it: for every positive finite bf16
// amax (blockIdx.x + 1 as magnitude bits) and every bf16 x with |x| <= amax, the e4m3
// code of div_by_scale(x, s, RN(1/s), amax >= 2^-95) must equal the code of the
// correctly rounded x / s.
__global__ void __launch_bounds__(256) e4m3_division_selftest_kernel(unsigned long long* mismatch) {
  const unsigned amax_bits = blockIdx.x + 1;  // 0x0001 .. 0x7F7F
  const float s = scale_from_amax_bits(amax_bits);
  const float y = __frcp_rn(s);
  const float amax = __uint_as_float(amax_bits << 16);
  unsigned long long bad = 0;
  for (unsigned m = threadIdx.x; m <= amax_bits; m += blockDim.x) {
    const float xp = __uint_as_float(m << 16);
    if (!(xp <= amax)) continue;
    const uint16_t want = e4m3x2_rn_satfinite(__fdiv_rn(xp, s), __fdiv_rn(-xp, s));
    const bool fast = amax_bits >= kFastDivMinBits;
    const uint16_t got =
        e4m3x2_rn_satfinite(div_by_scale(xp, s, y, fast), div_by_scale(-xp, s, y, fast));
    bad += want != got;
  }
  if (bad) atomicAdd(mismatch, bad);
}

}  // namespace bca
