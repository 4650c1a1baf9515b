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
// HBM-bound: 16-byte vector loads, coalesced along [t, h, c]; the absmax pass is a
// separate read so that the encode pass sees the final scale.  The running absmax
// is kept as bf16 magnitude bits (|x| bit patterns of finite bf16 values order like
// the values) in the slot's own scale array, which the last pass overwrites with
// s_h -- no scratch memory.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace bca {

struct KvStoreParams {
  const uint16_t* src[2];  // K, V (bf16 bits), token t head h at t*row_stride + h*128
  void* dst[2];            // [H, cap, 128] bf16 or e4m3
  float* scale[2];         // [H] (e4m3 tensors only)
  int32_t quant[2];        // 1: e4m3, 0: bf16 copy
  int64_t row_stride;      // elements
  int32_t n_prefix;
  int32_t heads;
  int32_t cap;
};

constexpr int kStoreThreads = 256;

// Zero the running absmax of every e4m3 tensor.
__global__ void kv_amax_init_kernel(KvStoreParams p) {
  const int t = blockIdx.y;
  if (!(t ? p.quant[1] : p.quant[0])) return;
  unsigned* a = reinterpret_cast<unsigned*>(t ? p.scale[1] : p.scale[0]);
  for (int h = threadIdx.x; h < p.heads; h += blockDim.x) a[h] = 0u;
}

__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t m, uint32_t w) {
  return max(m, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
}

// Pass 1: per-head absmax.  blockIdx.y = tensor; a block covers a token range and
// every (head, 16-byte chunk) pair; 16 lanes share a head.
__global__ void __launch_bounds__(kStoreThreads) kv_amax_kernel(KvStoreParams p, int tokens_per_block) {
  const int tsel = blockIdx.y;
  if (!(tsel ? p.quant[1] : p.quant[0])) return;
  const uint16_t* src = tsel ? p.src[1] : p.src[0];
  unsigned* amax = reinterpret_cast<unsigned*>(tsel ? p.scale[1] : p.scale[0]);
  const int t0 = blockIdx.x * tokens_per_block;
  const int t1 = min(p.n_prefix, t0 + tokens_per_block);
  const int pairs = p.heads * 16;
  for (int base = 0; base < pairs; base += blockDim.x) {
    const int pr = base + threadIdx.x;
    const int h = pr >> 4, c = pr & 15;
    uint32_t m = 0;
    if (pr < pairs) {
      const uint16_t* s = src + static_cast<int64_t>(h) * 128 + c * 8;
      for (int t = t0; t < t1; ++t) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(s + static_cast<int64_t>(t) * p.row_stride));
        m = max_abs_bf16x2(m, v.x);
        m = max_abs_bf16x2(m, v.y);
        m = max_abs_bf16x2(m, v.z);
        m = max_abs_bf16x2(m, v.w);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (pr < pairs && c == 0 && t1 > t0)
      atomicMax(amax + h, m);
  }
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

// Pass 2: copy (bf16) or encode (e4m3).  One thread per 16-byte source chunk
// (8 elements); grid-stride over [t, h, chunk].
__global__ void __launch_bounds__(kStoreThreads) kv_write_kernel(KvStoreParams p) {
  const int tsel = blockIdx.y;
  const uint16_t* src = tsel ? p.src[1] : p.src[0];
  void* dst = tsel ? p.dst[1] : p.dst[0];
  const int64_t total = static_cast<int64_t>(p.n_prefix) * p.heads * 16;
  const bool quant = (tsel ? p.quant[1] : p.quant[0]) != 0;
  const unsigned* amax_bits = reinterpret_cast<const unsigned*>(tsel ? p.scale[1] : p.scale[0]);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i & 15);
    int h;
    int64_t t;
    if (total < (int64_t{1} << 31)) {  // 32-bit index arithmetic when it fits
      const uint32_t th = static_cast<uint32_t>(i) >> 4;
      t = th / static_cast<uint32_t>(p.heads);
      h = static_cast<int>(th - static_cast<uint32_t>(t) * static_cast<uint32_t>(p.heads));
    } else {
      const int64_t th = i >> 4;
      h = static_cast<int>(th % p.heads);
      t = th / p.heads;
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + t * p.row_stride + h * 128 + c * 8));
    const int64_t drow = static_cast<int64_t>(h) * p.cap + t;
    if (!quant) {
      reinterpret_cast<uint4*>(static_cast<uint16_t*>(dst) + drow * 128)[c] = v;
    } else {
      const unsigned ab = amax_bits[h];
      const float s = scale_from_amax_bits(ab);
      const float y = __frcp_rn(s);
      const bool fast = ab >= kFastDivMinBits;
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
      reinterpret_cast<uint2*>(static_cast<uint8_t*>(dst) + drow * 128)[c] =
          make_uint2(out[0], out[1]);
    }
  }
}

// Pass 3: running absmax bits -> final fp32 scale.
__global__ void kv_scale_finalize_kernel(KvStoreParams p) {
  const int t = blockIdx.y;
  if (!(t ? p.quant[1] : p.quant[0])) return;
  float* sc = t ? p.scale[1] : p.scale[0];
  for (int h = threadIdx.x; h < p.heads; h += blockDim.x)
    sc[h] = scale_from_amax_bits(__float_as_uint(sc[h]));
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
