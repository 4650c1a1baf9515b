// qk_norm_rope_kernel.cuh -- Q/K RMS normalisation + rotary position embedding of
// the rows that enter the attention, in one pass over each tensor.
//
// What it computes.  "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll" (section
// "Siffrorna, och vad de inte säger") names a Q/K-norm change among the steps
// around the DiT's attention; the pages give no formula, so the plain reading is
// used: for every row t and head h of x in {Q, K} ([rows, H, 128] bf16),
//   r        = 1 / sqrt(mean_c x[t,h,c]^2 + eps)
//   y_c      = x[t,h,c] * r * gamma_x[c]                      (gamma shared by the heads)
//   out_{2i}   = y_{2i} cos[t,i] - y_{2i+1} sin[t,i]            (pair i = channels 2i, 2i+1
//   out_{2i+1} = y_{2i} sin[t,i] + y_{2i+1} cos[t,i]             turned by angle theta[t,i])
// with the caller's cos/sin tables [rows, 64] (any 1-D or multi-axis position
// scheme), fp32 arithmetic and one round-to-nearest-even to bf16 at the end.
//
// HBM-bound.  One warp per (tensor, row): the row's cos/sin (shared by its heads)
// and the weights are loaded once; the two half-warps take alternate heads, 16
// lanes per 256-byte head vector (16 bytes = 8 channels = 4 pairs each), and every
// lane issues kNormHeadsInFlight vectors' loads before it reduces (a 16-lane
// shuffle sum of squares per vector) and stores.  Warps take consecutive
// rows, so the loads of a warp cover whole 256-byte rows of the [rows, H, 128]
// tensor.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace bca {

struct QkNormRopeParams {
  uint16_t* x[2];          // Q, K (bf16 bits, in place); a NULL tensor is skipped
  const float* gamma[2];   // [128] each
  const float* cos_t;      // [rows, 64]
  const float* sin_t;      // [rows, 64]
  int64_t rows;
  int32_t heads;
  float eps;
};

constexpr int kNormThreads = 256;
constexpr int kNormWarpsPerBlock = kNormThreads / 32;
// Head vectors each half-warp loads before it reduces (2 per warp per slot).
// Measured on B200, GB/s as a fraction of the HBM copy bandwidth, at 4096 / 32768
// rows x 32 heads: 2 -> 0.76 / 0.93, 4 -> 0.68 / 0.87, 8 -> 0.59 / 0.75 (more
// registers, fewer resident warps); a cp.async ring of 2-6 chunks per warp in
// shared memory measured 0.63-0.77 / 0.72-0.86.
constexpr int kNormHeadsInFlight = 2;

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t to_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void __launch_bounds__(kNormThreads) qk_norm_rope_kernel(QkNormRopeParams p) {
  const int lane16 = threadIdx.x & 15;
  const int half = (threadIdx.x >> 4) & 1;
  const int64_t n_items = 2 * p.rows;  // (tensor, row): all Q rows, then all K rows
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kNormWarpsPerBlock;
  // Every loop bound below is uniform across the warp, so all 32 lanes reach every
  // shuffle; lanes without a vector this round only skip their loads and stores.
  for (int64_t item = warp_id; item < n_items; item += n_warps) {
    const int t = item >= p.rows ? 1 : 0;
    const int64_t row = item - t * p.rows;
    uint16_t* x = t ? p.x[1] : p.x[0];
    if (x == nullptr) continue;  // warp-uniform
    const float4 c = __ldg(reinterpret_cast<const float4*>(p.cos_t + row * 64) + lane16);
    const float4 s = __ldg(reinterpret_cast<const float4*>(p.sin_t + row * 64) + lane16);
    const float4* g = reinterpret_cast<const float4*>(t ? p.gamma[1] : p.gamma[0]) + 2 * lane16;
    const float4 g0 = __ldg(g), g1 = __ldg(g + 1);
    uint4* xrow = reinterpret_cast<uint4*>(x + row * p.heads * 128);
    for (int h0 = 0; h0 < p.heads; h0 += 2 * kNormHeadsInFlight) {
      uint4 w[kNormHeadsInFlight];
#pragma unroll
      for (int j = 0; j < kNormHeadsInFlight; ++j) {
        const int h = h0 + 2 * j + half;
        w[j] = h < p.heads ? xrow[h * 16 + lane16] : make_uint4(0u, 0u, 0u, 0u);
      }
      float r[kNormHeadsInFlight];
#pragma unroll
      for (int j = 0; j < kNormHeadsInFlight; ++j) {
        float ss = 0.f;
        for (uint32_t word : {w[j].x, w[j].y, w[j].z, w[j].w}) {
          const float a = lo_bf16(word), b = hi_bf16(word);
          ss = fmaf(a, a, fmaf(b, b, ss));
        }
        r[j] = ss;
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1)  // within each 16-lane half
#pragma unroll
        for (int j = 0; j < kNormHeadsInFlight; ++j) r[j] += __shfl_xor_sync(0xffffffffu, r[j], o);
#pragma unroll
      for (int j = 0; j < kNormHeadsInFlight; ++j) {
        const int h = h0 + 2 * j + half;
        if (h >= p.heads) continue;
        const float inv = rsqrtf(r[j] * (1.0f / 128.0f) + p.eps);
        // pair (2i, 2i+1): normalise, weight, rotate, round
        auto pair = [&](uint32_t word, float ga, float gb, float cs, float sn) {
          const float a = lo_bf16(word) * inv * ga;
          const float b = hi_bf16(word) * inv * gb;
          return to_bf16x2(a * cs - b * sn, a * sn + b * cs);
        };
        xrow[h * 16 + lane16] =
            make_uint4(pair(w[j].x, g0.x, g0.y, c.x, s.x), pair(w[j].y, g0.z, g0.w, c.y, s.y),
                       pair(w[j].z, g1.x, g1.y, c.z, s.z), pair(w[j].w, g1.z, g1.w, c.w, s.w));
      }
    }
  }
}

}  // namespace bca
