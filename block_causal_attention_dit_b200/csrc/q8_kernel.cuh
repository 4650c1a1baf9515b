// q8_kernel.cuh -- e4m3 quantisation of the target rows' Q for the e4m3-Q cached
// step (bca_step_attend_q8).
//
// What it computes: each request's Q rows are quantised per head exactly like a
// prefix K/V tensor of an "fp8" cache slot ("Qwen/Qwen-Image-2.1" vLLM recipe,
// "Prefix KV cache"; OFP8 E4M3):
//   amax_{r,h} = max_{t < T_r, c} |q[q_start_r + t, h, c]|
//   s_{r,h}    = fp32(amax_{r,h}) / 448 (correctly rounded; 1 if amax is 0)
//   codes[h, q_start_r + t, c] = e4m3_rn_satfinite(q / s_{r,h})   (t < T_r)
// The codes are laid out [H, rows, 128] (one 128-byte row per (head, row), the
// layout the attention kernel's Q8 tiles load from); scales [n_req][H] by the
// caller's request index.  The encoder is the cache's (kv_store_kernel.cuh).
// HBM-bound: an absmax pass over Q, then an encode pass; three launches per call
// whatever the number of requests.
#pragma once
#include <cstdint>

#include "../../include/bca.h"
#include "kv_store_kernel.cuh"

namespace bca {

struct Q8Params {
  const uint16_t* q;  // [rows, H, 128] bf16 bits (packed target rows)
  uint8_t* codes;     // [H, rows, 128]
  float* scale;       // [n_req][H]
  unsigned* amax;     // [n_req][H] scratch: running absmax as bf16 magnitude bits
  int32_t rows;
  int32_t heads;
  int32_t n_req;
  int32_t q_start[BCA_MAX_BATCH];
  int32_t q_len[BCA_MAX_BATCH];
};

constexpr int kQ8Threads = 256;
constexpr int kQ8RowsPerBlock = 32;  // absmax pass

__global__ void q8_amax_init_kernel(Q8Params p) {
  const int n = p.n_req * p.heads;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    p.amax[i] = 0u;
}

// Pass 1: blockIdx.y = request, blockIdx.x = a range of kQ8RowsPerBlock of its rows;
// 16 lanes share a head (one 16-byte chunk each), as in the cache's absmax pass.
__global__ void __launch_bounds__(kQ8Threads) q8_amax_kernel(Q8Params p) {
  const int r = blockIdx.y;
  const int t0 = blockIdx.x * kQ8RowsPerBlock;
  const int t1 = min(p.q_len[r], t0 + kQ8RowsPerBlock);
  if (t0 >= t1) return;
  const int64_t row_elems = static_cast<int64_t>(p.heads) * 128;
  const uint16_t* src = p.q + static_cast<int64_t>(p.q_start[r]) * row_elems;
  const int pairs = p.heads * 16;
  for (int base = 0; base < pairs; base += blockDim.x) {
    const int pr = base + threadIdx.x;
    const int h = pr >> 4, c = pr & 15;
    uint32_t m = 0;
    if (pr < pairs) {
      const uint16_t* s = src + h * 128 + c * 8;
      for (int t = t0; t < t1; ++t) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(s + t * row_elems));
        m = max_abs_bf16x2(m, v.x);
        m = max_abs_bf16x2(m, v.y);
        m = max_abs_bf16x2(m, v.z);
        m = max_abs_bf16x2(m, v.w);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (pr < pairs && c == 0) atomicMax(p.amax + r * p.heads + h, m);
  }
}

// Pass 2: blockIdx.y = request; grid-stride over its (row, head, 16-byte chunk)
// triples.  Block 0 of each request also writes the request's fp32 scales.
__global__ void __launch_bounds__(kQ8Threads) q8_encode_kernel(Q8Params p) {
  const int r = blockIdx.y;
  const unsigned* amax = p.amax + r * p.heads;
  if (blockIdx.x == 0)
    for (int h = threadIdx.x; h < p.heads; h += blockDim.x)
      p.scale[r * p.heads + h] = scale_from_amax_bits(amax[h]);
  const int64_t total = static_cast<int64_t>(p.q_len[r]) * p.heads * 16;
  const int64_t row0 = p.q_start[r];
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i & 15);
    const int64_t th = i >> 4;
    const int64_t t = th / p.heads;
    const int h = static_cast<int>(th - t * p.heads);
    const int64_t row = row0 + t;
    const uint4 v =
        __ldg(reinterpret_cast<const uint4*>(p.q + (row * p.heads + h) * 128 + c * 8));
    const unsigned ab = amax[h];
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
    reinterpret_cast<uint2*>(p.codes + (static_cast<int64_t>(h) * p.rows + row) * 128)[c] =
        make_uint2(out[0], out[1]);
  }
}

}  // namespace bca
