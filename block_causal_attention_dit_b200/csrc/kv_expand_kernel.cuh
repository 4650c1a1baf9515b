// kv_expand_kernel.cuh -- e4m3 prefix cache tensors expanded once per cached step
// into a bf16 scratch, for bca_step_attend_dq.
//
// What it computes: for every e4m3 cache tensor of the call (K and/or V of each
// request's slot, "Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV cache"),
//   out[h, t, c] = decode(code[h, t, c])        t < n_tokens   (exact in bf16)
// The per-head scale is not applied here: the attention folds it in exactly as it
// does for e4m3 tiles it converts itself (K's into the score scale, V's into P).
// Every e4m3 value (3 mantissa bits, exponents 2^-9 .. 2^8) is exact in bf16.
//
// HBM-bound: each thread reads 16 codes (16 bytes) and writes 32 bytes; the code ->
// bf16 table (256 entries) sits in shared memory, filled by the block from the
// exact e4m3 -> f16 -> f32 -> bf16 conversions.
#pragma once
#include <cstdint>

namespace bca {

struct ExpandTensor {
  const uint8_t* src;  // [heads, cap, 128] e4m3; rows [0, rows) of every head are read
  uint16_t* dst;       // [heads, rows, 128] bf16
  int64_t cap;
  int32_t rows;
  int32_t heads;
};

constexpr int kMaxExpandTensors = 128;
constexpr int kExpandThreads = 256;

struct ExpandParams {
  ExpandTensor t[kMaxExpandTensors];
  int32_t n_tensors;
};

__device__ __forceinline__ uint16_t e4m3_to_bf16_bits(uint32_t code) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(code & 0xFFu)));
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(static_cast<uint16_t>(h & 0xFFFFu)));
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);  // exact: 3 mantissa bits
}

// blockIdx.y = tensor; the blocks of x stride over its (head, row, 16-byte chunk) triples.
__global__ void __launch_bounds__(kExpandThreads) kv_expand_kernel(const __grid_constant__ ExpandParams p) {
  __shared__ uint16_t lut[256];
  lut[threadIdx.x] = e4m3_to_bf16_bits(threadIdx.x);
  __syncthreads();
  const ExpandTensor& T = p.t[blockIdx.y];
  // 16-byte chunks per head and in all (rows <= 2^20, heads <= 256: 32 bits suffice)
  const uint32_t per_head = static_cast<uint32_t>(T.rows) * 8u;
  const uint32_t total = per_head * static_cast<uint32_t>(T.heads);
  for (uint32_t i = blockIdx.x * kExpandThreads + threadIdx.x; i < total;
       i += gridDim.x * kExpandThreads) {
    const uint32_t h = i / per_head, r = i - h * per_head;  // r: chunk within the head's rows
    const uint4 v =
        __ldcs(reinterpret_cast<const uint4*>(T.src + static_cast<int64_t>(h) * T.cap * 128) + r);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = lut[w[j] & 0xFFu] | (static_cast<uint32_t>(lut[(w[j] >> 8) & 0xFFu]) << 16);
      o[2 * j + 1] = lut[(w[j] >> 16) & 0xFFu] | (static_cast<uint32_t>(lut[w[j] >> 24]) << 16);
    }
    uint4* d = reinterpret_cast<uint4*>(T.dst + static_cast<int64_t>(h) * T.rows * 128) + 2 * r;
    __stcs(d, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(d + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

}  // namespace bca
