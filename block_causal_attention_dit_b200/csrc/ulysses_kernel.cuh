// ulysses_kernel.cuh -- re-sharding copies around the all-to-all of head-sharded
// (Ulysses) sequence parallelism.
//
// "Qwen/Qwen-Image-2.1" (recipes.vllm.ai), "Overview" and "Limitations": the
// engine's sequence parallelism is Ulysses; "SGLang-Diffusion stöder Qwen-Image-2.1
// på dag noll", "Hur en driftsättning faktiskt ser ut": Ulysses attention is among
// the verified multi-GPU modes.  With N ranks each holding rows_local rows of all
// H heads, one all-to-all gives every rank all rows of H/N heads, attention runs per
// head locally, and a second all-to-all returns O to the row shards.
//
// pack   : x[t, g*Hn + j, :]  -> send[g, t, j, :]   (block g goes to rank g)
// unpack : recv[g, t, j, :]   -> x[t, g*Hn + j, :]  (block g came from rank g)
// with Hn = H / N.  After the first all-to-all, rank r's receive buffer
// [N][rows_local][Hn][d] is already the [N*rows_local, Hn, d] row-major layout the
// attention calls take, so only the send side of Q/K/V and the receive side of O
// need a copy.  HBM-bound: one 16-byte chunk per thread, reads coalesced along x,
// writes in contiguous runs of Hn*256 bytes.
#pragma once
#include <cstdint>

namespace bca {

constexpr int kUlyssesThreads = 256;

template <bool kPack>
__global__ void __launch_bounds__(kUlyssesThreads)
    ulysses_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t rows,
                        int32_t heads, int32_t n_ranks) {
  const int32_t hn = heads / n_ranks;
  const int64_t n = rows * heads * 16;  // 16-byte chunks of x (head_dim 128, bf16)
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kUlyssesThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kUlyssesThreads) {
    const int32_t c = static_cast<int32_t>(i & 15);
    const int64_t th = i >> 4;  // t * heads + h
    const int64_t t = th / heads;
    const int32_t h = static_cast<int32_t>(th - t * heads);
    const int32_t g = h / hn, j = h - g * hn;
    const int64_t s = ((static_cast<int64_t>(g) * rows + t) * hn + j) * 16 + c;  // sharded index
    if (kPack)
      dst[s] = src[i];
    else
      dst[i] = src[s];
  }
}

}  // namespace bca
