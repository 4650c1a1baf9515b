// qkv_proj_kernel.cuh -- projection of the target rows into Q, K and V with the
// Q/K RMS norm and the rotary embedding in the epilogue, for sm_100a.
//
// What it computes.  "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll"
// (orcarouter.ai), section "Siffrorna, och vad de inte säger", puts a Q/K-norm change
// between the projection of the rows and the attention; the pages give no formula,
// so the plain reading is used (the same as bca_qk_norm_rope's):
//   y[t, n]    = sum_c x[t, c] w[n, c]           x [T, D] bf16, w [3*H*128, D] bf16
//                                                (torch Linear layout: Q heads, K
//                                                heads, V heads; no bias)
//   q[t, h, :] = rope(rms_norm(y[t, 128h .. 128h+127], gamma_q), cos[t], sin[t])
//   k[t, h, :] = rope(rms_norm(y[t, 128(H+h) ..], gamma_k), cos[t], sin[t])
//   v[t, h, :] = y[t, 128(2H+h) ..]
// with rms_norm(z, g)_c = z_c / sqrt(mean(z^2) + eps) * g_c and rope turning pair
// (2i, 2i+1) by the angle whose cos/sin the caller gives per (row, pair).  fp32
// accumulation (tensor cores), fp32 epilogue, one round-to-nearest-even to bf16.
// Q, K and V land in the [T, H, 128] layout bca_step_attend reads.
//
// Design (B200).  A dense contraction: tcgen05.mma kind::f16, M = 128 rows, N = 256
// output features (two heads), K = 16 per instruction, fp32 accumulators in TMEM
// (two 256-column buffers, so one tile's epilogue overlaps the next tile's
// mainloop).  Persistent CTAs walk the tiles feature-block-major (CTAs working at
// the same time share a block of w).  Roles:
//  * warp 0: TMA producer, a 4-stage ring of (x 128 x 64, w 256 x 64) bf16 tiles,
//    128-byte swizzle;
//  * warp 1: MMA issuer (one elected lane), 4 MMAs per k-step;
//  * warps 2..5: epilogue, one TMEM lane (one row) per thread.  For a Q or K head the
//    thread sums the squares of its 128 values (first TMEM pass), then scales,
//    weights and turns each pair (second pass); the bf16 row goes to a 128-byte-
//    swizzled staging box and one TMA store writes 128 rows x 64 features.
// Every mbarrier wait is bounded; on expiry the CTA reports BCA_ERR_DEVICE_TIMEOUT,
// drains and frees TMEM.
#pragma once
#include <cuda_bf16.h>

#include "../../include/bca.h"
#include "ptx.cuh"

namespace bca {

constexpr int kPBM = 128;
constexpr int kPBN = 256;
constexpr int kPBK = 64;
constexpr int kPStages = 4;
constexpr int kPThreads = 192;
constexpr int kPATile = kPBM * kPBK * 2;  // 16 KiB
constexpr int kPBTile = kPBN * kPBK * 2;  // 32 KiB
constexpr int kPStageBytes = kPATile + kPBTile;

struct ProjSmem {
  static constexpr int kStage = kPStages * kPStageBytes;  // output staging: two 64-feature boxes
  static constexpr int kGamma = kStage + 2 * 128 * 128;   // gamma_q | gamma_k, 256 fp32
  static constexpr int kBars = kGamma + 2 * 128 * 4;
  static constexpr int bFull = 0;      // kPStages
  static constexpr int bEmpty = 4;     // kPStages
  static constexpr int bAccFull = 8;   // 2
  static constexpr int bAccEmpty = 10; // 2 (128 epilogue arrivals)
  static constexpr int bDone = 12;
  static constexpr int bStgFull = 13;  // a head's rows are in the staging boxes (128 arrivals)
  static constexpr int bStgFree = 14;  // their TMA store has read them (1 arrival)
  static constexpr int kNumBars = 15;
  static constexpr int kTmemSlot = kBars + 8 * kNumBars;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kDynamicBytes = kBytes + 1024;
};
static_assert(kPStages == 4, "barrier table assumes 4 stages");

struct ProjParams {
  CUtensorMap tm_x;       // x [T, D]: dims (D, T), box (64, 128)
  CUtensorMap tm_w;       // w [N, D]: dims (D, N), box (64, 256)
  CUtensorMap tm_out[3];  // q, k, v [T, H, 128]: dims (128, H, T), box (64, 1, 128)
  const float* gamma_q;
  const float* gamma_k;
  const float* cos_t;  // [T, 64]
  const float* sin_t;
  int32_t rows;
  int32_t heads;
  int32_t m_tiles;
  int32_t n_tiles;
  int32_t k_steps;
  float eps;
  int32_t* dev_status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void proj_abort(volatile int* abort, int32_t* dev_status) {
  *abort = 1;
  if (dev_status) atomicExch(dev_status, static_cast<int32_t>(BCA_ERR_DEVICE_TIMEOUT));
}

__global__ void __launch_bounds__(kPThreads, 1)
    qkv_proj_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + ProjSmem::kBars;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  volatile int* abort = reinterpret_cast<volatile int*>(smem + ProjSmem::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + ProjSmem::kTmemSlot);
  float* s_gamma = reinterpret_cast<float*>(smem + ProjSmem::kGamma);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles_all = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(bar(ProjSmem::bFull + i), 1);
      mbar_init(bar(ProjSmem::bEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ProjSmem::bAccFull + i), 1);
      mbar_init(bar(ProjSmem::bAccEmpty + i), 128);
    }
    mbar_init(bar(ProjSmem::bDone), 1);
    mbar_init(bar(ProjSmem::bStgFull), 128);
    mbar_init(bar(ProjSmem::bStgFree), 1);
    *abort = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 256; i += kPThreads)
    s_gamma[i] = i < 128 ? __ldg(p.gamma_q + i) : __ldg(p.gamma_k + i - 128);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_all && ok; tile += gridDim.x) {
        const int n = tile / p.m_tiles, m = tile % p.m_tiles;
        for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
          const int st = it % kPStages;
          if (!mbar_wait_bounded(bar(ProjSmem::bEmpty + st),
                                 (static_cast<uint32_t>(it / kPStages) & 1u) ^ 1u, abort,
                                 p.timeout_ns)) {
            proj_abort(abort, p.dev_status);
            ok = false;
            break;
          }
          const uint32_t a = sbase + st * kPStageBytes;
          mbar_arrive_expect_tx(bar(ProjSmem::bFull + st), kPStageBytes);
          tma_load_2d(a, &p.tm_x, bar(ProjSmem::bFull + st), ks * kPBK, m * kPBM);
          tma_load_2d(a + kPATile, &p.tm_w, bar(ProjSmem::bFull + st), ks * kPBK, n * kPBN);
        }
      }
      if (!ok) {
        // Drain: the copies this thread may still have in flight (bounded waits).
        constexpr unsigned long long kDrainNs = 20000000ull;
        for (int i = it > kPStages ? it - kPStages : 0; i < it; ++i)
          mbar_wait_bounded(bar(ProjSmem::bFull + i % kPStages),
                            static_cast<uint32_t>(i / kPStages) & 1u, nullptr, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t kIdesc = idesc_bf16_f32(kPBM, kPBN, false);
    bool ok = true;
    auto wait = [&](int b, uint32_t parity) {
      if (ok) {
        const bool got = mbar_wait_bounded(bar(b), parity, abort, p.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (elect_one()) proj_abort(abort, p.dev_status);
          ok = false;
        }
      }
      return ok;
    };
    int it = 0, lt = 0;
    for (int tile = blockIdx.x; tile < n_tiles_all && ok; tile += gridDim.x, ++lt) {
      const int a = lt & 1;
      if (!wait(ProjSmem::bAccEmpty + a, (static_cast<uint32_t>(lt >> 1) & 1u) ^ 1u)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(a * kPBN);
      for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
        const int st = it % kPStages;
        if (!wait(ProjSmem::bFull + st, static_cast<uint32_t>(it / kPStages) & 1u)) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sa = sbase + st * kPStageBytes;
          const uint64_t da = sdesc_sw128(sa, 16, 1024);
          const uint64_t db = sdesc_sw128(sa + kPATile, 16, 1024);
#pragma unroll
          for (int s = 0; s < kPBK / 16; ++s)  // 32 bytes of each row per K = 16 step
            mma_bf16_ss(d_tmem, da + ((s * 32) >> 4), db + ((s * 32) >> 4), kIdesc,
                        (ks > 0 || s > 0) ? 1u : 0u);
          mma_commit(bar(ProjSmem::bEmpty + st));
          if (ks == p.k_steps - 1) mma_commit(bar(ProjSmem::bAccFull + a));
        }
        __syncwarp();
      }
    }
    // Everything issued is complete before TMEM is released.
    if (elect_one()) mma_commit(bar(ProjSmem::bDone));
    __syncwarp();
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(ProjSmem::bDone), 0, nullptr,
                                                    p.timeout_ns))) {
      if (elect_one()) proj_abort(abort, p.dev_status);
      mbar_wait_bounded(bar(ProjSmem::bDone), 0, nullptr, p.timeout_ns);
    }
  } else {
    // ---------------- epilogue: warps 2..5, thread = TMEM lane = tile row ----------------
    const int q4 = warp % 4;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t stage = sbase + ProjSmem::kStage;
    const int feats = 3 * p.heads * 128;
    int lt = 0, ns = 0;  // tiles, heads stored (staging barrier phases)
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_all && ok; tile += gridDim.x, ++lt) {
      const int n = tile / p.m_tiles, m = tile % p.m_tiles;
      const int a = lt & 1;
      const bool got = mbar_wait_bounded(bar(ProjSmem::bAccFull + a),
                                         static_cast<uint32_t>(lt >> 1) & 1u, abort,
                                         p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        proj_abort(abort, p.dev_status);
        break;
      }
      tc_fence_after();
      const int grow = m * kPBM + row;
      const bool in_rows = grow < p.rows;
#pragma unroll 1
      for (int hh = 0; hh < kPBN / 128 && ok; ++hh, ++ns) {
        const int col0 = n * kPBN + hh * 128;
        if (col0 >= feats) break;  // uniform over the CTA
        const int which = col0 / (p.heads * 128);  // 0 q, 1 k, 2 v
        const int head = (col0 - which * p.heads * 128) / 128;
        const uint32_t tacc = tmem + lane_off + static_cast<uint32_t>(a * kPBN + hh * 128);
        float inv = 1.0f;
        if (which < 2) {
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tacc + 32 * c, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
          }
          inv = rsqrtf(ss * (1.0f / 128.0f) + p.eps);
        }
        const float* g = s_gamma + (which == 1 ? 128 : 0);
        // The previous head's TMA store must have read the staging boxes.
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(bar(ProjSmem::bStgFree),
                                          (static_cast<uint32_t>(ns) & 1u) ^ 1u, abort,
                                          p.timeout_ns))) {
          proj_abort(abort, p.dev_status);
          ok = false;
          break;
        }
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tacc + 32 * c, r);
          tmem_wait_ld();
          uint32_t pk[16];
          if (which < 2) {
            float cs[16], sn[16];
            if (in_rows) {
              const float4* pc = reinterpret_cast<const float4*>(p.cos_t + static_cast<size_t>(grow) * 64) + 4 * c;
              const float4* ps = reinterpret_cast<const float4*>(p.sin_t + static_cast<size_t>(grow) * 64) + 4 * c;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 u = __ldg(pc + j), w4 = __ldg(ps + j);
                cs[4 * j] = u.x; cs[4 * j + 1] = u.y; cs[4 * j + 2] = u.z; cs[4 * j + 3] = u.w;
                sn[4 * j] = w4.x; sn[4 * j + 1] = w4.y; sn[4 * j + 2] = w4.z; sn[4 * j + 3] = w4.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) cs[j] = sn[j] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x0 = __uint_as_float(r[2 * e]) * inv * g[32 * c + 2 * e];
              const float x1 = __uint_as_float(r[2 * e + 1]) * inv * g[32 * c + 2 * e + 1];
              pk[e] = pack_bf16x2(x0 * cs[e] - x1 * sn[e], x0 * sn[e] + x1 * cs[e]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
          }
          // features 32c..32c+31: box c/2, 16-byte chunks 4(c%2)..4(c%2)+3 of the row
          const uint32_t box = stage + (c >> 1) * (128 * 128) + row * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int q = 4 * (c & 1) + j;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             box + ((q ^ (row & 7)) << 4)),
                         "r"(pk[4 * j]), "r"(pk[4 * j + 1]), "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(ProjSmem::bStgFull));
        if (row == 0) {
          if (!mbar_wait_bounded(bar(ProjSmem::bStgFull), static_cast<uint32_t>(ns) & 1u, abort,
                                 p.timeout_ns)) {
            proj_abort(abort, p.dev_status);
          } else {
            tma_store_3d(&p.tm_out[which], stage, 0, head, m * kPBM);
            tma_store_3d(&p.tm_out[which], stage + 128 * 128, 64, head, m * kPBM);
            bulk_commit();
            bulk_wait_read();  // the staging boxes may be written again
          }
          mbar_arrive(bar(ProjSmem::bStgFree));
        }
      }
      // This accumulator buffer has been read: the MMA may reuse it.
      tc_fence_before();
      mbar_arrive(bar(ProjSmem::bAccEmpty + a));
    }
    if (row == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bca
