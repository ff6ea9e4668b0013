// Decode-shaped W1.58A8 product (M <= 8 tokens) on CUDA cores.
//
// The ternary product is "the sum of the inputs with weight +1 minus the sum
// of those with weight -1" (Habr repost on juhe.plus, section "Когда - три
// лучше двух"); here each group of four weights is expanded to four bytes
// and combined with four int8 activations by one dp4a, which is that
// add/subtract exactly, in integers.  With the per-token sum of x_q at hand
// the bytes hold the unsigned codes c = q + 1 in {0, 1, 2} and the row sum
// is subtracted once per output (sum c*x - sum x = sum q*x), which saves two
// instructions per four weights.
//
// Work split: CTA c owns the contiguous rows [N*c/G, N*(c+1)/G) (G = grid,
// one CTA per SM); its warps take groups of 4 consecutive rows round-robin.
// A group is streamed in items of up to 4096 weights per row (4 KB): lane 0
// of the warp issues the bulk asynchronous copies of an item into a 2-slot
// ring of shared memory owned by that warp.  The activations x_q (M*K bytes)
// are copied into shared memory once per CTA when they fit.  Lane l handles
// 16 consecutive weights of each of the 4 rows per 512-weight step, so the
// warp's loads of codes (4 bytes per lane) and of activations (16 bytes per
// lane) are contiguous and free of bank conflicts, and each activation load
// serves 4 rows.  Lane partial sums are reduced with warp shuffles.
//
// The first weight items are requested before waiting on the previous
// kernel (programmatic dependent launch), because the weights never depend
// on it; under 100 KB of shared memory per CTA lets the next kernel's CTA sit
// on the same SM and do the same.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 4;                                 // rows per group
constexpr int kGemvSlots = 2;                                // ring depth per warp
constexpr int kGemvSlotBytes = 4096;                         // one item: 4 rows x 1 KB
constexpr int kGemvKChunk = kGemvSlotBytes * 4 / kGemvRows;  // 4096 weights per row per item
constexpr int kGemvRingBytes = kGemvWarps * kGemvSlots * kGemvSlotBytes;
constexpr int kGemvXMaxBytes = 21504;  // x_q is staged in shared memory when M*K fits
constexpr int kGemvBarBytes = 256;

__host__ __device__ constexpr int gemv_smem_bytes(bool xs) {
  return kGemvRingBytes + kGemvBarBytes + (xs ? kGemvXMaxBytes : 0);
}

// FUSED: the kernel takes the unquantised activations x (M x K of type T)
// and the optional RMSNorm gain instead of x_q / a_scale / rowsum, and
// quantises every token row itself, with all 256 threads, straight into its
// shared-memory copy of x_q (quant_row_cta: the same arithmetic and order as
// the standalone quantisation kernel).  Every CTA repeats this small step
// (M*K <= 21504 values, read from L2), which removes a dependent kernel
// launch and the x_q round trip through global memory from each decode
// linear.
template <int MT, bool U8, bool XS, bool FUSED = false, typename T = float, int MAXC = 1>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const uint8_t* __restrict__ Wp,
                                                               const float* __restrict__ gamma_ptr, int N, int K,
                                                               const int8_t* __restrict__ xq,
                                                               const float* __restrict__ a_scale,
                                                               const int32_t* __restrict__ rowsum,
                                                               const T* __restrict__ xin, const T* __restrict__ gain,
                                                               float rms_eps, void* __restrict__ y, int y_dtype) {
  static_assert(!FUSED || (XS && U8), "the fused kernel keeps x_q in shared memory and uses its row sums");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = smem + warp * kGemvSlots * kGemvSlotBytes;
  uint64_t* all_bars = reinterpret_cast<uint64_t*>(smem + kGemvRingBytes);
  uint64_t* bars = all_bars + warp * kGemvSlots;
  uint64_t* xbar = all_bars + kGemvWarps * kGemvSlots;
  uint8_t* xs = smem + kGemvRingBytes + kGemvBarBytes;

  const int64_t row_lo = static_cast<int64_t>(N) * blockIdx.x / gridDim.x;
  const int64_t row_hi = static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x;
  const int ngroups = static_cast<int>((row_hi - row_lo + kGemvRows - 1) / kGemvRows);
  const int my_groups = ngroups > warp ? (ngroups - warp + kGemvWarps - 1) / kGemvWarps : 0;
  const int kchunk = K < kGemvKChunk ? K : kGemvKChunk;
  const int nkc = (K + kchunk - 1) / kchunk;
  const int items = my_groups * nkc;
  const int64_t row_bytes = K >> 2;
  const int slot_row = kchunk >> 2;  // bytes per row inside a slot

  if (lane == 0) {
    for (int s = 0; s < kGemvSlots; ++s) mbar_init(&bars[s], 1);
    if (warp == 0) mbar_init(xbar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  const uint64_t policy = policy_evict_first();
  // Issue item j into ring slot j % kGemvSlots (lane 0 only).
  auto issue = [&](int j) {
    const int gi = j / nkc, kc = j - gi * nkc;
    const int64_t r0 = row_lo + static_cast<int64_t>(warp + gi * kGemvWarps) * kGemvRows;
    const int64_t left = row_hi - r0;
    const int nr = left < kGemvRows ? static_cast<int>(left) : kGemvRows;
    const int k0 = kc * kchunk;
    const int len = min(kchunk, K - k0) >> 2;  // bytes per row
    uint64_t* bar = &bars[j % kGemvSlots];
    uint8_t* dst = ring + (j % kGemvSlots) * kGemvSlotBytes;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nr * len));
    if (len == row_bytes) {
      // whole rows: the group's rows are contiguous in memory, one copy
      bulk_copy_g2s(dst, Wp + r0 * row_bytes, static_cast<uint32_t>(nr * len), bar, policy);
    } else {
      for (int r = 0; r < nr; ++r)
        bulk_copy_g2s(dst + r * slot_row, Wp + (r0 + r) * row_bytes + (k0 >> 2), static_cast<uint32_t>(len), bar,
                      policy);
    }
  };
  if (lane == 0)
    for (int j = 0; j < kGemvSlots && j < items; ++j) issue(j);

  // Everything below reads the outputs of the previous kernel.
  pdl_launch_dependents();
  pdl_wait();
  if constexpr (XS && !FUSED) {
    if (warp == 0 && lane == 0) {
      mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(MT * K));
      bulk_copy_g2s(xs, xq, static_cast<uint32_t>(MT * K), xbar, policy_evict_last());
    }
  }
  const float gamma = __ldg(gamma_ptr);
  float asc[MT];
  int rsum[MT];
  bool xok = true;
  if constexpr (FUSED) {
    __shared__ QuantScratch qsc;
#pragma unroll 1
    for (int m = 0; m < MT; ++m) {
      float amax;
      int sum;
      quant_row_cta<T, MAXC>(xin + static_cast<int64_t>(m) * K, K, gain, rms_eps,
                             reinterpret_cast<int8_t*>(xs) + m * K, qsc, amax, sum);
      asc[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
      rsum[m] = sum;
    }
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      asc[m] = __ldg(a_scale + m);
      rsum[m] = U8 ? __ldg(rowsum + m) : 0;
    }
    if constexpr (XS) xok = __all_sync(0xffffffffu, mbar_wait(xbar, 0));
  }

  int acc[kGemvRows][MT];
#pragma unroll
  for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0;

  int failed_at = xok ? -1 : 0;
  for (int j = 0; xok && j < items; ++j) {
    const int slot = j % kGemvSlots;
    // Every lane acquires the barrier itself; the warp leaves together if any gave up.
    const bool got = mbar_wait(&bars[slot], (j / kGemvSlots) & 1);
    if (!__all_sync(0xffffffffu, got)) {
      failed_at = j;
      break;
    }
    const int gi = j / nkc, kc = j - gi * nkc;
    const int k0 = kc * kchunk;
    const int len = min(kchunk, K - k0);  // weights per row in this item
    const uint32_t sw = smem_addr(ring + slot * kGemvSlotBytes);
#pragma unroll 1
    for (int kk = lane * 16; kk < len; kk += 512) {
      // This lane: weights k0+kk .. k0+kk+15 of the 4 rows.
      uint32_t xv[MT][4];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        uint4 u;
        if constexpr (XS) {
          u = lds128(smem_addr(xs) + m * K + k0 + kk);
        } else {
          u = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K + k0 + kk));
        }
        xv[m][0] = u.x;
        xv[m][1] = u.y;
        xv[m][2] = u.z;
        xv[m][3] = u.w;
      }
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r) {
        uint32_t w;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(sw + r * slot_row + (kk >> 2)));
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint32_t c4 = (w >> (2 * jj)) & 0x03030303u;
#pragma unroll
          for (int m = 0; m < MT; ++m)
            acc[r][m] = U8 ? dp4a_us(c4, xv[m][jj], acc[r][m]) : dp4a_ss(codes_to_signed(c4), xv[m][jj], acc[r][m]);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && j + kGemvSlots < items) {
      fence_proxy_async_smem();
      issue(j + kGemvSlots);
    }
    if (kc == nkc - 1) {
      // Row group finished: reduce over lanes, dequantise, store.
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int v = acc[r][m];
#pragma unroll
          for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
          acc[r][m] = v;
        }
      const int64_t r0 = row_lo + static_cast<int64_t>(warp + gi * kGemvWarps) * kGemvRows;
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == r * MT + m && r0 + r < row_hi) {
            const int a = acc[r][m] - rsum[m];
            const int64_t o = static_cast<int64_t>(m) * N + r0 + r;
            if (y_dtype == 2) {
              static_cast<int32_t*>(y)[o] = a;
            } else {
              const float v = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), asc[m]);
              if (y_dtype == 0) static_cast<float*>(y)[o] = v;
              else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
            }
          }
          acc[r][m] = 0;
        }
    }
  }
  if (failed_at >= 0 && lane == 0) {
    // Let copies still in flight land before the CTA's shared memory goes away.
    for (int j = failed_at; j < items && j < failed_at + kGemvSlots; ++j)
      mbar_wait(&bars[j % kGemvSlots], (j / kGemvSlots) & 1);
    if (XS && !FUSED && warp == 0) mbar_wait(xbar, 0);
  }
}

}  // namespace bitnet
