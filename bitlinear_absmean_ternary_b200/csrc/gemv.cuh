// Decode-shaped W1.58A8 product (M <= 8 tokens) on CUDA cores.
//
// The ternary product is "the sum of the inputs with weight +1 minus the sum
// of those with weight -1" (Habr repost on juhe.plus, section "Когда - три
// лучше двух"); here each group of four weights is expanded to four signed
// bytes and combined with four int8 activations by one dp4a, which is that
// add/subtract exactly, in integers.
//
// Work split: CTA c owns the contiguous rows [N*c/G, N*(c+1)/G) (G = grid);
// inside a CTA, warps take groups of 4 consecutive rows round-robin.  A row
// group is streamed in K-chunks of up to 4096 weights (4 x 1 KB): lane 0 of
// the warp issues one bulk asynchronous copy per row into a 4-slot ring of
// shared memory owned by that warp; all 32 lanes then read 16-byte pieces
// (64 weights) of the 4 rows, so every activation load is reused 4 times.
// Lane partial sums are reduced with warp shuffles.  The first ring slots are
// requested before waiting on the previous kernel (programmatic dependent
// launch), because the weights never depend on it.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bitnet {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 4;       // rows per group
constexpr int kGemvSlots = 4;      // ring depth per warp
constexpr int kGemvKChunk = 4096;  // weights per row per slot
constexpr int kGemvSlotBytes = kGemvRows * kGemvKChunk / 4;
constexpr int kGemvSmemBytes = kGemvWarps * kGemvSlots * kGemvSlotBytes + kGemvWarps * kGemvSlots * 8;

template <int MT, bool U8>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const uint8_t* __restrict__ Wp,
                                                               const float* __restrict__ gamma_ptr, int N, int K,
                                                               const int8_t* __restrict__ xq,
                                                               const float* __restrict__ a_scale,
                                                               const int32_t* __restrict__ rowsum, void* __restrict__ y,
                                                               int y_dtype) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = smem + warp * kGemvSlots * kGemvSlotBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * kGemvSlots * kGemvSlotBytes) + warp * kGemvSlots;

  const int64_t row_lo = static_cast<int64_t>(N) * blockIdx.x / gridDim.x;
  const int64_t row_hi = static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x;
  const int ngroups = static_cast<int>((row_hi - row_lo + kGemvRows - 1) / kGemvRows);
  const int my_groups = ngroups > warp ? (ngroups - warp + kGemvWarps - 1) / kGemvWarps : 0;
  const int kchunk = K < kGemvKChunk ? K : kGemvKChunk;
  const int nkc = (K + kchunk - 1) / kchunk;
  const int items = my_groups * nkc;
  const int row_bytes = K >> 2;

  if (lane == 0) {
    for (int s = 0; s < kGemvSlots; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

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
    for (int r = 0; r < nr; ++r)
      bulk_copy_g2s(dst + r * (kchunk >> 2), Wp + (r0 + r) * row_bytes + (k0 >> 2), static_cast<uint32_t>(len), bar,
                    policy);
  };
  if (lane == 0)
    for (int j = 0; j < kGemvSlots && j < items; ++j) issue(j);

  // Everything below reads the outputs of the previous kernel.
  pdl_wait();
  pdl_launch_dependents();
  const float gamma = *gamma_ptr;

  int acc[kGemvRows][MT];
#pragma unroll
  for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0;

  int failed_at = -1;
  for (int j = 0; j < items; ++j) {
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
    const uint32_t sbase = smem_addr(ring + slot * kGemvSlotBytes);
    for (int ci = lane; ci < (len >> 6); ci += 32) {
      // 64 weights per row: 16 bytes of codes per row, 64 bytes of x per token.
      uint32_t wq[kGemvRows][16];
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r) {
        const uint4 p = lds128(sbase + r * (kchunk >> 2) + ci * 16);
        const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t c4 = (pw[wi] >> (2 * jj)) & 0x03030303u;
            wq[r][4 * wi + jj] = U8 ? c4 : codes_to_signed(c4);
          }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* xp = reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K + k0 + ci * 64);
        uint32_t xv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 u = __ldg(xp + q);
          xv[4 * q + 0] = u.x;
          xv[4 * q + 1] = u.y;
          xv[4 * q + 2] = u.z;
          xv[4 * q + 3] = u.w;
        }
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            acc[r][m] = U8 ? dp4a_us(wq[r][e], xv[e], acc[r][m]) : dp4a_ss(wq[r][e], xv[e], acc[r][m]);
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
            const int a = U8 ? acc[r][m] - __ldg(rowsum + m) : acc[r][m];
            const int64_t o = static_cast<int64_t>(m) * N + r0 + r;
            if (y_dtype == 2) {
              static_cast<int32_t*>(y)[o] = a;
            } else {
              const float v = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), __ldg(a_scale + m));
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
  }
}

}  // namespace bitnet
