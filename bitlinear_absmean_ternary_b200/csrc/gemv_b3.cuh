// Fused decode BitLinear (M <= 8 tokens) on base-3 packed weights.
//
// Five ternary codes per byte as a base-3 number (inferownia.pl, "BitNet
// b1.58: era 1-bitowych LLM-ów", "Skąd te 1,58 bita": a ternary weight holds
// log2(3) ~ 1.58 bits), 1.6 bits per weight: 20% fewer weight bytes than the
// 2-bit layout.  A row is padded with zero weights to Kp = ceil(K/80)*80 and
// stored as 16-byte groups; byte i of group g holds weight 80g + 16t + i as
// base-3 digit t.  Digit t of four consecutive bytes is therefore four
// consecutive weights, which dp4a combines with four consecutive activations.
//
// Digits come out without division or tables: two bytes sit in the 16-bit
// halves of a register and floor(v / 3) = (171 v) >> 9, exact for v <= 255,
// is evaluated for both halves with one multiply (the products stay inside
// their halves).  Four such steps give digits 0..3, the last quotient is
// digit 4.  The rest is the fused decode GEMV of gemv.cuh: every CTA
// quantises the token rows into shared memory (zero-padded to Kp), the
// weights stream through per-warp rings of bulk copies (items of 4 rows by up
// to 40 groups), the first of them requested before the dependency wait.
#pragma once

#include <cuda_bf16.h>

#include "gemv.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kB3GroupWeights = 80;  // weights per 16-byte group
constexpr int kB3ChunkGroups = kGemvSlotBytes / (kGemvRows * 16);  // 40 groups per row per item

__host__ __device__ inline int b3_padded_k(int K) { return (K + kB3GroupWeights - 1) / kB3GroupWeights * kB3GroupWeights; }

// Groups per row per item: equal chunks of at most kB3ChunkGroups.
__host__ __device__ inline int b3_chunk_groups(int groups) {
  const int n = (groups + kB3ChunkGroups - 1) / kB3ChunkGroups;
  return (groups + n - 1) / n;
}

__host__ __device__ inline int gemv_b3_smem_bytes(int mt, int kp) {
  return kGemvRingBytes + kGemvBarBytes + kGemvWaveRows * mt * 4 + ((mt * kp + 15) / 16) * 16;
}

template <int MT, typename T, int MAXC>
__global__ void __launch_bounds__(kGemvThreads) gemv_b3_kernel(const uint8_t* __restrict__ Wp,
                                                               const float* __restrict__ gamma_ptr, int N, int K,
                                                               const T* __restrict__ xin, const T* __restrict__ gain,
                                                               float rms_eps, void* __restrict__ y, int y_dtype) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ QuantScratch qsc;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = smem + warp * kGemvSlots * kGemvSlotBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvRingBytes) + warp * kGemvSlots;
  int* accs = reinterpret_cast<int*>(smem + kGemvRingBytes + kGemvBarBytes);  // [kGemvWaveRows][MT]
  uint8_t* xs = smem + kGemvRingBytes + kGemvBarBytes + kGemvWaveRows * MT * 4;

  const int Kp = b3_padded_k(K);
  const int groups = Kp / kB3GroupWeights;
  const int64_t row_bytes = Kp / 5;
  const int cg = b3_chunk_groups(groups), nkc = (groups + cg - 1) / cg;
  const int slot_row = cg * 16;  // bytes per row inside a slot
  const int64_t row_lo = static_cast<int64_t>(N) * blockIdx.x / gridDim.x;
  const int64_t row_hi = static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x;
  const int nrows = static_cast<int>(row_hi - row_lo);
  const int ngroups = (nrows + kGemvRows - 1) / kGemvRows;
  const int items = ngroups * nkc;  // item j -> (row group j / nkc, chunk j % nkc), warp j % 16

  if (lane == 0) {
    for (int s = 0; s < kGemvSlots; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kGemvWaveRows * MT; i += kGemvThreads) accs[i] = 0;
  __syncthreads();

  const uint64_t policy = policy_evict_first();
  auto issue = [&](int k) {
    const int j = warp + k * kGemvWarps;
    const int gi = j / nkc, kc = j - gi * nkc;
    const int64_t r0 = row_lo + static_cast<int64_t>(gi) * kGemvRows;
    const int64_t left = row_hi - r0;
    const int nr = left < kGemvRows ? static_cast<int>(left) : kGemvRows;
    const int g0 = kc * cg;
    const int len = (groups - g0 < cg ? groups - g0 : cg) * 16;  // bytes per row
    uint64_t* bar = &bars[k % kGemvSlots];
    uint8_t* dst = ring + (k % kGemvSlots) * kGemvSlotBytes;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nr * len));
    if (len == row_bytes) {
      bulk_copy_g2s(dst, Wp + r0 * row_bytes, static_cast<uint32_t>(nr * len), bar, policy);
    } else {
      for (int r = 0; r < nr; ++r)
        bulk_copy_g2s(dst + r * slot_row, Wp + (r0 + r) * row_bytes + g0 * 16, static_cast<uint32_t>(len), bar,
                      policy);
    }
  };
  const int my_items = items > warp ? (items - warp + kGemvWarps - 1) / kGemvWarps : 0;
  if (lane == 0)
    for (int k = 0; k < kGemvSlots && k < my_items; ++k) issue(k);

  // Everything below reads the outputs of the previous kernel.
  pdl_launch_dependents();
  pdl_wait();
  const float gamma = __ldg(gamma_ptr);
  float asc[MT];
  int rsum[MT];
  for (int i = threadIdx.x; i < MT * (Kp - K); i += kGemvThreads) {
    const int m = i / (Kp - K);
    xs[m * Kp + K + (i - m * (Kp - K))] = 0;  // padded activations are zero
  }
#pragma unroll 1
  for (int m = 0; m < MT; ++m) {
    float amax;
    int sum;
    quant_row_cta<T, MAXC>(xin + static_cast<int64_t>(m) * K, K, gain, rms_eps,
                           reinterpret_cast<int8_t*>(xs) + m * Kp, qsc, amax, sum);
    asc[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    rsum[m] = sum;
  }

  constexpr int kWaveGroups = kGemvWaveRows / kGemvRows;
  const int nwaves = (ngroups + kWaveGroups - 1) / kWaveGroups;
  int k = 0;
  int failed_at = -1;
  for (int wv = 0; wv < nwaves; ++wv) {
    const int j_end = min(items, (wv + 1) * kWaveGroups * nkc);
    for (; failed_at < 0 && warp + k * kGemvWarps < j_end; ++k) {
      const int j = warp + k * kGemvWarps;
      const int slot = k % kGemvSlots;
      const bool got = mbar_wait(&bars[slot], (k / kGemvSlots) & 1);
      if (!__all_sync(0xffffffffu, got)) {
        failed_at = k;
        break;
      }
      const int gi = j / nkc, kc = j - gi * nkc;
      const int g0 = kc * cg;
      const int ng = groups - g0 < cg ? groups - g0 : cg;
      const uint32_t sw = smem_addr(ring + slot * kGemvSlotBytes);
      const uint32_t xa = smem_addr(xs) + g0 * kB3GroupWeights;
      int acc[kGemvRows][MT];
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll 1
      for (int gg = lane; gg < ng; gg += 32) {
        // Digit state of the group's 16 bytes of each row: even bytes (0, 2)
        // and odd bytes (1, 3) of every word in 16-bit halves.
        uint32_t ev[kGemvRows][4], od[kGemvRows][4];
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r) {
          const uint4 u = lds128(sw + r * slot_row + gg * 16);
          const uint32_t wv4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            ev[r][q] = wv4[q] & 0x00FF00FFu;
            od[r][q] = (wv4[q] >> 8) & 0x00FF00FFu;
          }
        }
#pragma unroll
        for (int t = 0; t < 5; ++t) {
          uint32_t xw[MT][4];
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 u = lds128(xa + m * Kp + gg * kB3GroupWeights + 16 * t);
            xw[m][0] = u.x;
            xw[m][1] = u.y;
            xw[m][2] = u.z;
            xw[m][3] = u.w;
          }
#pragma unroll
          for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t ce, co;
              if (t < 4) {
                const uint32_t qe = ((ev[r][q] * 171u) >> 9) & 0x007F007Fu;
                const uint32_t qo = ((od[r][q] * 171u) >> 9) & 0x007F007Fu;
                ce = ev[r][q] - 3u * qe;
                co = od[r][q] - 3u * qo;
                ev[r][q] = qe;
                od[r][q] = qo;
              } else {
                ce = ev[r][q];
                co = od[r][q];
              }
              const uint32_t c4 = ce | (co << 8);  // codes of weights 80g + 16t + 4q + (0..3)
#pragma unroll
              for (int m = 0; m < MT; ++m) acc[r][m] = dp4a_us(c4, xw[m][q], acc[r][m]);
            }
        }
      }
      __syncwarp();
      if (lane == 0 && k + kGemvSlots < my_items) {
        fence_proxy_async_smem();
        issue(k + kGemvSlots);
      }
      const int wrow0 = (gi - wv * kWaveGroups) * kGemvRows;
      const int grow0 = gi * kGemvRows;
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int v = __reduce_add_sync(0xffffffffu, acc[r][m]);
          if (lane == r * MT + m && grow0 + r < nrows) atomicAdd(&accs[(wrow0 + r) * MT + m], v);
        }
    }
    __syncthreads();
    const int wrows = min(kGemvWaveRows, nrows - wv * kGemvWaveRows);
    for (int i = threadIdx.x; i < wrows * MT; i += kGemvThreads) {
      const int rr = i / MT, m = i - rr * MT;
      const int a = accs[i] - rsum[m];
      const int64_t o = static_cast<int64_t>(m) * N + row_lo + wv * kGemvWaveRows + rr;
      if (y_dtype == 2) {
        static_cast<int32_t*>(y)[o] = a;
      } else {
        const float v = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), asc[m]);
        if (y_dtype == 0) static_cast<float*>(y)[o] = v;
        else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
      }
      accs[i] = 0;
    }
    __syncthreads();
  }
  if (failed_at >= 0 && lane == 0) {
    for (int kk = failed_at; kk < my_items && kk < failed_at + kGemvSlots; ++kk)
      if (!mbar_wait(&bars[kk % kGemvSlots], (kk / kGemvSlots) & 1)) break;
  }
}

}  // namespace bitnet
