// Decode-shaped W1.58A8 product (M <= 8 tokens) on CUDA cores.
//
// The ternary product is "the sum of the inputs with weight +1 minus the sum
// of those with weight -1" (Habr repost on juhe.plus, section "Когда - три
// лучше двух"); here each group of four weights is expanded to four bytes
// and combined with four int8 activations by one dp4a, which is that
// add/subtract exactly, in integers.  With the per-token sum of x_q at hand
// the bytes hold the unsigned codes c = q + 1 in {0, 1, 2} and the row sum
// is subtracted once per output (sum c*x - sum x = sum q*x), which saves two
// instructions per four weights.  For one token the four 2-bit fields of a
// code word are not even shifted down: field j masked in place is 4^j * c,
// a byte of at most 128, and its dp4a goes to an accumulator of its own that
// is divided by 4^j (an exact shift: it holds a multiple of 4^j) when the
// item is done -- 8 instructions per 16 weights instead of 12.
//
// Work split: CTA c owns the contiguous rows [N*c/G, N*(c+1)/G) (G = grid,
// one CTA per SM).  Its rows are cut into groups of 4 and K into equal
// chunks of at most `kcmax` weights (multiples of 64); an item is one (group,
// chunk) pair, and item j goes to warp j % 16.  Lane 0 of each warp streams
// the warp's items with bulk asynchronous copies (L2 evict-first) into a
// ring of `nslots` slots of shared memory it owns, refilling a slot as soon
// as the warp has consumed it.  The chunk size and the ring depth are chosen
// by the host per shape (the launch plan): small matrices are cut finely so
// that a CTA's few rows still spread over all 16 warps, large ones get long
// chunks and a deep ring, so that every SM keeps tens of KB of weights in
// flight (Little's law at HBM latency) without issuing many small copies.
// The activations x_q (M*K bytes) sit in shared memory, copied once per CTA.
// Lane l handles 16 consecutive weights of each of the 4 rows per 512-weight
// step, so the warp's loads of codes (4 bytes per lane) and of activations
// (16 bytes per lane) are contiguous and free of bank conflicts, and each
// activation load serves 4 rows.  A warp reduces its partial sums with one
// redux per row and token and adds them to the row's shared-memory
// accumulator (integer atomics: exact and order-free); the rows' outputs are
// dequantised and stored once all items of a wave of up to 256 rows are in.
//
// The first weight items are requested before waiting on the previous
// kernel (programmatic dependent launch), because the weights never depend
// on it.  The caller must therefore not write W_packed with the kernel that
// runs just before this one on the same stream.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvRows = 4;         // rows per group
constexpr int kGemvWaveRows = 256;   // rows accumulated in shared memory at a time
constexpr int kGemvXMaxBytes = 21504;  // x_q is staged in shared memory when M*K fits
constexpr int kGemvMaxSlots = 8;     // ring slots per warp (at most)
// The fixed ring of the kernels built on this one (decode FFN, base-3 GEMV):
// 2 slots per warp of 4 rows x at most 2560 weights.
constexpr int kGemvSlots = 2;
constexpr int kGemvKChunkMax = 2560;
constexpr int kGemvSlotBytes = kGemvRows * kGemvKChunkMax / 4;  // 2560 bytes
constexpr int kGemvRingBytes = kGemvWarps * kGemvSlots * kGemvSlotBytes;
constexpr int kGemvBarBytes = 512;
// Barrier block of gemv_kernel: one mbarrier per slot of every warp + x_q's.
constexpr int kGemvPlanBarBytes = 1152;

// Equal K-chunks of at most `cmax` weights, multiples of 64.
__host__ __device__ constexpr int gemv_kchunk_max(int K, int cmax) {
  return ((K + (K + cmax - 1) / cmax - 1) / ((K + cmax - 1) / cmax) + 63) / 64 * 64;
}

// Equal K-chunks of at most kGemvKChunkMax weights, multiples of 64.
__host__ __device__ constexpr int gemv_kchunk(int K) { return gemv_kchunk_max(K, kGemvKChunkMax); }

// Dynamic shared memory of gemv_kernel: ring (16 warps x nslots x kchunk
// bytes: a slot holds 4 rows x kchunk/4 bytes), barriers, the wave's row
// accumulators and (XS) x_q.
__host__ __device__ constexpr int gemv_plan_smem_bytes(int mt, int k, bool xs, int kchunk, int nslots) {
  return kGemvWarps * nslots * kchunk + kGemvPlanBarBytes + kGemvWaveRows * mt * 4 +
         (xs ? ((mt * k + 15) / 16) * 16 : 0);
}

__host__ __device__ constexpr int gemv_smem_bytes(int mt, int k, bool xs) {
  return kGemvRingBytes + kGemvBarBytes + kGemvWaveRows * mt * 4 + (xs ? ((mt * k + 15) / 16) * 16 : 0);
}

// FUSED: the kernel takes the unquantised activations x (M x K of type T)
// and the optional RMSNorm gain instead of x_q / a_scale / rowsum, and
// quantises every token row itself straight into its shared-memory copy of
// x_q (quant_row_cta: the same arithmetic and order as the standalone
// quantisation kernel).  Every CTA repeats this small step (M*K <= 21504
// values, read from L2), which removes a dependent kernel launch and the x_q
// round trip through global memory from each decode linear.
// kchunk: weights per row per item (a multiple of 64); nslots: ring slots
// per warp (1 .. kGemvMaxSlots).
template <int MT, bool U8, bool XS, bool FUSED = false, typename T = float, int MAXC = 1>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const uint8_t* __restrict__ Wp,
                                                            const float* __restrict__ gamma_ptr, int N, int K,
                                                            const int8_t* __restrict__ xq,
                                                            const float* __restrict__ a_scale,
                                                            const int32_t* __restrict__ rowsum,
                                                            const T* __restrict__ xin, const T* __restrict__ gain,
                                                            float rms_eps, void* __restrict__ y, int y_dtype,
                                                            int kchunk, int nslots, int l2_prefetch) {
  static_assert(!FUSED || (XS && U8), "the fused kernel keeps x_q in shared memory and uses its row sums");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ring_bytes = kGemvWarps * nslots * kchunk;
  uint8_t* ring = smem + warp * nslots * kchunk;
  uint64_t* all_bars = reinterpret_cast<uint64_t*>(smem + ring_bytes);
  uint64_t* bars = all_bars + warp * kGemvMaxSlots;
  uint64_t* xbar = all_bars + kGemvWarps * kGemvMaxSlots;
  int* accs = reinterpret_cast<int*>(smem + ring_bytes + kGemvPlanBarBytes);  // [kGemvWaveRows][MT]
  uint8_t* xs = smem + ring_bytes + kGemvPlanBarBytes + kGemvWaveRows * MT * 4;

  const int64_t row_lo = static_cast<int64_t>(N) * blockIdx.x / gridDim.x;
  const int64_t row_hi = static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x;
  const int nrows = static_cast<int>(row_hi - row_lo);
  const int ngroups = (nrows + kGemvRows - 1) / kGemvRows;
  const int nkc = (K + kchunk - 1) / kchunk;
  const int items = ngroups * nkc;  // item j -> (group j / nkc, chunk j % nkc), done by warp j % kGemvWarps
  const int64_t row_bytes = K >> 2;
  const int slot_row = kchunk >> 2;  // bytes per row inside a slot

  if (lane == 0) {
    for (int s = 0; s < nslots; ++s) mbar_init(&bars[s], 1);
    if (warp == 0) mbar_init(xbar, 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kGemvWaveRows * MT; i += kGemvThreads) accs[i] = 0;
  __syncthreads();

  const uint64_t policy = policy_evict_first();
  // Issue this warp's k-th item (item j = warp + k * kGemvWarps) into slot k % nslots (lane 0 only).
  auto issue = [&](int k) {
    const int j = warp + k * kGemvWarps;
    const int gi = j / nkc, kc = j - gi * nkc;
    const int64_t r0 = row_lo + static_cast<int64_t>(gi) * kGemvRows;
    const int64_t left = row_hi - r0;
    const int nr = left < kGemvRows ? static_cast<int>(left) : kGemvRows;
    const int k0 = kc * kchunk;
    const int len = min(kchunk, K - k0) >> 2;  // bytes per row
    const int slot = k % nslots;
    uint64_t* bar = &bars[slot];
    uint8_t* dst = ring + slot * kchunk;
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
  const int my_items = items > warp ? (items - warp + kGemvWarps - 1) / kGemvWarps : 0;
  if (lane == 0) {
    for (int k = 0; k < nslots && k < my_items; ++k) issue(k);
    if (l2_prefetch) {
      // The CTA's rows are contiguous in memory: request all of them into L2 now, one slice
      // per warp.  Under programmatic dependent launch this runs while the previous kernel
      // still works, so the weights stream from HBM across the kernel boundary and the ring
      // refills after the dependency wait hit L2.
      const int64_t share = static_cast<int64_t>(nrows) * row_bytes;
      const int64_t slice = (share / kGemvWarps + 15) / 16 * 16;
      const int64_t lo = slice * warp, hi = lo + slice < share ? lo + slice : share;
      for (int64_t o = lo; o < hi; o += 65536) {
        const int64_t n = hi - o < 65536 ? hi - o : 65536;
        bulk_prefetch_l2(Wp + row_lo * row_bytes + o, static_cast<uint32_t>(n));
      }
    }
  }

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

  // Waves of up to kGemvWaveRows rows (kGemvWaveRows / 4 groups).
  constexpr int kWaveGroups = kGemvWaveRows / kGemvRows;
  // one token with unsigned codes: the fields of a code word are masked in place
  constexpr bool kMasked = MT == 1 && U8;
  const int nwaves = (ngroups + kWaveGroups - 1) / kWaveGroups;
  int k = 0;  // this warp's item counter (ring position)
  int failed_at = -1;
  for (int wv = 0; wv < nwaves; ++wv) {
    const int j_end = min(items, (wv + 1) * kWaveGroups * nkc);
    for (; xok && failed_at < 0 && warp + k * kGemvWarps < j_end; ++k) {
      const int j = warp + k * kGemvWarps;
      const int slot = k % nslots;
      // Every lane acquires the barrier itself; the warp leaves together if any gave up.
      const bool got = mbar_wait(&bars[slot], (k / nslots) & 1);
      if (!__all_sync(0xffffffffu, got)) {
        failed_at = k;
        break;
      }
      const int gi = j / nkc, kc = j - gi * nkc;
      const int k0 = kc * kchunk;
      const int len = min(kchunk, K - k0);  // weights per row in this item
      const uint32_t sw = smem_addr(ring + slot * kchunk);
      int acc[kGemvRows][MT];
      int accf[kGemvRows][kMasked ? 4 : 1];  // kMasked: accumulator of field j, in units of 4^j
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r) {
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll
        for (int f = 0; f < (kMasked ? 4 : 1); ++f) accf[r][f] = 0;
      }
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
          if constexpr (kMasked) {
            accf[r][0] = dp4a_us(w & 0x03030303u, xv[0][0], accf[r][0]);
            accf[r][1] = dp4a_us(w & 0x0C0C0C0Cu, xv[0][1], accf[r][1]);
            accf[r][2] = dp4a_us(w & 0x30303030u, xv[0][2], accf[r][2]);
            accf[r][3] = dp4a_us(w & 0xC0C0C0C0u, xv[0][3], accf[r][3]);
          } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const uint32_t c4 = (w >> (2 * jj)) & 0x03030303u;
#pragma unroll
              for (int m = 0; m < MT; ++m)
                acc[r][m] = U8 ? dp4a_us(c4, xv[m][jj], acc[r][m])
                               : dp4a_ss(codes_to_signed(c4), xv[m][jj], acc[r][m]);
            }
          }
        }
      }
      if constexpr (kMasked) {
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r)
          acc[r][0] = accf[r][0] + (accf[r][1] >> 2) + (accf[r][2] >> 4) + (accf[r][3] >> 6);
      }
      __syncwarp();
      if (lane == 0 && k + nslots < my_items) {
        fence_proxy_async_smem();
        issue(k + nslots);
      }
      // Item partial sums -> the rows' shared accumulators.
      const int wrow0 = (gi - wv * kWaveGroups) * kGemvRows;  // row of the group inside the wave
      const int grow0 = gi * kGemvRows;                       // row of the group inside the CTA
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int v = __reduce_add_sync(0xffffffffu, acc[r][m]);
          if (lane == r * MT + m && grow0 + r < nrows) atomicAdd(&accs[(wrow0 + r) * MT + m], v);
        }
    }
    // Wave finished: dequantise and store its rows, then clear the accumulators.
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
  if ((failed_at >= 0 || !xok) && lane == 0) {
    // Let copies still in flight land before the CTA's shared memory goes away.
    const int from = failed_at >= 0 ? failed_at : 0;
    for (int kk = from; kk < my_items && kk < from + nslots; ++kk) mbar_wait(&bars[kk % nslots], (kk / nslots) & 1);
    if (XS && !FUSED && warp == 0) mbar_wait(xbar, 0);
  }
}

}  // namespace bitnet
