// Per-token absmax int8 quantisation (with the optional RMSNorm before it) of
// many long token rows: the same arithmetic and summation order as
// quant_row_cta (comrad404.com review, "Метод: как устроен BitNet b1.58":
// normalise, then quantise the activations to 8 bits), organised for
// throughput instead of latency.
//
// A CTA per row holds the row in registers and does nothing while its loads
// are in flight; with long rows few fit on an SM, so HBM idles between the
// reductions.  Here persistent CTAs walk the rows m = blockIdx.x, + gridDim.x,
// ...; each row (and, once, the norm gain) comes into shared memory with one
// bulk copy, into a ring of two row buffers, so the next row streams in while
// the current one is reduced and quantised, and every pass reads shared
// memory only.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

template <typename T>
BN_DEV Chunk8<T> qs_chunk(uint32_t addr) {
  Chunk8<T> c;
  if constexpr (sizeof(T) == 2) {
    c.u = lds128(addr);
  } else {
    const uint4 a = lds128(addr), b = lds128(addr + 16);
    c.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w));
    c.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w));
  }
  return c;
}

// One row from shared memory (row at shared address `rs`, the gain at `gs`
// when NORM) by the NTHR threads of the CTA: writes x_q to xq_row (global),
// returns max|h| and sum(x_q) to every thread.  Ends with a CTA barrier after
// the last read of the row.
template <typename T, bool NORM, int NTHR>
BN_DEV void qs_row(uint32_t rs, uint32_t gs, int K, float rms_eps, int8_t* __restrict__ xq_row, QuantScratch& sc,
                   float& amax_out, int& sum_out) {
  static_assert(NTHR >= kQuantThreads && NTHR % 32 == 0, "the fixed-order sum needs 256 threads");
  constexpr uint32_t CB = sizeof(Chunk8<T>);  // bytes per 8-element chunk
  constexpr int kWarps = NTHR / 32;
  const int t = static_cast<int>(threadIdx.x), lane = t & 31, warp = t >> 5;
  const int nchunks = K >> 3;

  float r = 1.0f;
  if constexpr (NORM) {
    // sum of squares: thread t < 256 adds RN32(v*v) over its chunks t, t+256,
    // ... in increasing order, then the fixed tree
    if (t < kQuantThreads) {
      float ss = 0.0f;
      for (int c = t; c < nchunks; c += kQuantThreads) {
        const Chunk8<T> ch = qs_chunk<T>(rs + CB * c);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = ch.get(e);
          ss = __fadd_rn(ss, __fmul_rn(v, v));
        }
      }
      sc.red[t] = ss;
    }
    __syncthreads();
    const float* R = sc.red;
    float p = __fadd_rn(__fadd_rn(__fadd_rn(R[lane], R[lane + 128]), __fadd_rn(R[lane + 64], R[lane + 192])),
                        __fadd_rn(__fadd_rn(R[lane + 32], R[lane + 160]), __fadd_rn(R[lane + 96], R[lane + 224])));
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const float o = __shfl_down_sync(0xffffffffu, p, s);
      if (lane < s) p = __fadd_rn(p, o);
    }
    p = __shfl_sync(0xffffffffu, p, 0);
    const float ms = __fdiv_rn(p, static_cast<float>(K));
    r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, rms_eps)));
  }

  // max|h| (order-free): h = RN32(RN32(v * r) * g) with the norm, else v
  float amax = 0.0f;
  for (int c = t; c < nchunks; c += NTHR) {
    const Chunk8<T> ch = qs_chunk<T>(rs + CB * c);
    if constexpr (NORM) {
      const Chunk8<T> g = qs_chunk<T>(gs + CB * c);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(ch.get(e), r), g.get(e))));
    } else if constexpr (sizeof(T) == 2) {
      // |v| of bf16 orders like its bit pattern with the sign cleared
      uint32_t m2 = max_u16x2(max_u16x2(ch.u.x & 0x7FFF7FFFu, ch.u.y & 0x7FFF7FFFu),
                              max_u16x2(ch.u.z & 0x7FFF7FFFu, ch.u.w & 0x7FFF7FFFu));
      const uint32_t mb = (m2 & 0xFFFFu) > (m2 >> 16) ? (m2 & 0xFFFFu) : (m2 >> 16);
      amax = fmaxf(amax, __uint_as_float(mb << 16));
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(ch.get(e)));
    }
  }
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if (lane == 0) sc.amx[warp] = amax;
  __syncthreads();
  amax = lane < kWarps ? sc.amx[lane] : 0.0f;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));

  int sum = 0;
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax);
  for (int c = t; c < nchunks; c += NTHR) {
    uint32_t lo = 0, hi = 0;
    if (amax != 0.0f) {
      const Chunk8<T> ch = qs_chunk<T>(rs + CB * c);
      Chunk8<T> g;
      if constexpr (NORM) g = qs_chunk<T>(gs + CB * c);
      uint32_t q[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = ch.get(e);
        const float h = NORM ? __fmul_rn(__fmul_rn(v, r), g.get(e)) : v;
        q[e] = f32_to_s8_rne_bits(__fmul_rn(h, s));
      }
      lo = pack4_s8(q[0], q[1], q[2], q[3]);
      hi = pack4_s8(q[4], q[5], q[6], q[7]);
      sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
      sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
    }
    *reinterpret_cast<uint2*>(xq_row + 8 * c) = make_uint2(lo, hi);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) sc.ired[warp] = sum;
  __syncthreads();
  int tot = lane < kWarps ? sc.ired[lane] : 0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  amax_out = amax;
  sum_out = tot;
}

// Dynamic shared memory: two row buffers, then (NORM) the gain.
template <typename T, bool NORM>
__host__ __device__ constexpr int quant_stream_smem_bytes(int K) {
  return (NORM ? 3 : 2) * K * static_cast<int>(sizeof(T));
}

// Rows m = blockIdx.x, + gridDim.x, ... of x (M x K), through a ring of two
// shared-memory row buffers, NTHR threads per CTA (256 for rows of at most
// 24 KB, four CTAs per SM; 512 for longer rows).  Every wait is bounded; after
// a timeout (the device error word is set) the CTA lets its copies in flight
// land and exits.
template <typename T, bool NORM, int NTHR>
__global__ void __launch_bounds__(NTHR, NTHR == 256 ? 4 : 2)
    quant_stream_kernel(const T* __restrict__ x, int M, int K, const T* __restrict__ gain, float rms_eps,
                        int8_t* __restrict__ xq, float* __restrict__ a_out, int32_t* __restrict__ rowsum_out) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ QuantScratch sc;
  __shared__ __align__(8) uint64_t full[2];
  const uint32_t rb = static_cast<uint32_t>(K) * static_cast<uint32_t>(sizeof(T));  // bytes per row
  const uint32_t base = smem_addr(smem);
  const int G = static_cast<int>(gridDim.x);
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // x comes from the previous kernel
  const uint64_t once = policy_evict_first();  // every row is read once
  int issued[2] = {0, 0};  // fills requested per buffer (thread 0)
  auto fill = [&](int b, int64_t m, bool with_gain) {
    mbar_arrive_expect_tx(&full[b], with_gain ? 2 * rb : rb);
    bulk_copy_g2s(smem + b * rb, x + m * K, rb, &full[b], once);
    if (with_gain) bulk_copy_g2s(smem + 2 * rb, gain, rb, &full[b], policy_evict_last());
    ++issued[b];
  };
  if (threadIdx.x == 0) {
    for (int j = 0; j < 2; ++j) {
      const int64_t m = static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(j) * G;
      if (m < M) fill(j, m, NORM && j == 0);
    }
  }
  int it = 0;
  for (int64_t m = blockIdx.x; m < M; m += G, ++it) {
    const int b = it & 1;
    if (!__syncthreads_and(mbar_wait(&full[b], static_cast<uint32_t>(it >> 1) & 1u))) break;
    float amax;
    int sum;
    qs_row<T, NORM, NTHR>(base + b * rb, base + 2 * rb, K, rms_eps, xq + m * K, sc, amax, sum);
    if (threadIdx.x == 0) {
      a_out[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
      if (rowsum_out != nullptr) rowsum_out[m] = sum;
      // every thread's reads of buffer b came before qs_row's last barrier
      const int64_t next = m + 2 * static_cast<int64_t>(G);
      if (next < M) {
        fence_proxy_async_smem();
        fill(b, next, false);
      }
    }
  }
  if (threadIdx.x == 0) {
    // after a timeout: the copies still in flight land before shared memory goes away
    for (int b = 0; b < 2; ++b)
      if (issued[b] > 0) mbar_wait(&full[b], static_cast<uint32_t>(issued[b] - 1) & 1u);
  }
  pdl_launch_dependents();
}

}  // namespace bitnet
