// Per-token absmax int8 activation quantisation fused with the RMSNorm that
// precedes it (comrad404.com review, "Метод: как устроен BitNet b1.58":
// 8-bit activations; RMSNorm; "normalise the input, then quantise").
//
// One CTA of 256 threads per token row; thread t owns the 8-element chunks
// c = t, t+256, ... and keeps them in registers, so x is read from HBM once.
// The sum of squares uses the fixed order of the oracle: each thread adds
// RN32(v*v) over its chunks in increasing k, then the halving tree
// l += l+128, +64, +32 (shared memory), +16 .. +1 (shuffles).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bitnet {

template <typename T>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
  uint4 u;
  BN_DEV void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  BN_DEV float get(int e) const {
    const uint32_t w = e < 2 ? u.x : (e < 4 ? u.y : (e < 6 ? u.z : u.w));
    return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
};

template <>
struct Chunk8<float> {
  float4 a, b;
  BN_DEV void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  BN_DEV float get(int e) const {
    switch (e) {
      case 0: return a.x;
      case 1: return a.y;
      case 2: return a.z;
      case 3: return a.w;
      case 4: return b.x;
      case 5: return b.y;
      case 6: return b.z;
      default: return b.w;
    }
  }
};

constexpr int kQuantThreads = 256;

template <typename T, int MAXC>
__global__ void __launch_bounds__(kQuantThreads) quant_act_kernel(const T* __restrict__ x, int K,
                                                                  const T* __restrict__ gain, float rms_eps,
                                                                  int8_t* __restrict__ xq, float* __restrict__ a_out,
                                                                  int32_t* __restrict__ rowsum_out) {
  __shared__ float red[kQuantThreads];
  __shared__ float bcast;
  __shared__ int ired[kQuantThreads / 32];

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int64_t m = blockIdx.x;
  const int nchunks = K >> 3;
  const T* row = x + m * K;

  pdl_wait();

  Chunk8<T> ch[MAXC];
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = t + kQuantThreads * i;
    if (c < nchunks) ch[i].load(row + 8 * c);
  }

  float r = 1.0f;
  if (gain != nullptr) {
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = t + kQuantThreads * i;
      if (c < nchunks) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = ch[i].get(e);
          ss = __fadd_rn(ss, __fmul_rn(v, v));
        }
      }
    }
    red[t] = ss;
    __syncthreads();
#pragma unroll
    for (int s = kQuantThreads / 2; s >= 32; s >>= 1) {
      if (t < s) red[t] = __fadd_rn(red[t], red[t + s]);
      __syncthreads();
    }
    if (warp == 0) {
      float p = red[lane];
#pragma unroll
      for (int s = 16; s >= 1; s >>= 1) {
        const float o = __shfl_down_sync(0xffffffffu, p, s);
        if (lane < s) p = __fadd_rn(p, o);
      }
      if (lane == 0) {
        const float ms = __fdiv_rn(p, static_cast<float>(K));
        bcast = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, rms_eps)));
      }
    }
    __syncthreads();
    r = bcast;
  }

  // h = RN32(RN32(v * r) * g) or v; amax = max |h| (order-free).
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = t + kQuantThreads * i;
    if (c < nchunks) {
      Chunk8<T> g;
      if (gain != nullptr) g.load(gain + 8 * c);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = ch[i].get(e);
        const float h = gain != nullptr ? __fmul_rn(__fmul_rn(v, r), g.get(e)) : v;
        amax = fmaxf(amax, fabsf(h));
      }
    }
  }
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  __syncthreads();  // red[] reuse
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red[w]);

  int sum = 0;
  if (amax == 0.0f) {
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = t + kQuantThreads * i;
      if (c < nchunks) *reinterpret_cast<uint2*>(xq + m * K + 8 * c) = make_uint2(0u, 0u);
    }
  } else {
    const float s = __fdiv_rn(127.0f, amax);
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = t + kQuantThreads * i;
      if (c < nchunks) {
        Chunk8<T> g;
        if (gain != nullptr) g.load(gain + 8 * c);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = ch[i].get(e);
          const float h = gain != nullptr ? __fmul_rn(__fmul_rn(v, r), g.get(e)) : v;
          int q = __float2int_rn(__fmul_rn(h, s));
          q = q < -127 ? -127 : (q > 127 ? 127 : q);
          sum += q;
          const uint32_t b = static_cast<uint32_t>(q) & 0xFFu;
          if (e < 4) lo |= b << (8 * e);
          else hi |= b << (8 * (e - 4));
        }
        *reinterpret_cast<uint2*>(xq + m * K + 8 * c) = make_uint2(lo, hi);
      }
    }
  }
  pdl_launch_dependents();

  if (rowsum_out != nullptr) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, s);
    if (lane == 0) ired[warp] = sum;
  }
  __syncthreads();
  if (t == 0) {
    a_out[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    if (rowsum_out != nullptr) {
      int tot = 0;
#pragma unroll
      for (int w = 0; w < kQuantThreads / 32; ++w) tot += ired[w];
      rowsum_out[m] = tot;
    }
  }
}

}  // namespace bitnet
