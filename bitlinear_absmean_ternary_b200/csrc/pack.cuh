// Absmean ternarisation and 2-bit packing of a latent fp32 weight matrix
// (inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", section "Trenowany
// od zera": scale the whole matrix by its mean absolute value, then round
// every entry to the nearest of {-1, 0, +1}).  Offline: runs once per model.
//
// gamma is reproducible bit for bit because its summation order is fixed:
// one warp per row, lane l summing k = l, l+32, ... in fp64 in increasing k,
// the 32 lane partials combined by the halving tree p[l] += p[l+s]
// (s = 16..1, which is what shfl_down with lanes l < s computes), and the row
// sums added in increasing row order by a single thread.
#pragma once

#include "ptx.cuh"

namespace bitnet {

// Pass 1: per-row sum of |w| in fp64 (canonical order) + non-finite check.
__global__ void __launch_bounds__(256) pack_rowsum_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                          double* __restrict__ rowsum,
                                                          unsigned int* __restrict__ nonfinite) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t n = warp; n < N; n += nwarps) {
    const float* row = W + n * K;
    double p = 0.0;
    bool bad = false;
    for (int64_t k = lane; k < K; k += 32) {
      const float w = __ldg(row + k);
      bad |= !isfinite(w);
      p = __dadd_rn(p, fabs(static_cast<double>(w)));
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const double o = __shfl_down_sync(0xffffffffu, p, s);
      if (lane < s) p = __dadd_rn(p, o);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(nonfinite, 1u);
    if (lane == 0) rowsum[n] = p;
  }
}

// Pass 2: S = sum of row sums in increasing n; gamma = RN32(S / (N*K));
// divisor d = RN32(gamma + eps).
__global__ void pack_gamma_kernel(const double* __restrict__ rowsum, int64_t N, int64_t K, float eps,
                                  float* __restrict__ gamma_out, float* __restrict__ d_out) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  double S = 0.0;
  for (int64_t n = 0; n < N; ++n) S = __dadd_rn(S, rowsum[n]);
  const float g = __double2float_rn(__ddiv_rn(S, static_cast<double>(N * K)));
  *gamma_out = g;
  *d_out = __fadd_rn(g, eps);
}

// Pass 3: one thread per packed 32-bit word (16 consecutive weights of one
// row).  q = clamp(RNE(RN32(w / d)), -1, 1); code q + 1 of weight 4j + b goes
// to byte b, bits 2j..2j+1.
__global__ void __launch_bounds__(256) pack_codes_kernel(const float* __restrict__ W, int64_t nwords,
                                                         const float* __restrict__ d_ptr,
                                                         uint32_t* __restrict__ packed) {
  const float d = *d_ptr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords; i += stride) {
    const float4* src = reinterpret_cast<const float4*>(W + i * 16);
    float v[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 f = __ldg(src + c);
      v[4 * c + 0] = f.x;
      v[4 * c + 1] = f.y;
      v[4 * c + 2] = f.z;
      v[4 * c + 3] = f.w;
    }
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      int q = __float2int_rn(__fdiv_rn(v[e], d));
      q = q < -1 ? -1 : (q > 1 ? 1 : q);
      word |= static_cast<uint32_t>(q + 1) << (8 * (e & 3) + 2 * (e >> 2));
    }
    packed[i] = word;
  }
}

// Base-3 storage: five codes c = q + 1 per byte as a base-3 number (a
// ternary weight holds log2(3) ~ 1.58 bits: inferownia.pl, "Skąd te 1,58
// bita"), 1.6 bits per weight.  A row is padded with zero weights (c = 1) to
// Kp = ceil(K/80)*80 and stored as groups of 16 bytes; byte i of group g is
// sum_t c[80g + 16t + i] * 3^t.  One thread per packed byte; q uses the same
// operations as pack_codes_kernel.
__global__ void __launch_bounds__(256) pack_codes_b3_kernel(const float* __restrict__ W, int64_t N, int K,
                                                            int row_bytes, const float* __restrict__ d_ptr,
                                                            uint8_t* __restrict__ packed) {
  const float d = *d_ptr;
  const int64_t total = N * row_bytes;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total; idx += stride) {
    const int64_t n = idx / row_bytes;
    const int j = static_cast<int>(idx - n * row_bytes);
    const int g = j >> 4, i = j & 15;
    const float* row = W + n * K;
    int v = 0, p3 = 1;
#pragma unroll
    for (int t = 0; t < 5; ++t) {
      const int k = 80 * g + 16 * t + i;
      int c = 1;
      if (k < K) {
        int q = __float2int_rn(__fdiv_rn(__ldg(row + k), d));
        q = q < -1 ? -1 : (q > 1 ? 1 : q);
        c = q + 1;
      }
      v += c * p3;
      p3 *= 3;
    }
    packed[idx] = static_cast<uint8_t>(v);
  }
}

}  // namespace bitnet
