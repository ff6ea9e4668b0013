// Per-token absmax int8 activation quantisation (with the optional RMSNorm
// in front of it) for many token rows at once: one warp per row (comrad404.com
// review, "Метод: как устроен BitNet b1.58": 8-bit activations; the input is
// normalised, then quantised).
//
// The CTA-per-row kernel of quant.cuh passes three CTA barriers per row (one
// per reduction).  Here a warp owns a row: lane l holds the 8-element chunks
// c = l, l+32, ... in registers (MAXC of them, read once with 16-byte loads:
// the warp reads 512 contiguous bytes per load), and every reduction is a
// handful of shuffles, so rows proceed independently of one another; an SM
// holds 16 of them at K = 6144 and 28 at K = 2560 (by register use), more
// for shorter rows.  Back to back over 4096 rows of K = 2560 it moved
// 4.45 TB/s against 3.62 TB/s for the CTA-per-row kernel.  bf16 input only,
// K <= 32 * 8 * MAXC.
//
// The arithmetic, and with RMSNorm the order of the sum of squares, are those
// of quant_row_cta, so the two kernels give the same bits.  That order is
// defined on 256 virtual lanes: virtual lane v owns the chunks c = v (mod 256)
// and adds RN32(x*x) over them in increasing k; the 256 partial sums are then
// added by the halving tree v += v+128, +64, ..., +1.  Lane l of the warp
// stands for the virtual lanes l + 32j (j = 0..7), whose chunks are exactly
// its chunks i = j (mod 8), so it keeps eight partial sums; the tree's first
// three levels (128, 64, 32) pair partial sums of the same lane and the last
// five are shuffles, as in quant_row_cta.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kQuantRowsWarps = 4;  // rows per CTA
constexpr int kQuantRowsThreads = kQuantRowsWarps * 32;
// Chunks per lane, K <= 6144.  At K = 6912 (27 chunks, 140 registers, 12 warps
// per SM) the CTA-per-row kernel was faster (20.5 us against 23.5 us for 4096
// rows back to back); at K = 5376 (21 chunks) this one still wins.
constexpr int kQuantRowsMaxChunks = 24;

BN_DEV float bf16_elem(const uint4& u, int e) {
  const uint32_t w = e < 2 ? u.x : (e < 4 ? u.y : (e < 6 ? u.z : u.w));
  return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

template <int MAXC, bool NORM>
__global__ void __launch_bounds__(kQuantRowsThreads)
    quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int K, const __nv_bfloat16* __restrict__ gain,
                      float rms_eps, int8_t* __restrict__ xq, float* __restrict__ a_out,
                      int32_t* __restrict__ rowsum_out) {
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * kQuantRowsWarps + (threadIdx.x >> 5);
  pdl_wait();
  if (m < M) {
    const int nchunks = K >> 3;
    const __nv_bfloat16* row = x + m * K;
    uint4 ch[MAXC];
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = lane + 32 * i;
      if (c < nchunks) ch[i] = __ldg(reinterpret_cast<const uint4*>(row + 8 * c));
    }

    float r = 1.0f;
    if constexpr (NORM) {
      float p[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) p[j] = 0.0f;
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        if (lane + 32 * i < nchunks) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v = bf16_elem(ch[i], e);
            p[i & 7] = __fadd_rn(p[i & 7], __fmul_rn(v, v));
          }
        }
      }
      // levels 128, 64 and 32 of the tree: virtual lanes l + 32j, j = 0..7
      float s = __fadd_rn(__fadd_rn(__fadd_rn(p[0], p[4]), __fadd_rn(p[2], p[6])),
                          __fadd_rn(__fadd_rn(p[1], p[5]), __fadd_rn(p[3], p[7])));
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) {
        const float o = __shfl_down_sync(0xffffffffu, s, d);
        if (lane < d) s = __fadd_rn(s, o);
      }
      s = __shfl_sync(0xffffffffu, s, 0);
      const float ms = __fdiv_rn(s, static_cast<float>(K));
      r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, rms_eps)));
    }

    // amax = max |h| with h = RN32(RN32(v * r) * g), or max |v| without the norm
    float amax = 0.0f;
    if constexpr (NORM) {
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        const int c = lane + 32 * i;
        if (c < nchunks) {
          const uint4 g = __ldg(reinterpret_cast<const uint4*>(gain + 8 * c));
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float h = __fmul_rn(__fmul_rn(bf16_elem(ch[i], e), r), bf16_elem(g, e));
            amax = fmaxf(amax, fabsf(h));
          }
        }
      }
    } else {
      // |v| orders like the bf16 bit pattern with the sign cleared
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        if (lane + 32 * i < nchunks) {
          m2 = max_u16x2(m2, ch[i].x & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, ch[i].y & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, ch[i].z & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, ch[i].w & 0x7FFF7FFFu);
        }
      }
      const uint32_t mb = (m2 & 0xFFFFu) > (m2 >> 16) ? (m2 & 0xFFFFu) : (m2 >> 16);
      amax = __uint_as_float(mb << 16);
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));

    const float s = amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax);
    int8_t* out = xq + m * K;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = lane + 32 * i;
      if (c < nchunks) {
        uint32_t lo = 0, hi = 0;
        if (amax != 0.0f) {
          uint4 g = make_uint4(0, 0, 0, 0);
          if constexpr (NORM) g = __ldg(reinterpret_cast<const uint4*>(gain + 8 * c));
          uint32_t q[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v = bf16_elem(ch[i], e);
            const float h = NORM ? __fmul_rn(__fmul_rn(v, r), bf16_elem(g, e)) : v;
            q[e] = f32_to_s8_rne_bits(__fmul_rn(h, s));
          }
          lo = pack4_s8(q[0], q[1], q[2], q[3]);
          hi = pack4_s8(q[4], q[5], q[6], q[7]);
          sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
          sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
        }
        *reinterpret_cast<uint2*>(out + 8 * c) = make_uint2(lo, hi);
      }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
    if (lane == 0) {
      a_out[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
      if (rowsum_out != nullptr) rowsum_out[m] = sum;
    }
  }
  pdl_launch_dependents();
}

}  // namespace bitnet
