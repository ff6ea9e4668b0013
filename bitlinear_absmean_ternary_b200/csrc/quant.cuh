// Per-token absmax int8 activation quantisation fused with the RMSNorm that
// precedes it (comrad404.com review, "Метод: как устроен BitNet b1.58":
// 8-bit activations; RMSNorm; the input is normalised, then quantised).
//
// 256 threads per token row; thread t owns the 8-element chunks c = t,
// t+256, ... and keeps them in registers, so x is read from HBM once (a long
// row with RMSNorm is read in three passes, the later ones from L1 or L2).
// The sum of squares uses the fixed order of the oracle: each thread adds
// RN32(v*v) over its chunks in increasing k, then the halving tree
// l += l+128, +64, +32 (shared memory), +16 .. +1 (shuffles).
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "ptx.cuh"

namespace bitnet {

template <typename T>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
  uint4 u;
  BN_DEV void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  // For data written earlier in the same kernel by other CTAs: L2 only.
  BN_DEV void load_cg(const __nv_bfloat16* p) { u = __ldcg(reinterpret_cast<const uint4*>(p)); }
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
  BN_DEV void load_cg(const float* p) {
    a = __ldcg(reinterpret_cast<const float4*>(p));
    b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
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

struct QuantScratch {
  float red[kQuantThreads];  // per-thread sums of squares (the first 256 threads)
  float amx[32];             // per-warp max|h|
  int ired[32];              // per-warp sums of x_q
};

// Round half to even of an fp32 value v with |v| < 2^22, returned as a bit
// pattern whose low byte is the integer in two's complement.  The sum
// v + 1.5 * 2^23 lies where the fp32 spacing is 1, so the addition's single
// rounding is the round-half-to-even of v (1.5 * 2^23 is even) and the sum's
// bit pattern is 0x4B400000 + RNE(v).  One fp32 add takes the place of a
// float-to-integer conversion, which issues at a lower rate.  For
// |v| <= 127 * (1 + 2^-23), as RN32(h * RN32(127 / amax)) always is, the low
// byte is clamp(RNE(v), -127, 127) (the clamp never binds).
BN_DEV uint32_t f32_to_s8_rne_bits(float v) { return __float_as_uint(__fadd_rn(v, 12582912.0f)); }

// The low bytes of four words packed into one word, byte 0 = a's.
BN_DEV uint32_t pack4_s8(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

BN_DEV void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// Unsigned 16-bit maximum of both halves.
BN_DEV uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Barrier over the first NT threads of the CTA (named barrier 1), or over
// the whole CTA when NT == 0.
template <int NT>
BN_DEV void sync_threads() {
  if constexpr (NT == 0) __syncthreads();
  else asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// The RMSNorm path of quant_row_cta for rows too long to keep in registers:
// three passes over the row, each reading it again (from L1 or L2), with a
// bounded number of chunks in registers at a time.  Pass 1 is the sum of
// squares in the fixed order (thread t < 256 adds its chunks t, t+256, ...
// in increasing order, then the same tree); passes 2 (max|h|) and 3 (x_q)
// are order-free and use every thread.  The first batch of a pass is
// requested before the barrier that ends the previous one, so each barrier
// overlaps one memory round trip.  Same arguments, results and barrier
// discipline as quant_row_cta.  Not inlined: compiled into the caller next to
// the register-resident path, it made the register allocator spill the
// callers' own loops; as a call it costs a few registers' save and restore
// once per row.
template <typename T, bool COHERENT, int NT, int T0>
__device__ __noinline__ void quant_row_norm_stream(const T* __restrict__ row, int K, const T* __restrict__ gain, float rms_eps,
                                  int8_t* xq_row, QuantScratch& sc, float& amax_out, int& sum_out) {
  const int t = static_cast<int>(threadIdx.x) - T0;
  const int lane = t & 31, warp = t >> 5;
  const int nthreads = NT == 0 ? static_cast<int>(blockDim.x) : NT;
  const int nwarps = nthreads >> 5;
  const int nchunks = K >> 3;
  // Chunks in flight per thread: 128 bytes of x in pass 1, 64 bytes each of
  // x and the gain in passes 2 and 3 (more spills under a 64-register budget).
  constexpr int NB1 = 128 / static_cast<int>(sizeof(Chunk8<T>));
  constexpr int NB2 = 64 / static_cast<int>(sizeof(Chunk8<T>));
  auto load_x = [&](Chunk8<T>& d, int c) {
    if constexpr (COHERENT) d.load_cg(row + 8 * c);
    else d.load(row + 8 * c);
  };

  float ss = 0.0f;
  if (t < kQuantThreads) {
#pragma unroll 1
    for (int c0 = t; c0 < nchunks; c0 += NB1 * kQuantThreads) {
      Chunk8<T> b[NB1];
#pragma unroll
      for (int j = 0; j < NB1; ++j)
        if (c0 + j * kQuantThreads < nchunks) load_x(b[j], c0 + j * kQuantThreads);
#pragma unroll
      for (int j = 0; j < NB1; ++j) {
        if (c0 + j * kQuantThreads < nchunks) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v = b[j].get(e);
            ss = __fadd_rn(ss, __fmul_rn(v, v));
          }
        }
      }
    }
    sc.red[t] = ss;
  }

  // Batches of passes 2 and 3: thread t takes chunks t + nthreads * i.
  Chunk8<T> xb[NB2], gb[NB2];
  const int step = NB2 * nthreads;
  auto load_batch = [&](int c0) {
#pragma unroll
    for (int j = 0; j < NB2; ++j) {
      const int c = c0 + j * nthreads;
      if (c < nchunks) {
        load_x(xb[j], c);
        gb[j].load(gain + 8 * c);
      }
    }
  };
  load_batch(t);
  sync_threads<NT>();
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
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, rms_eps)));

  float amax = 0.0f;
#pragma unroll 1
  for (int c0 = t; c0 < nchunks; c0 += step) {
    if (c0 != t) load_batch(c0);
#pragma unroll
    for (int j = 0; j < NB2; ++j) {
      if (c0 + j * nthreads < nchunks) {
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(xb[j].get(e), r), gb[j].get(e))));
      }
    }
  }
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if (lane == 0) sc.amx[warp] = amax;
  load_batch(t);
  sync_threads<NT>();
  amax = lane < nwarps ? sc.amx[lane] : 0.0f;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));

  int sum = 0;
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax);
#pragma unroll 1
  for (int c0 = t; c0 < nchunks; c0 += step) {
    if (c0 != t) load_batch(c0);
#pragma unroll
    for (int j = 0; j < NB2; ++j) {
      const int c = c0 + j * nthreads;
      if (c < nchunks) {
        uint32_t lo = 0, hi = 0;
        if (amax != 0.0f) {
          uint32_t q[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            q[e] = f32_to_s8_rne_bits(__fmul_rn(__fmul_rn(__fmul_rn(xb[j].get(e), r), gb[j].get(e)), s));
          lo = pack4_s8(q[0], q[1], q[2], q[3]);
          hi = pack4_s8(q[4], q[5], q[6], q[7]);
          sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
          sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
        }
        *reinterpret_cast<uint2*>(xq_row + 8 * c) = make_uint2(lo, hi);
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) sc.ired[warp] = sum;
  sync_threads<NT>();
  int tot = lane < nwarps ? sc.ired[lane] : 0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  amax_out = amax;
  sum_out = tot;
}

// Resident footprint (bytes of x per thread) above which the RMSNorm path
// streams the row instead of keeping it in registers.
#ifndef BN_QUANT_STREAM_BYTES
#define BN_QUANT_STREAM_BYTES 64
#endif

// Quantises one token row with the threads of the CTA.  Every thread must
// call it (it holds CTA-wide barriers).  Thread t owns the 8-element chunks
// c = t, t+nt, ... (nt = all threads without RMSNorm, the first 256 with it)
// and keeps them in registers, so the row is read once (with RMSNorm and
// more than BN_QUANT_STREAM_BYTES of x per thread, quant_row_norm_stream
// reads it in three passes instead).  Writes x_q through
// xq_row (global or shared memory; complete and visible to the whole CTA on
// return); returns max|h| and sum(x_q) to every thread.  COHERENT reads the
// row through L2 only, for a row that other CTAs of the same kernel wrote.
//
// The work is a chain of dependent steps, so the code keeps the chain short:
// the row and the gain are requested together at the start (one memory
// round trip), and each of the three reductions (sum of squares, max|h|,
// sum of x_q) costs one CTA barrier.  For the sum of squares every warp
// evaluates the same fixed tree from the 256 per-thread sums in shared
// memory -- level 128, 64 and 32 pairings, then shuffles 16 .. 1 -- so each
// warp obtains the norm itself, with the oracle's order of additions.
// Consecutive calls may reuse the scratch: every write to a scratch array
// comes after a barrier that all readers of its previous contents passed.
// NT: the threads taking part are the NT threads from T0 on (T0 a multiple of
// 32; synchronised by named barrier 1), or all of the CTA's when NT == 0.
// MAXC == 0 instantiates the streamed RMSNorm path alone (gain required): a
// kernel built for long normalised rows then carries no register-resident
// chunk arrays, which otherwise shape the register allocation of the rest of
// the kernel even where they are never used.
template <typename T, int MAXC, bool COHERENT = false, int NT = 0, int T0 = 0>
BN_DEV void quant_row_cta(const T* __restrict__ row, int K, const T* __restrict__ gain, float rms_eps,
                          int8_t* xq_row, QuantScratch& sc, float& amax_out, int& sum_out);

template <typename T, int MAXC, bool COHERENT, int NT, int T0>
BN_DEV void quant_row_regs(const T* __restrict__ row, int K, const T* __restrict__ gain, float rms_eps,
                           int8_t* xq_row, QuantScratch& sc, float& amax_out, int& sum_out) {
  static_assert(T0 % 32 == 0 && (T0 == 0 || NT != 0), "a thread offset needs a fixed thread count");
  if constexpr (sizeof(Chunk8<T>) * MAXC > BN_QUANT_STREAM_BYTES) {
    if (gain != nullptr) {
      quant_row_norm_stream<T, COHERENT, NT, T0>(row, K, gain, rms_eps, xq_row, sc, amax_out, sum_out);
      return;
    }
  }
  const int t = static_cast<int>(threadIdx.x) - T0;
  const int lane = t & 31, warp = t >> 5;
  const int nthreads = NT == 0 ? static_cast<int>(blockDim.x) : NT;
  const int nwarps = nthreads >> 5;
  // Without RMSNorm nothing depends on which thread owns which chunk (max and
  // integer sums are order-free), so every thread of the CTA takes part; with
  // it, the first 256 threads keep the fixed ownership the summation order is
  // defined on.
  const int nt = gain == nullptr ? nthreads : kQuantThreads;
  const int nchunks = t < nt ? (K >> 3) : 0;  // threads beyond nt own no chunk
  // The gain stays in registers when that is cheap, else it is prefetched
  // into L1 and read again there.
  constexpr bool kGainRegs = sizeof(Chunk8<T>) * MAXC <= 64;

  Chunk8<T> ch[MAXC];
  Chunk8<T> gch[kGainRegs ? MAXC : 1];
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = t + nt * i;
    if (c < nchunks) {
      if constexpr (COHERENT) ch[i].load_cg(row + 8 * c);
      else ch[i].load(row + 8 * c);
      if (gain != nullptr) {
        if constexpr (kGainRegs) gch[i].load(gain + 8 * c);
        else prefetch_l1(gain + 8 * c);
      }
    }
  }
  auto gain_chunk = [&](int i, int c) {
    if constexpr (kGainRegs) {
      return gch[i];
    } else {
      Chunk8<T> g;
      g.load(gain + 8 * c);
      return g;
    }
  };

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
    if (t < kQuantThreads) sc.red[t] = ss;
    sync_threads<NT>();
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

  // h = RN32(RN32(v * r) * g) or v; amax = max |h| (order-free).
  float amax = 0.0f;
  if constexpr (sizeof(T) == 2) {
    if (gain == nullptr) {
      // bf16 without a norm: |v| orders like the bit pattern with the sign
      // cleared, so two values take one 16-bit integer max.
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        const int c = t + nt * i;
        if (c < nchunks) {
          const uint4 u = reinterpret_cast<const uint4&>(ch[i]);
          m2 = max_u16x2(m2, u.x & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, u.y & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, u.z & 0x7FFF7FFFu);
          m2 = max_u16x2(m2, u.w & 0x7FFF7FFFu);
        }
      }
      const uint32_t mb = (m2 & 0xFFFFu) > (m2 >> 16) ? (m2 & 0xFFFFu) : (m2 >> 16);
      amax = __uint_as_float(mb << 16);
    }
  }
  // The branch on the gain is taken once, outside the element loops.
  auto amax_chunks = [&](auto has_gain) {
    constexpr bool HG = decltype(has_gain)::value;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = t + nt * i;
      if (c < nchunks) {
        Chunk8<T> g;
        if constexpr (HG) g = gain_chunk(i, c);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = ch[i].get(e);
          const float h = HG ? __fmul_rn(__fmul_rn(v, r), g.get(e)) : v;
          amax = fmaxf(amax, fabsf(h));
        }
      }
    }
  };
  if (gain != nullptr) amax_chunks(std::true_type{});
  else if (sizeof(T) != 2) amax_chunks(std::false_type{});
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if (lane == 0) sc.amx[warp] = amax;
  sync_threads<NT>();
  amax = lane < nwarps ? sc.amx[lane] : 0.0f;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));

  int sum = 0;
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax);
  auto quantise_chunks = [&](auto has_gain) {
    constexpr bool HG = decltype(has_gain)::value;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = t + nt * i;
      if (c < nchunks) {
        uint32_t lo = 0, hi = 0;
        if (amax != 0.0f) {
          Chunk8<T> g;
          if constexpr (HG) g = gain_chunk(i, c);
          uint32_t q[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v = ch[i].get(e);
            const float h = HG ? __fmul_rn(__fmul_rn(v, r), g.get(e)) : v;
            q[e] = f32_to_s8_rne_bits(__fmul_rn(h, s));
          }
          lo = pack4_s8(q[0], q[1], q[2], q[3]);
          hi = pack4_s8(q[4], q[5], q[6], q[7]);
          sum = __dp4a(static_cast<int>(lo), 0x01010101, sum);
          sum = __dp4a(static_cast<int>(hi), 0x01010101, sum);
        }
        *reinterpret_cast<uint2*>(xq_row + 8 * c) = make_uint2(lo, hi);
      }
    }
  };
  if (gain != nullptr) quantise_chunks(std::true_type{});
  else quantise_chunks(std::false_type{});
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) sc.ired[warp] = sum;
  sync_threads<NT>();
  int tot = lane < nwarps ? sc.ired[lane] : 0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  amax_out = amax;
  sum_out = tot;
}

template <typename T, int MAXC, bool COHERENT, int NT, int T0>
BN_DEV void quant_row_cta(const T* __restrict__ row, int K, const T* __restrict__ gain, float rms_eps,
                          int8_t* xq_row, QuantScratch& sc, float& amax_out, int& sum_out) {
  if constexpr (MAXC == 0) {
    static_assert(T0 % 32 == 0 && (T0 == 0 || NT != 0), "a thread offset needs a fixed thread count");
    quant_row_norm_stream<T, COHERENT, NT, T0>(row, K, gain, rms_eps, xq_row, sc, amax_out, sum_out);
  } else {
    quant_row_regs<T, MAXC, COHERENT, NT, T0>(row, K, gain, rms_eps, xq_row, sc, amax_out, sum_out);
  }
}

// Standalone kernel: one CTA per token row.  256 threads with RMSNorm (the
// fixed summation order is defined on 256 lanes); without it the launcher
// takes the fewest whole warps that give every thread the same number of
// chunks (160 threads x 2 chunks for K = 2560, 224 x 4 for K = 6912).
// early: every CTA of the grid is resident at once (a decode-sized batch),
// so the next kernel on the stream may be launched right away -- the
// product kernels then fetch their weights while this one runs; with more
// rows than fit at once, the next kernel launches once every CTA is past
// its quantisation, so that it takes no SM from the rows still waiting.
template <typename T, int MAXC, int NTHR = kQuantThreads>
__global__ void __launch_bounds__(NTHR) quant_act_kernel(const T* __restrict__ x, int K,
                                                                  const T* __restrict__ gain, float rms_eps,
                                                                  int8_t* __restrict__ xq, float* __restrict__ a_out,
                                                                  int32_t* __restrict__ rowsum_out, int early) {
  __shared__ QuantScratch sc;
  const int64_t m = blockIdx.x;
  if (early) pdl_launch_dependents();
  pdl_wait();
  float amax;
  int sum;
  quant_row_cta<T, MAXC>(x + m * K, K, gain, rms_eps, xq + m * K, sc, amax, sum);
  if (!early) pdl_launch_dependents();
  if (threadIdx.x == 0) {
    a_out[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    if (rowsum_out != nullptr) rowsum_out[m] = sum;
  }
}

}  // namespace bitnet
