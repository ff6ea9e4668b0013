// Decode product for ONE token (M = 1) on CUDA cores, streaming each CTA's
// share of the packed weights in whole-row slots.
//
// Arithmetic as gemv.cuh (the ternary product as the exact integer
// add/subtract of the activations, Habr repost on juhe.plus, "Когда - три
// лучше двух"; one dp4a per 4 weights on the in-place masked 2-bit fields,
// the row sum of x_q subtracted once per output).  What differs is how the
// weights reach the SM.  At one token the kernel does one dp4a per four
// weights, so it must take its weights at the SM's share of HBM bandwidth
// (about 23 bytes per clock) with little work per byte, and two costs
// dominate if nothing is done about them: the issue cost of a bulk copy
// (tens of ns each, whatever its size) and shared-memory bandwidth.  Hence:
//
//   * CTA c owns the contiguous rows [N*c/G, N*(c+1)/G) (G = grid, one CTA
//     per SM), i.e. one contiguous byte range of W_packed.  It streams that
//     range in slots of R whole rows (about 40 KB, ONE bulk copy each)
//     through a ring of `nslots` slots shared by the CTA.  The first slots
//     are requested before the dependency wait (programmatic dependent
//     launch: the weights never depend on the previous kernel), and with
//     l2_prefetch the rest of the range is requested into L2 at the same
//     time, so HBM keeps streaming across the kernel boundary.
//   * A row of K/4 bytes is cut into S column segments; warp w takes
//     segment w % S of the rows w / S, w / S + 16/S, ... of every slot, two
//     rows at a time (twice the independent loads and dp4a chains).  Lane l
//     of the warp owns the word pairs 2l + 64p (p < NP) of its segment, and
//     keeps the matching 32 bytes of x_q per pair in REGISTERS for the whole
//     launch: shared memory carries only the 2-bit codes (a quarter byte per
//     weight), and one 16-weight code word costs half an 8-byte shared load,
//     four masks and four dp4a.  Words past the segment have x_q = 0.
//   * A row's partial sums are reduced across the warp (one redux) and
//     stored to the row's slot for that segment; the epilogue adds the S
//     segments (integers: exact, in any order).  Each warp arrives on the
//     slot's "empty" barrier when done with it, and the last one refills it
//     (no warp ever waits for another to free a slot, and only the warps that
//     see the slot free take part in a one-atomic election).
//   * After the last slot, the CTA dequantises its rows and stores them.
//
// FUSED: the kernel quantises the token row itself after the dependency
// wait (quant_row_cta, the same arithmetic and order as bitnet_quant_act)
// into shared memory, then takes its registers' x_q from there.
#pragma once

#include <cuda_bf16.h>

#include "gemv.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kGemv1MaxPairs = 4;     // word pairs a lane keeps x_q for in registers (8 words, 32 registers)
constexpr int kGemv1MaxSlots = 8;     // ring slots (at most)
constexpr int kGemv1BarBytes = 256;   // full and empty barriers, refill elections, issue counts

// Dynamic shared memory of gemv1_kernel: ring, barrier block, the row sums
// per column segment (S x rows_max, twice with GATE) and (FUSED) x_q.
__host__ __device__ constexpr int gemv1_acc_bytes(int rows_max, int S, bool gate = false) {
  return (((gate ? 2 : 1) * S * rows_max * 4 + 15) / 16) * 16;
}
__host__ __device__ constexpr int gemv1_smem_bytes(int K, bool xs, int slot_bytes, int nslots, int rows_max, int S,
                                                  bool gate = false) {
  return nslots * slot_bytes + kGemv1BarBytes + gemv1_acc_bytes(rows_max, S, gate) + (xs ? K : 0);
}

// NWARPS: 16 (two CTAs per SM, so that consecutive launches overlap) or 32
// (one CTA per SM with a deeper ring).
// GATE: the FFN's up and gate projections at once (Wp = W_up, Wp2 = W_gate,
// the same N x K shape): a slot holds R rows of W_up then the same R rows of
// W_gate, a pass takes up row r and gate row r against the same x_q
// registers, and the epilogue writes h = bf16(RN32(RN32(r*r)*u)), r = g if
// g > 0 else +0 (u, g dequantised as the plain product's fp32 output) to y
// (bf16, M = 1 x N) -- the squared-ReLU gate of the FFN (inferownia.pl,
// "BitNet b1.58: era 1-bitowych LLM-ów", "Zrób to sam"; kripta.biz 2B4T news).
// NP: word pairs per lane (segments of at most 64 * NP words).  S: column
// segments per row (a power of two <= 16; a segment is ceil(K/16 / S)
// words rounded up to even); R: rows per slot; nslots: ring depth; rows_max
// = ceil(N / gridDim.x); l2_prefetch: request the part of the CTA's range
// beyond the ring into L2 up front.
template <bool U8, int NP, int NWARPS, bool FUSED = false, typename T = float, int MAXC = 1, bool GATE = false>
__global__ void __launch_bounds__(NWARPS * 32, 1024 / (NWARPS * 32))
    gemv1_kernel(const uint8_t* __restrict__ Wp, const float* __restrict__ gamma_ptr,
                 const uint8_t* __restrict__ Wp2, const float* __restrict__ gamma2_ptr, int N, int K,
                 const int8_t* __restrict__ xq, const float* __restrict__ a_scale,
                 const int32_t* __restrict__ rowsum, const T* __restrict__ xin, const T* __restrict__ gain,
                 float rms_eps, void* __restrict__ y, int y_dtype, int S, int R, int nslots, int rows_max,
                 int l2_prefetch) {
  static_assert(!FUSED || U8, "the fused kernel computes the row sum of x_q");
  static_assert(!GATE || U8, "the gated kernel takes the row sum of x_q");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int B = K >> 2;  // bytes per packed row
  const int slot_bytes = (GATE ? 2 : 1) * R * B;  // GATE: R up rows, then the same R gate rows
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + nslots * slot_bytes);
  uint64_t* empty = full + kGemv1MaxSlots;
  unsigned int* elect = reinterpret_cast<unsigned int*>(empty + kGemv1MaxSlots);
  unsigned int* issued = elect + kGemv1MaxSlots;
  int* failed = reinterpret_cast<int*>(issued + kGemv1MaxSlots);
  int* accs = reinterpret_cast<int*>(smem + nslots * slot_bytes + kGemv1BarBytes);
  uint8_t* xs = smem + nslots * slot_bytes + kGemv1BarBytes + gemv1_acc_bytes(rows_max, S, GATE);

  const int64_t row_lo = static_cast<int64_t>(N) * blockIdx.x / gridDim.x;
  const int64_t row_hi = static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x;
  const int nrows = static_cast<int>(row_hi - row_lo);
  const int nsl = (nrows + R - 1) / R;  // slots of this CTA
  const uint8_t* wbase = Wp + row_lo * B;
  const uint8_t* wbase2 = GATE ? Wp2 + row_lo * B : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nslots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NWARPS);
      elect[s] = 0;
      issued[s] = 0;
    }
    *failed = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const uint64_t policy = policy_evict_first();
  // Slot j of this CTA: rows [j*R, min(nrows, (j+1)*R)), one contiguous copy.
  auto issue = [&](int j) {
    const int s = j % nslots;
    const int r0 = j * R;
    const int nr = nrows - r0 < R ? nrows - r0 : R;
    const uint32_t bytes = static_cast<uint32_t>(nr) * static_cast<uint32_t>(B);
    issued[s] += 1u;
    mbar_arrive_expect_tx(&full[s], GATE ? 2 * bytes : bytes);
    bulk_copy_g2s(ring + s * slot_bytes, wbase + static_cast<int64_t>(r0) * B, bytes, &full[s], policy);
    if constexpr (GATE)
      bulk_copy_g2s(ring + s * slot_bytes + R * B, wbase2 + static_cast<int64_t>(r0) * B, bytes, &full[s], policy);
  };
  if (threadIdx.x == 0)
    for (int j = 0; j < nslots && j < nsl; ++j) issue(j);
  if (l2_prefetch && lane == 0) {
    // the part of the range beyond the ring, one slice per warp
    const int64_t share = static_cast<int64_t>(nrows) * B;
    const int64_t ring_part = static_cast<int64_t>(nslots) * R * B;
    const int64_t from = ring_part < share ? ring_part : share;
    const int64_t slice = ((share - from) / NWARPS + 15) / 16 * 16;
    const int64_t lo = from + slice * warp;
    const int64_t hi = lo + slice < share ? lo + slice : share;
    for (int64_t o = lo; o < hi; o += 65536) {
      const int64_t n = hi - o < 65536 ? hi - o : 65536;
      bulk_prefetch_l2(wbase + o, static_cast<uint32_t>(n));
      if constexpr (GATE) bulk_prefetch_l2(wbase2 + o, static_cast<uint32_t>(n));
    }
  }

  // Everything below reads the outputs of the previous kernel.
  pdl_launch_dependents();
  pdl_wait();
  const float gamma = __ldg(gamma_ptr);
  const int Bw = B >> 2;  // 16-weight code words per row (a multiple of 4)
  const int segw = ((Bw + S - 1) / S + 1) & ~1;  // words per segment, even: 8-byte pair loads
  const int seg = warp % S, grp = warp / S, RG = NWARPS / S;
  const int c_lo = seg * segw;
  const int c_hi = c_lo + segw < Bw ? c_lo + segw : Bw;
  // Lane l's words: the pairs c_lo + 2l + 64p (+0, +1), p < NP.  Words past
  // the segment get x = 0 (they add nothing) and read a valid pair of the row.
  float asc;
  int rsum;
  uint4 xr[2 * NP];
  uint32_t woff[NP];  // byte offset of each pair inside a row
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int c = c_lo + 2 * lane + 64 * p;
    woff[p] = 4u * static_cast<uint32_t>(c < Bw - 2 ? c : Bw - 2);
  }
  if constexpr (FUSED) {
    __shared__ QuantScratch qsc;
    float amax;
    int sum;
    quant_row_cta<T, MAXC>(xin, K, gain, rms_eps, reinterpret_cast<int8_t*>(xs), qsc, amax, sum);
    asc = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    rsum = sum;
    // (x_q in shared memory is complete: quant_row_cta ends with a CTA barrier)
#pragma unroll
    for (int i = 0; i < 2 * NP; ++i) {
      const int c = c_lo + 2 * lane + 64 * (i >> 1) + (i & 1);
      xr[i] = c < c_hi ? lds128(smem_addr(xs) + 16 * c) : make_uint4(0, 0, 0, 0);
    }
  } else {
    asc = __ldg(a_scale);
    rsum = U8 ? __ldg(rowsum) : 0;
#pragma unroll
    for (int i = 0; i < 2 * NP; ++i) {
      const int c = c_lo + 2 * lane + 64 * (i >> 1) + (i & 1);
      xr[i] = c < c_hi ? __ldg(reinterpret_cast<const uint4*>(xq) + c) : make_uint4(0, 0, 0, 0);
    }
  }

  // One row's partial dot product over this lane's words (4 in-place fields
  // per word for U8, each an exact multiple of 4^j; signed codes otherwise).
  auto row_dot = [&](const uint2 (&w)[NP]) {
    int f0 = 0, f1 = 0, f2 = 0, f3 = 0;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ww = h ? w[p].y : w[p].x;
        const uint4 xv = xr[2 * p + h];
        if constexpr (U8) {
          // field j of byte b is weight 4j + b, met in place (4^j * code)
          f0 = dp4a_us(ww & 0x03030303u, xv.x, f0);
          f1 = dp4a_us(ww & 0x0C0C0C0Cu, xv.y, f1);
          f2 = dp4a_us(ww & 0x30303030u, xv.z, f2);
          f3 = dp4a_us(ww & 0xC0C0C0C0u, xv.w, f3);
        } else {
          f0 = dp4a_ss(codes_to_signed(ww & 0x03030303u), xv.x, f0);
          f1 = dp4a_ss(codes_to_signed((ww >> 2) & 0x03030303u), xv.y, f1);
          f2 = dp4a_ss(codes_to_signed((ww >> 4) & 0x03030303u), xv.z, f2);
          f3 = dp4a_ss(codes_to_signed((ww >> 6) & 0x03030303u), xv.w, f3);
        }
      }
    }
    return U8 ? f0 + (f1 >> 2) + (f2 >> 4) + (f3 >> 6) : f0 + f1 + f2 + f3;
  };

  int* part = accs;  // [S][rows_max]: each row's sum per column segment
  for (int j = 0; j < nsl; ++j) {
    const int s = j % nslots;
    const int r0 = j * R;
    const int nr = nrows - r0 < R ? nrows - r0 : R;
    // A warp that gave up stops the others at their next slot (its slots are never refilled).
    if (*reinterpret_cast<volatile int*>(failed)) break;
    // Every lane acquires the barrier itself; the warp leaves together if any gave up.
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (j / nslots) & 1))) {
      if (lane == 0) *failed = 1;
      break;
    }
    const uint32_t sbase = smem_addr(ring + s * slot_bytes);
    // two rows at a time: r and r + RG, or (GATE) up row r and gate row r -- twice the
    // independent loads and chains
    for (int r = grp; r < nr; r += (GATE ? 1 : 2) * RG) {
      const bool two = GATE || r + RG < nr;
      const uint32_t rb0 = sbase + r * B;
      const uint32_t rb1 = GATE ? rb0 + R * B : (two ? rb0 + RG * B : rb0);
      uint2 w0[NP], w1[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0[p].x), "=r"(w0[p].y) : "r"(rb0 + woff[p]));
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w1[p].x), "=r"(w1[p].y) : "r"(rb1 + woff[p]));
      }
      const int v0 = __reduce_add_sync(0xffffffffu, row_dot(w0));
      const int v1 = __reduce_add_sync(0xffffffffu, row_dot(w1));
      if (lane == 0) {
        part[seg * rows_max + r0 + r] = v0;
        if constexpr (GATE) part[(S + seg) * rows_max + r0 + r] = v1;  // the gate rows' sums after the up rows'
        else if (two) part[seg * rows_max + r0 + r + RG] = v1;
      }
    }
    __syncwarp();
    if (lane == 0 && j + nslots < nsl) {
      // This warp's reads of the slot are done (the arrival releases them).  A
      // warp that then finds the phase complete (acquire: every warp's reads
      // came first) -- always the last to arrive, rarely one more -- takes
      // part in an election for the refill (a compare-and-swap from the fill's
      // number: one winner per fill); the winner issues it.
      mbar_arrive(&empty[s]);
      const unsigned int fill = static_cast<unsigned int>(j / nslots);
      if (mbar_test_wait(&empty[s], fill & 1u) && atomicCAS(&elect[s], fill, fill + 1u) == fill) {
        fence_proxy_async_smem();
        issue(j + nslots);
      }
    }
  }
  __syncthreads();
  if (*failed) {
    // Let the copies in flight land before the CTA's shared memory goes away.
    if (threadIdx.x == 0)
      for (int s = 0; s < nslots; ++s)
        if (issued[s] > 0) mbar_wait(&full[s], (issued[s] - 1u) & 1u);
    return;
  }
  if constexpr (GATE) {
    const float gamma2 = __ldg(gamma2_ptr);
    for (int i = threadIdx.x; i < nrows; i += NWARPS * 32) {
      int au = -rsum, ag = -rsum;
      for (int g = 0; g < S; ++g) {
        au += part[g * rows_max + i];
        ag += part[(S + g) * rows_max + i];
      }
      const float u = __fmul_rn(__fmul_rn(__int2float_rn(au), gamma), asc);
      const float g = __fmul_rn(__fmul_rn(__int2float_rn(ag), gamma2), asc);
      const float r = g > 0.0f ? g : 0.0f;
      static_cast<__nv_bfloat16*>(y)[row_lo + i] = __float2bfloat16_rn(__fmul_rn(__fmul_rn(r, r), u));
    }
  } else {
    for (int i = threadIdx.x; i < nrows; i += NWARPS * 32) {
      int a = -rsum;
      for (int g = 0; g < S; ++g) a += part[g * rows_max + i];
      const int64_t o = row_lo + i;
      if (y_dtype == 2) {
        static_cast<int32_t*>(y)[o] = a;
      } else {
        const float v = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), asc);
        if (y_dtype == 0) static_cast<float*>(y)[o] = v;
        else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
      }
    }
  }
}

}  // namespace bitnet
