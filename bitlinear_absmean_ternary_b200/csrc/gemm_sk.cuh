// W1.58A8 product for decode-sized batches (M <= 64 tokens) on the Blackwell
// tensor cores, balanced by splitting the work stream, not the tiles.
//
// Same operands and arithmetic as gemm.cuh (the pages' "low-bit matrix
// product followed by rescaling", comrad404.com review, "Метод: как устроен
// BitNet b1.58"): A = the ternary codes of 128 weight rows expanded to 8 bits
// in registers and written to tensor memory, B = the int8 activations of the
// BN token columns in shared memory (128-byte swizzled, K-major), int32
// accumulators in tensor memory, 256 bytes of K per stage (8 MMAs of K = 32).
//
// At these sizes the product is bound by streaming the packed weights from
// HBM (Habr repost on juhe.plus, "Но есть одно - НО": the weights are the
// cost), so the design keeps every SM streaming an equal share of them:
//
//   * Work split (stream-K): the units are (row tile, K stage) pairs in
//     tile-major order, U = ceil(N/128) * ceil(K/256) of them, and CTA c of
//     the G CTAs (one per SM) takes the contiguous range [U*c/G, U*(c+1)/G).
//     A range is a run of segments, one per row tile it touches.  A tile
//     that lies wholly in one range is finished by that CTA.  A tile cut by
//     range boundaries has one "finisher", the CTA holding its first K stage
//     (the tile is the last segment of that CTA's range), and helpers, the
//     later CTAs holding its other stages (for each helper the tile is its
//     FIRST segment, so a CTA is the helper of at most one tile).  A helper
//     adds its int32 partial tile into the finisher's slot of the workspace
//     with reductions at L2 (integer adds: exact and order-free, and the
//     helpers' latencies overlap instead of adding up at the finisher) and
//     raises its flag; the finisher, which reaches the tile last, waits for
//     the flags of its helpers, reads the summed partials once (the result is
//     bit-identical to an unsplit product), dequantises, stores y and zeroes
//     its slot and the flags again, so the workspace is all zero between
//     calls.
//
//   * Feed: the packed weights have a ring of their own (SW stages of 8 KB),
//     freed as soon as the unpack warps have read a stage into registers, so
//     the weight producer runs SW stages ahead of the tensor-memory writes.
//     Its first SW stages are requested before waiting on the previous
//     kernel (programmatic dependent launch): the weights never depend on it.
//     The activations (a few KB per stage, read from L2) come through a
//     shallower ring freed by the MMA commits.  The unpacked A operand has T
//     tensor-memory slots of 64 columns, freed by the MMA commits.
//
//   * Token tiles: the tiles are (row tile, token tile) pairs, row tiles
//     fastest, so consecutive units share their activation tile in L2.
//
//   * XT (fused quantisation, bitnet_bitlinear_gemm, M <= 64: the four
//     BitLinear steps of the comrad404.com review, "Метод", in one launch):
//     the unpack warps (256 threads: the fixed 256-lane order of the RMSNorm
//     sum) of CTA c quantise the token rows c, c+G, ... into the workspace
//     (x_q, scales, row sums), while every CTA's weight producer already
//     streams.  A sense-reversal grid barrier in the workspace (arrival
//     count, generation) then releases the activation producers and the
//     epilogues of all CTAs: every CTA of the launch is resident at once (one
//     per SM), and every wait is bounded.
//
//   * GATE (the FFN's up and gate projections in one product, inferownia.pl,
//     "BitNet b1.58: era 1-bitowych LLM-ów", "Zrób to sam": squared ReLU in
//     the FFN; kripta.biz 2B4T news: ReLU^2 in the FFN layers): a tile is 64
//     features, its rows 0..63 the up rows and 64..127 the gate rows of those
//     features (two 64-row weight boxes per stage), so the epilogue holds u
//     and g of every feature: the gate quarters dequantise g into shared
//     memory and the up quarters write h = bf16(RN32(RN32(r*r)*u)), r = g if
//     g > 0 else +0, straight into the down projection's input; u and g never
//     reach memory.
//
// Warp roles (480 threads):
//   warp 0, lane 0     weight producer (TMA, one 128-row x 64-byte box per stage);
//   warp 1, lane 0     activation producer (TMA, two BN x 128-byte boxes per stage);
//   warp 2             tensor-memory allocator; lane 0 issues the MMAs;
//   warps 3..10        unpack: two warps per TMEM lane quarter (warp % 4),
//                      taking alternate stages; thread = weight row;
//   warps 11..14       epilogue, one per lane quarter; thread = weight row.
// Every wait is bounded; a timeout flags the device error word, the role
// stops, and the kernel drains what is in flight and exits.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "gemm.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kSkFirstUnpack = 3;
constexpr int kSkUnpackWarps = 8;
constexpr int kSkFirstEpi = kSkFirstUnpack + kSkUnpackWarps;
constexpr int kSkEpiWarps = 4;
constexpr int kSkThreads = (kSkFirstEpi + kSkEpiWarps) * 32;

template <int BN, bool GATE = false>
struct SkCfg {
  static constexpr int kWStage = kGemmBM * (kGemmBK / 4);  // packed codes of 128 rows x 256 K: 8 KB
  static constexpr int kXSub = BN * 128;                   // one 128-byte-wide activation box
  static constexpr int kXStage = kXSub * (kGemmBK / 128);  // activations of a stage
  static constexpr int SW = BN <= 32 ? 16 : 12;            // weight ring stages
  static constexpr int SX = BN <= 32 ? 8 : 6;              // activation ring stages
  static constexpr int kAslot = kGemmBK / 4;               // TMEM columns per A slot
  static constexpr int kAcol = 2 * BN;                     // two accumulators first
  static constexpr int T = (512 - kAcol) / kAslot;         // A slots in TMEM
  static constexpr int kXOff = SW * kWStage;
  static constexpr int kBarOff = kXOff + SX * kXStage;
  static constexpr int kNumBars = 2 * SW + 2 * SX + 2 * T + 7;
  static constexpr int kScaleOff = kBarOff + ((kNumBars * 8 + 8 + 127) / 128) * 128;
  static constexpr int kGateOff = kScaleOff + 2 * BN * 8;  // (GATE) g of a tile, fp32 [BN][64]
  static constexpr int kRowsPerTile = GATE ? 64 : kGemmBM;  // output features per tile
  static constexpr int kNeeded = 1024 + kGateOff + (GATE ? BN * 64 * 4 : 0);
  // The CTA holds all 512 TMEM columns: ask for enough shared memory that a
  // second CTA never fits on the SM, so none waits in tcgen05.alloc.
  static constexpr int kMinSmem = 233472 / 2;
  static constexpr int kSmemBytes = kNeeded > kMinSmem ? kNeeded : kMinSmem;
  // workspace: G flags (rounded to 256 bytes), then G accumulation slots of kSkSlotInts (this tile
  // uses the first BN x 128 of its slot as int32 [BN][128]), zero between calls
  static_assert(kWStage % 1024 == 0 && kXStage % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(kAcol + T * kAslot <= 512 && T >= 2, "TMEM budget");
  static_assert(kNeeded <= 232448, "shared memory budget");
  static_assert(BN == 16 || BN == 32 || BN == 64, "token tile (at most the slot's 64)");
};

__host__ __device__ inline size_t sk_flag_bytes(int G) { return (static_cast<size_t>(G) * 4 + 255) / 256 * 256; }

// Whether a product of M <= 64 tokens runs stream-K.  Every CTA pays a fixed
// cost (the pipeline's fill, then partial tiles exchanged through L2 and the
// finisher's wait), which a share of a few K steps does not repay: below
// kSkMinUnitsPerCta (row tile, K step) units per SM the tile kernel, which
// exchanges no partials, is faster (measured: the 2.5B-class block's
// matrices, 1.4 to 7.3 units per SM, ran in 7.7 to 10.2 us on tiles against
// 13 to 15.5 us stream-K; the 27B FFN's, 24 units per SM, in 19.3 to 21.6
// us stream-K against 20.6 to 31 us on tiles).
constexpr int kSkMinUnitsPerCta = 12;
inline bool sk_preferred(int64_t M, int64_t N, int64_t K, int sms) {
  if (M > 64) return false;
  const int64_t bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  const int64_t units = ((N + 127) / 128) * ((M + bn - 1) / bn) * ((K + 255) / 256);
  return units >= static_cast<int64_t>(kSkMinUnitsPerCta) * sms;
}

// One accumulation slot per CTA, sized for the widest token tile whatever
// the call's tile, so that calls of any token count can share a workspace
// (each leaves its slots zero).
constexpr int kSkSlotInts = 64 * kGemmBM;
__host__ __device__ inline size_t sk_slot_bytes(int G) { return static_cast<size_t>(G) * kSkSlotInts * 4; }

// CTA (of G) whose unit range [U*c/G, U*(c+1)/G) holds unit u.
__device__ __forceinline__ int sk_cta_of(long long u, long long U, int G) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

// Integer add at L2, no result returned (the helpers' partial tiles).
BN_DEV void red_add_gpu_u32(unsigned int* p, unsigned int v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
BN_DEV void st_release_gpu_u32(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
BN_DEV unsigned int ld_acquire_gpu_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier over the four epilogue warps on an mbarrier of 4 arrivals, with
// a bounded wait (a warp that gave up earlier cannot hang the others).
// `phase` counts the uses; every epilogue warp makes the same calls.
BN_DEV bool sk_epi_sync(uint64_t* bar, int& phase) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, static_cast<uint32_t>(phase & 1));
  ++phase;
  return ok;
}

// In-kernel quantisation of the token rows (XT != void): the unquantised
// rows, the optional RMSNorm gain, where the quantised rows, scales and row
// sums go (the workspace), and the grid barrier's words (arrivals,
// generation; both start at zero, and the barrier leaves the arrival count
// at zero).
template <typename XT>
struct SkQuant {
  const XT* x;
  const XT* gain;
  float eps;
  int8_t* xq;
  float* a;
  int32_t* rs;
  unsigned int* bar;
};
template <typename XT>
using sk_qx_t = std::conditional_t<std::is_void_v<XT>, float, XT>;

BN_DEV unsigned int atom_add_acq_rel_gpu_u32(unsigned int* p, unsigned int v) {
  unsigned int old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Waits (bounded) until the grid barrier's generation differs from gen0.
// Polls back off briefly (__nanosleep), so that the hundreds of waiting
// threads leave the word's L2 line to the arrivals.
BN_DEV bool sk_wait_generation(const unsigned int* gen, unsigned int gen0) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1; ld_acquire_gpu_u32(gen) == gen0; ++i) {
    __nanosleep(64);
    if ((i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
      flag_timeout();
      return false;
    }
  }
  return true;
}

// N: output features (rows of W; for GATE the rows of W_up and of W_gate).
// tmap_w2 / gamma2_ptr: W_gate and its scale (GATE only).  y: M x N outputs
// of y_dtype, or for GATE the bf16 h (M x N).
// XT, MAXC: fused quantisation of x of type XT (void: x_q, a_scale and
// rowsum are given), MAXC 8-element chunks per unpack thread.
template <int BN, bool U8, bool GATE = false, typename XT = void, int MAXC = 1>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_sk_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_w2, const float* __restrict__ gamma_ptr,
                   const float* __restrict__ gamma2_ptr, const float* __restrict__ a_scale,
                   const int32_t* __restrict__ rowsum, int M, int N, int K, void* __restrict__ y, int y_dtype,
                   unsigned int* __restrict__ flags, int* __restrict__ parts, const SkQuant<sk_qx_t<XT>> qa) {
  constexpr bool FQ = !std::is_void_v<XT>;
  static_assert(!FQ || (U8 && !GATE), "the fused quantisation computes the row sums; no gate");
  using C = SkCfg<BN, GATE>;
  constexpr int RPT = C::kRowsPerTile;
  constexpr int SW = C::SW, SX = C::SX, T = C::T;
  constexpr int NMMA = kGemmBK / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* w_full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* w_empty = w_full + SW;
  uint64_t* x_full = w_empty + SW;
  uint64_t* x_empty = x_full + SX;
  uint64_t* a_full = x_empty + SX;
  uint64_t* a_empty = a_full + T;
  uint64_t* acc_full = a_empty + T;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint64_t* epi_bar = done + 1;
  uint64_t* qdone = epi_bar + 1;  // FQ: the generation the grid barrier starts from is in s_gen0
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qdone + 1);
  uint32_t* s_gen0 = tmem_holder + 1;
  float* s_a = reinterpret_cast<float*>(smem + C::kScaleOff);  // [2][BN]: double-buffered per segment
  int* s_rs = reinterpret_cast<int*>(s_a + 2 * BN);           // [2][BN]
  float* gbuf = reinterpret_cast<float*>(smem + C::kGateOff);  // GATE: [BN][64]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + RPT - 1) / RPT;
  const int m_tiles = (M + BN - 1) / BN;
  const int nk = (K + kGemmBK - 1) / kGemmBK;
  const long long U = static_cast<long long>(n_tiles) * m_tiles * nk;
  const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  const long long u0 = U * cta / G, u1 = U * (cta + 1) / G;
  const int total = static_cast<int>(u1 - u0);  // stages of this CTA

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 4);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    for (int s = 0; s < T; ++s) {
      mbar_init(&a_full[s], 4);
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kSkEpiWarps);
    }
    mbar_init(done, 1);
    mbar_init(epi_bar, kSkEpiWarps);
    mbar_init(qdone, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    if constexpr (GATE) tma_prefetch_desc(&tmap_w2);
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ weight producer
      // The packed weights never depend on the previous kernel: no wait at all.
      bool ok = true;
      int g = 0;
      for (; g < total; ++g) {
        const int s = g % SW;
        if (g >= SW && !mbar_wait(&w_empty[s], ((g / SW) & 1) ^ 1)) {
          ok = false;
          break;
        }
        const long long u = u0 + g;
        const long long t = u / nk;
        const int kb = static_cast<int>(u - t * nk);
        const int row0 = static_cast<int>(t % n_tiles) * RPT;
        mbar_arrive_expect_tx(&w_full[s], C::kWStage);
        if constexpr (GATE) {
          // up rows of the tile's 64 features, then their gate rows
          tma_load_2d(smem + s * C::kWStage, &tmap_w, kb * (kGemmBK / 4), row0, &w_full[s]);
          tma_load_2d(smem + s * C::kWStage + C::kWStage / 2, &tmap_w2, kb * (kGemmBK / 4), row0, &w_full[s]);
        } else {
          tma_load_2d(smem + s * C::kWStage, &tmap_w, kb * (kGemmBK / 4), row0, &w_full[s]);
        }
      }
      if (!ok)  // let the copies in flight land before the shared memory goes away
        for (int h = g - SW > 0 ? g - SW : 0; h < g; ++h) mbar_wait(&w_full[h % SW], (h / SW) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ activation producer
      pdl_wait();  // x_q comes from the previous kernel
      bool ok = true;
      if constexpr (FQ) {
        // x_q comes from this launch: wait for every CTA's quantisation
        ok = mbar_wait(qdone, 0) && sk_wait_generation(qa.bar + 1, *s_gen0);
        asm volatile("fence.proxy.async.global;" ::: "memory");  // generic writes -> TMA reads
      }
      int g = 0;
      for (; ok && g < total; ++g) {
        const int s = g % SX;
        if (g >= SX && !mbar_wait(&x_empty[s], ((g / SX) & 1) ^ 1)) {
          ok = false;
          break;
        }
        const long long u = u0 + g;
        const long long t = u / nk;
        const int kb = static_cast<int>(u - t * nk);
        const int m0 = static_cast<int>(t / n_tiles) * BN;
        uint8_t* xs = smem + C::kXOff + s * C::kXStage;
        mbar_arrive_expect_tx(&x_full[s], C::kXStage);
#pragma unroll
        for (int i = 0; i < kGemmBK / 128; ++i)
          tma_load_2d(xs + i * C::kXSub, &tmap_x, kb * kGemmBK + 128 * i, m0, &x_full[s]);
      }
      if (!ok)
        for (int h = g - SX > 0 ? g - SX : 0; h < g; ++h) mbar_wait(&x_full[h % SX], (h / SX) & 1);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_i8(kGemmBM, BN, !U8);
      bool ok = true;
      int g = 0, seg = 0;
      for (long long u = u0; ok && u < u1; ++seg) {
        const long long t = u / nk;
        const long long seg_end = (t + 1) * nk < u1 ? (t + 1) * nk : u1;
        const int b = seg & 1;
        if (!mbar_wait(&acc_empty[b], ((seg >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (long long v = u; v < seg_end; ++v, ++g) {
          const int a = g % T, sx = g % SX;
          if (!mbar_wait(&a_full[a], (g / T) & 1) || !mbar_wait(&x_full[sx], (g / SX) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xaddr = smem_addr(smem + C::kXOff + sx * C::kXStage);
#pragma unroll
          for (int kk = 0; kk < NMMA; ++kk)
            mma_i8_tmemA(tmem + b * BN, tmem + C::kAcol + C::kAslot * a + 8 * kk,
                         smem_desc_k_sw128(xaddr + (kk >> 2) * C::kXSub + 32 * (kk & 3)), idesc,
                         (v > u || kk > 0) ? 1u : 0u);
          tc_commit(&a_empty[a]);
          tc_commit(&x_empty[sx]);
        }
        if (ok) tc_commit(&acc_full[b]);
        u = seg_end;
      }
      tc_commit(done);  // arrives once every MMA issued above has finished
      mbar_wait(done, 0);
    }
  } else if (warp < kSkFirstEpi) {
    // ------------------------------------------------------------ unpack
    if constexpr (FQ) {
      // first the quantisation of the token rows cta, cta + G, ... (256 threads: the
      // unpack warps are threads 96 .. 351), then one arrival on the grid barrier
      __shared__ QuantScratch qsc;
      constexpr int kT0 = kSkFirstUnpack * 32;
      const int ut = static_cast<int>(threadIdx.x) - kT0;
      pdl_wait();
      unsigned int gen0 = 0;
      if (ut == 0) {
        gen0 = *reinterpret_cast<volatile unsigned int*>(qa.bar + 1);
        *s_gen0 = gen0;
        mbar_arrive(qdone);
      }
      for (int m = cta; m < M; m += G) {
        float amax;
        int sum;
        quant_row_cta<sk_qx_t<XT>, MAXC, false, 256, kT0>(qa.x + static_cast<int64_t>(m) * K, K, qa.gain, qa.eps,
                                                          qa.xq + static_cast<int64_t>(m) * K, qsc, amax, sum);
        if (ut == 0) {
          qa.a[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
          qa.rs[m] = sum;
        }
      }
      __threadfence();
      sync_threads<256>();
      if (ut == 0) {
        const unsigned int old = atom_add_acq_rel_gpu_u32(qa.bar, 1u);
        if (old == static_cast<unsigned int>(G) - 1u) {
          qa.bar[0] = 0u;  // the last arrival: count back to zero, then the new generation
          st_release_gpu_u32(qa.bar + 1, gen0 + 1u);
        }
      }
    }
    const int q = warp & 3;
    const int par = (warp - kSkFirstUnpack) >> 2;  // this warp takes stages with g % 2 == par
    const int r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    // 64-byte swizzle of the packed tile: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
    const uint32_t swz = static_cast<uint32_t>((r >> 1) & 3);
    for (int g = par; g < total; g += 2) {
      const int s = g % SW;
      if (!__all_sync(0xffffffffu, mbar_wait(&w_full[s], (g / SW) & 1))) break;
      const uint32_t wrow = smem_addr(smem + s * C::kWStage) + r * (kGemmBK / 4);
      uint4 p[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) p[c] = lds128(wrow + ((static_cast<uint32_t>(c) ^ swz) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(&w_empty[s]);  // the weight slot may be refilled
      const int a = g % T;
      if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[a], ((g / T) & 1) ^ 1))) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // two halves of 128 K each -> 32 TMEM columns each
        const uint32_t pw[8] = {p[2 * h].x, p[2 * h].y, p[2 * h].z, p[2 * h].w,
                                p[2 * h + 1].x, p[2 * h + 1].y, p[2 * h + 1].z, p[2 * h + 1].w};
        uint32_t v[32];
#pragma unroll
        for (int wi = 0; wi < 8; ++wi)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t c4 = (pw[wi] >> (2 * j)) & 0x03030303u;
            v[4 * wi + j] = U8 ? c4 : codes_to_signed(c4);
          }
        tmem_st_32x32b_x32(lane_base + C::kAcol + C::kAslot * a + 32 * h, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[a]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;  // accumulator row (TMEM lane) of this thread
    const int et = (warp - kSkFirstEpi) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    pdl_wait();  // a_scale, rowsum and the workspace follow the previous kernel
    // row r's scale: W_up's (or W's) for the first 64 rows of a gated tile, W_gate's for the others
    const float gamma = (GATE && r >= 64) ? __ldg(gamma2_ptr) : __ldg(gamma_ptr);
    int ephase = 0;
    if constexpr (FQ) {
      // the scales and row sums come from this launch's quantisation (every CTA's)
      if (et == 0) {
        if (mbar_wait(qdone, 0)) sk_wait_generation(qa.bar + 1, *s_gen0);
      }
      sk_epi_sync(epi_bar, ephase);
    }
    int seg = 0;
    for (long long u = u0; u < u1; ++seg) {
      const long long t = u / nk;
      const int kb_lo = static_cast<int>(u - t * nk);
      const long long seg_end = (t + 1) * nk < u1 ? (t + 1) * nk : u1;
      const int kb_hi = static_cast<int>(seg_end - t * nk);
      u = seg_end;
      const int m0 = static_cast<int>(t / n_tiles) * BN;
      const int f0 = static_cast<int>(t % n_tiles) * RPT;
      const int sb = (seg & 1) * BN;  // this segment's half of the scale buffers
      if (et < BN) {  // requested before the accumulator wait, so the loads overlap it
        const int m = m0 + et;
        s_a[sb + et] = m < M ? __ldcg(a_scale + m) : 0.0f;
        s_rs[sb + et] = (U8 && m < M) ? __ldcg(rowsum + m) : 0;
      }
      const int b = seg & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[b], (seg >> 1) & 1))) break;
      tc_fence_after();
      uint32_t v[BN];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t w16[16];
        tmem_ld_32x32b_x16(lane_base + b * BN + c0, w16);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) v[c0 + j] = w16[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);  // the accumulator may be reused
      if (kb_lo > 0) {
        // helper: this CTA's partial of a tile finished by an earlier CTA (the one holding the tile's
        // first stage), added into that finisher's accumulation slot [BN][128] by integer reductions at
        // L2 -- exact and order-free, and none of the helpers' latencies adds up at the finisher
        unsigned int* acc = reinterpret_cast<unsigned int*>(parts) +
                            static_cast<size_t>(sk_cta_of(t * nk, U, G)) * kSkSlotInts;
#pragma unroll
        for (int j = 0; j < BN; ++j) red_add_gpu_u32(acc + j * kGemmBM + r, v[j]);
        __threadfence();
        if (sk_epi_sync(epi_bar, ephase) && et == 0) st_release_gpu_u32(&flags[cta], 1u);
        continue;
      }
      if (kb_hi < nk) {
        // finisher: add the partials of the helpers (the CTAs after this one that hold the tile's other stages)
        const int last = sk_cta_of(t * nk + nk - 1, U, G);
        bool ok = true;
        if (et == 0) {
          const uint64_t t0 = global_timer_ns();
          for (int h = cta + 1; h <= last && ok; ++h) {
            for (uint32_t i = 1; ld_acquire_gpu_u32(&flags[h]) == 0u; ++i) {
              __nanosleep(64);
              if ((i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
                flag_timeout();
                ok = false;
                break;
              }
            }
          }
        }
        sk_epi_sync(epi_bar, ephase);
        __threadfence();
        {
          // the helpers' partials, already summed in this CTA's slot: one read, then the slot is
          // zeroed again for the next call (a warp moves 128 contiguous bytes per access)
          unsigned int* acc = reinterpret_cast<unsigned int*>(parts) + static_cast<size_t>(cta) * kSkSlotInts;
          uint32_t pv[BN];
#pragma unroll
          for (int j = 0; j < BN; ++j) pv[j] = __ldcg(acc + j * kGemmBM + r);
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            v[j] += pv[j];
            __stcg(acc + j * kGemmBM + r, 0u);
          }
        }
        if (et == 0)  // every thread has read the partials once the next barrier completes
          for (int h = cta + 1; h <= last; ++h) flags[h] = 0u;  // all zero again for the next call
      }
      sk_epi_sync(epi_bar, ephase);  // this segment's scales are in shared memory
      if constexpr (GATE) {
        // g of the tile's features through shared memory to the up quarters
        const int f = f0 + (r & 63);
        if (r >= 64) {
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            const int a = static_cast<int>(v[j]) - s_rs[sb + j];
            gbuf[j * 64 + (r - 64)] = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), s_a[sb + j]);
          }
        }
        sk_epi_sync(epi_bar, ephase);
        if (r < 64 && f < N) {
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            if (m0 + j < M) {
              const int a = static_cast<int>(v[j]) - s_rs[sb + j];
              const float uu = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), s_a[sb + j]);
              const float gg = gbuf[j * 64 + r];
              const float rr = gg > 0.0f ? gg : 0.0f;
              static_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m0 + j) * N + f] =
                  __float2bfloat16_rn(__fmul_rn(__fmul_rn(rr, rr), uu));
            }
          }
        }
      } else {
        // dequantise and store: thread = output feature n, columns = tokens (the output type and the
        // token count decided once per segment, outside the store loop)
        const int n = f0 + r;
        const int jn = M - m0 < BN ? M - m0 : BN;
        auto store_all = [&](auto* out, auto conv) {
          auto* p = out + static_cast<int64_t>(m0) * N + n;
#pragma unroll
          for (int j = 0; j < BN; ++j)
            if (j < jn) p[static_cast<int64_t>(j) * N] = conv(static_cast<int>(v[j]) - s_rs[sb + j], j);
        };
        if (n < N) {
          if (y_dtype == 2) {
            store_all(static_cast<int32_t*>(y), [](int a, int) { return a; });
          } else if (y_dtype == 0) {
            store_all(static_cast<float*>(y),
                      [&](int a, int j) { return __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), s_a[sb + j]); });
          } else {
            store_all(static_cast<__nv_bfloat16*>(y), [&](int a, int j) {
              return __float2bfloat16_rn(__fmul_rn(__fmul_rn(__int2float_rn(a), gamma), s_a[sb + j]));
            });
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bitnet
