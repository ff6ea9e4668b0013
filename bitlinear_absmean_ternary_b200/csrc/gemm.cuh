// W1.58A8 product on the Blackwell tensor cores (tcgen05.mma kind::i8).
//
// The pages' "low-bit matrix product followed by rescaling" (comrad404.com
// review, "Метод: как устроен BitNet b1.58") with exact int32 accumulation.
//
// Tile: 128 weight rows (the MMA's M) x BN tokens (the MMA's N).  Operands:
//   A = ternary weights, 128 rows x 128 K per stage, expanded from 2-bit
//       codes to 8-bit in registers by "unpack" warps and written with
//       tcgen05.st into tensor memory (TMEM), so the expanded bytes never
//       pass through shared memory.  Warp w may only touch TMEM lanes
//       32*(w%4)..+31, so thread t of warp w owns weight row 32*(w%4)+t.
//   B = int8 activations, BN tokens x 128 K per stage, loaded by TMA into
//       shared memory in the 128-byte swizzled K-major layout the MMA reads.
//   D = int32 accumulator, 128 lanes x BN columns of TMEM, double-buffered
//       when two fit next to the A slots (BN <= 128), single otherwise.
// Packed weights arrive by TMA too (128 rows x 32 bytes per stage, 32-byte
// swizzle, which makes the unpack warps' 16-byte reads bank-conflict free).
// With the per-token sums of x_q available, A holds the unsigned codes
// c = q + 1 and the epilogue subtracts rowsum[m] (sum c*x - sum x = sum q*x).
//
// Persistent: one CTA per SM walks tiles t = blockIdx.x, +gridDim.x, ...
// (weight-row tiles fastest).  Warp roles:
//   warp 0 and warps 14.., lane 0   TMA producers over an S-deep ring;
//   warp 1           TMEM allocator; lane 0 issues the MMAs;
//   warps 2..9       unpack: two warps per TMEM lane quarter, taking
//                    alternate stages;
//   warps 10..13     epilogue: tcgen05.ld of a finished accumulator,
//                    dequantise, store, then hand the buffer back.
// Barriers: full[s] (TMA bytes landed), afull[s] (4 unpack warps wrote A
// slot s), empty[s] (MMAs of stage s done; tcgen05.commit), accfull[b] (tile
// accumulated in buffer b), accempty[b] (epilogue drained buffer b).  Every
// wait is bounded; a timeout flags the device error word, the CTA stops
// issuing work, drains what is in flight and exits.
//
// Epilogue: y = RN32(RN32(float(acc) * gamma) * a[m]) as fp32 / bf16, or acc
// as int32; for a fixed token the 32 lanes of a warp write 32 consecutive n.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bitnet {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;  // K bytes per stage = 4 MMAs of K = 32
constexpr int kGemmUnpackWarps = 8;
constexpr int kGemmEpiWarps = 4;
// TMA issue warps: one issuing thread streams a stage roughly every 270 ns
// whatever its size, so several warps share the ring (warp p issues the
// stages g with g % kGemmProducers == p).
constexpr int kGemmProducers = 2;
constexpr int kGemmThreads = (1 + kGemmProducers + kGemmUnpackWarps + kGemmEpiWarps) * 32;

// BN tokens per tile, S ring stages.  TMEM holds the accumulator(s) (BN
// columns each; two when they fit, so the epilogue of one tile overlaps the
// MMAs of the next) and one 32-column A slot per stage.
template <int BN, int S>
struct GemmCfg {
  static constexpr int kXBytes = BN * kGemmBK;           // activation tile
  static constexpr int kWBytes = kGemmBM * kGemmBK / 4;  // packed weight tile
  static constexpr int kStageBytes = kXBytes + kWBytes;  // multiple of 1024
  static constexpr int kTmemCols = 512;
  static constexpr int kBufs = 2 * BN + 32 * S <= kTmemCols ? 2 : 1;
  static constexpr int kAcol = kBufs * BN;  // first A slot column
  static constexpr int kBarOffset = S * kStageBytes;
  static constexpr int kNeeded = 1024 + kBarOffset + 256;
  // The CTA holds all 512 TMEM columns: ask for enough shared memory that a
  // second CTA never fits on the SM (228 KB), so none waits in tcgen05.alloc.
  static constexpr int kMinSmem = 233472 / 2;
  static constexpr int kSmemBytes = kNeeded > kMinSmem ? kNeeded : kMinSmem;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(kAcol + S * 32 <= kTmemCols, "TMEM budget");
  static_assert(kNeeded <= 232448, "shared memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(S % kGemmProducers == 0, "each ring slot belongs to one producer");
};

template <int BN, int S, bool U8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const float* __restrict__ gamma_ptr, const float* __restrict__ a_scale,
                const int32_t* __restrict__ rowsum, int M, int N, int K, void* __restrict__ y, int y_dtype) {
  using C = GemmCfg<BN, S>;
  constexpr int NB = C::kBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;
  uint64_t* accfull = afull + S;
  uint64_t* accempty = accfull + 2;
  uint64_t* done = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + kGemmBM - 1) / kGemmBM;
  const int tiles = n_tiles * ((M + BN - 1) / BN);
  const int nk = (K + kGemmBK - 1) / kGemmBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kGemmEpiWarps);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();

  const int prod = warp == 0 ? 0 : warp - (1 + kGemmUnpackWarps + kGemmEpiWarps);  // producer index or < 1
  if (warp == 0 || warp >= 2 + kGemmUnpackWarps + kGemmEpiWarps) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      // The weights never depend on the previous kernel: the first ring's
      // worth of weight tiles is requested before waiting on it.
      const int my_tiles = blockIdx.x < tiles ? (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
      const int total = my_tiles * nk;
      const int pre = total < S ? total : S;
      for (int g = prod; g < pre; g += kGemmProducers) {
        const int t = blockIdx.x + (g / nk) * gridDim.x, kb = g % nk;
        mbar_arrive_expect_tx(&full[g], C::kStageBytes);
        tma_load_2d(smem + g * C::kStageBytes + C::kXBytes, &tmap_w, kb * (kGemmBK / 4), (t % n_tiles) * kGemmBM,
                    &full[g]);
      }
      pdl_wait();
      int issued = prod;
      bool ok = true;
      for (int g = prod; g < total; g += kGemmProducers) {
        const int s = g % S;
        const int t = blockIdx.x + (g / nk) * gridDim.x, kb = g % nk;
        const int n0 = (t % n_tiles) * kGemmBM, m0 = (t / n_tiles) * BN;
        uint8_t* xs = smem + s * C::kStageBytes;
        if (g >= pre) {
          if (!mbar_wait(&empty[s], ((g / S) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          tma_load_2d(xs + C::kXBytes, &tmap_w, kb * (kGemmBK / 4), n0, &full[s]);
        }
        tma_load_2d(xs, &tmap_x, kb * kGemmBK, m0, &full[s]);
        issued = g + kGemmProducers;
      }
      if (!ok) {
        // weight tiles were requested for stages up to max(issued, pre)
        const int last = issued > pre ? issued : pre;
        for (int g = prod; g < last; g += kGemmProducers)
          if (g + S >= last) mbar_wait(&full[g % S], (g / S) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_i8(kGemmBM, BN, !U8);
      bool ok = true;
      int g = 0, tc = 0;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tc) {
        const int b = tc % NB;
        if (!mbar_wait(&accempty[b], ((tc / NB) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait(&full[s], ph) || !mbar_wait(&afull[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xaddr = smem_addr(smem + s * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk)
            mma_i8_tmemA(dcol, tmem + C::kAcol + 32 * s + 8 * kk, smem_desc_k_sw128(xaddr + 32 * kk), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accfull[b]);
      }
      tc_commit(done);  // arrives once every MMA issued above has finished
      mbar_wait(done, 0);
    }
  } else if (warp < 2 + kGemmUnpackWarps) {
    // ------------------------------------------------------------ unpack
    const int q = warp & 3;
    const int par = (warp - 2) >> 2;  // this warp takes stages with g % 2 == par
    const int r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const uint32_t sw = static_cast<uint32_t>((r >> 2) & 1) << 4;  // 32-byte swizzle of the packed tile
    const int my_tiles = blockIdx.x < tiles ? (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int total = my_tiles * nk;
    for (int g = par; g < total; g += 2) {
      const int s = g % S;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (g / S) & 1))) break;
      const uint32_t wrow = smem_addr(smem + s * C::kStageBytes + C::kXBytes) + r * 32;
      const uint4 p0 = lds128(wrow + (0u ^ sw));
      const uint4 p1 = lds128(wrow + (16u ^ sw));
      const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      uint32_t v[32];
#pragma unroll
      for (int wi = 0; wi < 8; ++wi)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t c4 = (pw[wi] >> (2 * j)) & 0x03030303u;
          v[4 * wi + j] = U8 ? c4 : codes_to_signed(c4);
        }
      tmem_st_32x32b_x32(lane_base + C::kAcol + 32 * s, v);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    pdl_wait();  // a_scale and rowsum come from the previous kernel
    const float gamma = __ldg(gamma_ptr);
    int tc = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
      const int b = tc % NB;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], (tc / NB) & 1))) break;
      tc_fence_after();
      const int n = (t % n_tiles) * kGemmBM + 32 * q + lane;
      const int m0 = (t / n_tiles) * BN;
      constexpr int CW = BN < 32 ? BN : 32;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += CW) {
        uint32_t v[CW];
        if constexpr (CW == 32) {
          tmem_ld_32x32b_x32(lane_base + b * BN + cc, v);
        } else {
          tmem_ld_32x32b_x16(lane_base + b * BN + cc, v);
        }
        // per-token scale and row sum of the CW tokens of this chunk, one per lane
        const int mm = m0 + cc + (lane < CW ? lane : 0);
        const bool inb = lane < CW && mm < M;
        const float my_a = inb ? __ldg(a_scale + mm) : 0.0f;
        const int my_rs = (U8 && inb) ? __ldg(rowsum + mm) : 0;
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const float aj = __shfl_sync(0xffffffffu, my_a, j);
          const int rsj = __shfl_sync(0xffffffffu, my_rs, j);
          const int m = m0 + cc + j;
          if (m < M && n < N) {
            const int a = static_cast<int>(v[j]) - rsj;
            const int64_t o = static_cast<int64_t>(m) * N + n;
            if (y_dtype == 2) {
              static_cast<int32_t*>(y)[o] = a;
            } else {
              const float val = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), aj);
              if (y_dtype == 0) static_cast<float*>(y)[o] = val;
              else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(val);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bitnet
