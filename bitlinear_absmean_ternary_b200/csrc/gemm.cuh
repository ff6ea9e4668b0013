// W1.58A8 product on the Blackwell tensor cores (tcgen05.mma kind::i8).
//
// The pages' "low-bit matrix product followed by rescaling" (comrad404.com
// review, "Метод: как устроен BitNet b1.58") with exact int32 accumulation.
//
// Tile: 128 weight rows (the MMA's M) x BN tokens (the MMA's N).  Operands:
//   A = ternary weights, 128 rows x 128 K per stage, expanded from 2-bit
//       codes to int8 in registers by four "unpack" warps and written with
//       tcgen05.st into tensor memory (TMEM), so the expanded bytes never
//       pass through shared memory.  Warp w may only touch TMEM lanes
//       32*(w%4)..+31, so thread t of warp w owns weight row 32*(w%4)+t.
//   B = int8 activations, BN tokens x 128 K per stage, loaded by TMA into
//       shared memory in the 128-byte swizzled K-major layout the MMA reads.
//   D = int32 accumulator, 128 lanes x BN columns of TMEM.
// Packed weights arrive by TMA too (128 rows x 32 bytes per stage, 32-byte
// swizzle, which makes the unpack warps' 16-byte reads bank-conflict free).
//
// Warp roles (192 threads): warp 0 lane 0 = TMA producer; warp 1 = TMEM
// allocator and lane 0 = MMA issuer; warps 2..5 = unpack, then epilogue.
// Barriers per stage s: full[s] (TMA bytes landed), afull[s] (4 unpack warps
// wrote A slot s), empty[s] (MMAs of stage s done: tcgen05.commit), plus
// accfull (all MMAs done).  Every wait is bounded; a timeout flags the
// device error word and the CTA drains in-flight work and exits.
//
// Epilogue: tcgen05.ld of the accumulator (thread = weight row n, 32 tokens
// at a time), acc -= rowsum[m] when unsigned codes were used, then
// y = RN32(RN32(float(acc) * gamma) * a[m]) stored as fp32 / bf16 / int32;
// for a fixed token the 32 lanes of a warp write 32 consecutive n.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bitnet {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;  // K bytes per stage = 4 MMAs of K = 32
constexpr int kGemmThreads = 192;

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int BN, int STAGES>
struct GemmCfg {
  static constexpr int kXBytes = BN * kGemmBK;               // activation tile
  static constexpr int kWBytes = kGemmBM * kGemmBK / 4;      // packed weight tile
  static constexpr int kStageBytes = kXBytes + kWBytes;      // multiple of 1024
  static constexpr int kTmemCols = pow2_at_least(BN + STAGES * 32);
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kScaleOffset = kBarOffset + 256;
  static constexpr int kNeeded = 1024 + kScaleOffset + BN * 8;
  // Each resident CTA holds kTmemCols of the SM's 512 TMEM columns; ask for
  // enough shared memory that no more CTAs than that fit on one SM (228 KB),
  // so a CTA never waits in tcgen05.alloc for another CTA's columns.
  static constexpr int kMaxCtasByTmem = 512 / kTmemCols;
  static constexpr int kMinSmem = 233472 / (kMaxCtasByTmem + 1);
  static constexpr int kSmemBytes = kNeeded > kMinSmem ? kNeeded : kMinSmem;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(kTmemCols <= 512, "TMEM has 512 columns");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
};

template <int BN, int STAGES, bool U8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const float* __restrict__ gamma_ptr, const float* __restrict__ a_scale,
                const int32_t* __restrict__ rowsum, int M, int N, int K, void* __restrict__ y, int y_dtype) {
  using C = GemmCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;
  uint64_t* accfull = afull + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accfull + 1);
  float* s_a = reinterpret_cast<float*>(smem + C::kScaleOffset);
  int* s_rs = reinterpret_cast<int*>(s_a + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kGemmBM;
  const int m0 = blockIdx.y * BN;
  const int nk = (K + kGemmBK - 1) / kGemmBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], 4);
    }
    mbar_init(accfull, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }

  // Activations, scales and row sums come from the previous kernel.
  pdl_wait();
  for (int j = threadIdx.x; j < BN; j += kGemmThreads) {
    const bool in = m0 + j < M;
    s_a[j] = in ? __ldg(a_scale + m0 + j) : 0.0f;
    s_rs[j] = (U8 && in) ? __ldg(rowsum + m0 + j) : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          ok = false;
          break;
        }
        uint8_t* xs = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        tma_load_2d(xs, &tmap_x, i * kGemmBK, m0, &full[s]);
        tma_load_2d(xs + C::kXBytes, &tmap_w, i * (kGemmBK / 4), n0, &full[s]);
        issued = i + 1;
      }
      if (!ok)
        for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_i8(kGemmBM, BN, !U8);
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[s], ph) || !mbar_wait(&afull[s], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t xaddr = smem_addr(smem + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 32; ++kk)
          mma_i8_tmemA(tmem, tmem + BN + 32 * s + 8 * kk, smem_desc_k_sw128(xaddr + 32 * kk), idesc,
                       (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accfull);  // arrives once every MMA issued above has finished
      if (!ok) mbar_wait(accfull, 0);
    }
  } else {
    // -------------------------------------------------- unpack, then epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const uint32_t sw = static_cast<uint32_t>((r >> 2) & 1) << 4;  // 32-byte swizzle of the packed tile
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) {
        ok = false;
        break;
      }
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
      tmem_st_32x32b_x32(lane_base + BN + 32 * s, v);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(accfull, 0))) {
      tc_fence_after();
      const float gamma = __ldg(gamma_ptr);
      const int n = n0 + r;
      constexpr int CW = BN < 32 ? BN : 32;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += CW) {
        uint32_t v[CW];
        if constexpr (CW == 32) {
          tmem_ld_32x32b_x32(lane_base + cc, v);
        } else {
          tmem_ld_32x32b_x16(lane_base + cc, v);
        }
        tmem_ld_wait();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            const int m = m0 + cc + j;
            if (m < M) {
              const int a = static_cast<int>(v[j]) - s_rs[cc + j];
              const int64_t o = static_cast<int64_t>(m) * N + n;
              if (y_dtype == 2) {
                static_cast<int32_t*>(y)[o] = a;
              } else {
                const float val = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), s_a[cc + j]);
                if (y_dtype == 0) static_cast<float*>(y)[o] = val;
                else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(val);
              }
            }
          }
        }
      }
    }
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bitnet
