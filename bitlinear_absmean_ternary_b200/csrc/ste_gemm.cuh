// Straight-through-estimator (STE) backward of the BitLinear on the Blackwell
// tensor cores (tcgen05.mma kind::f16: bf16 operands, fp32 accumulation).
//
// Training keeps precise latent weights and computes with the rounded ones;
// the rounding has no useful derivative, so the backward pass lets the
// gradient through as if it were absent (Habr repost on juhe.plus, sections
// "А откуда взялась сама идея?" and "Когда - три лучше двух").  With the
// forward's W_hat = gamma * q and x_hat[m] = a[m] * x_q[m]:
//   MODE 0 (input gradient):  dX[m, k] = gamma * sum_n dY[m, n] q[n, k]
//   MODE 1 (weight gradient): dW[n, k] = sum_m dYs[m, n] x_q[m, k],
//                             dYs = bf16(dY[m, n] * a[m]) (a pre-pass writes it transposed)
//
// Both are D[r, c] = sum_j A[r, j] B[c, j] with output rows r = k (a stage
// carries 128 contraction elements, 8 MMAs, to amortise the stage handoff): a tile is
// 128 values of k (the MMA's M, one TMEM lane each) by BN = 128 columns
// (m for dX, n for dW), so that the epilogue's 32 lanes store 32 consecutive
// k of one output row.
//   A (128 x 128 per stage) is built in tensor memory by converter warps from
//     a tile that TMA brings into shared memory with the contraction index j
//     along its rows: MODE 0 packed weight rows n (32 bytes = 128 codes of k
//     each; code -> bf16 -1/0/+1 through one byte permute per pair),
//     MODE 1 int8 activation rows m (128 bytes of k; exact int8 -> bf16).
//   B (BN x 128 per stage, two 64-wide boxes) is bf16, K-major (j
//     contiguous), loaded by TMA in the 128-byte swizzled layout: MODE 0 dY as stored ([M][N]), MODE 1 the
//     pre-pass output dYs^T ([N][M padded]).
// Warp roles, barriers and bounded waits follow the int8 GEMM (gemm.cuh):
// two TMA producer warps, an MMA warp that also allocates TMEM, eight
// converter warps (two per TMEM lane quarter, alternate stages), four
// epilogue warps; the accumulator is double-buffered in TMEM.
#pragma once

#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace bitnet {

constexpr int kSteBM = 128;   // output rows (k) per tile
constexpr int kSteBN = 128;   // output columns per tile
constexpr int kSteBJ = 128;   // contraction elements per stage (8 MMAs of K = 16)
constexpr int kSteBox = 64;   // bf16 per 128-byte swizzled B box
constexpr int kSteStages = 4;

template <int MODE>
struct SteCfg {
  static constexpr int kBSub = kSteBN * 128;                      // one B box: bf16 [BN][64]
  static constexpr int kBBytes = kBSub * (kSteBJ / kSteBox);
  static constexpr int kARow = MODE == 0 ? kSteBM / 4 : kSteBM;   // source bytes per contraction row
  static constexpr int kABytes = kSteBJ * kARow;                  // [BJ rows j][kARow]
  static constexpr int kStageBytes = kBBytes + kABytes;
  static constexpr int kAslot = kSteBJ / 2;  // TMEM columns per A slot (two bf16 per column)
  static constexpr int kTmemCols = 512;
  static constexpr int kAcol = 2 * kSteBN;   // two accumulator buffers first
  static constexpr int kBarOffset = kSteStages * kStageBytes;
  static constexpr int kSmemBytes = 1024 + kBarOffset + 256;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(kAcol + kSteStages * kAslot <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kSteStages % kGemmProducers == 0, "each ring slot belongs to one producer");
};

// Instruction descriptor for kind::f16 with bf16 A and B (both K-major) and
// fp32 accumulation: D format F32 (bits 4-5 = 1), A format BF16 (bits 7-9 =
// 1), B format BF16 (bits 10-12 = 1), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D (tmem) [+]= A (tmem) x B (smem descriptor), kind::f16, fp32 accumulate.
BN_DEV void mma_bf16_tmemA(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// R output rows (k), C output columns, J contraction length.  out is [C][R]
// row-major (fp32 or bf16); scale_ptr: gamma (MODE 0) or null (scale 1).
template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    ste_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_a,
                    const float* __restrict__ scale_ptr, int R, int C, int J, void* __restrict__ out, int out_dtype) {
  using Cfg = SteCfg<MODE>;
  constexpr int S = kSteStages;
  constexpr int NB = 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;
  uint64_t* accfull = afull + S;
  uint64_t* accempty = accfull + 2;
  uint64_t* done = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_tiles = (R + kSteBM - 1) / kSteBM;
  const int tiles = r_tiles * ((C + kSteBN - 1) / kSteBN);
  const int nk = (J + kSteBJ - 1) / kSteBJ;
  const int cid = blockIdx.x, ncl = gridDim.x;
  const int my_tiles = cid < tiles ? (tiles - cid + ncl - 1) / ncl : 0;
  const int total = my_tiles * nk;

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
    tma_prefetch_desc(&tmap_b);
    tma_prefetch_desc(&tmap_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();

  const int prod = warp == 0 ? 0 : warp - (1 + kGemmUnpackWarps + kGemmEpiWarps);
  if (warp == 0 || warp >= 2 + kGemmUnpackWarps + kGemmEpiWarps) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producers
      pdl_wait();  // dY and x_q come from earlier kernels
      int issued = prod;
      bool ok = true;
      for (int g = prod; g < total; g += kGemmProducers) {
        const int s = g % S;
        const int t = cid + (g / nk) * ncl, kb = g % nk;
        const int r0 = (t % r_tiles) * kSteBM, c0 = (t / r_tiles) * kSteBN;
        uint8_t* st = smem + s * Cfg::kStageBytes;
        if (g >= S && !mbar_wait(&empty[s], ((g / S) & 1) ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
#pragma unroll
        for (int i = 0; i < kSteBJ / kSteBox; ++i)
          tma_load_2d(st + i * Cfg::kBSub, &tmap_b, kb * kSteBJ + i * kSteBox, c0, &full[s]);
        tma_load_2d(st + Cfg::kBBytes, &tmap_a, MODE == 0 ? r0 / 4 : r0, kb * kSteBJ, &full[s]);
        issued = g + kGemmProducers;
      }
      if (!ok) {
        for (int g = prod; g < issued; g += kGemmProducers)
          if (g + S >= issued) mbar_wait(&full[g % S], (g / S) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16(kSteBM, kSteBN);
      bool ok = true;
      int g = 0, tc = 0;
      for (int t = cid; ok && t < tiles; t += ncl, ++tc) {
        const int b = tc % NB;
        if (!mbar_wait(&accempty[b], ((tc / NB) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * kSteBN;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait(&full[s], ph) || !mbar_wait(&afull[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t baddr = smem_addr(smem + s * Cfg::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kSteBJ / 16; ++kk)
            mma_bf16_tmemA(dcol, tmem + Cfg::kAcol + Cfg::kAslot * s + 8 * kk,
                           smem_desc_k_sw128(baddr + (kk >> 2) * Cfg::kBSub + 32 * (kk & 3)), idesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accfull[b]);
      }
      tc_commit(done);
      mbar_wait(done, 0);
    }
  } else if (warp < kGemmFirstEpiWarp) {
    // ------------------------------------------------------------ converters
    const int q = warp & 3;
    const int par = (warp - 2) >> 2;  // stages with g % 2 == par
    const int r = 32 * q + lane;      // output row (k - r0) of this thread = its TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    // MODE 0: weight k0 + r sits in 32-bit word r / 16 of a 32-byte packed row, at bit 8 (r % 4) + 2 ((r / 4) % 4)
    const uint32_t woff = MODE == 0 ? static_cast<uint32_t>(r >> 4) * 4u : static_cast<uint32_t>(r & ~3);
    const uint32_t sh = MODE == 0 ? 8u * (r & 3) + 2u * ((r >> 2) & 3) : 8u * (r & 3);
    for (int g = par; g < total; g += 2) {
      const int s = g % S;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (g / S) & 1))) break;
      const uint32_t src = smem_addr(smem + s * Cfg::kStageBytes + Cfg::kBBytes) + woff;
#pragma unroll
      for (int h = 0; h < kSteBJ / 64; ++h) {  // 64 contraction elements -> 32 TMEM columns per pass
        uint32_t v[32];
#pragma unroll
        for (int p = 0; p < 32; ++p) {
          const int j = 64 * h + 2 * p;
          uint32_t w0, w1;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(src + j * Cfg::kARow));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w1) : "r"(src + (j + 1) * Cfg::kARow));
          if constexpr (MODE == 0) {
            // codes c in {0,1,2} -> bf16 of q = c - 1: bytes (0x80,0xBF), (0,0), (0x80,0x3F) at pool
            // positions (2c, 2c+1) of {0x0000BF80, 0x00003F80}
            uint32_t c0, c1;
            asm("bfe.u32 %0, %1, %2, 2;" : "=r"(c0) : "r"(w0), "r"(sh));
            asm("bfe.u32 %0, %1, %2, 2;" : "=r"(c1) : "r"(w1), "r"(sh));
            v[p] = __byte_perm(0x0000BF80u, 0x00003F80u, 0x1010u + 0x22u * c0 + 0x2200u * c1);
          } else {
            // signed byte -> float exactly: the bits of 1.5 * 2^23 plus x are the float 1.5 * 2^23 + x
            // (unit spacing in [2^23, 2^24)), minus 1.5 * 2^23; |x| <= 127 leaves the low 16 bits of the
            // float zero, so its high half is the bf16 value
            int x0, x1;
            asm("bfe.s32 %0, %1, %2, 8;" : "=r"(x0) : "r"(w0), "r"(sh));
            asm("bfe.s32 %0, %1, %2, 8;" : "=r"(x1) : "r"(w1), "r"(sh));
            const float f0 = __fsub_rn(__int_as_float(0x4B400000 + x0), 12582912.0f);
            const float f1 = __fsub_rn(__int_as_float(0x4B400000 + x1), 12582912.0f);
            v[p] = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
          }
        }
        tmem_st_32x32b_x32(lane_base + Cfg::kAcol + Cfg::kAslot * s + 32 * h, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const float scale = scale_ptr != nullptr ? __ldg(scale_ptr) : 1.0f;
    int tc = 0;
    for (int t = cid; t < tiles; t += ncl, ++tc) {
      const int b = tc % NB;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], (tc / NB) & 1))) break;
      tc_fence_after();
      const int k = (t % r_tiles) * kSteBM + 32 * q + lane;
      const int c0 = (t / r_tiles) * kSteBN;
#pragma unroll 1
      for (int cc = 0; cc < kSteBN; cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + b * kSteBN + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = c0 + cc + j;
          if (c < C && k < R) {
            const float acc = __uint_as_float(v[j]);
            const float val = scale_ptr != nullptr ? __fmul_rn(acc, scale) : acc;
            const int64_t o = static_cast<int64_t>(c) * R + k;
            if (out_dtype == 0) static_cast<float*>(out)[o] = val;
            else static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(val);
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
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// Pre-pass of the weight gradient: dYsT[n][m] = bf16_RNE(RN32(dY[m][n] * a[m]))
// for m < M, 0 for M <= m < Mp (Mp a multiple of 64).  32 x 32 tiles through
// shared memory so that both the reads of dY rows and the writes of dYsT rows
// are coalesced.
__global__ void __launch_bounds__(256) ste_scale_transpose_kernel(const __nv_bfloat16* __restrict__ dY,
                                                                  const float* __restrict__ a, int M, int N, int Mp,
                                                                  __nv_bfloat16* __restrict__ out) {
  __shared__ float tile[32][33];
  pdl_wait();
  const int n0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  for (int i = ty; i < 32; i += 8) {
    const int m = m0 + i, n = n0 + tx;
    float v = 0.0f;
    if (m < M && n < N) v = __fmul_rn(__bfloat162float(dY[static_cast<int64_t>(m) * N + n]), __ldg(a + m));
    tile[i][tx] = v;
  }
  __syncthreads();
  pdl_launch_dependents();
  for (int i = ty; i < 32; i += 8) {
    const int n = n0 + i, m = m0 + tx;
    if (n < N && m < Mp) out[static_cast<int64_t>(n) * Mp + m] = __float2bfloat16_rn(tile[tx][i]);
  }
}

}  // namespace bitnet
