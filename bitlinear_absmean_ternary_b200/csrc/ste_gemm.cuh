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
// Both are D[r, c] = sum_j A[r, j] B[c, j] with output rows r = k, on a plain
// bf16 GEMM whose operands both come from shared memory by TMA (128-byte
// swizzled, K-major): expansion pre-passes first write the ternary codes
// transposed as bf16 -1/0/+1 (MODE 0: WT[k][n]) or the int8 activations
// transposed as exact bf16 (MODE 1: XT[k][m]), and dY * a transposed and
// rounded to bf16 (MODE 1: dYs^T[n][m]).  Training GEMMs are bound by the
// tensor pipe, so expanding each operand once beats re-expanding a weight
// tile for every tile of tokens inside the GEMM (an in-GEMM expansion into
// tensor memory kept the integer pipe 80% busy and the tensor pipe 30%).
// Tile: 128 rows k (TMEM lanes) x BN columns (m for dX, n for dW), 64
// contraction elements (4 MMAs) per stage in a ring of four (deeper rings of
// smaller stages fed the MMAs better than two stages of 128); the epilogue's
// 32 lanes store 32 consecutive k of one output row.  Warps: two TMA producers (alternate
// stages), one MMA issuer that also allocates TMEM, four epilogue warps; the
// fp32 accumulator is double-buffered in TMEM; every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace bitnet {

constexpr int kSteBM = 128;  // output rows (k) per tile
constexpr int kSteBJ = 64;   // contraction elements per stage (4 MMAs of K = 16)
constexpr int kSteBox = 64;  // bf16 per 128-byte swizzled box
constexpr int kStePad = 64;  // contraction lengths of the expanded operands are padded to this
constexpr int kSteEpiWarps = 8;  // two per TMEM lane quarter, half of a tile's columns each
constexpr int kSteThreads = (3 + kSteEpiWarps) * 32;  // producer, MMA, epilogue warps, producer

// BN output columns per tile, S ring stages.  TMEM holds two accumulators of
// BN fp32 columns.
template <int BN, int S>
struct SteCfg {
  static constexpr int kASub = kSteBM * 128;                // one A box: bf16 [128][64]
  static constexpr int kBSub = BN * 128;                    // one B box: bf16 [BN][64]
  static constexpr int kBoxes = kSteBJ / kSteBox;           // boxes per operand per stage
  static constexpr int kStageBytes = kBoxes * (kASub + kBSub);
  static constexpr int kTmemCols = 2 * BN <= 256 ? 256 : 512;
  static constexpr int kBarOffset = S * kStageBytes;
  static constexpr int kSmemBytes = 1024 + kBarOffset + 256;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "MMA N; two 32-column-multiple halves");
  static_assert(S % 2 == 0 || S == 3, "ring");
};

// Instruction descriptor for kind::f16 with bf16 A and B (both K-major) and
// fp32 accumulation: D format F32 (bits 4-5 = 1), A format BF16 (bits 7-9 =
// 1), B format BF16 (bits 10-12 = 1), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D (tmem) [+]= A (smem descriptor) x B (smem descriptor), kind::f16, fp32 accumulate.
BN_DEV void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[r][c] = sum_j A[r][j] B[c][j] for R output rows, C columns, contraction J;
// A [R][J] and B [C][J] bf16 row-major (j contiguous) behind the tensor maps.
// out is [C][R] row-major (fp32 or bf16), times *scale_ptr when given.
template <int BN, int S>
__global__ void __launch_bounds__(kSteThreads, 1)
    ste_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const float* __restrict__ scale_ptr, int R, int C, int J, void* __restrict__ out, int out_dtype) {
  using Cfg = SteCfg<BN, S>;
  constexpr int NB = 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* accfull = empty + S;
  uint64_t* accempty = accfull + 2;
  uint64_t* done = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_tiles = (R + kSteBM - 1) / kSteBM;
  const int tiles = r_tiles * ((C + BN - 1) / BN);
  const int nk = (J + kSteBJ - 1) / kSteBJ;
  const int cid = blockIdx.x, ncl = gridDim.x;
  const int my_tiles = cid < tiles ? (tiles - cid + ncl - 1) / ncl : 0;
  const int total = my_tiles * nk;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kSteEpiWarps);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
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

  if (warp == 0 || warp == 2 + kSteEpiWarps) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producers (stage g by producer g % 2)
      const int prod = warp == 0 ? 0 : 1;
      pdl_wait();  // the operands come from earlier kernels
      int issued = prod;
      bool ok = true;
      for (int g = prod; g < total; g += 2) {
        const int s = g % S;
        const int t = cid + (g / nk) * ncl, kb = g % nk;
        const int r0 = (t % r_tiles) * kSteBM, c0 = (t / r_tiles) * BN;
        uint8_t* st = smem + s * Cfg::kStageBytes;
        if (g >= S && !mbar_wait(&empty[s], ((g / S) & 1) ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
#pragma unroll
        for (int i = 0; i < Cfg::kBoxes; ++i) {
          tma_load_2d(st + i * Cfg::kASub, &tmap_a, kb * kSteBJ + i * kSteBox, r0, &full[s]);
          tma_load_2d(st + Cfg::kBoxes * Cfg::kASub + i * Cfg::kBSub, &tmap_b, kb * kSteBJ + i * kSteBox, c0,
                      &full[s]);
        }
        issued = g + 2;
      }
      if (!ok) {
        for (int g = prod; g < issued; g += 2)
          if (g + S >= issued) mbar_wait(&full[g % S], (g / S) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16(kSteBM, BN);
      bool ok = true;
      int g = 0, tc = 0;
      for (int t = cid; ok && t < tiles; t += ncl, ++tc) {
        const int b = tc % NB;
        if (!mbar_wait(&accempty[b], ((tc / NB) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % S;
          if (!mbar_wait(&full[s], (g / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t abase = smem_addr(smem + s * Cfg::kStageBytes);
          const uint32_t bbase = abase + Cfg::kBoxes * Cfg::kASub;
#pragma unroll
          for (int kk = 0; kk < kSteBJ / 16; ++kk)
            mma_bf16_ss(dcol, smem_desc_k_sw128(abase + (kk >> 2) * Cfg::kASub + 32 * (kk & 3)),
                        smem_desc_k_sw128(bbase + (kk >> 2) * Cfg::kBSub + 32 * (kk & 3)), idesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accfull[b]);
      }
      tc_commit(done);
      mbar_wait(done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2 .. 2 + kSteEpiWarps - 1)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // which half of the tile's columns
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const float scale = scale_ptr != nullptr ? __ldg(scale_ptr) : 1.0f;
    int tc = 0;
    for (int t = cid; t < tiles; t += ncl, ++tc) {
      const int b = tc % NB;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], (tc / NB) & 1))) break;
      tc_fence_after();
      const int k = (t % r_tiles) * kSteBM + 32 * q + lane;
      const int c0 = (t / r_tiles) * BN;
#pragma unroll 1
      for (int cc = half * (BN / 2); cc < (half + 1) * (BN / 2); cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + b * BN + cc, v);
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

// Expansion of the ternary codes for the input gradient: WT[k][n] = q[n][k]
// as bf16 (-1, 0, +1) for n < N, 0 for N <= n < Np.  One 64 x 64 tile per
// CTA through shared memory: packed words of 16 codes read along k, bf16
// rows written along n.
__global__ void __launch_bounds__(256) ste_expand_wt_kernel(const uint8_t* __restrict__ Wp, int N, int K, int Np,
                                                            __nv_bfloat16* __restrict__ wt) {
  __shared__ int8_t tile[64][65];  // [n][k]
  pdl_wait();
  const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  {
    const int n = threadIdx.x >> 2, w = threadIdx.x & 3;  // 64 rows x 4 words of 16 codes
    uint32_t word = 0x55555555u;  // code 1 (q = 0) in every field: padding rows
    if (n0 + n < N && k0 + 16 * w < K)
      word = __ldg(reinterpret_cast<const uint32_t*>(Wp + static_cast<int64_t>(n0 + n) * (K / 4) + k0 / 4) + w);
#pragma unroll
    for (int e = 0; e < 16; ++e)  // weight 16w + e: byte e % 4, bits 2 (e / 4)
      tile[n][16 * w + e] = static_cast<int8_t>(((word >> (8 * (e & 3) + 2 * (e >> 2))) & 3u) - 1);
  }
  __syncthreads();
  pdl_launch_dependents();
  const int nn = threadIdx.x & 63, kr = threadIdx.x >> 6;  // 64 n x 4 rows of k per pass
  for (int k = kr; k < 64; k += 4)
    if (k0 + k < K && n0 + nn < Np)
      wt[static_cast<int64_t>(k0 + k) * Np + n0 + nn] = __float2bfloat16_rn(static_cast<float>(tile[nn][k]));
}

// Expansion of the activations for the weight gradient: XT[k][m] = x_q[m][k]
// as bf16 (exact) for m < M, 0 for M <= m < Mp.  One 64 x 64 tile per CTA:
// 16-byte reads of x_q rows (16 values of k), 16-byte writes of XT rows
// (8 values of m) through a padded bf16 tile in shared memory.
__global__ void __launch_bounds__(256) ste_expand_xt_kernel(const int8_t* __restrict__ xq, int M, int K, int Mp,
                                                            __nv_bfloat16* __restrict__ xt) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];  // [m][k]
  pdl_wait();
  const int m0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  {
    const int m = threadIdx.x >> 2, kc = (threadIdx.x & 3) * 16;  // 64 rows x 4 chunks of 16
    int4 v = make_int4(0, 0, 0, 0);
    if (m0 + m < M) v = __ldg(reinterpret_cast<const int4*>(xq + static_cast<int64_t>(m0 + m) * K + k0 + kc));
    const uint32_t w[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y), static_cast<uint32_t>(v.z),
                           static_cast<uint32_t>(v.w)};
#pragma unroll
    for (int e = 0; e < 16; ++e)
      tile[m][kc + e] = __float2bfloat16_rn(static_cast<float>(static_cast<int8_t>(w[e >> 2] >> (8 * (e & 3)))));
  }
  __syncthreads();
  pdl_launch_dependents();
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int idx = threadIdx.x + 256 * p;  // 64 rows of k x 8 chunks of 8 m
    const int k = idx >> 3, mc = (idx & 7) * 8;
    if (k0 + k < K && m0 + mc < Mp) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = static_cast<uint32_t>(__bfloat16_as_ushort(tile[mc + 2 * e][k])) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(tile[mc + 2 * e + 1][k])) << 16);
      *reinterpret_cast<uint4*>(xt + static_cast<int64_t>(k0 + k) * Mp + m0 + mc) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Pre-pass of the weight gradient: dYsT[n][m] = bf16_RNE(RN32(dY[m][n] * a[m]))
// for m < M, 0 for M <= m < Mp (Mp a multiple of 64).  One 64 x 64 tile per
// CTA: 16-byte reads of dY rows (8 values of n), 16-byte writes of dYsT rows
// (8 values of m) through a padded bf16 tile in shared memory.
__global__ void __launch_bounds__(256) ste_scale_transpose_kernel(const __nv_bfloat16* __restrict__ dY,
                                                                  const float* __restrict__ a, int M, int N, int Mp,
                                                                  __nv_bfloat16* __restrict__ out) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];  // [m][n]
  pdl_wait();
  const int n0 = blockIdx.x * 64, m0 = blockIdx.y * 64;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int idx = threadIdx.x + 256 * p;  // 64 rows of m x 8 chunks of 8 n
    const int m = idx >> 3, nc = (idx & 7) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    float am = 0.0f;
    if (m0 + m < M && n0 + nc < N) {
      v = __ldg(reinterpret_cast<const uint4*>(dY + static_cast<int64_t>(m0 + m) * N + n0 + nc));
      am = __ldg(a + m0 + m);
    }
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t bits = (e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16);
      tile[m][nc + e] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(bits), am));
    }
  }
  __syncthreads();
  pdl_launch_dependents();
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int idx = threadIdx.x + 256 * p;  // 64 rows of n x 8 chunks of 8 m
    const int n = idx >> 3, mc = (idx & 7) * 8;
    if (n0 + n < N && m0 + mc < Mp) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = static_cast<uint32_t>(__bfloat16_as_ushort(tile[mc + 2 * e][n])) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(tile[mc + 2 * e + 1][n])) << 16);
      *reinterpret_cast<uint4*>(out + static_cast<int64_t>(n0 + n) * Mp + m0 + mc) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace bitnet
