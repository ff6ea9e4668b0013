// W1.58A8 product on the Blackwell tensor cores (tcgen05.mma kind::i8).
//
// The pages' "low-bit matrix product followed by rescaling" (comrad404.com
// review, "Метод: как устроен BitNet b1.58") with exact int32 accumulation.
//
// Tile: 128 weight rows (the MMA's M) x BN tokens (the MMA's N); a stage
// covers BK = 256 bytes of K (8 MMAs of K = 32).  Operands:
//   A = ternary weights, 128 rows x BK per stage, expanded from 2-bit codes
//       to 8-bit in registers by "unpack" warps and written with tcgen05.st
//       into tensor memory (TMEM), so the expanded bytes never pass through
//       shared memory.  Warp w may only touch TMEM lanes 32*(w%4)..+31, so
//       thread t of warp w owns weight row 32*(w%4)+t.
//   B = int8 activations, BN tokens x BK per stage, loaded by TMA (one box
//       per 128 bytes of K) into shared memory in the 128-byte swizzled
//       K-major layout the MMA reads.
//   D = int32 accumulator, 128 lanes x BN columns of TMEM, double-buffered
//       when two fit next to the A slots.
// Packed weights arrive by TMA as one 128-row x BK/4-byte box per stage,
// swizzled (64-byte pattern) so that the unpack warps' 16-byte reads are
// bank-conflict free.  With the per-token sums of x_q available, A holds the
// unsigned codes c = q + 1 and the epilogue subtracts rowsum[m]
// (sum c*x - sum x = sum q*x).
//
// A stage is handed from the TMA producers to the unpack warps to the MMA
// issuer and back through mbarriers; measured on B200, this handoff, not the
// bytes moved, bounds the feed, which is why a stage carries 256 bytes of K.
//
// Persistent: clusters of KSPLIT CTAs walk the tiles t = cluster, +clusters,
// ...; with KSPLIT > 1 every CTA of a cluster accumulates its own range of
// K for the same tile and the partial sums are added exactly in integers
// through distributed shared memory (each CTA reduces a slice of rows from
// all its peers' partial tiles), which keeps every SM busy when there are
// fewer tiles than SMs (decode-sized M).
//
// Warp roles (544 threads):
//   warp 0 and warp 14, lane 0   TMA producers (stage g by producer g % 2);
//   warp 1                       TMEM allocator; lane 0 issues the MMAs;
//   warps 2..9                   unpack: two warps per TMEM lane quarter,
//                                taking alternate stages;
//   warps 10..13                 epilogue.
// Barriers: full[s] (TMA bytes landed), afull[s] (4 unpack warps wrote A
// slot s), empty[s] (MMAs of stage s done; tcgen05.commit), accfull[b] /
// accempty[b] (accumulator buffer b), ready / consumed (split-K exchange).
// Every wait is bounded; a timeout flags the device error word, the CTA
// stops issuing work, drains what is in flight and exits.
//
// Epilogue: y = RN32(RN32(float(acc) * gamma) * a[m]) as fp32 / bf16, or acc
// as int32; for a fixed token consecutive threads write consecutive n.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bitnet {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 256;  // K bytes per stage = 8 MMAs of K = 32
constexpr int kGemmUnpackWarps = 8;
constexpr int kGemmEpiWarps = 8;  // two per TMEM lane quarter, each draining half of the columns
// TMA issue warps: one issuing thread streams a stage roughly every 270 ns
// whatever its size, so two warps share the ring (warp p issues the stages g
// with g % kGemmProducers == p).
constexpr int kGemmProducers = 2;
constexpr int kGemmThreads = (1 + kGemmProducers + kGemmUnpackWarps + kGemmEpiWarps) * 32;
constexpr int kGemmFirstEpiWarp = 2 + kGemmUnpackWarps;

// BN tokens per tile, S ring stages, KSPLIT CTAs per cluster.  TMEM holds the
// accumulator(s) (BN columns each; two when they fit, so the epilogue of one
// tile overlaps the MMAs of the next) and one BK/4-column A slot per stage.
template <int BN, int S, int KSPLIT = 1>
struct GemmCfg {
  static constexpr int kXSub = BN * 128;                   // one 128-byte-wide activation box
  static constexpr int kXBytes = kXSub * (kGemmBK / 128);  // activation tile of a stage
  static constexpr int kWRow = kGemmBK / 4;                // packed bytes per weight row per stage
  static constexpr int kWBytes = kGemmBM * kWRow;          // packed weight tile of a stage
  static constexpr int kStageBytes = kXBytes + kWBytes;    // multiple of 1024
  static constexpr int kTmemCols = 512;
  static constexpr int kAslot = kGemmBK / 4;  // TMEM columns per A slot
  static constexpr int kBufs = 2 * BN + kAslot * S <= kTmemCols ? 2 : 1;
  static constexpr int kAcol = kBufs * BN;  // first A slot column
  static constexpr int kBarOffset = S * kStageBytes;
  // split-K: this CTA's partial accumulator tile, int32 [BN tokens][128 rows]
  static constexpr int kPartOffset = kBarOffset + 256;
  static constexpr int kPartBytes = KSPLIT > 1 ? kGemmBM * BN * 4 : 0;
  static constexpr int kNeeded = 1024 + kPartOffset + kPartBytes;
  // The CTA holds all 512 TMEM columns: ask for enough shared memory that a
  // second CTA never fits on the SM (228 KB), so none waits in tcgen05.alloc.
  static constexpr int kMinSmem = 233472 / 2;
  static constexpr int kSmemBytes = kNeeded > kMinSmem ? kNeeded : kMinSmem;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(kAcol + S * kAslot <= kTmemCols, "TMEM budget");
  static_assert(kNeeded <= 232448, "shared memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(S % kGemmProducers == 0, "each ring slot belongs to one producer");
  static_assert(KSPLIT == 1 || KSPLIT == 2 || KSPLIT == 4 || KSPLIT == 8, "row slices of a multiple of 4 rows");
  static_assert(kWRow == 64, "the unpack swizzle below is the 64-byte pattern");
};

template <int BN, int S, bool U8, int KSPLIT = 1>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const float* __restrict__ gamma_ptr, const float* __restrict__ a_scale,
                const int32_t* __restrict__ rowsum, int M, int N, int K, void* __restrict__ y, int y_dtype) {
  using C = GemmCfg<BN, S, KSPLIT>;
  constexpr int NB = C::kBufs;
  constexpr int KSUB = kGemmBK / 128;  // activation boxes per stage
  constexpr int NMMA = kGemmBK / 32;   // MMAs per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;
  uint64_t* accfull = afull + S;
  uint64_t* accempty = accfull + 2;
  uint64_t* done = accempty + 2;
  uint64_t* ready = done + 1;      // split-K: every CTA's partial of the current tile is in its shared memory
  uint64_t* consumed = ready + 1;  // split-K: every CTA has finished reading the partials of that tile
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(consumed + 1);
  int* part = reinterpret_cast<int*>(smem + C::kPartOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + kGemmBM - 1) / kGemmBM;
  const int tiles = n_tiles * ((M + BN - 1) / BN);
  const int nk = (K + kGemmBK - 1) / kGemmBK;
  // The CTAs of a cluster of KSPLIT share each tile; rank r accumulates the
  // K-steps [kb0, kb1).  Clusters walk the tiles persistently.
  const int rank = KSPLIT > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int cid = static_cast<int>(blockIdx.x) / KSPLIT, ncl = static_cast<int>(gridDim.x) / KSPLIT;
  const int kb0 = rank * nk / KSPLIT, kb1 = (rank + 1) * nk / KSPLIT;
  const int nkr = kb1 - kb0;
  const int my_tiles = cid < tiles ? (tiles - cid + ncl - 1) / ncl : 0;

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
    mbar_init(ready, kGemmEpiWarps * KSPLIT);
    mbar_init(consumed, kGemmEpiWarps * KSPLIT);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  if constexpr (KSPLIT > 1) {
    cluster_sync();  // every CTA's barriers initialised before any remote arrival
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();

  const int prod = warp == 0 ? 0 : warp - (1 + kGemmUnpackWarps + kGemmEpiWarps);  // producer index
  if (warp == 0 || warp >= 2 + kGemmUnpackWarps + kGemmEpiWarps) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producers
      // The weights never depend on the previous kernel: the first ring's
      // worth of weight tiles is requested before waiting on it.
      const int total = my_tiles * nkr;
      const int pre = total < S ? total : S;
      for (int g = prod; g < pre; g += kGemmProducers) {
        const int t = cid + (g / nkr) * ncl, kb = kb0 + g % nkr;
        mbar_arrive_expect_tx(&full[g], C::kStageBytes);
        tma_load_2d(smem + g * C::kStageBytes + C::kXBytes, &tmap_w, kb * C::kWRow, (t % n_tiles) * kGemmBM,
                    &full[g]);
      }
      pdl_wait();
      int issued = prod;
      bool ok = true;
      for (int g = prod; g < total; g += kGemmProducers) {
        const int s = g % S;
        const int t = cid + (g / nkr) * ncl, kb = kb0 + g % nkr;
        const int n0 = (t % n_tiles) * kGemmBM, m0 = (t / n_tiles) * BN;
        uint8_t* xs = smem + s * C::kStageBytes;
        if (g >= pre) {
          if (!mbar_wait(&empty[s], ((g / S) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          tma_load_2d(xs + C::kXBytes, &tmap_w, kb * C::kWRow, n0, &full[s]);
        }
#pragma unroll
        for (int i = 0; i < KSUB; ++i) tma_load_2d(xs + i * C::kXSub, &tmap_x, kb * kGemmBK + 128 * i, m0, &full[s]);
        issued = g + kGemmProducers;
      }
      if (!ok) {
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
      for (int t = cid; ok && t < tiles; t += ncl, ++tc) {
        const int b = tc % NB;
        if (!mbar_wait(&accempty[b], ((tc / NB) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * BN;
        for (int kb = 0; kb < nkr; ++kb, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait(&full[s], ph) || !mbar_wait(&afull[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xaddr = smem_addr(smem + s * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < NMMA; ++kk)
            mma_i8_tmemA(dcol, tmem + C::kAcol + C::kAslot * s + 8 * kk,
                         smem_desc_k_sw128(xaddr + (kk >> 2) * C::kXSub + 32 * (kk & 3)), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accfull[b]);
      }
      tc_commit(done);  // arrives once every MMA issued above has finished
      mbar_wait(done, 0);
    }
  } else if (warp < kGemmFirstEpiWarp) {
    // ------------------------------------------------------------ unpack
    const int q = warp & 3;
    const int par = (warp - 2) >> 2;  // this warp takes stages with g % 2 == par
    const int r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    // 64-byte swizzle of the packed tile: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
    const uint32_t swz = static_cast<uint32_t>((r >> 1) & 3);
    const int total = my_tiles * nkr;
    for (int g = par; g < total; g += 2) {
      const int s = g % S;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (g / S) & 1))) break;
      const uint32_t wrow = smem_addr(smem + s * C::kStageBytes + C::kXBytes) + r * C::kWRow;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // two halves of 128 K each -> 32 TMEM columns each
        const uint4 p0 = lds128(wrow + ((static_cast<uint32_t>(2 * h) ^ swz) << 4));
        const uint4 p1 = lds128(wrow + ((static_cast<uint32_t>(2 * h + 1) ^ swz) << 4));
        const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        uint32_t v[32];
#pragma unroll
        for (int wi = 0; wi < 8; ++wi)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t c4 = (pw[wi] >> (2 * j)) & 0x03030303u;
            v[4 * wi + j] = U8 ? c4 : codes_to_signed(c4);
          }
        tmem_st_32x32b_x32(lane_base + C::kAcol + C::kAslot * s + 32 * h, v);
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
    pdl_wait();  // a_scale and rowsum come from the previous kernel
    const float gamma = __ldg(gamma_ptr);
    constexpr int EH = BN >= 64 ? 2 : 1;      // column halves per tile (one per warp of a quarter)
    constexpr int CW = BN / EH < 32 ? BN / EH : 32;
    const int half = (warp - kGemmFirstEpiWarp) >> 2;
    const int col_lo = half * (BN / EH), col_hi = half < EH ? (half + 1) * (BN / EH) : col_lo;
    constexpr int NCH = (BN / EH) / CW;  // column chunks of this warp per tile
    int tc = 0;
    for (int t = cid; t < tiles; t += ncl, ++tc) {
      const int b = tc % NB;
      const int n0 = (t % n_tiles) * kGemmBM;
      const int m0 = (t / n_tiles) * BN;
      // per-token scale and row sum of this warp's columns, one token per lane and
      // chunk, requested before the accumulator wait so the loads overlap it
      float pa[NCH];
      int prs[NCH];
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        const int mm = m0 + col_lo + ch * CW + (lane < CW ? lane : 0);
        const bool inb = col_lo < col_hi && lane < CW && mm < M;
        pa[ch] = inb ? __ldg(a_scale + mm) : 0.0f;
        prs[ch] = (U8 && inb) ? __ldg(rowsum + mm) : 0;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], (tc / NB) & 1))) break;
      tc_fence_after();
      if constexpr (KSPLIT > 1) {
        // ---- split-K: partial -> shared memory, exchange, reduce this CTA's slice of rows
        const int r = 32 * q + lane;  // accumulator row (TMEM lane) this thread drains
        if (tc > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(consumed, (tc - 1) & 1))) break;
#pragma unroll 1
        for (int cc = col_lo; cc < col_hi; cc += CW) {
          uint32_t v[CW];
          if constexpr (CW == 32) {
            tmem_ld_32x32b_x32(lane_base + b * BN + cc, v);
          } else {
            tmem_ld_32x32b_x16(lane_base + b * BN + cc, v);
          }
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < CW; ++j) part[(cc + j) * kGemmBM + r] = static_cast<int>(v[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&accempty[b]);  // the TMEM buffer may be reused
          for (int p = 0; p < KSPLIT; ++p) mbar_arrive_cluster(mapa_shared(smem_addr(ready), p));
        }
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(ready, tc & 1))) break;
        constexpr int RN = kGemmBM / KSPLIT;  // rows reduced by this CTA
        const int rlo = rank * RN;
        const int et = (warp - kGemmFirstEpiWarp) * 32 + lane;  // 0 .. 127
        const uint32_t part_addr = smem_addr(part);
        // four consecutive rows of one token per step: 16-byte loads from every CTA
        for (int e = et; e < (RN / 4) * BN; e += kGemmEpiWarps * 32) {
          const int ml = e / (RN / 4), r4 = rlo + 4 * (e - ml * (RN / 4));
          const uint32_t off = static_cast<uint32_t>((ml * kGemmBM + r4) * 4);
          int4 sum = make_int4(0, 0, 0, 0);
#pragma unroll
          for (int p = 0; p < KSPLIT; ++p) {
            const int4 v = ld_shared_cluster_v4(mapa_shared(part_addr + off, p));
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
          }
          const int m = m0 + ml;
          if (m < M) {
            const int rsm = U8 ? __ldg(rowsum + m) : 0;
            const float am = __ldg(a_scale + m);
            const int sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int n = n0 + r4 + i;
              if (n < N) {
                const int a = sv[i] - rsm;
                const int64_t o = static_cast<int64_t>(m) * N + n;
                if (y_dtype == 2) {
                  static_cast<int32_t*>(y)[o] = a;
                } else {
                  const float val = __fmul_rn(__fmul_rn(__int2float_rn(a), gamma), am);
                  if (y_dtype == 0) static_cast<float*>(y)[o] = val;
                  else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(val);
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0)
          for (int p = 0; p < KSPLIT; ++p) mbar_arrive_cluster(mapa_shared(smem_addr(consumed), p));
      } else {
        // ---- one CTA per tile: dequantise straight from TMEM
        const int n = n0 + 32 * q + lane;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const int cc = col_lo + ch * CW;
          if (cc >= col_hi) break;
          uint32_t v[CW];
          if constexpr (CW == 32) {
            tmem_ld_32x32b_x32(lane_base + b * BN + cc, v);
          } else {
            tmem_ld_32x32b_x16(lane_base + b * BN + cc, v);
          }
          const float my_a = pa[ch];
          const int my_rs = prs[ch];
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
  }

  if constexpr (KSPLIT > 1) {
    tc_fence_before();
    cluster_sync();  // no CTA leaves while a peer may still read its partial tile
  } else {
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bitnet
