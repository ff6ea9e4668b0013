// Decode feed-forward block of BitNet b1.58 in one launch, for M <= 8 tokens.
//
// The block is three BitLinears with squared-ReLU gating between them
// (inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", "Zrób to sam":
// squared ReLU in the FFN, subln normalisation, no biases; kripta.biz 2B4T
// news: ReLU^2 in the FFN layers).  Every BitLinear normalises and
// quantises its input, multiplies by the ternary weights and rescales
// (comrad404.com review, "Метод: как устроен BitNet b1.58"):
//
//   phase 1:  u = BitLinear_up(x), g = BitLinear_gate(x)   (RMSNorm gain_in)
//             h = bf16(RN32(RN32(r*r)*u)), r = g if g > 0 else +0
//   phase 2:  y = BitLinear_down(h)                        (RMSNorm gain_sub)
//
// Both phases are the decode GEMV of gemv.cuh (dp4a over the unsigned codes,
// x_q in shared memory, each CTA quantising the token rows itself), inside
// one cooperative launch of one CTA per SM, with one grid-wide barrier
// between the phases: phase 2 normalises and quantises all of h, which every
// CTA writes a slice of.
//
// Work split.  Phase 1: CTA c owns the features [F*c/G, F*(c+1)/G); an item
// is (pair of features, K chunk), and its 4 slot rows are up f, up f+1,
// gate f, gate f+1, so the CTA holds u and g of its features and computes h
// in the epilogue.  Phase 2: CTA c owns the rows [D*c/G, D*(c+1)/G) of W_down
// in groups of 4.  The CTA's items are numbered phase 1 first, then phase 2,
// and item j belongs to compute warp j % 16.  K is cut into as few chunks
// as the slot size allows (whole rows for K <= 2560): every extra chunk adds
// a bulk copy per row, and issuing copies costs more than the imbalance of
// items between warps that finer chunks would remove.  Each compute warp consumes its
// items from a ring of S slots (S chosen by the host, up to all of the
// warp's items), so the weights of phase 2 are requested while phase 1 still
// computes: for the 2.5B block at M = 1 every weight byte of the whole FFN
// (13.3 MB, 90 KB per CTA) is in flight from the start of the kernel.
//
// A 17th warp makes the initial fill: its lane w issues the first S items of
// compute warp w.  Issuing tens of copies per SM takes microseconds (each
// waits for room in the memory system), so the compute warps do not do it
// themselves: they go straight to the quantisation, and synchronise among
// themselves with a named barrier that the producer warp does not take part
// in.  When a warp has more items than slots (large FFNs), the warp itself
// refills a slot as soon as it has consumed it.
#pragma once

#include <cuda_bf16.h>

#include "gemv.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace bitnet {

constexpr int kFfnWarps = kGemvWarps;                 // compute warps
constexpr int kFfnComputeThreads = kFfnWarps * 32;
constexpr int kFfnThreads = kFfnComputeThreads + 32;  // + the producer warp
constexpr int kFfnSlotBytes = kGemvSlotBytes;  // 4 rows x at most 2560 weights
constexpr int kFfnMaxK = 24576;                // token rows quantised with at most 12 chunks per thread
constexpr int kFfnSmemMax = 227 * 1024 - 2048;  // dynamic shared memory (static scratch beside it)

struct FfnArgs {
  const __nv_bfloat16* x;         // M x D
  const __nv_bfloat16* gain_in;   // D or null
  const uint8_t* w_up;            // F x D/4
  const uint8_t* w_gate;          // F x D/4
  const float* gamma_up;
  const float* gamma_gate;
  const __nv_bfloat16* gain_sub;  // F or null
  const uint8_t* w_down;          // D x F/4
  const float* gamma_down;
  __nv_bfloat16* h;               // M x F
  void* y;                        // M x D
  uint64_t* sync;                 // grid barrier arrival counter
  float eps_in, eps_sub;
  int D, F, y_dtype, slots;
};

// Per-CTA accumulator rows: 2 per feature in phase 1, 1 per row in phase 2.
__host__ __device__ inline int ffn_acc_rows(int D, int F, int G) {
  const int f = (F + G - 1) / G, d = (D + G - 1) / G;
  const int r = 2 * f > d ? 2 * f : d;
  return (r + 3) / 4 * 4;
}

// one mbarrier per ring slot
__host__ __device__ inline int ffn_bar_bytes(int slots) { return kFfnWarps * slots * 8; }

__host__ __device__ inline int ffn_smem_bytes(int mt, int D, int F, int G, int slots) {
  const int kmax = D > F ? D : F;
  return kFfnWarps * slots * kFfnSlotBytes + ffn_bar_bytes(slots) + ffn_acc_rows(D, F, G) * mt * 4 +
         (mt * kmax + 15) / 16 * 16;
}

template <int MT, int MAXC>
__global__ void __launch_bounds__(kFfnThreads, 1) ffn_kernel(const FfnArgs p) {
  constexpr int NT = kFfnComputeThreads;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ QuantScratch qsc;
  __shared__ int barrier_ok;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = p.slots, D = p.D, F = p.F, G = gridDim.x, cta = blockIdx.x;
  uint64_t* full_bars = reinterpret_cast<uint64_t*>(smem + kFfnWarps * S * kFfnSlotBytes);  // [warp][slot]
  const int acc_rows = ffn_acc_rows(D, F, G);
  int* accs = reinterpret_cast<int*>(smem + kFfnWarps * S * kFfnSlotBytes + ffn_bar_bytes(S));
  uint8_t* xs = reinterpret_cast<uint8_t*>(accs) + acc_rows * MT * 4;

  // phase 1: features [f_lo, f_hi)
  const int f_lo = static_cast<int>(static_cast<int64_t>(F) * cta / G);
  const int f_hi = static_cast<int>(static_cast<int64_t>(F) * (cta + 1) / G);
  const int nfeat = f_hi - f_lo;
  const int kc1 = gemv_kchunk(D), nkc1 = (D + kc1 - 1) / kc1;
  const int items1 = (nfeat + 1) / 2 * nkc1;
  // phase 2: rows [r_lo, r_hi) of W_down
  const int r_lo = static_cast<int>(static_cast<int64_t>(D) * cta / G);
  const int r_hi = static_cast<int>(static_cast<int64_t>(D) * (cta + 1) / G);
  const int nrows2 = r_hi - r_lo;
  const int kc2 = gemv_kchunk(F), nkc2 = (F + kc2 - 1) / kc2;
  const int items = items1 + (nrows2 + 3) / 4 * nkc2;
  const int64_t rb1 = D >> 2, rb2 = F >> 2;  // packed row bytes
  auto items_of = [&](int w) { return items > w ? (items - w + kFfnWarps - 1) / kFfnWarps : 0; };

  if (threadIdx.x < kFfnWarps) {
    for (int s = 0; s < S; ++s) mbar_init(&full_bars[threadIdx.x * S + s], 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < acc_rows * MT; i += kFfnThreads) accs[i] = 0;
  __syncthreads();  // the last barrier of the whole CTA; below, only the compute warps synchronise

  // Issue item k of compute warp w into its slot k % S (one thread).
  auto issue = [&](int w, int k, uint64_t policy) {
    const int slot = k % S;
    const int j = w + k * kFfnWarps;
    uint64_t* bar = &full_bars[w * S + slot];
    uint8_t* dst = smem + (w * S + slot) * kFfnSlotBytes;
    if (j < items1) {
      const int gi = j / nkc1, kc = j - gi * nkc1;
      const int f0 = f_lo + 2 * gi;
      const int nf = f_hi - f0 < 2 ? f_hi - f0 : 2;
      const int k0 = kc * kc1;
      const int len = min(kc1, D - k0) >> 2;  // bytes per row
      const int slot_row = kc1 >> 2;
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(2 * nf * len));
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint8_t* base = which ? p.w_gate : p.w_up;
        if (len == rb1) {
          bulk_copy_g2s(dst + which * 2 * slot_row, base + f0 * rb1, static_cast<uint32_t>(nf * len), bar, policy);
        } else {
          for (int r = 0; r < nf; ++r)
            bulk_copy_g2s(dst + (which * 2 + r) * slot_row, base + (f0 + r) * rb1 + (k0 >> 2),
                          static_cast<uint32_t>(len), bar, policy);
        }
      }
    } else {
      const int j2 = j - items1;
      const int gi = j2 / nkc2, kc = j2 - gi * nkc2;
      const int r0 = r_lo + 4 * gi;
      const int nr = r_hi - r0 < 4 ? r_hi - r0 : 4;
      const int k0 = kc * kc2;
      const int len = min(kc2, F - k0) >> 2;
      const int slot_row = kc2 >> 2;
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nr * len));
      if (len == rb2) {
        bulk_copy_g2s(dst, p.w_down + r0 * rb2, static_cast<uint32_t>(nr * len), bar, policy);
      } else {
        for (int r = 0; r < nr; ++r)
          bulk_copy_g2s(dst + r * slot_row, p.w_down + (r0 + r) * rb2 + (k0 >> 2), static_cast<uint32_t>(len), bar,
                        policy);
      }
    }
  };

  if (warp == kFfnWarps) {
    // ---- producer: lane w makes the initial fill of compute warp w's ring.
    // The weights never depend on the previous kernel, so this starts at once.
    if (lane < kFfnWarps) {
      const int n = items_of(lane);
      const uint64_t policy = policy_evict_first();
      for (int k = 0; k < S && k < n; ++k) issue(lane, k, policy);
    }
    return;
  }

  // ---- compute warps.  Everything below reads the outputs of the previous kernel.
  pdl_launch_dependents();
  pdl_wait();
  uint8_t* ring = smem + warp * S * kFfnSlotBytes;
  uint64_t* full = full_bars + warp * S;
  const int my_items = items_of(warp);
  const uint64_t policy = policy_evict_first();

  int k = 0;  // this warp's item counter (ring position)
  bool failed = false;
  // This warp's items with index below j_end: dp4a over the slot, partial
  // sums into the CTA's accumulators, the slot refilled with item k + S.
  auto run_items = [&](int j_end, bool phase1) {
    const int K = phase1 ? D : F;
    const int kchunk = phase1 ? kc1 : kc2, nkc = phase1 ? nkc1 : nkc2;
    const int slot_row = kchunk >> 2;
    for (; !failed && warp + k * kFfnWarps < j_end; ++k) {
      const int j = warp + k * kFfnWarps;
      const int slot = k % S;
      const bool got = mbar_wait(&full[slot], (k / S) & 1);
      if (!__all_sync(0xffffffffu, got)) {
        failed = true;
        break;
      }
      const int jj = phase1 ? j : j - items1;
      const int gi = jj / nkc, kc = jj - gi * nkc;
      const int k0 = kc * kchunk;
      const int len = min(kchunk, K - k0);
      const uint32_t sw = smem_addr(ring + slot * kFfnSlotBytes);
      const uint32_t xa = smem_addr(xs) + k0;
      int acc[4][MT];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll 1
      for (int kk = lane * 16; kk < len; kk += 512) {
        uint32_t xv[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4 u = lds128(xa + m * K + kk);
          xv[m][0] = u.x;
          xv[m][1] = u.y;
          xv[m][2] = u.z;
          xv[m][3] = u.w;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          uint32_t w;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(sw + r * slot_row + (kk >> 2)));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t c4 = (w >> (2 * q)) & 0x03030303u;
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = dp4a_us(c4, xv[m][q], acc[r][m]);
          }
        }
      }
      __syncwarp();
      if (lane == 0 && k + S < my_items) {
        // the slot's generic-proxy reads are done before the next bulk copy into it
        fence_proxy_async_smem();
        issue(warp, k + S, policy);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // phase 1: slot row r is (feature 2gi + (r & 1), branch r >> 1) -> accumulator 2 * feature + branch
        const int fl = 2 * gi + (r & 1);
        const bool valid = phase1 ? fl < nfeat : 4 * gi + r < nrows2;
        const int arow = phase1 ? 2 * fl + (r >> 1) : 4 * gi + r;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int v = __reduce_add_sync(0xffffffffu, acc[r][m]);
          if (lane == r * MT + m && valid) atomicAdd(&accs[arow * MT + m], v);
        }
      }
    }
  };

  // ---- phase 1: quantise x (RMSNorm with gain_in), up and gate products
  float asc[MT];
  int rsum[MT];
#pragma unroll 1
  for (int m = 0; m < MT; ++m) {
    float amax;
    int sum;
    quant_row_cta<__nv_bfloat16, MAXC, false, NT>(p.x + static_cast<int64_t>(m) * D, D, p.gain_in, p.eps_in,
                                                  reinterpret_cast<int8_t*>(xs) + m * D, qsc, amax, sum);
    asc[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    rsum[m] = sum;
  }
  run_items(items1, true);
  sync_threads<NT>();
  {
    const float gu = __ldg(p.gamma_up), gg = __ldg(p.gamma_gate);
    for (int i = threadIdx.x; i < nfeat * MT; i += NT) {
      const int fl = i / MT, m = i - fl * MT;
      const int au = accs[(2 * fl) * MT + m] - rsum[m];
      const int ag = accs[(2 * fl + 1) * MT + m] - rsum[m];
      // each entry is read by exactly one thread, which clears it for phase 2
      // (entries past 2 * nfeat are never written in phase 1)
      accs[(2 * fl) * MT + m] = 0;
      accs[(2 * fl + 1) * MT + m] = 0;
      const float u = __fmul_rn(__fmul_rn(__int2float_rn(au), gu), asc[m]);
      const float g = __fmul_rn(__fmul_rn(__int2float_rn(ag), gg), asc[m]);
      const float r = g > 0.0f ? g : 0.0f;
      p.h[static_cast<int64_t>(m) * F + f_lo + fl] = __float2bfloat16_rn(__fmul_rn(__fmul_rn(r, r), u));
    }
  }

  // ---- every CTA's slice of h is written; phase 2 reads all of it
  const bool synced = grid_barrier<NT>(p.sync, &barrier_ok);

  if (synced) {
#pragma unroll 1
    for (int m = 0; m < MT; ++m) {
      float amax;
      int sum;
      quant_row_cta<__nv_bfloat16, MAXC, true, NT>(p.h + static_cast<int64_t>(m) * F, F, p.gain_sub, p.eps_sub,
                                                   reinterpret_cast<int8_t*>(xs) + m * F, qsc, amax, sum);
      asc[m] = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
      rsum[m] = sum;
    }
    run_items(items, false);
    sync_threads<NT>();
    const float gd = __ldg(p.gamma_down);
    for (int i = threadIdx.x; i < nrows2 * MT; i += NT) {
      const int rr = i / MT, m = i - rr * MT;
      const int a = accs[rr * MT + m] - rsum[m];
      const int64_t o = static_cast<int64_t>(m) * D + r_lo + rr;
      if (p.y_dtype == 2) {
        static_cast<int32_t*>(p.y)[o] = a;
      } else {
        const float v = __fmul_rn(__fmul_rn(__int2float_rn(a), gd), asc[m]);
        if (p.y_dtype == 0) static_cast<float*>(p.y)[o] = v;
        else static_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
      }
    }
  }
  if ((failed || !synced) && lane == 0) {
    // Let copies still in flight land before the CTA's shared memory goes away
    // (a wait that runs out means the copy was never issued).
    for (int kk = k; kk < my_items && kk < k + S; ++kk)
      if (!mbar_wait(&full[kk % S], (kk / S) & 1)) break;
  }
}

}  // namespace bitnet
