// Host side of the decode products on CUDA cores: bitnet_linear_gemv and the
// fused decode BitLinear bitnet_bitlinear_gemv (gemv.cuh).
#include "host_common.h"
#include "gemv.cuh"
#include "gemv1.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

// Launch plan of gemv_kernel (grid, K-chunk, ring depth, shared memory).
//
// A CTA whose share of W is small (the 2.5B-class decode shapes, about
// 30 KB per SM) has all of it in flight from the start with the default
// ring, and its few rows are cut into chunks of at most 2560 weights so
// that they spread over all 16 warps.  A large share (the 27B-class shapes,
// about 195 KB per SM) is streamed with long chunks through a deep ring, so
// that each SM keeps tens of KB of weights in flight with few, large bulk
// copies.  The thresholds are compile-time constants (a tuning build may
// define them).
#ifndef BITNET_GEMV_SMALL_SHARE
#define BITNET_GEMV_SMALL_SHARE (64 * 1024)
#endif
#ifndef BITNET_GEMV_BIG_CHUNK
#define BITNET_GEMV_BIG_CHUNK 2688
#endif
#ifndef BITNET_GEMV_BIG_RING
#define BITNET_GEMV_BIG_RING (86 * 1024)
#endif
constexpr int kGemvSmemMax = 232448 - 2048;  // 227 KB less the fused kernel's static scratch

struct GemvPlan {
  int grid, kchunk, nslots, smem, l2_prefetch;
};

GemvPlan gemv_plan(int mt, int N, int K, bool xs) {
  GemvPlan p;
  const int64_t groups = (N + kGemvRows - 1) / kGemvRows;
  p.grid = static_cast<int>(groups < sm_count() ? groups : sm_count());
  const int64_t rows = (N + p.grid - 1) / p.grid;
  const int64_t share = rows * (K / 4);
  p.l2_prefetch = share > BITNET_GEMV_SMALL_SHARE ? 1 : 0;
  if (share <= BITNET_GEMV_SMALL_SHARE) {
    p.kchunk = gemv_kchunk(K);
    p.nslots = kGemvSlots;
  } else {
    p.kchunk = gemv_kchunk_max(K, BITNET_GEMV_BIG_CHUNK);
    const int per_warp = BITNET_GEMV_BIG_RING / (kGemvWarps * p.kchunk);
    p.nslots = per_warp < 2 ? 2 : (per_warp > kGemvMaxSlots ? kGemvMaxSlots : per_warp);
  }
  while (p.nslots > 1 && gemv_plan_smem_bytes(mt, K, xs, p.kchunk, p.nslots) > kGemvSmemMax) --p.nslots;
  p.smem = gemv_plan_smem_bytes(mt, K, xs, p.kchunk, p.nslots);
  return p;
}

// Launch plan of gemv1_kernel (one token): S column segments per row (the
// fewest that leave each lane at most kGemv1MaxPairs word pairs), NP pairs
// per lane, slots of R whole rows (a multiple of the 16/S rows the warps take
// at once, about BITNET_GEMV1_SLOT_TARGET bytes), a ring of about
// BITNET_GEMV1_RING_TARGET bytes, and the rest of a large share prefetched
// into L2.  The kernel's shared memory stays under half an SM's (two CTAs
// per SM, so that a launch overlaps the previous one).  Returns false for a
// share of at most BITNET_GEMV_SMALL_SHARE bytes per CTA and when K is beyond
// the register budget (K > 16 * 16 * 64 * kGemv1MaxPairs); those shapes take
// gemv_kernel.
#ifndef BITNET_GEMV1_SLOT_TARGET
#define BITNET_GEMV1_SLOT_TARGET (48 * 1024)
#endif
#ifndef BITNET_GEMV1_RING_TARGET
#define BITNET_GEMV1_RING_TARGET (88 * 1024)
#endif
#ifndef BITNET_GEMV1_RING_TARGET1
#define BITNET_GEMV1_RING_TARGET1 (176 * 1024)
#endif
#ifndef BITNET_GEMV1_WARPS
#define BITNET_GEMV1_WARPS 16
#endif
constexpr int kGemv1SmemMax = 232448 / 2 - 2048 - 1024;  // two CTAs per SM, each with static scratch
constexpr int kGemv1SmemMax1 = 232448 - 2048;            // one CTA per SM

struct Gemv1Plan {
  int grid, warps, S, NP, R, nslots, rows_max, smem, l2_prefetch;
};

int gemv1_segw(int Bw, int S) { return ((Bw + S - 1) / S + 1) & ~1; }

bool gemv1_plan(int N, int K, bool xs, Gemv1Plan& p, bool gate = false) {
  const int B = K / 4, Bw = B / 4;
  p.warps = BITNET_GEMV1_WARPS;
  const int smem_max = p.warps == 16 ? kGemv1SmemMax : kGemv1SmemMax1;
  p.S = 1;
  while (p.S < kGemvWarps && gemv1_segw(Bw, p.S) > 64 * kGemv1MaxPairs) p.S *= 2;
  const int segw = gemv1_segw(Bw, p.S);
  if (segw > 64 * kGemv1MaxPairs) return false;
  p.NP = (segw + 63) / 64;
  p.grid = N < sm_count() ? N : sm_count();
  p.rows_max = (N + p.grid - 1) / p.grid;
  // a small share (a few rows per SM) is latency-bound: the item kernel, whose
  // 16 warps each start on their own first item at once, serves it better
  if (static_cast<int64_t>(p.rows_max) * B <= BITNET_GEMV_SMALL_SHARE) return false;
  const int RG = p.warps / p.S;
  const int mats = gate ? 2 : 1;  // GATE: a slot holds the rows of both matrices
  const int per = BITNET_GEMV1_SLOT_TARGET / (mats * RG * B);
  p.R = RG * (per > 1 ? per : 1);
  if (p.R > p.rows_max) p.R = p.rows_max;
  const int slot_bytes = mats * p.R * B;
  const int slots_per_cta = (p.rows_max + p.R - 1) / p.R;
  p.nslots = (p.warps == 16 ? BITNET_GEMV1_RING_TARGET : BITNET_GEMV1_RING_TARGET1) / slot_bytes;
  if (p.nslots < 2) p.nslots = 2;
  if (p.nslots > kGemv1MaxSlots) p.nslots = kGemv1MaxSlots;
  if (p.nslots > slots_per_cta) p.nslots = slots_per_cta;
  while (p.nslots > 1 && gemv1_smem_bytes(K, xs, slot_bytes, p.nslots, p.rows_max, p.S, gate) > smem_max) --p.nslots;
  p.smem = gemv1_smem_bytes(K, xs, slot_bytes, p.nslots, p.rows_max, p.S, gate);
  if (p.smem > smem_max) return false;
#ifndef BITNET_GEMV1_L2_PREFETCH
#define BITNET_GEMV1_L2_PREFETCH 1
#endif
  p.l2_prefetch = BITNET_GEMV1_L2_PREFETCH &&
                  static_cast<int64_t>(p.rows_max) * B > static_cast<int64_t>(p.nslots) * p.R * B;
  return true;
}

template <bool U8, int NP, int NWARPS, bool FUSED, typename T, int MAXC, bool GATE = false>
cudaError_t launch_gemv1_w(const Gemv1Plan& p, const uint8_t* Wp, const float* gamma, int N, int K,
                            const int8_t* xq, const float* a, const int32_t* rs, const T* x, const T* gain,
                            float eps, void* y, int yd, cudaStream_t s, const uint8_t* Wp2 = nullptr,
                            const float* gamma2 = nullptr) {
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemv1_kernel<U8, NP, NWARPS, FUSED, T, MAXC, GATE>;
  const cudaError_t e = set_smem(kern, NWARPS == 16 ? kGemv1SmemMax : kGemv1SmemMax1, done);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(p.grid), dim3(NWARPS * 32), p.smem, s, Wp, gamma, Wp2, gamma2, N, K, xq, a, rs, x,
                    gain, eps, y, yd, p.S, p.R, p.nslots, p.rows_max, p.l2_prefetch);
}

template <bool U8, int NP, bool FUSED, typename T, int MAXC>
cudaError_t launch_gemv1_np(const Gemv1Plan& p, const uint8_t* Wp, const float* gamma, int N, int K,
                            const int8_t* xq, const float* a, const int32_t* rs, const T* x, const T* gain,
                            float eps, void* y, int yd, cudaStream_t s) {
  static_assert(BITNET_GEMV1_WARPS == 16 || BITNET_GEMV1_WARPS == 32, "16 or 32 warps");
  return launch_gemv1_w<U8, NP, BITNET_GEMV1_WARPS, FUSED, T, MAXC>(p, Wp, gamma, N, K, xq, a, rs, x, gain, eps, y,
                                                                    yd, s);
}

template <bool U8, bool FUSED, typename T = float, int MAXC = 1>
cudaError_t launch_gemv1(const Gemv1Plan& p, const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq,
                         const float* a, const int32_t* rs, const T* x, const T* gain, float eps, void* y, int yd,
                         cudaStream_t s) {
  switch (p.NP) {
    case 1: return launch_gemv1_np<U8, 1, FUSED, T, MAXC>(p, Wp, gamma, N, K, xq, a, rs, x, gain, eps, y, yd, s);
    case 2: return launch_gemv1_np<U8, 2, FUSED, T, MAXC>(p, Wp, gamma, N, K, xq, a, rs, x, gain, eps, y, yd, s);
    case 3: return launch_gemv1_np<U8, 3, FUSED, T, MAXC>(p, Wp, gamma, N, K, xq, a, rs, x, gain, eps, y, yd, s);
    default: return launch_gemv1_np<U8, 4, FUSED, T, MAXC>(p, Wp, gamma, N, K, xq, a, rs, x, gain, eps, y, yd, s);
  }
}

template <int MT, bool U8, bool XS>
cudaError_t launch_gemv_x(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                          const int32_t* rs, void* y, int yd, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(gemv_kernel<MT, U8, XS>, kGemvSmemMax, done);
  if (e != cudaSuccess) return e;
  const GemvPlan p = gemv_plan(MT, N, K, XS);
  if (p.smem > kGemvSmemMax) return cudaErrorInvalidValue;
  return launch_pdl(gemv_kernel<MT, U8, XS>, dim3(p.grid), dim3(kGemvThreads), p.smem, s, Wp, gamma, N, K, xq, a, rs,
                    static_cast<const float*>(nullptr), static_cast<const float*>(nullptr), 0.0f, y, yd, p.kchunk,
                    p.nslots, p.l2_prefetch);
}

template <int MT, bool U8>
cudaError_t launch_gemv_t(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                          const int32_t* rs, void* y, int yd, cudaStream_t s) {
  if constexpr (MT == 1) {
    Gemv1Plan p;
    if (gemv1_plan(N, K, false, p))
      return launch_gemv1<U8, false>(p, Wp, gamma, N, K, xq, a, rs, static_cast<const float*>(nullptr),
                                     static_cast<const float*>(nullptr), 0.0f, y, yd, s);
  }
  if (static_cast<int64_t>(MT) * K <= kGemvXMaxBytes)
    return launch_gemv_x<MT, U8, true>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
  return launch_gemv_x<MT, U8, false>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
}

template <bool U8>
cudaError_t launch_gemv_u(int M, const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                          const int32_t* rs, void* y, int yd, cudaStream_t s) {
  switch (M) {
    case 1: return launch_gemv_t<1, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 2: return launch_gemv_t<2, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 3: return launch_gemv_t<3, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 4: return launch_gemv_t<4, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 5: return launch_gemv_t<5, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 6: return launch_gemv_t<6, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 7: return launch_gemv_t<7, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    case 8: return launch_gemv_t<8, U8>(Wp, gamma, N, K, xq, a, rs, y, yd, s);
    default: return cudaErrorInvalidValue;
  }
}

// Fused decode BitLinear: quantisation (and RMSNorm) of M <= 8 token rows in
// every CTA's prologue, then the GEMV.
template <int MT, typename T, int MAXC>
cudaError_t launch_fused_t(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                           int K, void* y, int yd, cudaStream_t s) {
  if constexpr (MT == 1) {
    Gemv1Plan p;
    if (gemv1_plan(N, K, true, p))
      return launch_gemv1<true, true, T, MAXC>(p, Wp, gamma, N, K, static_cast<const int8_t*>(nullptr),
                                               static_cast<const float*>(nullptr),
                                               static_cast<const int32_t*>(nullptr), static_cast<const T*>(x),
                                               static_cast<const T*>(gain), eps, y, yd, s);
  }
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemv_kernel<MT, true, true, true, T, MAXC>;
  const cudaError_t e = set_smem(kern, kGemvSmemMax, done);
  if (e != cudaSuccess) return e;
  const GemvPlan p = gemv_plan(MT, N, K, true);
  if (p.smem > kGemvSmemMax) return cudaErrorInvalidValue;
  return launch_pdl(kern, dim3(p.grid), dim3(kGemvThreads), p.smem, s, Wp, gamma, N, K,
                    static_cast<const int8_t*>(nullptr), static_cast<const float*>(nullptr),
                    static_cast<const int32_t*>(nullptr), static_cast<const T*>(x), static_cast<const T*>(gain), eps, y,
                    yd, p.kchunk, p.nslots, p.l2_prefetch);
}

template <int MT, typename T>
cudaError_t launch_fused_c(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                           int K, void* y, int yd, cudaStream_t s) {
  // 8-element chunks per thread of the quantisation prologue: the fixed-order
  // RMSNorm sum is defined on 256 threads; without a norm all 512 take part
  // (fewer registers, so the next launch's CTA can share the SM)
  const int nthr = gain != nullptr ? kQuantThreads : kGemvThreads;
  const int per_thread = (K / 8 + nthr - 1) / nthr;
  if constexpr (MT == 1) {
    // one token, a row past the norm's register budget: the instantiation
    // with the streamed normalisation alone (MAXC 0), so that no unused
    // register-resident chunks weigh on the kernel's register allocation
    constexpr int kResident = BN_QUANT_STREAM_BYTES / static_cast<int>(sizeof(Chunk8<T>));
    if (gain != nullptr && per_thread > kResident)
      return launch_fused_t<1, T, 0>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  }
  if (per_thread <= 1) return launch_fused_t<MT, T, 1>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 2) return launch_fused_t<MT, T, 2>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 4) return launch_fused_t<MT, T, 4>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 8) return launch_fused_t<MT, T, 8>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if constexpr (sizeof(T) == 2 && MT > 1) return launch_fused_t<MT, T, 16>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_fused(int M, const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma,
                         int N, int K, void* y, int yd, cudaStream_t s) {
  switch (M) {
    case 1: return launch_fused_c<1, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 2: return launch_fused_c<2, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 3: return launch_fused_c<3, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 4: return launch_fused_c<4, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 5: return launch_fused_c<5, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 6: return launch_fused_c<6, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 7: return launch_fused_c<7, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 8: return launch_fused_c<8, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int NP, int MAXC>
cudaError_t launch_upgate1_np(const Gemv1Plan& p, const __nv_bfloat16* x, const __nv_bfloat16* gain, float eps,
                              const uint8_t* Wu, const float* gu, const uint8_t* Wg, const float* gg, int F, int D,
                              __nv_bfloat16* h, cudaStream_t s) {
  return launch_gemv1_w<true, NP, BITNET_GEMV1_WARPS, true, __nv_bfloat16, MAXC, true>(
      p, Wu, gu, F, D, static_cast<const int8_t*>(nullptr), static_cast<const float*>(nullptr),
      static_cast<const int32_t*>(nullptr), x, gain, eps, h, BITNET_BF16, s, Wg, gg);
}

template <int MAXC>
cudaError_t launch_upgate1_c(const Gemv1Plan& p, const __nv_bfloat16* x, const __nv_bfloat16* gain, float eps,
                             const uint8_t* Wu, const float* gu, const uint8_t* Wg, const float* gg, int F, int D,
                             __nv_bfloat16* h, cudaStream_t s) {
  switch (p.NP) {
    case 1: return launch_upgate1_np<1, MAXC>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
    case 2: return launch_upgate1_np<2, MAXC>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
    case 3: return launch_upgate1_np<3, MAXC>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
    default: return launch_upgate1_np<4, MAXC>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
  }
}

}  // namespace

// The decode FFN's up and gate projections for one token with the gating
// in the epilogue (gemv1_kernel<..., GATE>): x (D bf16, optional RMSNorm
// gain) -> h (F bf16).  *used = false (nothing launched) where the
// one-token whole-row-slot plan does not apply.
cudaError_t bitnet_host::launch_ffn_upgate_gemv1(const __nv_bfloat16* x, const __nv_bfloat16* gain, float eps,
                                                 const uint8_t* Wu, const float* gu, const uint8_t* Wg,
                                                 const float* gg, int F, int D, __nv_bfloat16* h, cudaStream_t s,
                                                 bool* used) {
  Gemv1Plan p;
  *used = false;
  if (D > kGemvXMaxBytes || !gemv1_plan(F, D, true, p, true)) return cudaSuccess;
  const int nthr = gain != nullptr ? kQuantThreads : kGemvThreads;
  const int per_thread = (D / 8 + nthr - 1) / nthr;
  *used = true;
  // a long normalised input row: the streamed normalisation alone (MAXC 0); without a norm
  // D <= 21504 gives at most 6 chunks per thread
  if (gain != nullptr && per_thread > BN_QUANT_STREAM_BYTES / static_cast<int>(sizeof(Chunk8<__nv_bfloat16>)))
    return launch_upgate1_c<0>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
  if (per_thread <= 1) return launch_upgate1_c<1>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
  if (per_thread <= 2) return launch_upgate1_c<2>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
  if (per_thread <= 4) return launch_upgate1_c<4>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
  return launch_upgate1_c<8>(p, x, gain, eps, Wu, gu, Wg, gg, F, D, h, s);
}

BITNET_DEFINE_TAKE_ERROR(gemv)

extern "C" {

bitnet_status bitnet_linear_gemv(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, const int8_t* x_q,
                                 const float* a_scale, const int32_t* x_rowsum, int64_t M, void* y, int y_dtype,
                                 void* stream) {
  const bitnet_status st = check_linear(W_packed, gamma, N, K, x_q, a_scale, x_rowsum, M, y, y_dtype);
  if (st != BITNET_OK) return st;
  if (M > 8) return BITNET_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  const cudaError_t e = x_rowsum != nullptr
                            ? launch_gemv_u<true>(m, W_packed, gamma, n, k, x_q, a_scale, x_rowsum, y, y_dtype, s)
                            : launch_gemv_u<false>(m, W_packed, gamma, n, k, x_q, a_scale, x_rowsum, y, y_dtype, s);
  return from_cuda(e);
}

}  // extern "C"

namespace {

bitnet_status check_bitlinear_gemv(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                   const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                   const void* y, int y_dtype) {
  if (x == nullptr || W_packed == nullptr || gamma == nullptr || y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rms_gain, 16) || !aligned(W_packed, 16) || !aligned(y, 16) || !aligned(gamma, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (rms_gain != nullptr && (!std::isfinite(rms_eps) || !(rms_eps > 0.0f))) return BITNET_ERR_INVALID_ARG;
  const int64_t kmax = x_dtype == BITNET_BF16 ? 32768 : 16384;
  if (!valid_k(K) || K > kmax || N < 1 || N > INT32_MAX || M < 1 || M > 8 || M * K > kGemvXMaxBytes)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

cudaError_t launch_bitlinear_gemv(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                  const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                  void* y, int y_dtype, cudaStream_t s) {
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  return x_dtype == BITNET_BF16
             ? launch_fused<__nv_bfloat16>(m, x, rms_gain, rms_eps, W_packed, gamma, n, k, y, y_dtype, s)
             : launch_fused<float>(m, x, rms_gain, rms_eps, W_packed, gamma, n, k, y, y_dtype, s);
}

}  // namespace

extern "C" {

bitnet_status bitnet_bitlinear_gemv(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                    const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                    void* y, int y_dtype, void* stream) {
  const bitnet_status st = check_bitlinear_gemv(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype);
  if (st != BITNET_OK) return st;
  return from_cuda(launch_bitlinear_gemv(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype,
                                         static_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_bitlinear_gemv_host(const void* x_host, void* x, int x_dtype, const void* rms_gain,
                                         float rms_eps, const uint8_t* W_packed, const float* gamma, int64_t N,
                                         int64_t K, int64_t M, void* y, void* y_host, int y_dtype, void* stream) {
  if (x_host == nullptr || y_host == nullptr) return BITNET_ERR_INVALID_ARG;
  const bitnet_status st = check_bitlinear_gemv(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(M * K) * (x_dtype == BITNET_BF16 ? 2 : 4);
  const size_t yb = static_cast<size_t>(M * N) * (y_dtype == BITNET_BF16 ? 2 : 4);
  cudaError_t e = cudaMemcpyAsync(x, x_host, xb, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = launch_bitlinear_gemv(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(y_host, y, yb, cudaMemcpyDeviceToHost, s);
  return from_cuda(e);
}

}  // extern "C"
