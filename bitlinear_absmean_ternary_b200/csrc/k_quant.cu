// Host side of bitnet_quant_act: per-token absmax int8 quantisation with the
// optional fused RMSNorm (quant.cuh: a CTA per row; quant_rows.cuh: a warp
// per row for many bf16 rows).
#include "host_common.h"
#include "quant.cuh"
#include "quant_rows.cuh"
#include "quant_stream.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

template <typename T, int MAXC, int NTHR = kQuantThreads>
cudaError_t launch_quant_t(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                           int32_t* rs, cudaStream_t s, int threads = kQuantThreads) {
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(quant_act_kernel<T, MAXC, NTHR>, 0, done);
  if (e != cudaSuccess) return e;
  const int early = M <= sm_count() ? 1 : 0;  // the whole grid is resident at once
  return launch_pdl(quant_act_kernel<T, MAXC, NTHR>, dim3(static_cast<unsigned>(M)), dim3(threads), 0, s,
                    static_cast<const T*>(x), K, static_cast<const T*>(gain), eps, xq, a, rs, early);
}

template <int MAXC, bool NORM>
cudaError_t launch_quant_rows_t(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                                int32_t* rs, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(quant_rows_kernel<MAXC, NORM>, 0, done);
  if (e != cudaSuccess) return e;
  const int64_t grid = (M + kQuantRowsWarps - 1) / kQuantRowsWarps;
  return launch_pdl(quant_rows_kernel<MAXC, NORM>, dim3(static_cast<unsigned>(grid)), dim3(kQuantRowsThreads), 0, s,
                    static_cast<const __nv_bfloat16*>(x), M, K, static_cast<const __nv_bfloat16*>(gain), eps, xq, a,
                    rs);
}

template <bool NORM>
cudaError_t launch_quant_rows(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                              int32_t* rs, cudaStream_t s) {
  const int per_lane = (K / 8 + 31) / 32;
#define BN_QROWS(C) \
  if (per_lane <= C) return launch_quant_rows_t<C, NORM>(x, M, K, gain, eps, xq, a, rs, s);
  BN_QROWS(2) BN_QROWS(4) BN_QROWS(6) BN_QROWS(8) BN_QROWS(10) BN_QROWS(12) BN_QROWS(16) BN_QROWS(20)
  BN_QROWS(24)
#undef BN_QROWS
  return cudaErrorInvalidValue;
}

template <typename T, bool NORM, int NTHR>
cudaError_t launch_quant_stream_n(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                                  int32_t* rs, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  // the largest ring: three 64-KB rows (bf16 K = 32768 or f32 K = 16384 with the gain)
  const cudaError_t e = set_smem(quant_stream_kernel<T, NORM, NTHR>, 3 * 65536, done);
  if (e != cudaSuccess) return e;
  const int smem = quant_stream_smem_bytes<T, NORM>(K);
  const int fit = 232448 / (smem + 4096);  // rings per SM by shared memory
  const int most = NTHR == 256 ? 4 : 2;    // and by threads and registers
  const int per_sm = fit > most ? most : (fit < 1 ? 1 : fit);
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const int64_t grid = M < cap ? M : cap;
  return launch_pdl(quant_stream_kernel<T, NORM, NTHR>, dim3(static_cast<unsigned>(grid)), dim3(NTHR),
                    static_cast<size_t>(smem), s, static_cast<const T*>(x), static_cast<int>(M), K,
                    static_cast<const T*>(gain), eps, xq, a, rs);
}

// Rows of at least this many bytes, more than two per SM: the persistent
// kernel that streams rows through shared memory (quant_stream.cuh), with
// 256 threads per CTA up to kQuantStreamWideRowBytes and 512 beyond.  Shorter
// rows keep the CTA-per-row kernel (measured, bf16 rows, back to back:
// K = 6912 0.65 of HBM either way; K = 12288 0.86 streamed against 0.72;
// K = 21504 0.79 against 0.65).
constexpr int kQuantStreamMinRowBytes = 16384;
constexpr int kQuantStreamWideRowBytes = 24576;

template <typename T, bool NORM>
cudaError_t launch_quant_stream_t(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                                  int32_t* rs, cudaStream_t s) {
  if (K * static_cast<int>(sizeof(T)) <= kQuantStreamWideRowBytes)
    return launch_quant_stream_n<T, NORM, 256>(x, M, K, gain, eps, xq, a, rs, s);
  return launch_quant_stream_n<T, NORM, 512>(x, M, K, gain, eps, xq, a, rs, s);
}

// Token count from which the warp-per-row kernel takes over (bf16 input,
// K <= 6144): from there on it keeps more rows in flight per SM; below, a CTA
// per row spreads a short batch over more SMs.
constexpr int64_t kQuantRowsMinM = 512;

template <typename T>
cudaError_t launch_quant(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                         int32_t* rs, cudaStream_t s) {
  if (K * static_cast<int>(sizeof(T)) >= kQuantStreamMinRowBytes && M > 2 * static_cast<int64_t>(sm_count()))
    return gain != nullptr ? launch_quant_stream_t<T, true>(x, M, K, gain, eps, xq, a, rs, s)
                           : launch_quant_stream_t<T, false>(x, M, K, gain, eps, xq, a, rs, s);
  if constexpr (sizeof(T) == 2) {
    if (M >= kQuantRowsMinM && K <= 32 * 8 * kQuantRowsMaxChunks)
      return gain != nullptr ? launch_quant_rows<true>(x, M, K, gain, eps, xq, a, rs, s)
                             : launch_quant_rows<false>(x, M, K, gain, eps, xq, a, rs, s);
  }
  const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;
  if (gain == nullptr && M <= sm_count() && (K / 8 <= 768 || K / 8 > 4 * kQuantThreads)) {
    // No norm and a row per SM: up to 1024 threads per row (a shorter chain of
    // loads and arithmetic per row), one chunk each for rows of up to 768
    // chunks, four for rows too long for 256 threads at four (in between, the
    // 256-thread launch below; more warps there made the cross-warp reductions
    // cost more than they save, measured at M = 64, K = 6912).  Measured: one
    // row of K = 21504 3.21 -> 2.69 us, 16 rows 3.28 -> 2.77 us.
    const int nc = K / 8;
    const int mc = nc <= 768 ? 1 : 4;
    const int threads = ((nc + mc - 1) / mc + 31) / 32 * 32;
    if (mc == 1) return launch_quant_t<T, 1, 1024>(x, M, K, gain, eps, xq, a, rs, s, threads);
    return launch_quant_t<T, 4, 1024>(x, M, K, gain, eps, xq, a, rs, s, threads);
  }
  if (gain == nullptr) {
    // No norm, so no fixed order: the fewest whole warps (at most 256 threads)
    // that give every thread the same number of 8-element chunks.
    const int mc = per_thread <= 1 ? 1 : per_thread <= 2 ? 2 : per_thread <= 4 ? 4 : per_thread <= 8 ? 8 : 16;
    const int threads = ((K / 8 + mc - 1) / mc + 31) / 32 * 32;
    if (mc == 1) return launch_quant_t<T, 1>(x, M, K, gain, eps, xq, a, rs, s, threads);
    if (mc == 2) return launch_quant_t<T, 2>(x, M, K, gain, eps, xq, a, rs, s, threads);
    if (mc == 4) return launch_quant_t<T, 4>(x, M, K, gain, eps, xq, a, rs, s, threads);
    if (mc == 8) return launch_quant_t<T, 8>(x, M, K, gain, eps, xq, a, rs, s, threads);
    if constexpr (sizeof(T) == 2) return launch_quant_t<T, 16>(x, M, K, gain, eps, xq, a, rs, s, threads);
    return cudaErrorInvalidValue;
  }
  // With the norm, rows past the register budget are read in three passes
  // (quant_row_norm_stream); when every row has its own SM, 1024 threads per
  // row take the two order-free passes in one batch each.
  constexpr int kResidentChunks = BN_QUANT_STREAM_BYTES / static_cast<int>(sizeof(Chunk8<T>));
  if (per_thread > kResidentChunks && M <= sm_count())
    return launch_quant_t<T, kResidentChunks + 1, 1024>(x, M, K, gain, eps, xq, a, rs, s, 1024);
  if (per_thread <= 1) return launch_quant_t<T, 1>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 2) return launch_quant_t<T, 2>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 4) return launch_quant_t<T, 4>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 8) return launch_quant_t<T, 8>(x, M, K, gain, eps, xq, a, rs, s);
  if constexpr (sizeof(T) == 2) return launch_quant_t<T, 16>(x, M, K, gain, eps, xq, a, rs, s);
  return cudaErrorInvalidValue;
}

}  // namespace

BITNET_DEFINE_TAKE_ERROR(quant)

extern "C" {

bitnet_status bitnet_quant_act(const void* x, int x_dtype, int64_t M, int64_t K, const void* rms_gain, float rms_eps,
                               int8_t* x_q, float* a_scale, int32_t* x_rowsum, void* stream) {
  if (x == nullptr || x_q == nullptr || a_scale == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_q, 16) || !aligned(rms_gain, 16) || !aligned(a_scale, 4) || !aligned(x_rowsum, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (rms_gain != nullptr && (!std::isfinite(rms_eps) || !(rms_eps > 0.0f))) return BITNET_ERR_INVALID_ARG;
  const int64_t kmax = x_dtype == BITNET_BF16 ? 32768 : 16384;
  if (!valid_k(K) || K > kmax || M < 1 || M > INT32_MAX) return BITNET_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      x_dtype == BITNET_BF16
          ? launch_quant<__nv_bfloat16>(x, M, static_cast<int>(K), rms_gain, rms_eps, x_q, a_scale, x_rowsum, s)
          : launch_quant<float>(x, M, static_cast<int>(K), rms_gain, rms_eps, x_q, a_scale, x_rowsum, s);
  return from_cuda(e);
}

}  // extern "C"
