// Host side of bitnet_bitlinear_gemv_b3: the fused decode BitLinear on
// base-3 packed weights (gemv_b3.cuh).
#include "host_common.h"
#include "gemv_b3.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

template <int MT, typename T, int MAXC>
cudaError_t launch_b3_t(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                        int K, void* y, int yd, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemv_b3_kernel<MT, T, MAXC>;
  const cudaError_t e = set_smem(kern, gemv_b3_smem_bytes(MT, kGemvB3XMaxBytes / MT), done);
  if (e != cudaSuccess) return e;
  const int64_t groups = (N + kGemvRows - 1) / kGemvRows;
  const int grid = static_cast<int>(groups < sm_count() ? groups : sm_count());
  return launch_pdl(kern, dim3(grid), dim3(kGemvThreads), gemv_b3_smem_bytes(MT, b3_padded_k(K)), s, Wp, gamma, N,
                    K, static_cast<const T*>(x), static_cast<const T*>(gain), eps, y, yd);
}

template <int MT, typename T>
cudaError_t launch_b3_c(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                        int K, void* y, int yd, cudaStream_t s) {
  const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;
  if (per_thread <= 2) return launch_b3_t<MT, T, 2>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 4) return launch_b3_t<MT, T, 4>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if constexpr (sizeof(T) == 2) {
    if (per_thread <= 12) return launch_b3_t<MT, T, 12>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_b3(int M, const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma,
                      int N, int K, void* y, int yd, cudaStream_t s) {
  switch (M) {
    case 1: return launch_b3_c<1, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 2: return launch_b3_c<2, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 3: return launch_b3_c<3, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 4: return launch_b3_c<4, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 5: return launch_b3_c<5, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 6: return launch_b3_c<6, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 7: return launch_b3_c<7, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    case 8: return launch_b3_c<8, T>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

BITNET_DEFINE_TAKE_ERROR(b3)

extern "C" {

bitnet_status bitnet_bitlinear_gemv_b3(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                       const uint8_t* W_b3, const float* gamma, int64_t N, int64_t K, int64_t M,
                                       void* y, int y_dtype, void* stream) {
  if (x == nullptr || W_b3 == nullptr || gamma == nullptr || y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rms_gain, 16) || !aligned(W_b3, 16) || !aligned(y, 16) || !aligned(gamma, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (rms_gain != nullptr && (!std::isfinite(rms_eps) || !(rms_eps > 0.0f))) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 1 || N > INT32_MAX || M < 1 || M > 8) return BITNET_ERR_UNSUPPORTED_SHAPE;
  const int64_t kp = (K + 79) / 80 * 80;
  if (M * kp > kGemvB3XMaxBytes || (x_dtype == BITNET_F32 && K > 8192)) return BITNET_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  const cudaError_t e = x_dtype == BITNET_BF16
                            ? launch_b3<__nv_bfloat16>(m, x, rms_gain, rms_eps, W_b3, gamma, n, k, y, y_dtype, s)
                            : launch_b3<float>(m, x, rms_gain, rms_eps, W_b3, gamma, n, k, y, y_dtype, s);
  return from_cuda(e);
}

}  // extern "C"
