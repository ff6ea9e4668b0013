// Host side of bitnet_bitlinear_gemm: the BitLinear for decode-sized batches
// (M <= 64) -- quantisation of the token rows (with the optional RMSNorm)
// into the workspace, then bitnet_linear_gemm's product (two launches) -- and
// of bitnet_bitlinear_gemm_stream_k: the same in ONE launch, the quantisation
// inside the stream-K product (gemm_sk.cuh).  Measured on B200, the one-launch
// kernel was the slower of the two (27B FFN at M = 16: 23.6 and 26.7 us per
// linear against 21.2 and 25.2 us; its grid barrier costs more than the kernel
// boundary, which programmatic dependent launch overlaps with the product's
// weight prefetch), so the entry point without a suffix takes two launches.
#include "host_common.h"
#include "gemm_sk.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

// Workspace layout: stream-K flags and partial tiles (as bitnet_linear_gemm),
// the grid barrier's two words, the scales, the row sums, x_q.
struct FqLayout {
  size_t bar, a, rs, xq, total;
};

FqLayout fq_layout(int64_t M, int64_t K) {
  const int G = sm_count();
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  FqLayout L;
  L.bar = sk_flag_bytes(G) + sk_slot_bytes(G);
  L.a = L.bar + 256;
  L.rs = L.a + r256(static_cast<size_t>(M) * 4);
  L.xq = L.rs + r256(static_cast<size_t>(M) * 4);
  L.total = L.xq + r256(static_cast<size_t>(M) * K);
  return L;
}

template <int BN, typename XT, int MAXC>
cudaError_t launch_fq_t(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                        int K, int M, void* y, int yd, uint8_t* ws, cudaStream_t s) {
  using C = SkCfg<BN, false>;
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemm_sk_kernel<BN, true, false, XT, MAXC>;
  const cudaError_t e = set_smem(kern, C::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const FqLayout L = fq_layout(M, K);
  SkQuant<XT> qa;
  qa.x = static_cast<const XT*>(x);
  qa.gain = static_cast<const XT*>(gain);
  qa.eps = eps;
  qa.xq = reinterpret_cast<int8_t*>(ws + L.xq);
  qa.a = reinterpret_cast<float*>(ws + L.a);
  qa.rs = reinterpret_cast<int32_t*>(ws + L.rs);
  qa.bar = reinterpret_cast<unsigned int*>(ws + L.bar);
  CUtensorMap mx, mw;
  if (!make_map_u8(&mx, qa.xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&mw, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4),
                   kGemmBK / 4, kGemmBM, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  const int64_t units = static_cast<int64_t>((N + kGemmBM - 1) / kGemmBM) * ((K + kGemmBK - 1) / kGemmBK);
  const int sms = sm_count();
  const int G = static_cast<int>(units < sms ? units : sms);
  unsigned int* flags = reinterpret_cast<unsigned int*>(ws);
  int* parts = reinterpret_cast<int*>(ws + sk_flag_bytes(sms));
  return launch_pdl(kern, dim3(G), dim3(kSkThreads), C::kSmemBytes, s, mx, mw, mw, gamma, gamma,
                    static_cast<const float*>(qa.a), static_cast<const int32_t*>(qa.rs), M, N, K, y, yd, flags, parts,
                    qa);
}

template <int BN, typename XT>
cudaError_t launch_fq_c(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                        int K, int M, void* y, int yd, uint8_t* ws, cudaStream_t s) {
  const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;  // chunks per unpack thread
  if (per_thread <= 2) return launch_fq_t<BN, XT, 2>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  if (per_thread <= 4) return launch_fq_t<BN, XT, 4>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  if (per_thread <= 8) return launch_fq_t<BN, XT, 8>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  if constexpr (sizeof(XT) == 2) return launch_fq_t<BN, XT, 16>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  return cudaErrorInvalidValue;
}

template <typename XT>
cudaError_t launch_fq(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N, int K,
                      int M, void* y, int yd, uint8_t* ws, cudaStream_t s) {
  if (M <= 16) return launch_fq_c<16, XT>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  if (M <= 32) return launch_fq_c<32, XT>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
  return launch_fq_c<64, XT>(x, gain, eps, Wp, gamma, N, K, M, y, yd, ws, s);
}

}  // namespace

BITNET_DEFINE_TAKE_ERROR(gemm_fused)

extern "C" {

size_t bitnet_bitlinear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 64 || N < 1 || N > INT32_MAX || !valid_k(K) || K > 32768) return 0;
  return fq_layout(M, K).total;
}

}  // extern "C"

namespace {

// The fused BitLinear with the one-launch stream-K kernel forced (force_sk), or chosen by sk_preferred.
bitnet_status bitlinear_gemm(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                             const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M, void* y,
                             int y_dtype, void* workspace, size_t workspace_bytes, void* stream, bool force_sk) {
  if (x == nullptr || W_packed == nullptr || gamma == nullptr || y == nullptr || workspace == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rms_gain, 16) || !aligned(W_packed, 16) || !aligned(y, 16) ||
      !aligned(workspace, 16) || !aligned(gamma, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (rms_gain != nullptr && (!std::isfinite(rms_eps) || !(rms_eps > 0.0f))) return BITNET_ERR_INVALID_ARG;
  const int64_t kmax = x_dtype == BITNET_BF16 ? 32768 : 16384;
  if (!valid_k(K) || K > kmax || N < 1 || N > INT32_MAX || M < 1 || M > 64) return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < fq_layout(M, K).total) return BITNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (!force_sk) {
    // the quantisation into the workspace, then bitnet_linear_gemm's product with the rest of the
    // workspace (stream-K or tiles): two launches, chained by programmatic dependent launch
    const FqLayout L = fq_layout(M, K);
    int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
    float* a = reinterpret_cast<float*>(ws + L.a);
    int32_t* rs = reinterpret_cast<int32_t*>(ws + L.rs);
    const bitnet_status st = bitnet_quant_act(x, x_dtype, M, K, rms_gain, rms_eps, xq, a, rs, stream);
    if (st != BITNET_OK) return st;
    return bitnet_linear_gemm(W_packed, gamma, N, K, xq, a, rs, M, y, y_dtype, ws, L.bar, stream);
  }
  const cudaError_t e =
      x_dtype == BITNET_BF16
          ? launch_fq<__nv_bfloat16>(x, rms_gain, rms_eps, W_packed, gamma, n, k, m, y, y_dtype, ws, s)
          : launch_fq<float>(x, rms_gain, rms_eps, W_packed, gamma, n, k, m, y, y_dtype, ws, s);
  return from_cuda(e);
}

}  // namespace

extern "C" {

bitnet_status bitnet_bitlinear_gemm(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                    const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                    void* y, int y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bitlinear_gemm(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype, workspace,
                        workspace_bytes, stream, false);
}

bitnet_status bitnet_bitlinear_gemm_stream_k(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                             const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                             int64_t M, void* y, int y_dtype, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  return bitlinear_gemm(x, x_dtype, rms_gain, rms_eps, W_packed, gamma, N, K, M, y, y_dtype, workspace,
                        workspace_bytes, stream, true);
}

}  // extern "C"
