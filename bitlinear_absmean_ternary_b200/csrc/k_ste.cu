// Host side of the straight-through-estimator backward products
// (ste_gemm.cuh): operand expansion pre-passes and the bf16 tcgen05 GEMM.
#include "host_common.h"
#include "ste_gemm.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

// STE backward GEMMs (ste_gemm.cuh): persistent, one CTA per SM.
constexpr int kSteBN = 256;
constexpr int kSteStages = 4;

cudaError_t launch_ste(const CUtensorMap& ma, const CUtensorMap& mb, const float* scale, int R, int C, int J,
                       void* out, int od, cudaStream_t s) {
  using Cfg = SteCfg<kSteBN, kSteStages>;
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = ste_gemm_kernel<kSteBN, kSteStages>;
  const cudaError_t e = set_smem(kern, Cfg::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>((R + kSteBM - 1) / kSteBM) * ((C + kSteBN - 1) / kSteBN);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  return launch_pdl(kern, dim3(grid), dim3(kSteThreads), Cfg::kSmemBytes, s, ma, mb, scale, R, C, J, out, od);
}

int64_t ste_pad(int64_t n) { return (n + kStePad - 1) / kStePad * kStePad; }

}  // namespace

BITNET_DEFINE_TAKE_ERROR(ste)

extern "C" {

size_t bitnet_ste_input_workspace_bytes(int64_t N, int64_t K) {
  if (N < 1 || !valid_k(K)) return 0;
  return static_cast<size_t>(K) * static_cast<size_t>(ste_pad(N)) * 2;
}

bitnet_status bitnet_ste_backward_input(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                        const void* dY, int64_t M, void* dX, int dx_dtype, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (W_packed == nullptr || gamma == nullptr || dY == nullptr || dX == nullptr || workspace == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(W_packed, 16) || !aligned(dY, 16) || !aligned(dX, 16) || !aligned(workspace, 16) ||
      !aligned(gamma, 4))
    return BITNET_ERR_INVALID_ARG;
  if (dx_dtype != BITNET_F32 && dx_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 8 || N % 8 != 0 || N > INT32_MAX || M < 1 || M > INT32_MAX)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < bitnet_ste_input_workspace_bytes(N, K)) return BITNET_ERR_INVALID_ARG;
  const int64_t Np = ste_pad(N);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* wt = static_cast<__nv_bfloat16*>(workspace);
  const dim3 pgrid(static_cast<unsigned>(Np / 64), static_cast<unsigned>(K / 64));
  if (launch_pdl(ste_expand_wt_kernel, pgrid, dim3(256), 0, s, W_packed, static_cast<int>(N), static_cast<int>(K),
                 static_cast<int>(Np), wt) != cudaSuccess)
    return BITNET_ERR_CUDA;
  CUtensorMap ma, mb;
  if (!make_map_bf16(&ma, wt, static_cast<uint64_t>(Np), static_cast<uint64_t>(K), static_cast<uint64_t>(Np) * 2,
                     kSteBox, kSteBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_bf16(&mb, dY, static_cast<uint64_t>(N), static_cast<uint64_t>(M), static_cast<uint64_t>(N) * 2,
                     kSteBox, kSteBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  return from_cuda(launch_ste(ma, mb, gamma, static_cast<int>(K), static_cast<int>(M), static_cast<int>(Np), dX,
                              dx_dtype, s));
}

size_t bitnet_ste_weight_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || !valid_k(K)) return 0;
  return (static_cast<size_t>(N) + static_cast<size_t>(K)) * static_cast<size_t>(ste_pad(M)) * 2;
}

bitnet_status bitnet_ste_backward_weight(const void* dY, const int8_t* x_q, const float* a_scale, int64_t M,
                                         int64_t N, int64_t K, void* dW, int dw_dtype, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (dY == nullptr || x_q == nullptr || a_scale == nullptr || dW == nullptr || workspace == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(dY, 16) || !aligned(x_q, 16) || !aligned(dW, 16) || !aligned(workspace, 16) || !aligned(a_scale, 4))
    return BITNET_ERR_INVALID_ARG;
  if (dw_dtype != BITNET_F32 && dw_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 8 || N % 8 != 0 || N > INT32_MAX || M < 1 || M > INT32_MAX)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < bitnet_ste_weight_workspace_bytes(M, N, K)) return BITNET_ERR_INVALID_ARG;
  const int64_t Mp = ste_pad(M);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* dyst = static_cast<__nv_bfloat16*>(workspace);  // [N][Mp]
  __nv_bfloat16* xt = dyst + N * Mp;                              // [K][Mp]
  const dim3 g1(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>(Mp / 64));
  if (launch_pdl(ste_scale_transpose_kernel, g1, dim3(256), 0, s, static_cast<const __nv_bfloat16*>(dY), a_scale,
                 static_cast<int>(M), static_cast<int>(N), static_cast<int>(Mp), dyst) != cudaSuccess)
    return BITNET_ERR_CUDA;
  const dim3 g2(static_cast<unsigned>(Mp / 64), static_cast<unsigned>(K / 64));
  if (launch_pdl(ste_expand_xt_kernel, g2, dim3(256), 0, s, x_q, static_cast<int>(M), static_cast<int>(K),
                 static_cast<int>(Mp), xt) != cudaSuccess)
    return BITNET_ERR_CUDA;
  CUtensorMap ma, mb;
  if (!make_map_bf16(&ma, xt, static_cast<uint64_t>(Mp), static_cast<uint64_t>(K), static_cast<uint64_t>(Mp) * 2,
                     kSteBox, kSteBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_bf16(&mb, dyst, static_cast<uint64_t>(Mp), static_cast<uint64_t>(N), static_cast<uint64_t>(Mp) * 2,
                     kSteBox, kSteBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  return from_cuda(launch_ste(ma, mb, nullptr, static_cast<int>(K), static_cast<int>(N), static_cast<int>(Mp), dW,
                              dw_dtype, s));
}

}  // extern "C"
