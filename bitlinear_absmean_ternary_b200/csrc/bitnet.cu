// Host side of the BitLinear C ABI declared in include/bitnet.h: the weight
// packs (absmean ternarisation, pack.cuh), the pack without allocation, and
// the status calls.  The other entry points live beside their kernels:
// k_quant.cu, k_gemv.cu, k_gemm.cu, k_ffn.cu, k_b3.cu and k_ste.cu.
#include "host_common.h"
#include "pack.cuh"

#include <algorithm>

namespace {

using namespace bitnet;
using namespace bitnet_host;

// ------------------------------------------------ pack without allocation
//
// bitnet_pack_weights_noalloc keeps its scratch (one fp64 row sum per weight
// row, the divisor and the non-finite flag) in this fixed array instead of a
// caller buffer.  Every GPU that loads the library holds the array until the
// process exits.  All calls share it and it keeps the last call's contents,
// so the flag is cleared at the start of every call; calls that overlap on
// the GPU (for example from two host threads on two streams) race on it.
constexpr int64_t kNoAllocMaxRows = BITNET_PACK_NOALLOC_MAX_ROWS;
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(kNoAllocMaxRows) * sizeof(double) + 256;
static __device__ __align__(256) unsigned char g_pack_scratch[kNoAllocScratchBytes];

// Device address of g_pack_scratch on the current device, looked up once per
// device (the host-side name of the array is only a stand-in, not a device
// address).  Returns nullptr if the lookup fails.
void* pack_scratch_address() {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[d] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pack_scratch) != cudaSuccess) return nullptr;
    addr[d] = p;
  }
  return addr[d];
}

}  // namespace

extern "C" {

size_t bitnet_pack_workspace_bytes(int64_t N, int64_t K) {
  (void)K;
  if (N < 1) return 0;
  const size_t bytes = static_cast<size_t>(N) * sizeof(double) + 16;
  return (bytes + 255) & ~size_t(255);
}

bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, float eps, uint8_t* W_packed, float* gamma,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (W == nullptr || W_packed == nullptr || gamma == nullptr || workspace == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_packed, 16) || !aligned(gamma, 4) || !aligned(workspace, 16))
    return BITNET_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || !(eps > 0.0f)) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 1 || N > (int64_t{1} << 31) || N * K > (int64_t{1} << 40)) return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < bitnet_pack_workspace_bytes(N, K)) return BITNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* rowsum = static_cast<double*>(workspace);
  float* d = reinterpret_cast<float*>(rowsum + N);
  unsigned int* flag = reinterpret_cast<unsigned int*>(d + 1);

  if (cudaMemsetAsync(flag, 0, sizeof(unsigned int), s) != cudaSuccess) return BITNET_ERR_CUDA;
  const int64_t warps_wanted = N;
  const int blocks1 = static_cast<int>(std::min<int64_t>((warps_wanted + 7) / 8, int64_t{sm_count()} * 8));
  pack_rowsum_kernel<<<blocks1, 256, 0, s>>>(W, N, K, rowsum, flag);
  pack_gamma_kernel<<<1, 32, 0, s>>>(rowsum, N, K, eps, gamma, d);
  const int64_t nwords = N * K / 16;
  const int blocks3 = static_cast<int>(std::min<int64_t>((nwords + 255) / 256, int64_t{sm_count()} * 16));
  pack_codes_kernel<<<blocks3, 256, 0, s>>>(W, nwords, d, reinterpret_cast<uint32_t*>(W_packed));
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned int host_flag = 0;
  if (cudaMemcpyAsync(&host_flag, flag, sizeof(host_flag), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  return host_flag != 0 ? BITNET_ERR_NONFINITE : BITNET_OK;
}

size_t bitnet_b3_row_bytes(int64_t K) {
  if (!valid_k(K)) return 0;
  return static_cast<size_t>((K + 79) / 80 * 80 / 5);
}

bitnet_status bitnet_pack_weights_b3(const float* W, int64_t N, int64_t K, float eps, uint8_t* W_b3, float* gamma,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (W == nullptr || W_b3 == nullptr || gamma == nullptr || workspace == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_b3, 16) || !aligned(gamma, 4) || !aligned(workspace, 16))
    return BITNET_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || !(eps > 0.0f)) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || K > kGemvB3XMaxBytes || N < 1 || N > (int64_t{1} << 31) || N * K > (int64_t{1} << 40))
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < bitnet_pack_workspace_bytes(N, K)) return BITNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* rowsum = static_cast<double*>(workspace);
  float* d = reinterpret_cast<float*>(rowsum + N);
  unsigned int* flag = reinterpret_cast<unsigned int*>(d + 1);

  if (cudaMemsetAsync(flag, 0, sizeof(unsigned int), s) != cudaSuccess) return BITNET_ERR_CUDA;
  const int blocks1 = static_cast<int>(std::min<int64_t>((N + 7) / 8, int64_t{sm_count()} * 8));
  pack_rowsum_kernel<<<blocks1, 256, 0, s>>>(W, N, K, rowsum, flag);
  pack_gamma_kernel<<<1, 32, 0, s>>>(rowsum, N, K, eps, gamma, d);
  const int rb = static_cast<int>(bitnet_b3_row_bytes(K));
  const int blocks3 = static_cast<int>(std::min<int64_t>((N * rb + 255) / 256, int64_t{sm_count()} * 16));
  pack_codes_b3_kernel<<<blocks3, 256, 0, s>>>(W, N, static_cast<int>(K), rb, d, W_b3);
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned int host_flag = 0;
  if (cudaMemcpyAsync(&host_flag, flag, sizeof(host_flag), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  return host_flag != 0 ? BITNET_ERR_NONFINITE : BITNET_OK;
}

bitnet_status bitnet_pack_weights_noalloc(const float* W, int64_t N, int64_t K, float eps, uint8_t* W_packed,
                                          float* gamma, void* stream) {
  if (W == nullptr || W_packed == nullptr || gamma == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_packed, 16) || !aligned(gamma, 4)) return BITNET_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || !(eps > 0.0f)) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 1 || N > kNoAllocMaxRows || N * K > (int64_t{1} << 40)) return BITNET_ERR_UNSUPPORTED_SHAPE;
  void* scratch = pack_scratch_address();
  if (scratch == nullptr) return BITNET_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* rowsum = static_cast<double*>(scratch);
  float* d = reinterpret_cast<float*>(rowsum + kNoAllocMaxRows);
  unsigned int* flag = reinterpret_cast<unsigned int*>(d + 1);

  if (cudaMemsetAsync(flag, 0, sizeof(unsigned int), s) != cudaSuccess) return BITNET_ERR_CUDA;
  const int blocks1 = static_cast<int>(std::min<int64_t>((N + 7) / 8, int64_t{sm_count()} * 8));
  pack_rowsum_kernel<<<blocks1, 256, 0, s>>>(W, N, K, rowsum, flag);
  pack_gamma_kernel<<<1, 32, 0, s>>>(rowsum, N, K, eps, gamma, d);
  const int64_t nwords = N * K / 16;
  const int blocks3 = static_cast<int>(std::min<int64_t>((nwords + 255) / 256, int64_t{sm_count()} * 16));
  pack_codes_kernel<<<blocks3, 256, 0, s>>>(W, nwords, d, reinterpret_cast<uint32_t*>(W_packed));
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned int host_flag = 0;
  if (cudaMemcpyAsync(&host_flag, flag, sizeof(host_flag), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  return host_flag != 0 ? BITNET_ERR_NONFINITE : BITNET_OK;
}

bitnet_status bitnet_get_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  cudaError_t (*const takers[])(unsigned int*) = {take_error_gemv, take_error_gemm, take_error_gemm_fused,
                                                  take_error_ffn,  take_error_b3,   take_error_ste,
                                                  take_error_quant};
  bool timed_out = false;
  for (auto take : takers) {
    unsigned int v = 0;
    if (take(&v) != cudaSuccess) return BITNET_ERR_CUDA;
    timed_out |= v != 0;
  }
  return timed_out ? BITNET_ERR_TIMEOUT : BITNET_OK;
}

const char* bitnet_status_string(bitnet_status s) {
  switch (s) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad dtype or eps)";
    case BITNET_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (K must be a positive multiple of 64; M, N >= 1)";
    case BITNET_ERR_NONFINITE: return "weight matrix holds a non-finite value";
    case BITNET_ERR_CUDA: return "CUDA error";
    case BITNET_ERR_TIMEOUT: return "a kernel timed out waiting on a barrier";
  }
  return "unknown status";
}

}  // extern "C"
