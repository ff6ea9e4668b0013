// Host-side helpers shared by the translation units of the library: argument
// checks, per-device caches, launch helpers and TMA tensor-map encoding.
// Each kernel family lives in its own .cu file (built in parallel); every
// file that launches kernels with bounded waits owns a device error word and
// exports a function that reads and clears it, which
// bitnet_get_device_status calls for all of them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "bitnet.h"

namespace bitnet_host {

constexpr int kMaxDevices = 64;

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline bool valid_k(int64_t K) { return K >= 64 && K % 64 == 0 && K <= (int64_t{1} << 30); }

inline int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

inline int sm_count() {
  static std::atomic<int> cache[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  int n = cache[d].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    cache[d].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Opt a kernel into more than 48 KB of dynamic shared memory and ask for the
// largest shared-memory carveout (once per device; the flags are atomic, so
// host threads making their first calls at once at worst repeat these
// idempotent attribute calls).  With every kernel of the library on the same
// carveout, a kernel launched with programmatic dependent launch can place
// its CTAs next to the previous kernel's CTAs without the SM first draining
// to change its L1/shared split.
template <typename F>
cudaError_t set_smem(F* fn, int bytes, std::atomic<bool> (&done)[kMaxDevices]) {
  const int d = current_device();
  if (d >= 0 && d < kMaxDevices && done[d]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && d >= 0 && d < kMaxDevices) done[d] = true;
  return e;
}

// Launch with programmatic stream serialisation, so the kernel may start its
// independent prologue while the previous kernel on the stream finishes; the
// kernels call griddepcontrol.wait before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bitnet_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

// ------------------------------------------------------------ tensor maps

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor [rows][cols] of `dtype` with row pitch `pitch` bytes, box {box_cols, box_rows}.
inline bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t cols, uint64_t rows,
                        uint64_t pitch, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
                        uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, cols, rows, pitch, box_cols, box_rows, swz);
}

inline bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
                          uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, pitch, box_cols, box_rows, swz);
}

// Argument checks shared by the product entry points (gemv and gemm).
inline bitnet_status check_linear(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                                  const float* a, const int32_t* rs, int64_t M, void* y, int yd) {
  if (Wp == nullptr || gamma == nullptr || xq == nullptr || a == nullptr || y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(Wp, 16) || !aligned(xq, 16) || !aligned(y, 16) || !aligned(gamma, 4) || !aligned(a, 4) ||
      !aligned(rs, 4))
    return BITNET_ERR_INVALID_ARG;
  if (yd != BITNET_F32 && yd != BITNET_BF16 && yd != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 1 || M < 1 || N > INT32_MAX || M > INT32_MAX) return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

// Largest M * Kp (token rows x padded K) the base-3 decode kernel keeps in
// shared memory; the base-3 pack refuses K beyond it.
constexpr int kGemvB3XMaxBytes = 24000;

// The decode FFN's up and gate products for one token with the squared-ReLU
// gate in the epilogue (k_gemv.cu): *used = false, nothing launched, where
// that kernel's plan does not apply.
cudaError_t launch_ffn_upgate_gemv1(const __nv_bfloat16* x, const __nv_bfloat16* gain, float eps, const uint8_t* Wu,
                                    const float* gu, const uint8_t* Wg, const float* gg, int F, int D,
                                    __nv_bfloat16* h, cudaStream_t s, bool* used);

// Device error words, one per translation unit that launches kernels with
// bounded waits: each reads its word into *v and clears it when set.
cudaError_t take_error_gemv(unsigned int* v);
cudaError_t take_error_gemm(unsigned int* v);
cudaError_t take_error_gemm_fused(unsigned int* v);
cudaError_t take_error_ffn(unsigned int* v);
cudaError_t take_error_b3(unsigned int* v);
cudaError_t take_error_ste(unsigned int* v);
cudaError_t take_error_quant(unsigned int* v);

}  // namespace bitnet_host

// Defines the error-word reader of the including translation unit.
#define BITNET_DEFINE_TAKE_ERROR(NAME)                                                     \
  cudaError_t bitnet_host::take_error_##NAME(unsigned int* v) {                            \
    *v = 0;                                                                                \
    cudaError_t e = cudaMemcpyFromSymbol(v, bitnet::g_device_error, sizeof(*v));           \
    if (e == cudaSuccess && *v != 0) {                                                     \
      const unsigned int zero = 0;                                                         \
      e = cudaMemcpyToSymbol(bitnet::g_device_error, &zero, sizeof(zero));                 \
    }                                                                                      \
    return e;                                                                              \
  }
