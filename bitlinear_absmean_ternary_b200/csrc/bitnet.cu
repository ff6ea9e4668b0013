// Host side of the BitLinear C ABI declared in include/bitnet.h: argument
// checks, launch configuration and stream-ordered launches.  One translation
// unit holds every kernel so that the device error word has a single home.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "bitnet.h"
#include "ffn.cuh"
#include "gemm.cuh"
#include "gemv.cuh"
#include "gemv_b3.cuh"
#include "pack.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "quant_rows.cuh"
#include "ste_gemm.cuh"

namespace {

using namespace bitnet;

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_k(int64_t K) { return K >= 64 && K % 64 == 0 && K <= (int64_t{1} << 30); }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int sm_count() {
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
// idempotent attribute calls).  With every kernel of the
// library on the same carveout, a kernel launched with programmatic
// dependent launch can place its CTAs next to the previous kernel's CTAs
// without the SM first draining to change its L1/shared split.
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

bitnet_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

// ------------------------------------------------------------ tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D byte tensor [rows][cols] with row pitch `pitch` bytes, box {box_cols, box_rows}.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch, uint32_t box_cols,
                 uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows][cols] with row pitch `pitch` bytes, box {box_cols, box_rows}.
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
                   uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ launchers

template <typename T, int MAXC, int NTHR = kQuantThreads>
cudaError_t launch_quant_t(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                           int32_t* rs, cudaStream_t s, int threads = kQuantThreads) {
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(quant_act_kernel<T, MAXC, NTHR>, 0, done);
  if (e != cudaSuccess) return e;
  return launch_pdl(quant_act_kernel<T, MAXC, NTHR>, dim3(static_cast<unsigned>(M)), dim3(threads), 0, s,
                    static_cast<const T*>(x), K, static_cast<const T*>(gain), eps, xq, a, rs);
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

// Token count from which the warp-per-row kernel takes over (bf16 input,
// K <= 6144): from there on it keeps more rows in flight per SM; below, a CTA
// per row spreads a short batch over more SMs.
constexpr int64_t kQuantRowsMinM = 512;

template <typename T>
cudaError_t launch_quant(const void* x, int64_t M, int K, const void* gain, float eps, int8_t* xq, float* a,
                         int32_t* rs, cudaStream_t s) {
  if constexpr (sizeof(T) == 2) {
    if (M >= kQuantRowsMinM && K <= 32 * 8 * kQuantRowsMaxChunks)
      return gain != nullptr ? launch_quant_rows<true>(x, M, K, gain, eps, xq, a, rs, s)
                             : launch_quant_rows<false>(x, M, K, gain, eps, xq, a, rs, s);
  }
  const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;
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
  if (per_thread <= 1) return launch_quant_t<T, 1>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 2) return launch_quant_t<T, 2>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 4) return launch_quant_t<T, 4>(x, M, K, gain, eps, xq, a, rs, s);
  if (per_thread <= 8) return launch_quant_t<T, 8>(x, M, K, gain, eps, xq, a, rs, s);
  if constexpr (sizeof(T) == 2) return launch_quant_t<T, 16>(x, M, K, gain, eps, xq, a, rs, s);
  return cudaErrorInvalidValue;
}

template <int MT, bool U8, bool XS>
cudaError_t launch_gemv_x(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                          const int32_t* rs, void* y, int yd, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(gemv_kernel<MT, U8, XS>, gemv_smem_bytes(MT, kGemvXMaxBytes / MT, XS), done);
  if (e != cudaSuccess) return e;
  const int64_t groups = (N + kGemvRows - 1) / kGemvRows;
  const int grid = static_cast<int>(groups < sm_count() ? groups : sm_count());
  return launch_pdl(gemv_kernel<MT, U8, XS>, dim3(grid), dim3(kGemvThreads), gemv_smem_bytes(MT, K, XS), s, Wp, gamma,
                    N, K, xq, a, rs, static_cast<const float*>(nullptr), static_cast<const float*>(nullptr), 0.0f, y,
                    yd);
}

template <int MT, bool U8>
cudaError_t launch_gemv_t(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                          const int32_t* rs, void* y, int yd, cudaStream_t s) {
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

// Launch configuration of a GEMM split over clusters of KS CTAs (KS = 1: plain persistent grid).
template <int BN, int S, bool U8, int KS>
cudaLaunchConfig_t gemm_config(int clusters, cudaStream_t s, cudaLaunchAttribute (&attr)[2]) {
  using C = GemmCfg<BN, S, KS>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * KS);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = KS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KS > 1 ? 2 : 1;
  return cfg;
}

// How many clusters of KS CTAs can be resident at once (clusters live inside
// one GPC, so this is not simply SMs / KS).  Cached per device.
template <int BN, int S, bool U8, int KS>
int gemm_cluster_capacity() {
  static std::atomic<int> cache[kMaxDevices] = {};
  const int d = current_device();
  if (d >= 0 && d < kMaxDevices && cache[d] > 0) return cache[d];
  static std::atomic<bool> done[kMaxDevices] = {};
  int n = 0;
  if (set_smem(gemm_kernel<BN, S, U8, KS>, GemmCfg<BN, S, KS>::kSmemBytes, done) == cudaSuccess) {
    if (KS == 1) {
      n = sm_count();
    } else {
      cudaLaunchAttribute attr[2];
      cudaLaunchConfig_t cfg = gemm_config<BN, S, U8, KS>(1, nullptr, attr);
      if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<BN, S, U8, KS>, &cfg) != cudaSuccess) n = 0;
    }
  }
  cudaGetLastError();
  if (n <= 0) n = sm_count() / KS;
  if (d >= 0 && d < kMaxDevices) cache[d] = n;
  return n;
}

template <int BN, int S, bool U8, int KS>
cudaError_t launch_gemm_ks(const CUtensorMap& mx, const CUtensorMap& mw, const float* gamma, const float* a,
                           const int32_t* rs, int M, int N, int K, void* y, int yd, cudaStream_t s) {
  using C = GemmCfg<BN, S, KS>;
  static std::atomic<bool> done[kMaxDevices] = {};
  const cudaError_t e = set_smem(gemm_kernel<BN, S, U8, KS>, C::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>((N + kGemmBM - 1) / kGemmBM) * ((M + BN - 1) / BN);
  const int cap = gemm_cluster_capacity<BN, S, U8, KS>();
  const int clusters = static_cast<int>(tiles < cap ? tiles : cap);
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = gemm_config<BN, S, U8, KS>(clusters, s, attr);
  return cudaLaunchKernelEx(&cfg, gemm_kernel<BN, S, U8, KS>, mx, mw, gamma, a, rs, M, N, K, y, yd);
}

// Split factor for a GEMM of `tiles` output tiles and nk K-steps: the one
// that keeps the most SMs busy over the whole launch (tiles spread over
// resident clusters in waves), with a small penalty per extra split for the
// partial-sum exchange.  Only used with unsigned codes (row sums given).
// Split factor for a GEMM of `tiles` output tiles and nk K-steps.  With two
// or more waves of tiles per SM the plain persistent grid is used; with fewer
// (decode-sized M) the factor in {1, 2, 4, 8} that keeps the most SMs busy
// over the launch (tiles spread over the resident clusters in waves), with a
// small penalty per extra split for the partial-sum exchange.  Only used with
// unsigned codes (row sums given).
template <int BN, int S>
int choose_ksplit(int64_t tiles, int nk) {
  const int sms = sm_count();
  const int cap1 = gemm_cluster_capacity<BN, S, true, 1>();
  if (tiles >= 2 * static_cast<int64_t>(cap1)) return 1;
  const int ks[4] = {1, 2, 4, 8};
  const int caps[4] = {cap1, gemm_cluster_capacity<BN, S, true, 2>(), gemm_cluster_capacity<BN, S, true, 4>(),
                       gemm_cluster_capacity<BN, S, true, 8>()};
  int best = 1;
  double best_score = -1.0;
  for (int i = 0; i < 4; ++i) {
    const int k = ks[i];
    if (k > nk) break;
    const int64_t cl = tiles < caps[i] ? tiles : caps[i];
    if (cl <= 0) continue;
    const int64_t waves = (tiles + cl - 1) / cl;
    const double busy = static_cast<double>(tiles) * k / (static_cast<double>(waves) * sms);
    const double score = busy - 0.03 * (k - 1);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = k;
    }
  }
  return best;
}

template <int BN, int S, bool U8>
cudaError_t launch_gemm_t(const CUtensorMap& mx, const CUtensorMap& mw, const float* gamma, const float* a,
                          const int32_t* rs, int M, int N, int K, void* y, int yd, cudaStream_t s) {
  if constexpr (U8) {
    const int64_t tiles = static_cast<int64_t>((N + kGemmBM - 1) / kGemmBM) * ((M + BN - 1) / BN);
    const int nk = (K + kGemmBK - 1) / kGemmBK;
    switch (choose_ksplit<BN, S>(tiles, nk)) {
      case 2: return launch_gemm_ks<BN, S, U8, 2>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
      case 4: return launch_gemm_ks<BN, S, U8, 4>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
      case 8: return launch_gemm_ks<BN, S, U8, 8>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
      default: break;
    }
  }
  return launch_gemm_ks<BN, S, U8, 1>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
}

template <int BN, int S>
cudaError_t launch_gemm_bn(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                           const int32_t* rs, int M, void* y, int yd, cudaStream_t s) {
  CUtensorMap mx, mw;
  // activations: 128-byte-wide boxes (two per stage); packed codes: one
  // 64-byte-wide box of 128 rows per stage
  if (!make_map_u8(&mx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map_u8(&mw, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4),
                   kGemmBK / 4, kGemmBM, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  if (rs != nullptr) return launch_gemm_t<BN, S, true>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
  return launch_gemm_t<BN, S, false>(mx, mw, gamma, a, rs, M, N, K, y, yd, s);
}

// Fused decode BitLinear: quantisation (and RMSNorm) of M <= 8 token rows in
// every CTA's prologue, then the GEMV.
template <int MT, typename T, int MAXC>
cudaError_t launch_fused_t(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                           int K, void* y, int yd, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemv_kernel<MT, true, true, true, T, MAXC>;
  const cudaError_t e = set_smem(kern, gemv_smem_bytes(MT, kGemvXMaxBytes / MT, true), done);
  if (e != cudaSuccess) return e;
  const int64_t groups = (N + kGemvRows - 1) / kGemvRows;
  const int grid = static_cast<int>(groups < sm_count() ? groups : sm_count());
  return launch_pdl(kern, dim3(grid), dim3(kGemvThreads), gemv_smem_bytes(MT, K, true), s, Wp, gamma, N, K,
                    static_cast<const int8_t*>(nullptr), static_cast<const float*>(nullptr),
                    static_cast<const int32_t*>(nullptr), static_cast<const T*>(x), static_cast<const T*>(gain), eps, y,
                    yd);
}

template <int MT, typename T>
cudaError_t launch_fused_c(const void* x, const void* gain, float eps, const uint8_t* Wp, const float* gamma, int N,
                           int K, void* y, int yd, cudaStream_t s) {
  const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;
  if (per_thread <= 1) return launch_fused_t<MT, T, 1>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 2) return launch_fused_t<MT, T, 2>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 4) return launch_fused_t<MT, T, 4>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if (per_thread <= 8) return launch_fused_t<MT, T, 8>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
  if constexpr (sizeof(T) == 2) return launch_fused_t<MT, T, 16>(x, gain, eps, Wp, gamma, N, K, y, yd, s);
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

// Decode FFN: one cooperative launch of one CTA per SM.  Cooperative, so
// that the driver guarantees every CTA is resident for the grid barrier;
// with programmatic stream serialisation, so that the weight prefetch may
// start while the previous kernel on the stream finishes.
template <int MT, int MAXC>
cudaError_t launch_ffn_t(const FfnArgs& a, int grid, size_t smem, cudaStream_t s) {
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = ffn_kernel<MT, MAXC>;
  const cudaError_t e = set_smem(kern, kFfnSmemMax, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFfnThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int MAXC>
cudaError_t launch_ffn_c(int M, const FfnArgs& a, int grid, size_t smem, cudaStream_t s) {
  switch (M) {
    case 1: return launch_ffn_t<1, MAXC>(a, grid, smem, s);
    case 2: return launch_ffn_t<2, MAXC>(a, grid, smem, s);
    case 3: return launch_ffn_t<3, MAXC>(a, grid, smem, s);
    case 4: return launch_ffn_t<4, MAXC>(a, grid, smem, s);
    case 5: return launch_ffn_t<5, MAXC>(a, grid, smem, s);
    case 6: return launch_ffn_t<6, MAXC>(a, grid, smem, s);
    case 7: return launch_ffn_t<7, MAXC>(a, grid, smem, s);
    case 8: return launch_ffn_t<8, MAXC>(a, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// Ring depth per warp for the FFN kernel: enough slots for every item of the
// busiest warp when that fits in shared memory (all weights in flight from
// the start), else as many as fit; 0 when not even two fit.
int ffn_slots(int M, int D, int F, int G) {
  // the busiest CTA has at most ceil(F/G) features and ceil(D/G) rows of W_down
  const int kc1 = gemv_kchunk(D), kc2 = gemv_kchunk(F);
  const int nkc1 = (D + kc1 - 1) / kc1, nkc2 = (F + kc2 - 1) / kc2;
  const int f = (F + G - 1) / G, d = (D + G - 1) / G;
  const int items = (f + 1) / 2 * nkc1 + (d + 3) / 4 * nkc2;
  const int want = (items + kFfnWarps - 1) / kFfnWarps;
  int sl = want < 2 ? 2 : want;
  while (sl >= 2 && ffn_smem_bytes(M, D, F, G, sl) > kFfnSmemMax) --sl;
  return sl >= 2 ? sl : 0;
}

// Fused decode BitLinear on base-3 packed weights.
constexpr int kGemvB3XMaxBytes = 24000;  // M * Kp: the quantised, zero-padded token rows in shared memory

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

bitnet_status check_linear(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                           const float* a, const int32_t* rs, int64_t M, void* y, int yd) {
  if (Wp == nullptr || gamma == nullptr || xq == nullptr || a == nullptr || y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(Wp, 16) || !aligned(xq, 16) || !aligned(y, 16) || !aligned(gamma, 4) || !aligned(a, 4) ||
      !aligned(rs, 4))
    return BITNET_ERR_INVALID_ARG;
  if (yd != BITNET_F32 && yd != BITNET_BF16 && yd != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || N < 1 || M < 1 || N > INT32_MAX || M > INT32_MAX) return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

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

bitnet_status bitnet_linear_gemm(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, const int8_t* x_q,
                                 const float* a_scale, const int32_t* x_rowsum, int64_t M, void* y, int y_dtype,
                                 void* stream) {
  const bitnet_status st = check_linear(W_packed, gamma, N, K, x_q, a_scale, x_rowsum, M, y, y_dtype);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  cudaError_t e;
  if (m <= 16) e = launch_gemm_bn<16, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  else if (m <= 32) e = launch_gemm_bn<32, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  else if (m <= 64) e = launch_gemm_bn<64, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  else e = launch_gemm_bn<128, 4>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  return from_cuda(e);
}

bitnet_status bitnet_bitlinear_gemv(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                    const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                    void* y, int y_dtype, void* stream) {
  if (x == nullptr || W_packed == nullptr || gamma == nullptr || y == nullptr) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rms_gain, 16) || !aligned(W_packed, 16) || !aligned(y, 16) || !aligned(gamma, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (rms_gain != nullptr && (!std::isfinite(rms_eps) || !(rms_eps > 0.0f))) return BITNET_ERR_INVALID_ARG;
  const int64_t kmax = x_dtype == BITNET_BF16 ? 32768 : 16384;
  if (!valid_k(K) || K > kmax || N < 1 || N > INT32_MAX || M < 1 || M > 8 || M * K > kGemvXMaxBytes)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  const cudaError_t e =
      x_dtype == BITNET_BF16
          ? launch_fused<__nv_bfloat16>(m, x, rms_gain, rms_eps, W_packed, gamma, n, k, y, y_dtype, s)
          : launch_fused<float>(m, x, rms_gain, rms_eps, W_packed, gamma, n, k, y, y_dtype, s);
  return from_cuda(e);
}

bitnet_status bitnet_bitlinear_ffn_gemv(const void* x, int x_dtype, int64_t M, int64_t D, int64_t F,
                                        const void* rms_gain_in, float rms_eps_in, const uint8_t* W_up,
                                        const float* gamma_up, const uint8_t* W_gate, const float* gamma_gate,
                                        const void* rms_gain_sub, float rms_eps_sub, const uint8_t* W_down,
                                        const float* gamma_down, void* h, void* y, int y_dtype, void* sync,
                                        void* stream) {
  if (x == nullptr || W_up == nullptr || gamma_up == nullptr || W_gate == nullptr || gamma_gate == nullptr ||
      W_down == nullptr || gamma_down == nullptr || h == nullptr || y == nullptr || sync == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rms_gain_in, 16) || !aligned(rms_gain_sub, 16) || !aligned(W_up, 16) ||
      !aligned(W_gate, 16) || !aligned(W_down, 16) || !aligned(h, 16) || !aligned(y, 16) || !aligned(sync, 8) ||
      !aligned(gamma_up, 4) || !aligned(gamma_gate, 4) || !aligned(gamma_down, 4))
    return BITNET_ERR_INVALID_ARG;
  if (x_dtype != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16 && y_dtype != BITNET_I32) return BITNET_ERR_INVALID_ARG;
  if (rms_gain_in != nullptr && (!std::isfinite(rms_eps_in) || !(rms_eps_in > 0.0f))) return BITNET_ERR_INVALID_ARG;
  if (rms_gain_sub != nullptr && (!std::isfinite(rms_eps_sub) || !(rms_eps_sub > 0.0f)))
    return BITNET_ERR_INVALID_ARG;
  if (!valid_k(D) || !valid_k(F) || D > kFfnMaxK || F > kFfnMaxK || M < 1 || M > 8)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  const int m = static_cast<int>(M), d = static_cast<int>(D), f = static_cast<int>(F);
  const int G = sm_count();
  const int slots = ffn_slots(m, d, f, G);
  if (slots == 0) return BITNET_ERR_UNSUPPORTED_SHAPE;
  FfnArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.gain_in = static_cast<const __nv_bfloat16*>(rms_gain_in);
  a.w_up = W_up;
  a.w_gate = W_gate;
  a.gamma_up = gamma_up;
  a.gamma_gate = gamma_gate;
  a.gain_sub = static_cast<const __nv_bfloat16*>(rms_gain_sub);
  a.w_down = W_down;
  a.gamma_down = gamma_down;
  a.h = static_cast<__nv_bfloat16*>(h);
  a.y = y;
  a.sync = static_cast<uint64_t*>(sync);
  a.eps_in = rms_eps_in;
  a.eps_sub = rms_eps_sub;
  a.D = d;
  a.F = f;
  a.y_dtype = y_dtype;
  a.slots = slots;
  const size_t smem = static_cast<size_t>(ffn_smem_bytes(m, d, f, G, slots));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int per_thread = ((d > f ? d : f) / 8 + kQuantThreads - 1) / kQuantThreads;
  const cudaError_t e = per_thread <= 4 ? launch_ffn_c<4>(m, a, G, smem, s) : launch_ffn_c<12>(m, a, G, smem, s);
  return from_cuda(e);
}

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

bitnet_status bitnet_get_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bitnet::g_device_error, sizeof(v)) != cudaSuccess) return BITNET_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(bitnet::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return BITNET_ERR_CUDA;
    return BITNET_ERR_TIMEOUT;
  }
  return BITNET_OK;
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
