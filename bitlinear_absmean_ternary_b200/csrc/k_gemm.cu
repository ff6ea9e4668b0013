// Host side of bitnet_linear_gemm: the tcgen05 tensor-core products --
// gemm_sk.cuh (stream-K, M <= 64 with a workspace) and gemm.cuh (persistent
// tiles, cluster split-K for few tiles): tensor maps, tile size by M, launch.
#include "host_common.h"
#include "gemm.cuh"
#include "gemm_sk.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

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

// Workspace of the stream-K kernel on the current device: a flag per CTA
// (one CTA per SM at most) and an accumulation slot per CTA, the same for
// every token count M <= 64.
size_t sk_workspace_bytes(int64_t) {
  const int G = sm_count();
  return sk_flag_bytes(G) + sk_slot_bytes(G);
}

template <int BN, bool U8, bool GATE>
cudaError_t launch_sk(const CUtensorMap& mx, const CUtensorMap& mw, const CUtensorMap& mw2, const float* gamma,
                      const float* gamma2, const float* a, const int32_t* rs, int M, int N, int K, void* y, int yd,
                      void* ws, cudaStream_t s) {
  using C = SkCfg<BN, GATE>;
  static std::atomic<bool> done[kMaxDevices] = {};
  auto kern = gemm_sk_kernel<BN, U8, GATE>;
  const cudaError_t e = set_smem(kern, C::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>((N + C::kRowsPerTile - 1) / C::kRowsPerTile) * ((M + BN - 1) / BN) *
                        ((K + kGemmBK - 1) / kGemmBK);
  const int sms = sm_count();
  const int G = static_cast<int>(units < sms ? units : sms);
  unsigned int* flags = static_cast<unsigned int*>(ws);
  int* parts = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + sk_flag_bytes(sms));
  return launch_pdl(kern, dim3(G), dim3(kSkThreads), C::kSmemBytes, s, mx, mw, mw2, gamma, gamma2, a, rs, M, N, K, y,
                    yd, flags, parts, SkQuant<float>{});
}

// Tensor maps of a stream-K product: activations in 128-byte-wide boxes of BN
// tokens (two per stage), packed codes in 64-byte-wide boxes of `rows` rows.
template <int BN>
bool sk_maps(const int8_t* xq, int M, int K, const uint8_t* Wp, int N, uint32_t rows, CUtensorMap* mx,
             CUtensorMap* mw) {
  return make_map_u8(mx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, BN,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map_u8(mw, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4),
                     kGemmBK / 4, rows, CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int BN>
cudaError_t launch_sk_bn(const uint8_t* Wp, const float* gamma, int N, int K, const int8_t* xq, const float* a,
                         const int32_t* rs, int M, void* y, int yd, void* ws, cudaStream_t s) {
  CUtensorMap mx, mw;
  if (!sk_maps<BN>(xq, M, K, Wp, N, kGemmBM, &mx, &mw)) return cudaErrorInvalidValue;
  if (rs != nullptr) return launch_sk<BN, true, false>(mx, mw, mw, gamma, gamma, a, rs, M, N, K, y, yd, ws, s);
  return launch_sk<BN, false, false>(mx, mw, mw, gamma, gamma, a, rs, M, N, K, y, yd, ws, s);
}

// Up and gate projections with the squared-ReLU gate in the epilogue: h (bf16, M x F).
template <int BN>
cudaError_t launch_upgate_bn(const uint8_t* Wu, const float* gu, const uint8_t* Wg, const float* gg, int F, int K,
                             const int8_t* xq, const float* a, const int32_t* rs, int M, void* h, void* ws,
                             cudaStream_t s) {
  CUtensorMap mx, mw, mw2, unused;
  if (!sk_maps<BN>(xq, M, K, Wu, F, 64, &mx, &mw) || !sk_maps<BN>(xq, M, K, Wg, F, 64, &unused, &mw2))
    return cudaErrorInvalidValue;
  if (rs != nullptr) return launch_sk<BN, true, true>(mx, mw, mw2, gu, gg, a, rs, M, F, K, h, 1, ws, s);
  return launch_sk<BN, false, true>(mx, mw, mw2, gu, gg, a, rs, M, F, K, h, 1, ws, s);
}

}  // namespace

BITNET_DEFINE_TAKE_ERROR(gemm)

extern "C" {

size_t bitnet_linear_upgate_workspace_bytes(int64_t M, int64_t F, int64_t K) {
  if (M < 1 || M > INT32_MAX || F < 1 || F > INT32_MAX || !valid_k(K)) return 0;
  return sk_workspace_bytes(M);
}

bitnet_status bitnet_linear_upgate_gemm(const uint8_t* W_up, const float* gamma_up, const uint8_t* W_gate,
                                        const float* gamma_gate, int64_t F, int64_t K, const int8_t* x_q,
                                        const float* a_scale, const int32_t* x_rowsum, int64_t M, void* h,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  if (W_up == nullptr || gamma_up == nullptr || W_gate == nullptr || gamma_gate == nullptr || x_q == nullptr ||
      a_scale == nullptr || h == nullptr || workspace == nullptr)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(W_up, 16) || !aligned(W_gate, 16) || !aligned(x_q, 16) || !aligned(h, 16) || !aligned(workspace, 16) ||
      !aligned(gamma_up, 4) || !aligned(gamma_gate, 4) || !aligned(a_scale, 4) || !aligned(x_rowsum, 4))
    return BITNET_ERR_INVALID_ARG;
  if (!valid_k(K) || F < 1 || F > INT32_MAX || M < 1 || M > INT32_MAX || K > INT32_MAX)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < sk_workspace_bytes(M)) return BITNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int f = static_cast<int>(F), k = static_cast<int>(K), m = static_cast<int>(M);
  cudaError_t e;
  if (m <= 16) e = launch_upgate_bn<16>(W_up, gamma_up, W_gate, gamma_gate, f, k, x_q, a_scale, x_rowsum, m, h, workspace, s);
  else if (m <= 32) e = launch_upgate_bn<32>(W_up, gamma_up, W_gate, gamma_gate, f, k, x_q, a_scale, x_rowsum, m, h, workspace, s);
  else e = launch_upgate_bn<64>(W_up, gamma_up, W_gate, gamma_gate, f, k, x_q, a_scale, x_rowsum, m, h, workspace, s);
  return from_cuda(e);
}

size_t bitnet_linear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 64 || N < 1 || N > INT32_MAX || !valid_k(K)) return 0;
  return sk_workspace_bytes(M);
}

}  // extern "C"

namespace {

// The product with the stream-K kernel forced (force_sk), or chosen by sk_preferred.
bitnet_status linear_gemm(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, const int8_t* x_q,
                          const float* a_scale, const int32_t* x_rowsum, int64_t M, void* y, int y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream, bool force_sk) {
  const bitnet_status st = check_linear(W_packed, gamma, N, K, x_q, a_scale, x_rowsum, M, y, y_dtype);
  if (st != BITNET_OK) return st;
  if (!aligned(workspace, 16)) return BITNET_ERR_INVALID_ARG;
  if (force_sk && (workspace == nullptr || M > 64)) return workspace == nullptr ? BITNET_ERR_INVALID_ARG
                                                                                 : BITNET_ERR_UNSUPPORTED_SHAPE;
  if (workspace != nullptr && M <= 64 && workspace_bytes < sk_workspace_bytes(M)) return BITNET_ERR_INVALID_ARG;
  const bool stream_k = force_sk || (workspace != nullptr && sk_preferred(M, N, K, sm_count()));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(N), k = static_cast<int>(K), m = static_cast<int>(M);
  cudaError_t e;
  if (stream_k) {
    if (m <= 16) e = launch_sk_bn<16>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, workspace, s);
    else if (m <= 32) e = launch_sk_bn<32>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, workspace, s);
    else e = launch_sk_bn<64>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, workspace, s);
  } else if (m <= 16) {
    e = launch_gemm_bn<16, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  } else if (m <= 32) {
    e = launch_gemm_bn<32, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  } else if (m <= 64) {
    e = launch_gemm_bn<64, 6>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  } else {
    e = launch_gemm_bn<128, 4>(W_packed, gamma, n, k, x_q, a_scale, x_rowsum, m, y, y_dtype, s);
  }
  return from_cuda(e);
}

}  // namespace

extern "C" {

bitnet_status bitnet_linear_gemm(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, const int8_t* x_q,
                                 const float* a_scale, const int32_t* x_rowsum, int64_t M, void* y, int y_dtype,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return linear_gemm(W_packed, gamma, N, K, x_q, a_scale, x_rowsum, M, y, y_dtype, workspace, workspace_bytes, stream,
                     false);
}

bitnet_status bitnet_linear_gemm_stream_k(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                          const int8_t* x_q, const float* a_scale, const int32_t* x_rowsum, int64_t M,
                                          void* y, int y_dtype, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  return linear_gemm(W_packed, gamma, N, K, x_q, a_scale, x_rowsum, M, y, y_dtype, workspace, workspace_bytes, stream,
                     true);
}

}  // extern "C"
