// Host side of bitnet_bitlinear_ffn_gemv: the one-launch decode feed-forward
// block (ffn.cuh).
#include "host_common.h"
#include "ffn.cuh"

namespace {

using namespace bitnet;
using namespace bitnet_host;

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

}  // namespace

BITNET_DEFINE_TAKE_ERROR(ffn)

extern "C" {

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
  if (m == 1) {
    // one token with large weight shares: the gated one-token GEMV (x -> h), then the fused
    // one-token GEMV on h (h -> y) -- two launches whose weights stream in whole-row slots, which on
    // the 27B FFN beat the one-launch kernel below (its per-warp rings issue many small copies)
    bool used = false;
    const cudaError_t e = launch_ffn_upgate_gemv1(static_cast<const __nv_bfloat16*>(x),
                                                  static_cast<const __nv_bfloat16*>(rms_gain_in), rms_eps_in, W_up,
                                                  gamma_up, W_gate, gamma_gate, f, d, static_cast<__nv_bfloat16*>(h),
                                                  static_cast<cudaStream_t>(stream), &used);
    if (e != cudaSuccess) return from_cuda(e);
    if (used)
      return bitnet_bitlinear_gemv(h, BITNET_BF16, rms_gain_sub, rms_eps_sub, W_down, gamma_down, D, F, 1, y, y_dtype,
                                   stream);
  }
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

}  // extern "C"
