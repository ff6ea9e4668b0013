// CPU oracle for the BitNet b1.58 BitLinear forward (W1.58A8).
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
// definition that the CUDA library is checked against.  Only the tests, the
// smoke check and the CPU-baseline leg of the benchmark may load it; the
// library itself never calls it and shares no code, header or table with it.
//
// Sources (web pages on BitNet b1.58), cited by title and section:
//   [Review]     comrad404.com, "BitNet b1.58: что показала работа Microsoft
//                об «эре 1-битных LLM»", section "Метод: как устроен BitNet b1.58"
//                (ternary weights {-1,0,1} via absmean, 8-bit activations,
//                LLaMA-like stack with RMSNorm, and the four BitLinear steps:
//                normalise the input, quantise activations, replace weights by
//                ternary ones, low-bit product followed by rescaling).
//   [Explainer]  inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów",
//                sections "Skąd te 1,58 bita" (three states stored on two bits
//                plus some structure), "Trenowany od zera" (absmean: the whole
//                matrix is scaled by its mean absolute value, then each entry
//                goes to the nearest integer in {-1,0,+1}) and "Mnożenie? Jakie
//                mnożenie" (products by +1/-1/0 become add/subtract/skip).
//   [Habr]       juhe.plus repost of a Habr article on 1-bit networks, section
//                "Когда - три лучше двух" (y = W x with ternary W is the sum of
//                the inputs with weight +1 minus the sum of those with -1).
//
// The pages give no formulas for the absmax activation scale, the 127
// constant, eps, rounding or the storage layout.  The readings taken here:
//   * gamma = mean|W| over the whole matrix, summed in a fixed canonical
//     order in fp64 (per row: 32 strided partials, then a halving tree; rows
//     added in increasing order), gamma = RN32(S / (N*K)).
//   * q = clamp(RNE(RN32(w / RN32(gamma + eps))), -1, 1).
//   * Storage: code c = q + 1 in {0,1,2}; one little-endian 32-bit word holds
//     16 consecutive weights k0..k0+15, weight k0+4j+b in byte b, bits 2j..2j+1.
//   * Activations, per token: optional RMSNorm h = RN32(RN32(v*r)*g) with
//     r = RN32(1 / RN32(sqrt(RN32(RN32(ss/K) + eps)))), ss the sum of RN32(v*v)
//     in a fixed order (256 lanes over 8-element chunks, then a halving tree);
//     amax = max|h|; s = RN32(127/amax); x_q = clamp(RNE(RN32(h*s)), -127, 127);
//     per-token dequant scale a = RN32(amax/127); a token with amax == 0 gets
//     x_q = 0 and a = 0.
//   * acc = sum_k q*x_q, exact in integers; y = RN32(RN32(float(acc)*gamma)*a).
// Every fp32 operation is a single correctly rounded IEEE operation; build
// with -ffp-contract=off so that no multiply-add is fused.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// Sum of |w| over one row in the canonical order: 32 fp64 partials, partial l
// taking k = l, l+32, l+64, ... in increasing k, then p[l] += p[l+s] for
// s = 16, 8, 4, 2, 1.
double row_abs_sum(const float* row, int64_t K) {
  double p[32];
  for (int l = 0; l < 32; ++l) p[l] = 0.0;
  for (int64_t k = 0; k < K; ++k) p[k % 32] = p[k % 32] + std::fabs(static_cast<double>(row[k]));
  for (int s = 16; s >= 1; s /= 2)
    for (int l = 0; l < s; ++l) p[l] = p[l] + p[l + s];
  return p[0];
}

float round_half_even(float t) { return std::nearbyint(t); }  // default rounding mode is RNE

float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

}  // namespace

extern "C" {

// absmean scale [Explainer, "Trenowany od zera"]: mean absolute value of the
// whole weight matrix W (N rows of K), canonical fp64 order, rounded to fp32.
float oracle_absmean_gamma(const float* W, int64_t N, int64_t K) {
  double S = 0.0;
  for (int64_t n = 0; n < N; ++n) S = S + row_abs_sum(W + n * K, K);
  return static_cast<float>(S / static_cast<double>(N * K));
}

// Ternary codes q in {-1, 0, 1} [Review, "Метод"; Explainer, "Trenowany od
// zera"]: every entry divided by (gamma + eps) and rounded to the nearest of
// {-1, 0, +1}.  Returns 0, or 3 if W holds a non-finite value.
int oracle_ternarize(const float* W, int64_t N, int64_t K, float eps, int8_t* q, float* gamma_out) {
  for (int64_t i = 0; i < N * K; ++i)
    if (!std::isfinite(W[i])) return 3;
  const float gamma = oracle_absmean_gamma(W, N, K);
  const float d = gamma + eps;
  for (int64_t i = 0; i < N * K; ++i) {
    const float t = W[i] / d;
    q[i] = static_cast<int8_t>(clampf(round_half_even(t), -1.0f, 1.0f));
  }
  *gamma_out = gamma;
  return 0;
}

// Two-bit storage of ternary codes [Explainer, "Skąd te 1,58 bita": three
// states kept on two bits]; the word layout is this library's own.
void oracle_pack_codes(const int8_t* q, int64_t N, int64_t K, uint8_t* packed) {
  const int64_t row_bytes = K / 4;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t w = 0; w < K / 16; ++w)
      for (int b = 0; b < 4; ++b) {
        unsigned byte = 0;
        for (int j = 0; j < 4; ++j) {
          const int c = q[n * K + 16 * w + 4 * j + b] + 1;
          byte |= static_cast<unsigned>(c) << (2 * j);
        }
        packed[n * row_bytes + 4 * w + b] = static_cast<uint8_t>(byte);
      }
}

// Inverse of oracle_pack_codes.  Returns how many 2-bit fields held the
// illegal code 3 (those decode to 0).
int64_t oracle_unpack_codes(const uint8_t* packed, int64_t N, int64_t K, int8_t* q) {
  const int64_t row_bytes = K / 4;
  int64_t illegal = 0;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t w = 0; w < K / 16; ++w)
      for (int b = 0; b < 4; ++b) {
        const unsigned byte = packed[n * row_bytes + 4 * w + b];
        for (int j = 0; j < 4; ++j) {
          const int c = (byte >> (2 * j)) & 3;
          if (c == 3) ++illegal;
          q[n * K + 16 * w + 4 * j + b] = static_cast<int8_t>(c == 3 ? 0 : c - 1);
        }
      }
  return illegal;
}

// The offline weight step: absmean ternarisation followed by 2-bit packing.
int oracle_pack_weights(const float* W, int64_t N, int64_t K, float eps, uint8_t* packed, float* gamma_out) {
  std::vector<int8_t> q(static_cast<size_t>(N * K));
  const int st = oracle_ternarize(W, N, K, eps, q.data(), gamma_out);
  if (st != 0) return st;
  oracle_pack_codes(q.data(), N, K, packed);
  return 0;
}

// RMSNorm of one token [Review, "Метод": RMSNorm in the LLaMA-like stack, and
// normalising the input is the first BitLinear step].
void oracle_rmsnorm_row(const float* v, const float* g, int64_t K, float eps, float* h) {
  float lane[256];
  for (int l = 0; l < 256; ++l) lane[l] = 0.0f;
  for (int64_t c = 0; c < K / 8; ++c)
    for (int e = 0; e < 8; ++e) {
      const float x = v[8 * c + e];
      const float sq = x * x;
      lane[c % 256] = lane[c % 256] + sq;
    }
  for (int s = 128; s >= 1; s /= 2)
    for (int l = 0; l < s; ++l) lane[l] = lane[l] + lane[l + s];
  const float ms = lane[0] / static_cast<float>(K);
  const float rms = std::sqrt(ms + eps);
  const float r = 1.0f / rms;
  for (int64_t k = 0; k < K; ++k) {
    const float t = v[k] * r;
    h[k] = t * g[k];
  }
}

// Per-token absmax int8 activation quantisation [Review, "Метод": 8-bit
// activations; second BitLinear step], optionally preceded by RMSNorm.
// x: M x K values (bf16 inputs are passed widened to fp32, which is exact).
// gain: K values or NULL (no norm).  Outputs x_q (M x K), a (M) and, when
// rowsum is not NULL, the per-token sum of x_q.
void oracle_quant_act(const float* x, int64_t M, int64_t K, const float* gain, float rms_eps,
                      int8_t* xq, float* a, int32_t* rowsum) {
  std::vector<float> h(static_cast<size_t>(K));
  for (int64_t m = 0; m < M; ++m) {
    const float* v = x + m * K;
    if (gain != nullptr) {
      oracle_rmsnorm_row(v, gain, K, rms_eps, h.data());
    } else {
      for (int64_t k = 0; k < K; ++k) h[k] = v[k];
    }
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) amax = std::fmax(amax, std::fabs(h[k]));
    int64_t sum = 0;
    if (amax == 0.0f) {
      for (int64_t k = 0; k < K; ++k) xq[m * K + k] = 0;
      a[m] = 0.0f;
    } else {
      const float s = 127.0f / amax;
      for (int64_t k = 0; k < K; ++k) {
        const float t = h[k] * s;
        const float r = clampf(round_half_even(t), -127.0f, 127.0f);
        xq[m * K + k] = static_cast<int8_t>(r);
        sum += static_cast<int64_t>(r);
      }
      a[m] = amax / 127.0f;
    }
    if (rowsum != nullptr) rowsum[m] = static_cast<int32_t>(sum);
  }
}

// One output of the W1.58A8 product and its dequantisation.  The integer
// result is formed twice, as the plain dot product sum_k q*x_q and as the
// add/subtract form [Habr, "Когда - три лучше двух"; Explainer, "Mnożenie?
// Jakie mnożenie"]: sum of x_q where q = +1 minus sum where q = -1.  Returns
// 0, or 1 if the two forms disagree or the result leaves int32.
int oracle_dot(const int8_t* qrow, const int8_t* xrow, int64_t K, float gamma, float a,
               int32_t* acc_out, float* y_out) {
  int64_t dot = 0, plus = 0, minus = 0;
  for (int64_t k = 0; k < K; ++k) {
    dot += static_cast<int64_t>(qrow[k]) * static_cast<int64_t>(xrow[k]);
    if (qrow[k] == 1) plus += xrow[k];
    if (qrow[k] == -1) minus += xrow[k];
  }
  if (dot != plus - minus) return 1;
  if (dot > INT32_MAX || dot < INT32_MIN) return 1;
  const int32_t acc = static_cast<int32_t>(dot);
  // low-bit product followed by rescaling [Review, "Метод"]
  const float t = static_cast<float>(acc) * gamma;
  *acc_out = acc;
  *y_out = t * a;
  return 0;
}

// Full BitLinear product for M tokens against packed weights (N x K).
// acc and y are M x N, row-major (y[m*N + n]).
int oracle_bitlinear(const uint8_t* packed, float gamma, int64_t N, int64_t K,
                     const int8_t* xq, const float* a, int64_t M, int32_t* acc, float* y) {
  std::vector<int8_t> q(static_cast<size_t>(K));
  for (int64_t n = 0; n < N; ++n) {
    oracle_unpack_codes(packed + n * (K / 4), 1, K, q.data());
    for (int64_t m = 0; m < M; ++m)
      if (oracle_dot(q.data(), xq + m * K, K, gamma, a[m], &acc[m * N + n], &y[m * N + n]) != 0) return 1;
  }
  return 0;
}

// The same product at the listed (m, n) positions only.
int oracle_bitlinear_sampled(const uint8_t* packed, float gamma, int64_t N, int64_t K,
                             const int8_t* xq, const float* a, int64_t M,
                             const int64_t* ms, const int64_t* ns, int64_t count,
                             int32_t* acc, float* y) {
  std::vector<int8_t> q(static_cast<size_t>(K));
  for (int64_t i = 0; i < count; ++i) {
    if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return 2;
    oracle_unpack_codes(packed + ns[i] * (K / 4), 1, K, q.data());
    if (oracle_dot(q.data(), xq + ms[i] * K, K, gamma, a[ms[i]], &acc[i], &y[i]) != 0) return 1;
  }
  return 0;
}

// Base-3 storage of the ternary codes ([Explainer, "Skąd te 1,58 bita": a
// ternary weight carries log2(3) ~ 1.58 bits of information; Habr repost,
// "Когда - три лучше двух": log2(3) bits per parameter).  Five codes
// c = q + 1 in {0,1,2} fit in one byte as a base-3 number (3^5 = 243 <= 256),
// 1.6 bits per weight.  Layout (this library's own): a row is padded with
// zero weights to Kp = ceil(K/80)*80 and stored as Kp/80 groups of 16 bytes;
// byte i of group g is sum_{t=0..4} c[80g + 16t + i] * 3^t.
int64_t oracle_b3_padded_k(int64_t K) { return (K + 79) / 80 * 80; }

void oracle_pack_codes_b3(const int8_t* q, int64_t N, int64_t K, uint8_t* packed) {
  const int64_t Kp = oracle_b3_padded_k(K), rb = Kp / 5;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < Kp / 80; ++g)
      for (int i = 0; i < 16; ++i) {
        int v = 0, p3 = 1;
        for (int t = 0; t < 5; ++t) {
          const int64_t k = 80 * g + 16 * t + i;
          const int c = k < K ? q[n * K + k] + 1 : 1;
          v += c * p3;
          p3 *= 3;
        }
        packed[n * rb + 16 * g + i] = static_cast<uint8_t>(v);
      }
}

// Inverse of oracle_pack_codes_b3 for the first K weights of each row;
// returns the number of bytes above 242 (not a valid base-3 group) plus the
// number of padded positions whose code is not 1 (q = 0).
int64_t oracle_unpack_codes_b3(const uint8_t* packed, int64_t N, int64_t K, int8_t* q) {
  const int64_t Kp = oracle_b3_padded_k(K), rb = Kp / 5;
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < Kp / 80; ++g)
      for (int i = 0; i < 16; ++i) {
        int v = packed[n * rb + 16 * g + i];
        if (v > 242) ++bad;
        for (int t = 0; t < 5; ++t) {
          const int c = v % 3;
          v /= 3;
          const int64_t k = 80 * g + 16 * t + i;
          if (k < K) q[n * K + k] = static_cast<int8_t>(c - 1);
          else if (c != 1) ++bad;
        }
      }
  return bad;
}

// The BitLinear product against base-3 packed weights: the same exact dot
// product and dequant as oracle_bitlinear, on the decoded codes.
int oracle_bitlinear_b3(const uint8_t* packed, float gamma, int64_t N, int64_t K,
                        const int8_t* xq, const float* a, int64_t M, int32_t* acc, float* y) {
  const int64_t rb = oracle_b3_padded_k(K) / 5;
  std::vector<int8_t> q(static_cast<size_t>(K));
  for (int64_t n = 0; n < N; ++n) {
    if (oracle_unpack_codes_b3(packed + n * rb, 1, K, q.data()) != 0) return 2;
    for (int64_t m = 0; m < M; ++m)
      if (oracle_dot(q.data(), xq + m * K, K, gamma, a[m], &acc[m * N + n], &y[m * N + n]) != 0) return 1;
  }
  return 0;
}

// Squared-ReLU gating of the feed-forward block: the FFN of BitNet b1.58
// uses a squared ReLU as its activation ([Explainer, "Zrób to sam": squared
// ReLU in the FFN, subln normalisation, no biases]; kripta.biz 2B4T news:
// ReLU^2 in the FFN layers).  The gate branch goes through the activation
// and multiplies the up branch elementwise:
//   out[i] = RN32(RN32(r * r) * u[i]),  r = g[i] if g[i] > 0, else +0.
// u and g are the fp32 outputs of the up and gate BitLinears.
void oracle_relu2_gate(const float* u, const float* g, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) {
    const float r = g[i] > 0.0f ? g[i] : 0.0f;
    const float sq = r * r;
    out[i] = sq * u[i];
  }
}

// fp32 -> bf16, round half to even, as bit patterns (NaN -> quiet NaN).
void oracle_f32_to_bf16(const float* y, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u;
    std::memcpy(&u, &y[i], 4);
    if (std::isnan(y[i])) {
      out[i] = 0x7FC0;
      continue;
    }
    const uint32_t lsb = (u >> 16) & 1u;
    out[i] = static_cast<uint16_t>((u + 0x7FFFu + lsb) >> 16);
  }
}

}  // extern "C"
