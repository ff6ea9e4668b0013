/*
 * bitnet.h -- C ABI of the BitNet b1.58 BitLinear forward (W1.58A8) for
 * NVIDIA B200 (sm_100a).
 *
 * The four steps of BitLinear, as the BitNet b1.58 pages describe them
 * (comrad404.com, "BitNet b1.58: что показала работа Microsoft об «эре
 * 1-битных LLM»", section "Метод: как устроен BitNet b1.58"): normalise the
 * input, quantise the activations to 8 bits, replace the weights by ternary
 * {-1, 0, 1} ones obtained by absmean, then a low-bit matrix product followed
 * by rescaling of the result.
 *
 * Conventions for every call below:
 *   - All array pointers are DEVICE pointers, allocated and owned by the
 *     caller.  The library allocates no memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is enqueued on that stream and returns without
 *     waiting, except bitnet_pack_weights and bitnet_get_device_status,
 *     which synchronise the stream.
 *   - Matrices are dense, row-major and contiguous.  W is N x K (row n is
 *     output feature n), activations are M x K (row m is token m), outputs
 *     are M x N.
 *   - K must be a positive multiple of 64 (so a packed row is a whole number
 *     of 16-byte units); M >= 1 and N >= 1 are arbitrary.
 *   - Every pointer must be 16-byte aligned.
 *   - Errors are returned as bitnet_status; nothing is launched when an
 *     argument is rejected.  No C++ exception crosses this boundary.
 *   - The product entry points (bitnet_linear_gemv, bitnet_linear_gemm and
 *     its _stream_k form, bitnet_linear_upgate_gemm, bitnet_bitlinear_gemv,
 *     bitnet_bitlinear_gemm and its _stream_k form, bitnet_bitlinear_ffn_gemv,
 *     bitnet_bitlinear_gemv_b3) are launched with programmatic dependent
 *     launch: they start while the previous kernel on the stream finishes,
 *     and request their first packed-weight tiles BEFORE waiting for it
 *     (the weights of a layer never depend on the layer before).  So the
 *     kernel launched immediately before one of them on the same stream must
 *     not write the packed weights it reads.  Any kernel between the writer
 *     and the product call, a synchronisation, or an event wait restores the
 *     ordering; a kernel that writes the weights and does not signal early
 *     completion (cudaTriggerProgrammaticLaunchCompletion) is also safe in
 *     practice, and the tests check a torch copy followed directly by the
 *     decode entry points.  Activations, scales and outputs are only touched
 *     after the wait.
 *
 * Packed weight layout (2 bits per weight; the pages say only that the three
 * states are stored on two bits plus some structure -- inferownia.pl,
 * "BitNet b1.58: era 1-bitowych LLM-ów", section "Skąd te 1,58 bita"):
 *   code c = q + 1 in {0, 1, 2} (3 never occurs); a row takes K/4 bytes; one
 *   little-endian 32-bit word holds 16 consecutive weights k0..k0+15, weight
 *   k0 + 4j + b in byte b, bits 2j..2j+1.  So (word >> 2j) & 0x03030303 gives
 *   the codes of weights k0+4j .. k0+4j+3 in its four bytes.
 */
#ifndef BITNET_H_
#define BITNET_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bitnet_status {
  BITNET_OK = 0,
  BITNET_ERR_INVALID_ARG = 1,       /* null/misaligned pointer, bad dtype, bad eps */
  BITNET_ERR_UNSUPPORTED_SHAPE = 2, /* K not a positive multiple of 64, M/N < 1, sizes too large */
  BITNET_ERR_NONFINITE = 3,         /* bitnet_pack_weights: W holds Inf or NaN */
  BITNET_ERR_CUDA = 4,              /* a CUDA runtime or driver call failed */
  BITNET_ERR_TIMEOUT = 5            /* a kernel gave up waiting on a barrier (see get_device_status) */
} bitnet_status;

typedef enum bitnet_dtype {
  BITNET_F32 = 0,
  BITNET_BF16 = 1,
  BITNET_I32 = 2 /* outputs only: the raw int32 accumulator, no dequantisation */
} bitnet_dtype;

/* Bytes of scratch memory bitnet_pack_weights needs for an N x K matrix. */
size_t bitnet_pack_workspace_bytes(int64_t N, int64_t K);

/*
 * Absmean ternarisation and 2-bit packing of a latent fp32 weight matrix
 * (inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", section "Trenowany
 * od zera": the whole matrix is scaled by its mean absolute value and every
 * entry goes to the nearest integer of {-1, 0, +1}).
 *
 *   gamma = mean |W| over all N*K entries.  Summation order is fixed, so the
 *           result is reproducible bit for bit: per row, 32 fp64 partials
 *           (partial l takes k = l, l+32, ... in increasing k) combined by the
 *           halving tree p[l] += p[l+s], s = 16, 8, 4, 2, 1; rows added in
 *           increasing n in fp64; gamma = RN32(S / (N*K)).
 *   q     = clamp(RNE(RN32(w / RN32(gamma + eps))), -1, 1), ties to even.
 *
 * W         [in]  N x K fp32, device.
 * eps       [in]  finite, > 0 (keeps the divisor positive for an all-zero W).
 * W_packed  [out] N x K/4 bytes, device, layout above.
 * gamma     [out] 1 fp32, device: the per-tensor scale used by the product.
 * workspace [in]  device scratch of at least bitnet_pack_workspace_bytes(N, K)
 *                 bytes; its contents on entry do not matter.
 * Synchronises `stream`.  Returns BITNET_ERR_NONFINITE (outputs unspecified)
 * if W holds a non-finite value.
 */
bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, float eps,
                                  uint8_t* W_packed, float* gamma,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * bitnet_pack_weights without a caller workspace.  The BitNet b1.58 pages
 * have no counterpart to this: it exists for callers that cannot allocate
 * device memory -- code that runs inside a host application whose memory
 * pool owns every device allocation, or services that must not allocate
 * once they have started -- and so cannot provide the workspace buffer.
 *
 * Same arguments (minus the workspace), results and error behaviour as
 * bitnet_pack_weights; it calls no cudaMalloc, cudaFree or allocating
 * library routine.  Its scratch is a fixed array inside the library,
 * 8 * BITNET_PACK_NOALLOC_MAX_ROWS + 256 bytes (about 512 KB), which every
 * GPU that loads the library holds until the process exits.
 *   - N above BITNET_PACK_NOALLOC_MAX_ROWS is rejected with
 *     BITNET_ERR_UNSUPPORTED_SHAPE before anything is launched.
 *   - The first call on each device looks up the device address of that
 *     array (cudaGetSymbolAddress) with that device current; make that first
 *     call before any stream capture.
 *   - All calls share the array and it keeps the previous call's contents;
 *     the call clears what must start at zero.  Calls that overlap on the GPU
 *     (for example from two host threads on two streams) race on it.
 *   - The looked-up address is kept for the life of the process, so the
 *     library must not be used on a device after cudaDeviceReset of that
 *     device (the array's address belongs to the destroyed context).
 * Synchronises `stream`.
 */
#define BITNET_PACK_NOALLOC_MAX_ROWS 65536
bitnet_status bitnet_pack_weights_noalloc(const float* W, int64_t N, int64_t K, float eps,
                                          uint8_t* W_packed, float* gamma, void* stream);

/*
 * Per-token absmax int8 quantisation of activations, optionally fused with
 * the RMSNorm that precedes it (comrad404.com review, section "Метод":
 * 8-bit activations, RMSNorm in the LLaMA-like stack, the input normalised
 * before it is quantised).  One pass over x.  For each token row v (values widened to
 * fp32 exactly):
 *   with rms_gain:  ss = sum of RN32(v_k^2) in a fixed order (256 lanes, lane
 *                   l owning the 8-element chunks c = l, l+256, ... summed in
 *                   increasing k; then the halving tree l += l+128, ..., l+1);
 *                   r = RN32(1 / RN32(sqrt(RN32(RN32(ss / K) + rms_eps))));
 *                   h_k = RN32(RN32(v_k * r) * g_k)
 *   without:        h = v
 *   amax = max |h|;  s = RN32(127 / amax);
 *   x_q  = clamp(RNE(RN32(h * s)), -127, 127);  a_scale = RN32(amax / 127);
 *   a token with amax == 0 gets x_q = 0 and a_scale = 0.
 *
 * x        [in]  M x K, dtype x_dtype (BITNET_F32 or BITNET_BF16), device.
 * rms_gain [in]  K values of the same dtype as x, or NULL for no RMSNorm.
 * rms_eps  [in]  finite, > 0 when rms_gain is given; ignored otherwise.
 * x_q      [out] M x K int8.
 * a_scale  [out] M fp32 per-token dequant scales.
 * x_rowsum [out] M int32 sums of x_q per token, or NULL to skip.
 * K <= 32768 for BF16 input, K <= 16384 for F32.  Non-finite inputs give
 * unspecified codes.  Asynchronous.
 */
bitnet_status bitnet_quant_act(const void* x, int x_dtype, int64_t M, int64_t K,
                               const void* rms_gain, float rms_eps,
                               int8_t* x_q, float* a_scale, int32_t* x_rowsum, void* stream);

/*
 * W1.58A8 product with exact int32 accumulation and fused dequant epilogue,
 * for small batches (decode), on CUDA cores: packed weights are streamed
 * once through shared memory with bulk asynchronous copies, each warp forms
 * byte dot products (dp4a) and reduces them with warp shuffles.
 * The ternary product is the sum of the inputs with weight +1 minus the sum
 * of those with weight -1 (Habr repost on juhe.plus, section "Когда - три
 * лучше двух"); the integer result is exact.
 *
 *   acc[m][n] = sum_k q[n][k] * x_q[m][k]              (exact, int32)
 *   y[m][n]   = RN32(RN32(float(acc) * gamma) * a_scale[m])   (F32), or its
 *               round-half-even bf16 (BF16), or acc itself (I32).
 *
 * W_packed [in]  N x K/4 bytes from bitnet_pack_weights.
 * gamma    [in]  1 fp32, device, from bitnet_pack_weights.
 * x_q, a_scale [in] from bitnet_quant_act (M x K int8, M fp32).
 * x_rowsum [in]  M int32 = sum_k x_q[m][k], or NULL.  When given, the kernel
 *                multiplies by the unsigned codes c = q + 1 and subtracts
 *                the row sum, which saves work; the result is identical.
 * M        [in]  1 <= M <= 8.
 * y        [out] M x N of dtype y_dtype (BITNET_F32, BITNET_BF16 or BITNET_I32).
 * Asynchronous.
 */
bitnet_status bitnet_linear_gemv(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                 const int8_t* x_q, const float* a_scale, const int32_t* x_rowsum,
                                 int64_t M, void* y, int y_dtype, void* stream);

/*
 * Bytes of workspace bitnet_linear_gemm uses for an M x K by N x K product on
 * the CURRENT device (it depends on the device's SM count): for M <= 64 a
 * flag per SM and one partial int32 tile of 128 rows x 16, 32 or 64 tokens
 * per SM (about 1.2, 2.4 or 4.8 MB on a B200); 0 for M > 64, where no
 * workspace is used.
 */
size_t bitnet_linear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * The same product for any M >= 1 on the 5th-generation tensor cores
 * (tcgen05 kind::i8, int32 accumulators in tensor memory): packed weight
 * tiles and activation tiles arrive in shared memory by TMA, the ternary
 * codes are expanded to 8-bit in registers and written to tensor memory as
 * the A operand, the activations are the B operand in shared memory.
 * Same formulas and results as bitnet_linear_gemv (the low-bit product
 * followed by rescaling of the comrad404.com review, section "Метод").
 *
 * workspace [in,out] device memory of at least
 *           bitnet_linear_gemm_workspace_bytes(M, N, K) bytes, 16-byte
 *           aligned, or NULL.  With M <= 64, a workspace, and at least 12
 *           (128-row tile, 256-K step) units of work per SM, the product
 *           runs "stream-K": every SM takes an equal share of the units and
 *           partial tiles cut between SMs are added exactly in int32 through
 *           the workspace, so decode-sized batches stream the packed weights
 *           on every SM (smaller products run on tiles: their fixed cost is
 *           lower).  Zero the workspace
 *           before its first use (e.g. cudaMemset): it holds flags and
 *           partial-tile accumulators that must start at zero, and every
 *           call leaves them zero again.  Two calls that may run at the same time (on two
 *           streams) must not share a workspace.  If a call reports
 *           BITNET_ERR_TIMEOUT through bitnet_get_device_status, zero the
 *           workspace again before reusing it.  The stream-K launch
 *           has one CTA per SM and its CTAs wait on one another (bounded
 *           waits), so it needs all the device's SMs to be available to it at
 *           once: where the process gets only part of the GPU (an MPS limit
 *           on active SMs), pass no workspace.  Without a workspace (NULL,
 *           with workspace_bytes ignored) or for M > 64, the product runs on
 *           persistent tiles, split over thread-block clusters when there
 *           are few tiles; the results are identical.
 * M <= 2^31 - 1, N <= 2^31 - 1, K <= 2^31 - 1 with M*N fitting the output.
 * Asynchronous.
 */
bitnet_status bitnet_linear_gemm(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                 const int8_t* x_q, const float* a_scale, const int32_t* x_rowsum,
                                 int64_t M, void* y, int y_dtype, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * bitnet_linear_gemm with the stream-K product forced for any size (the
 * automatic choice takes it only from 12 units of work per SM).  Same
 * arguments, results and errors; the workspace is required
 * (BITNET_ERR_INVALID_ARG without one) and M must be at most 64
 * (BITNET_ERR_UNSUPPORTED_SHAPE otherwise).
 */
bitnet_status bitnet_linear_gemm_stream_k(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                          const int8_t* x_q, const float* a_scale, const int32_t* x_rowsum, int64_t M,
                                          void* y, int y_dtype, void* workspace, size_t workspace_bytes,
                                          void* stream);

/*
 * Bytes of workspace bitnet_bitlinear_gemm uses on the CURRENT device: the
 * stream-K flags and partial tiles of bitnet_linear_gemm, 256 bytes of grid
 * barrier, and the quantised rows, scales and row sums; 0 for M outside
 * 1..64 or an invalid K.
 */
size_t bitnet_bitlinear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * BitLinear for decode-sized batches (1 <= M <= 64 tokens): bitnet_quant_act
 * into the workspace, then bitnet_linear_gemm's product with the rest of the
 * workspace (stream-K, or tiles for a small product), as two launches chained
 * by programmatic dependent launch (the four BitLinear steps of the
 * comrad404.com review, section "Метод").  bitnet_bitlinear_gemm_stream_k
 * does the same in ONE launch: the first CTAs quantise one token row each
 * (same arithmetic and summation order as bitnet_quant_act) into the
 * workspace while every CTA already streams its share of the packed weights,
 * and a grid barrier in the workspace then releases the stream-K product;
 * measured on B200 that launch is the slower one (its grid barrier costs more
 * than the kernel boundary it removes).  The results are identical either way
 * and to the two public calls.
 *
 * x, x_dtype, rms_gain, rms_eps   as bitnet_quant_act (K <= 32768 bf16, 16384 f32).
 * W_packed, gamma, N, K, y, y_dtype   as bitnet_linear_gemm.
 * workspace [in,out] at least bitnet_bitlinear_gemm_workspace_bytes(M, N, K)
 *           bytes, 16-byte aligned, zeroed before its first use; the calls
 *           leave its flags and barrier words zero-based again.  Same rules
 *           as bitnet_linear_gemm's workspace: not shared by calls that may
 *           overlap, zeroed again after a BITNET_ERR_TIMEOUT, and the launch
 *           needs every SM of the device at once (its CTAs wait on one
 *           another, with bounded waits).
 * Asynchronous.
 */
bitnet_status bitnet_bitlinear_gemm(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                    const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                    void* y, int y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * bitnet_bitlinear_gemm as ONE launch (quantisation inside the stream-K
 * product, see above), at any size.  Same arguments, results and errors.
 */
bitnet_status bitnet_bitlinear_gemm_stream_k(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                             const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                             int64_t M, void* y, int y_dtype, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace bitnet_linear_upgate_gemm uses on the CURRENT device
 * (a flag per SM and one partial int32 tile of 128 rows x 16, 32 or 64
 * tokens per SM); 0 for an invalid shape.
 */
size_t bitnet_linear_upgate_workspace_bytes(int64_t M, int64_t F, int64_t K);

/*
 * The feed-forward block's up and gate BitLinear products with the
 * squared-ReLU gate in their epilogue (inferownia.pl, "BitNet b1.58: era
 * 1-bitowych LLM-ów", section "Zrób to sam": squared ReLU in the FFN;
 * kripta.biz 2B4T news: ReLU^2 in the FFN layers), for any M, on the
 * tensor cores (the stream-K product of bitnet_linear_gemm: a 128-row tile
 * holds the up and the gate rows of 64 features, so one epilogue sees both):
 *
 *   u[m][f] = RN32(RN32(float(acc_up[m][f])   * gamma_up)   * a_scale[m])
 *   g[m][f] = RN32(RN32(float(acc_gate[m][f]) * gamma_gate) * a_scale[m])
 *   r = g if g > 0 else +0;   h[m][f] = bf16(RN32(RN32(r * r) * u))
 *
 * (acc as in bitnet_linear_gemv).  u and g never reach memory; h is the
 * down projection's bf16 input (quantise it with bitnet_quant_act, with the
 * sub-layer norm's gain, then bitnet_linear_gemm).
 *
 * W_up, W_gate     [in]  F x K/4 packed bytes each (bitnet_pack_weights).
 * gamma_up/gate    [in]  their fp32 scales (device).
 * x_q, a_scale, x_rowsum [in]  the quantised block input, as bitnet_linear_gemm.
 * h                [out] M x F bf16.
 * workspace        [in,out] at least bitnet_linear_upgate_workspace_bytes(M, F,
 *                  K) bytes, 16-byte aligned, zeroed before its first use;
 *                  same rules as bitnet_linear_gemm's workspace (required).
 * Asynchronous.
 */
bitnet_status bitnet_linear_upgate_gemm(const uint8_t* W_up, const float* gamma_up, const uint8_t* W_gate,
                                        const float* gamma_gate, int64_t F, int64_t K, const int8_t* x_q,
                                        const float* a_scale, const int32_t* x_rowsum, int64_t M, void* h,
                                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Fused decode BitLinear: bitnet_quant_act followed by bitnet_linear_gemv in
 * one kernel launch, for M <= 8 tokens.  Every CTA quantises the M token
 * rows itself (same arithmetic and summation order as bitnet_quant_act) into
 * its shared memory and then runs the GEMV, so the result is identical to
 * the two-call path while saving a dependent kernel launch and the x_q round
 * trip through global memory per linear (the four BitLinear steps of the
 * comrad404.com review, section "Метод", in one pass).
 *
 * x, x_dtype, rms_gain, rms_eps   as bitnet_quant_act.
 * W_packed, gamma, N, K, y, y_dtype   as bitnet_linear_gemv.
 * 1 <= M <= 8 and M * K <= 21504 (the quantised rows live in shared memory);
 * other shapes return BITNET_ERR_UNSUPPORTED_SHAPE (use the two calls).
 * Asynchronous.
 */
bitnet_status bitnet_bitlinear_gemv(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                    const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K, int64_t M,
                                    void* y, int y_dtype, void* stream);

/*
 * bitnet_bitlinear_gemv with the token rows and the output in host memory:
 * on `stream`, one cudaMemcpyAsync of x_host (M x K, x_dtype) into x, the
 * fused kernel, and one cudaMemcpyAsync of y (M x N, y_dtype) into y_host.
 * The decode step of a caller whose tokens live on the host, in one call.
 *
 * x_host  [in]  M x K host values; page-locked (cudaHostAlloc /
 *               cudaHostRegister) for the copy to be asynchronous, else the
 *               copy is synchronous with respect to the host.
 * x       [out] device staging buffer of M x K values (16-byte aligned); the
 *               kernel reads it after the copy.
 * y       [out] device M x N outputs; y_host [out] host copy of them, valid
 *               once `stream` has reached the end of the call.
 * Other arguments and errors as bitnet_bitlinear_gemv; NULL x_host or y_host
 * returns BITNET_ERR_INVALID_ARG.  Nothing is copied when an argument is
 * rejected.  Asynchronous: the caller synchronises `stream` before reading
 * y_host and must keep both host buffers alive until then.
 */
bitnet_status bitnet_bitlinear_gemv_host(const void* x_host, void* x, int x_dtype, const void* rms_gain,
                                         float rms_eps, const uint8_t* W_packed, const float* gamma, int64_t N,
                                         int64_t K, int64_t M, void* y, void* y_host, int y_dtype, void* stream);

/*
 * Base-3 storage of the ternary codes, 1.6 bits per weight (a ternary weight
 * holds log2(3) ~ 1.58 bits: inferownia.pl, "BitNet b1.58: era 1-bitowych
 * LLM-ów", section "Skąd te 1,58 bita"; Habr repost on juhe.plus, section
 * "Когда - три лучше двух").  Five codes c = q + 1 form one byte as a base-3
 * number.  A row is padded with zero weights to Kp = ceil(K/80)*80 and stored
 * as Kp/80 groups of 16 bytes; byte i of group g = sum_{t=0..4} c[80g+16t+i]
 * 3^t.  Rows are contiguous, bitnet_b3_row_bytes(K) = Kp/5 bytes each
 * (K = 2560: 512 bytes; K = 6912: 1392 bytes), 20% fewer than the 2-bit
 * layout when K is a multiple of 80.
 *
 * bitnet_b3_row_bytes: bytes per packed row, 0 for an unsupported K.
 * bitnet_pack_weights_b3: as bitnet_pack_weights (same gamma, same codes,
 *   same workspace and errors; K <= 24000), writing N x bitnet_b3_row_bytes(K)
 *   bytes to W_b3.  Synchronises.
 * bitnet_bitlinear_gemv_b3: as bitnet_bitlinear_gemv (fused quantisation and
 *   product for M <= 8 tokens) on base-3 packed weights; requires
 *   M * Kp <= 24000 (and K <= 8192 for fp32 x).  Results identical to
 *   bitnet_bitlinear_gemv on the 2-bit packing of the same matrix.
 *   Asynchronous.
 */
size_t bitnet_b3_row_bytes(int64_t K);
bitnet_status bitnet_pack_weights_b3(const float* W, int64_t N, int64_t K, float eps, uint8_t* W_b3, float* gamma,
                                     void* workspace, size_t workspace_bytes, void* stream);
bitnet_status bitnet_bitlinear_gemv_b3(const void* x, int x_dtype, const void* rms_gain, float rms_eps,
                                       const uint8_t* W_b3, const float* gamma, int64_t N, int64_t K, int64_t M,
                                       void* y, int y_dtype, void* stream);

/*
 * Backward pass of the BitLinear with the straight-through estimator.
 * Training keeps precise latent weights and computes with the rounded ones,
 * and the backward pass lets the gradient through the rounding as if it were
 * absent (Habr repost on juhe.plus, sections "А откуда взялась сама идея?"
 * and "Когда - три лучше двух").  The forward used W_hat = gamma * q and
 * x_hat[m] = a_scale[m] * x_q[m]; both products run on the tensor cores
 * (tcgen05 kind::f16: bf16 operands, fp32 accumulation) after short
 * pre-passes that write the operands as bf16 into the caller's workspace.
 *
 * bitnet_ste_backward_input: dX[m][k] = RN32(gamma * sum_n dY[m][n] q[n][k])
 *   up to the order of the fp32 accumulation.  W_packed, gamma, N, K as for
 *   the forward (N x K/4 packed codes); dY: M x N bf16, row-major; dX: M x K
 *   of dx_dtype (BITNET_F32 or BITNET_BF16).  N a multiple of 8.  workspace:
 *   bitnet_ste_input_workspace_bytes(N, K) device bytes (q transposed as bf16).
 * bitnet_ste_backward_weight: dW[n][k] = sum_m dYs[m][n] x_q[m][k] with
 *   dYs = bf16_RNE(RN32(dY[m][n] * a_scale[m])) (the product's bf16 left
 *   operand), up to the order of the fp32 accumulation.  dY: M x N bf16; x_q,
 *   a_scale: the forward's quantised activations (M x K int8, M fp32); dW:
 *   N x K of dw_dtype.  workspace: bitnet_ste_weight_workspace_bytes(M, N, K)
 *   device bytes (dYs and x_q transposed as bf16, tokens padded to 64).
 * Pointers 16-byte aligned (gamma, a_scale 4-byte).  Asynchronous.
 */
size_t bitnet_ste_input_workspace_bytes(int64_t N, int64_t K);
bitnet_status bitnet_ste_backward_input(const uint8_t* W_packed, const float* gamma, int64_t N, int64_t K,
                                        const void* dY, int64_t M, void* dX, int dx_dtype, void* workspace,
                                        size_t workspace_bytes, void* stream);
size_t bitnet_ste_weight_workspace_bytes(int64_t M, int64_t N, int64_t K);
bitnet_status bitnet_ste_backward_weight(const void* dY, const int8_t* x_q, const float* a_scale, int64_t M,
                                         int64_t N, int64_t K, void* dW, int dw_dtype, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* Bytes of the grid-barrier workspace that bitnet_bitlinear_ffn_gemv takes. */
#define BITNET_FFN_SYNC_BYTES 64

/*
 * Decode feed-forward block of BitNet b1.58 for M <= 8 tokens, in one
 * launch.  The block is three BitLinears with squared-ReLU gating
 * (inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", section "Zrób to
 * sam": squared ReLU in the FFN, subln normalisation, no biases; kripta.biz
 * BitNet b1.58 2B4T news: ReLU^2 in the FFN layers); each BitLinear
 * normalises and quantises its input, multiplies by the ternary weights and
 * rescales (comrad404.com review, section "Метод"):
 *
 *   u = BitLinear(x; W_up, gamma_up, rms_gain_in)      fp32, as bitnet_bitlinear_gemv
 *   g = BitLinear(x; W_gate, gamma_gate, rms_gain_in)  fp32
 *   h = bf16_RNE(RN32(RN32(r * r) * u)),  r = g if g > 0, else +0
 *   y = BitLinear(h; W_down, gamma_down, rms_gain_sub) y_dtype
 *
 * Results are identical to two bitnet_bitlinear_gemv calls with F32 output,
 * the gating step, and a third bitnet_bitlinear_gemv on h.
 *
 * x            [in]  M x D bf16 token rows (x_dtype must be BITNET_BF16).
 * M, D, F      [in]  1 <= M <= 8; D (hidden) and F (FFN width) positive
 *                    multiples of 64, each <= 24576; shapes whose working set
 *                    does not fit one SM's shared memory (roughly M * max(D, F)
 *                    above 140000 bytes) return BITNET_ERR_UNSUPPORTED_SHAPE.
 * rms_gain_in  [in]  D bf16 RMSNorm gain of x, or NULL for no norm; rms_eps_in
 *                    finite and > 0 when given.
 * W_up, W_gate [in]  F x D/4 packed (bitnet_pack_weights of F x D matrices),
 *                    gamma_up, gamma_gate their scales (device float[1]).
 * rms_gain_sub [in]  F bf16 RMSNorm gain of h (the sub-layer norm), or NULL;
 *                    rms_eps_sub finite and > 0 when given.
 * W_down       [in]  D x F/4 packed, gamma_down its scale.
 * h            [out] M x F bf16: the down projection's input.
 * y            [out] M x D of dtype y_dtype (BITNET_F32, BITNET_BF16, or
 *                    BITNET_I32 for the raw int32 accumulator of W_down).
 * sync         [in,out] BITNET_FFN_SYNC_BYTES bytes of device memory, 8-byte
 *                    aligned, zero-filled by the caller before the first call
 *                    (its first 8 bytes count barrier arrivals).  Calls in one
 *                    stream may share it; calls that can run at the same time
 *                    (other streams) must not.  The call leaves it ready for
 *                    the next call, except after a BITNET_ERR_TIMEOUT, when it
 *                    must be zero-filled again.
 * Pointers: x, gains, W_*, h, y 16-byte aligned; gammas 4-byte aligned; h
 * and y must not overlap the inputs.
 * The kernel is a cooperative launch of one CTA per SM (its CTAs wait for
 * one another once, between the gating and the down projection; that wait is
 * bounded and reports BITNET_ERR_TIMEOUT through bitnet_get_device_status).
 * For ONE token with large weight shares per SM (F rows x D/4 bytes above
 * 64 KB per SM, as in the 27B-class FFN) the block instead runs as two
 * launches of the one-token decode product: up and gate with the gating in
 * the epilogue (x -> h), then bitnet_bitlinear_gemv on h (h -> y); the results
 * are the same and `sync` is not touched.  Asynchronous.
 */
bitnet_status bitnet_bitlinear_ffn_gemv(const void* x, int x_dtype, int64_t M, int64_t D, int64_t F,
                                        const void* rms_gain_in, float rms_eps_in, const uint8_t* W_up,
                                        const float* gamma_up, const uint8_t* W_gate, const float* gamma_gate,
                                        const void* rms_gain_sub, float rms_eps_sub, const uint8_t* W_down,
                                        const float* gamma_down, void* h, void* y, int y_dtype, void* sync,
                                        void* stream);

/*
 * Synchronises `stream`, then reports and clears the device-side error word
 * that kernels set when a bounded wait on a barrier runs out (they then skip
 * their remaining work and exit instead of hanging).  Returns BITNET_OK,
 * BITNET_ERR_TIMEOUT, or BITNET_ERR_CUDA if the stream itself failed.
 */
bitnet_status bitnet_get_device_status(void* stream);

/* Static English description of a status code. */
const char* bitnet_status_string(bitnet_status s);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_H_ */
