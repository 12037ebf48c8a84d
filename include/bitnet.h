/*
 * bitnet.h -- C ABI of the sm_100a W1.58A8 BitLinear library.
 *
 * The library computes the BitNet b1.58 BitLinear forward pass: ternary
 * {-1,0,+1} weights stored 2 bits each, int8 activations, an int32 matmul
 * and an fp32 dequantisation stored as bf16, plus the fused FFN block built
 * from it.  Sources of each operation are cited per entry point by page and
 * section:
 *   [Y]  youngju.dev, "BitNet論文分析：1-Bit LLMの時代 — 三値重みからCPU推論まで"
 *   [D]  dashen-tech.com, "BitNet.cpp 深度解析：1-bit LLM 推論、CPU 上で 100B
 *        モデルを 6 倍高速実行"
 *   [A]  abeam.tech, review of "BitNet: 1-bit Pre-training for Large Language
 *        Models" (JMLR 2025)
 *   [R]  reinforz.co.jp, news article on "BitNet b1.58 2B4T"
 *
 * Conventions shared by every entry point
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or synchronises inside these calls.  Scratch
 *     memory, where needed, is a caller-provided device workspace whose size
 *     comes from the matching *_workspace_size() function.
 *   - bf16 values are passed as their raw 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it.  Kernels that only read
 *     weights before their first dependency are launched with programmatic
 *     dependent launch, so back-to-back calls overlap their weight streaming.
 *   - Row-major layouts: x [M,K], y [M,N], W [N,K] (out x in, like
 *     nn.Linear), packed [N, K/4].
 *   - Arguments are validated on the host before anything is launched; a
 *     non-OK status means nothing was enqueued.  Launch failures return
 *     BITNET_ERR_CUDA.  Device-side conditions (a bounded wait that expired,
 *     a non-finite weight) are recorded in a per-device status word that
 *     bitnet_last_device_status() reports.
 *   - Pointers to x, y, packed and the workspace must be 16-byte aligned.
 *   - The library keeps small per-device host caches (SM count, kernel
 *     shared-memory settings, occupancy, the no-alloc scratch address),
 *     filled on first use and safe across host threads.  They belong to the
 *     device's primary context: after cudaDeviceReset() (which destroys it)
 *     reload the library before calling it again on that device.
 */
#ifndef BITNET_B200_H_
#define BITNET_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BITNET_OK = 0,
  BITNET_ERR_INVALID_ARG = 1,  /* null pointer where one is required, eps < 0 */
  BITNET_ERR_SHAPE = 2,        /* M, N or K out of range, K % 4 != 0          */
  BITNET_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned            */
  BITNET_ERR_WORKSPACE = 4,    /* workspace null or smaller than required     */
  BITNET_ERR_UNSUPPORTED = 5,  /* device is not sm_100 / feature unavailable  */
  BITNET_ERR_CUDA = 6,         /* a CUDA runtime call failed                  */
  BITNET_ERR_TIMEOUT = 7,      /* a device-side bounded wait gave up          */
  BITNET_ERR_NONFINITE = 8     /* a weight was Inf or NaN (gamma set to NaN)  */
} bitnet_status;

/* Human-readable name of a status code (static string, never NULL). */
BITNET_API const char* bitnet_status_string(int status);

/* Library ABI version: 100 * major + minor. */
BITNET_API int bitnet_version(void);

/*
 * Absmean ternary weight quantisation + I2_S 2-bit packing.
 *   [Y] section "Absmean量子化関数" (weight_quant_ternary: gamma = mean|W|,
 *       W_q = clamp(round(W / (gamma + 1e-5)), -1, 1));
 *   [Y] section "アーキテクチャ概要" (I2_S: 00 = -1, 01 = 0, 10 = +1,
 *       16 weights per 32-bit register); [D] section "2.3 I2_S 形式".
 *
 * W       [N,K] fp32, device, read only.  Must be finite.
 * packed  [N,K/4] uint8, device, written.  Weight k of row n is code
 *         (W_q + 1) at bits 2*(k%4) of byte n*K/4 + k/4 (LSB first).
 *         Code 3 is never produced.
 * gamma   one fp32 on the device, written: the fp32 value nearest (ties to
 *         even) to the exact mean of |W| (independent of summation order).
 *         The ternary threshold divides by gamma + 1e-5 (fp32 add, IEEE
 *         division per element, round half to even); dequantisation later
 *         multiplies by gamma itself.
 * workspace  >= bitnet_pack_workspace_size(N, K) bytes of device memory; its
 *         contents are overwritten.
 * Requires K % 4 == 0, N >= 1, K >= 4, N*K < 2^39.  A non-finite weight sets
 * gamma to NaN and records BITNET_ERR_NONFINITE in the device status word.
 * Not performance-critical (run once per weight matrix).
 */
BITNET_API size_t bitnet_pack_workspace_size(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                  float* gamma, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * Per-token absmax int8 activation quantisation.
 *   [Y] section "Absmean量子化関数" (BitLinear_b158.activation_quant, per
 *       token absmax with rounding and clamping); [R] section
 *       "積極的量子化と三値化がもたらす学習効率の革新" (absmax, 8-bit, W1.58A8).
 *
 * s_t = 127 / max(max_k |x[t,k]|, 1e-5)          (fp32, IEEE division)
 * xq[t,k] = clamp(rint(x[t,k] * s_t), -128, 127)  (one fp32 multiply)
 * x       [M,K] bf16 bits, device.        xq   [M,K] int8, device, written.
 * scale   [M] fp32, device, written (s_t).
 * rowsum  [M] int32, device, written with sum_k xq[t,k]; may be NULL.
 * Requires M >= 1, K >= 1, K % 4 == 0.
 */
BITNET_API bitnet_status bitnet_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq,
                               float* scale, int32_t* rowsum, void* stream);

/*
 * BitLinear forward: y = dequant(quant(x) . W_q^T).
 *   [D] section "3.1 計算コア：整数行列乗算" (Y = sum_pos - sum_neg, no
 *       multiplications); [Y] section "Absmean量子化関数" (BitLinear_b158.forward:
 *       F.linear on the quantised operands, then the scale restore).
 *
 * acc[t,n] = sum_k xq[t,k] * W_q[n,k]   (exact int32)
 * d_t      = gamma / s_t                (fp32 division, once per token)
 * y32      = fp32(acc) * d_t            (one fp32 multiply)
 * y[t,n]   = bf16(y32), round to nearest even.
 * No bias, no normalisation (the caller applies any norm).
 *
 * packed  [N,K/4] from bitnet_pack_weights.   gamma  device fp32 scalar.
 * x       [M,K] bf16 bits.   y  [M,N] bf16 bits, written.
 * y_f32   [M,N] fp32, written with y32 when non-NULL (debug / parity).
 * acc     [M,N] int32, written with the exact accumulators when non-NULL.
 * workspace  >= bitnet_linear_workspace_size(M, N, K) bytes (0 bytes, and a
 *         NULL workspace, are accepted when that size is 0).
 * Requires M >= 1, N >= 1, K >= 4, K % 4 == 0, K <= 524288.  With
 * K % 64 == 0: M <= 8 runs a fused decode kernel (activation quantisation in
 * its prologue, no workspace); 9 <= M <= 32, on layers whose packed weights
 * spread over the SMs fit in shared memory (K <= 65536), runs an absmax pass
 * over x and the batched decode kernel (int8 mma.sync on weights held in
 * shared memory, split K through an int32 scratch in the workspace that the
 * kernel leaves zero); other M run the activation quantiser and the
 * tensor-core kernel.
 */
BITNET_API size_t bitnet_linear_workspace_size(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_linear(const uint8_t* packed, const float* gamma, int64_t N, int64_t K,
                            const uint16_t* x, int64_t M, uint16_t* y, float* y_f32,
                            int32_t* acc, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * Optional intermediate outputs of bitnet_ffn, for parity checking.  Every
 * member may be NULL.  Shapes: xq1 [M,H], acc_gate/acc_up [M,I], h [M,I]
 * (the folded h' below), xq2 [M,I], acc_down [M,H], y_f32 [M,H].
 */
typedef struct {
  int8_t* xq1;
  int32_t* acc_gate;
  int32_t* acc_up;
  float* h;
  int8_t* xq2;
  int32_t* acc_down;
  float* y_f32;
} bitnet_ffn_debug;

/*
 * Fused BitNet FFN block:
 *   RMSNorm(n1) -> act quant -> gate, up BitLinear -> ReLU(gate)^2 * up
 *   -> RMSNorm(n2) -> act quant -> down BitLinear.   No residual.
 *   [A] sections "モデル構造" (LLaMA-like FFN with RMSNorm) and
 *       "正規化で分散を安定させる" (normalise before BitLinear, subln);
 *   [R] section "BitNetが実現したCPU上での高効率AI処理" (ReLU^2);
 *   [Y] section "Absmean量子化関数" (RMSNorm before the activation quantiser).
 *
 * Folded evaluation (absmax quantisation ignores a positive per-token scale):
 *   r1 = 1/sqrt(mean(x^2) + eps);  u = x * n1;  xq1 = quant(u), s1
 *   g' = fp32(acc_gate) * (gamma_gate / s1);  u' = fp32(acc_up) * (gamma_up / s1)
 *   h' = (relu(g') * relu(g')) * u';  v = h' * n2;  xq2 = quant(v), s2
 *   r2 = 1/sqrt(r1^6 * mean(h'^2) + eps)
 *   y32 = (fp32(acc_down) * (gamma_down / s2)) * (r1^3 * r2);  y = bf16(y32)
 * Every quantised code and integer accumulator is exact; the r factors are
 * reductions whose rounding order is unspecified (y32 within 1e-5 relative).
 *
 * x [M,H] bf16 bits.  gate, up: packed [I, H/4]; down: packed [H, I/4];
 * gamma_* device fp32 scalars.  norm1_w [H], norm2_w [I] fp32 gains, NULL
 * means all ones.  eps >= 0.  y [M,H] bf16 bits written.
 * workspace >= bitnet_ffn_workspace_size(M, H, I) bytes.
 * debug  NULL or a host struct of optional device outputs (see above).
 * Requires M >= 1, H % 64 == 0, I % 64 == 0, H, I >= 64.  With M <= 8 and
 * M_pad * max(H, I) <= 65536 (M_pad = M rounded up to 1, 2 or a multiple of
 * 4) the block runs as two decode-kernel launches (gate/up with the h'
 * epilogue, then down); larger M runs the activation quantiser and the
 * tensor-core kernel per step.
 */
BITNET_API size_t bitnet_ffn_workspace_size(int64_t M, int64_t H, int64_t I);
BITNET_API bitnet_status bitnet_ffn(const uint16_t* x, int64_t M, int64_t H, int64_t I,
                         const float* norm1_w, const uint8_t* gate, const float* gamma_gate,
                         const uint8_t* up, const float* gamma_up, const float* norm2_w,
                         const uint8_t* down, const float* gamma_down, float eps,
                         uint16_t* y, const bitnet_ffn_debug* debug, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * A chain of BitLinear layers, each fed the previous one's output:
 *   y[0] = BitLinear(packed[0], gamma[0])(x),
 *   y[l] = BitLinear(packed[l], gamma[l])(y[l-1])   for l = 1 .. L-1,
 * every layer computed exactly as bitnet_linear computes it (same codes,
 * accumulators and bf16 outputs).  [A] section "モデル構造": the model is a
 * decoder-only Transformer whose nn.Linear layers are all BitLinear, so a
 * decode step runs them one after the other; the pages define no call that
 * runs several layers, this one only schedules them.
 *
 * The layers are launched one after the other on `stream`, each with the
 * kernel bitnet_linear would use (decode kernels start loading their weights
 * while the layer before them finishes).  When every layer runs the batched
 * decode kernel (9..32 tokens), x gets one absmax pass and each layer then
 * hands the per-token absmax of its bf16 outputs to the next through the
 * workspace, so the chain is one launch per layer plus one.
 *
 * L        number of layers, >= 1.
 * packed, gamma, N, K, y   HOST arrays of L entries; packed[l], gamma[l] and
 *          y[l] are device pointers.  Layer l maps [M, K[l]] to [M, N[l]];
 *          K[l] == N[l-1] for l >= 1.  The arrays are read during the call
 *          only.
 * x        [M, K[0]] bf16 bits, device.   y[l]  [M, N[l]] bf16 bits, written.
 * A layer's output may not overlap its input (y[l] vs y[l-1], y[0] vs x):
 * BITNET_ERR_INVALID_ARG.  Ping-pong buffers (y[l] == y[l-2]) are fine.
 * workspace  >= bitnet_linear_chain_workspace_size(L, N, K, M) bytes, device
 *          (the largest layer's bitnet_linear scratch, reused by every
 *          layer; 0 bytes, and a NULL workspace, when no layer needs any).
 * Other requirements and errors as bitnet_linear, per layer; all layers are
 * validated before anything is enqueued.
 */
BITNET_API size_t bitnet_linear_chain_workspace_size(int64_t L, const int64_t* N,
                                                     const int64_t* K, int64_t M);
BITNET_API bitnet_status bitnet_linear_chain(int64_t L, const uint8_t* const* packed,
                                             const float* const* gamma, const int64_t* N,
                                             const int64_t* K, const uint16_t* x, int64_t M,
                                             uint16_t* const* y, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * Several BitLinear layers applied to ONE input:
 *   y[l] = BitLinear(packed[l], gamma[l])(x)   for l = 0 .. L-1,
 * each identical, bit for bit, to what bitnet_linear computes for that
 * matrix and x.  [A] section "モデル構造": the model keeps the LLaMA-style
 * block (RMSNorm, SwiGLU, RoPE) with every nn.Linear a BitLinear, so the
 * gate and up projections of the SwiGLU read the same input, and so do the
 * query, key and value projections of the attention ([Y] section
 * "BitAttentionとMGQA" passes one x as query, key and value).  The
 * activation quantisation (per-token absmax, [Y] "Absmean量子化関数") does
 * not depend on the matrix, so it is done once where bitnet_linear runs the
 * tensor-core GEMM (K % 64 == 0 and more than 32 tokens, or fewer tokens on
 * rows too long for the decode kernels): one quantiser launch writes the
 * codes, then one GEMM per matrix reads them.  On the decode paths and for
 * K % 64 != 0 the kernels quantise in their own prologues and the call is
 * one bitnet_linear per matrix, in order.
 *
 * L        number of matrices, >= 1.
 * packed, gamma, N, y   HOST arrays of L entries; packed[l], gamma[l] and
 *          y[l] are device pointers.  Matrix l is [N[l], K] (all share K).
 *          The arrays are read during the call only.
 * x        [M, K] bf16 bits, device.   y[l]  [M, N[l]] bf16 bits, written.
 * No output may overlap x or another output: BITNET_ERR_INVALID_ARG.
 * workspace  >= bitnet_linear_multi_workspace_size(L, N, K, M) bytes,
 *          device (0, and NULL allowed, when nothing is needed).
 * Other requirements and errors as bitnet_linear, per matrix; everything is
 * validated before anything is enqueued.
 */
BITNET_API size_t bitnet_linear_multi_workspace_size(int64_t L, const int64_t* N, int64_t K,
                                                     int64_t M);
BITNET_API bitnet_status bitnet_linear_multi(int64_t L, const uint8_t* const* packed,
                                             const float* const* gamma, const int64_t* N,
                                             int64_t K, const uint16_t* x, int64_t M,
                                             uint16_t* const* y, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * BitLinear without a caller workspace, for callers that cannot allocate
 * device memory: code that issues work while a CUDA stream is being
 * captured into a graph (a cudaMalloc there is not part of the capture),
 * services that reserve a fixed memory budget at start-up and allocate
 * nothing afterwards, and plug-ins running inside another framework whose
 * allocator they cannot reach.  The pages describe no such variant; it has no
 * counterpart there.
 *
 * Computes exactly what bitnet_linear computes (same kernels, same results,
 * no y_f32 / acc outputs).  The scratch that bitnet_linear takes from the
 * workspace argument comes instead from one fixed array of
 * BITNET_NOALLOC_SCRATCH_BYTES in device memory that the library defines;
 * every GPU that loads the library holds that array until the process exits.
 * The function itself calls no allocator (no cudaMalloc, cudaFree or
 * allocating library routine).
 *   - Shapes whose scratch would exceed the array (see
 *     bitnet_linear_workspace_size) return BITNET_ERR_WORKSPACE and enqueue
 *     nothing.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (once per device, with that device current); make
 *     that first call before capturing any stream.  With lazy module loading
 *     (the CUDA default) the first launch of each kernel can load its code
 *     as well, so before capturing make one call for every kind of shape
 *     the capture will use (1-3 tokens, 4-8, 9-32, more tokens, K % 64 != 0:
 *     they run different kernels).
 *   - All calls share the one array, which keeps the last call's contents;
 *     whatever must start at zero is cleared by the call itself.  Calls that
 *     may overlap on the GPU (other streams, other host threads) race on the
 *     array: the caller must order them, e.g. on one stream.
 */
#define BITNET_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
BITNET_API bitnet_status bitnet_linear_noalloc(const uint8_t* packed, const float* gamma, int64_t N,
                                               int64_t K, const uint16_t* x, int64_t M,
                                               uint16_t* y, void* stream);

/*
 * BitNet v1 W1A8: sign weights, one bit each.
 *   [Y] section "BitNet v1：BitLinearの誕生" > "1-Bit重みとSign関数"
 *       (W_b = +1 where W >= 0, -1 where W < 0; alpha = mean |W_ij|; the
 *       output is restored with alpha and the activation scale).
 *
 * bitnet_pack_weights_w1:
 * W       [N,K] fp32, device, read only.  Must be finite.
 * packed  [N,K/8] uint8, device, written: bit (k % 8) of byte n*K/8 + k/8 is
 *         1 where W[n,k] >= 0 (including -0.0) and 0 where W[n,k] < 0.
 * alpha   one fp32 on the device, written: the fp32 value nearest (ties to
 *         even) to the exact mean of |W| (the same value bitnet_pack_weights
 *         writes as gamma).
 * workspace  >= bitnet_pack_w1_workspace_size(N, K) bytes.
 * Requires K % 8 == 0, N >= 1, K >= 8, N*K < 2^39.  A non-finite weight sets
 * alpha to NaN and records BITNET_ERR_NONFINITE.
 *
 * bitnet_linear_w1:  the activations are quantised exactly as in
 * bitnet_linear (per token, s_t = 127 / max(max|x|, 1e-5)); then
 *   acc[t,n] = sum_k xq[t,k] * W_b[n,k]   (exact int32)
 *   y32      = fp32(acc) * (alpha / s_t);  y = bf16(y32), nearest even.
 * (The page's v1 listing takes the absmax over the whole tensor; the library
 * keeps its per-token quantiser, identical for one token.)
 * Arguments as bitnet_linear, with packed [N,K/8] and alpha.
 * workspace  >= bitnet_linear_w1_workspace_size(M, N, K) bytes.  With 1-3
 * tokens, K % 128 == 0 and a per-SM slice that fits in shared memory the
 * decode kernel reads the sign bits directly and the workspace is unused;
 * otherwise the +-1 matrix is written into the workspace as I2_S codes
 * (a +-1 matrix is a ternary one) and bitnet_linear's kernels run on it.
 * Requires K % 8 == 0, K <= 524288.
 */
BITNET_API size_t bitnet_pack_w1_workspace_size(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_pack_weights_w1(const float* W, int64_t N, int64_t K,
                                                uint8_t* packed, float* alpha, void* workspace,
                                                size_t workspace_bytes, void* stream);
BITNET_API size_t bitnet_linear_w1_workspace_size(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_linear_w1(const uint8_t* packed, const float* alpha, int64_t N,
                                          int64_t K, const uint16_t* x, int64_t M, uint16_t* y,
                                          float* y_f32, int32_t* acc, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * BitLinear for one token through pair lookup tables instead of dp4a: the
 * same result as bitnet_linear (same codes, accumulators and outputs).
 *   [Y] section "I2_Sカーネルの内部動作" (TL2: two ternary weights, 3 x 3 = 9
 *       combinations, index one table entry).
 * For every activation pair (x_q[2i], x_q[2i+1]) a 16-entry table of
 * x0 (c0 - 1) + x1 (c1 - 1) is built in shared memory, indexed by the packed
 * nibble c0 + 4 c1 of two I2_S codes; a packed byte costs two lookups.
 * x [1,K] bf16 bits; y [1,N]; y_f32, acc optional [1,N].  No workspace.
 * Requires K % 64 == 0 and a per-SM slice of weights plus 16 K bytes of
 * tables that fits in shared memory (else BITNET_ERR_UNSUPPORTED).  Kept as
 * a measured alternative to the dp4a inner loop.
 */
BITNET_API bitnet_status bitnet_linear_tl2(const uint8_t* packed, const float* gamma, int64_t N,
                                           int64_t K, const uint16_t* x, uint16_t* y,
                                           float* y_f32, int32_t* acc, void* stream);

/*
 * BitNet a4.8: 4-bit activations with the largest values at 8 bits, on the
 * ternary I2_S weights.
 *   [Y] section "BitNet a4.8：ハイブリッド量子化戦略" (the top fraction of the
 *       activation values is split off and processed at 8 bits, the rest is
 *       quantised to 4 bits).
 * The pages give neither the fraction nor the scales.  Per token, the n_out
 * values of largest |x| (ties between equal |x| go to the lower channel) are
 * the 8-bit part, the rest the 4-bit part, each with its own absmax scale:
 *   s4 = 7 / max(max|x_in|, 1e-5),    q4 = clamp(rint(x s4), -8, 7) on inliers, 0 else
 *   s8 = 127 / max(max|x_out|, 1e-5), q8 = clamp(rint(x s8), -128, 127) on outliers, 0 else
 *   acc4 = q4 . W_q, acc8 = q8 . W_q   (exact int32)
 *   y32 = fp32(acc4) (gamma / s4) + fp32(acc8) (gamma / s8)  (two fp32
 *         products, one fp32 sum);  y = bf16(y32), nearest even.
 * The page's second technique, per-channel scaling, comes with no formula and
 * is not applied.
 *
 * bitnet_quant_act_a48: x [M,K] bf16 bits; q4, q8 [M,K] int8 (natural
 * order) and s4, s8 [M] fp32, device, written.  Requires K % 8 == 0,
 * 0 <= n_out <= K.
 * bitnet_linear_a48: packed [N,K/4], gamma as bitnet_linear; y [M,N] bf16
 * bits; y_f32, acc4, acc8 optional [M,N]; workspace >=
 * bitnet_linear_a48_workspace_size(M, N, K) bytes.  Requires K % 64 == 0,
 * 0 <= n_out <= K.  One token whose weight slices fit shared memory: the
 * resident decode kernel alone, quantising the token into its two code rows
 * in every CTA and combining them in its epilogue; otherwise the a4.8
 * quantiser (one CTA per token), the tensor-core kernel on the 2M code rows
 * and a combine kernel.
 */
BITNET_API bitnet_status bitnet_quant_act_a48(const uint16_t* x, int64_t M, int64_t K,
                                              int64_t n_out, int8_t* q4, float* s4, int8_t* q8,
                                              float* s8, void* stream);
BITNET_API size_t bitnet_linear_a48_workspace_size(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_linear_a48(const uint8_t* packed, const float* gamma, int64_t N,
                                           int64_t K, const uint16_t* x, int64_t M,
                                           int64_t n_out, uint16_t* y, float* y_f32,
                                           int32_t* acc4, int32_t* acc8, void* workspace,
                                           size_t workspace_bytes, void* stream);

/*
 * The FFN block split over G devices (tensor parallel), for models too large
 * for one GPU: [D] (100B-class models), [A] section
 * "推論コストはどれだけ下がったのか" (70B-class serving).  Gate and up are split
 * by rows (shard r holds intermediate features [I_r0, I_r1), Ir of them),
 * down by columns (the same features), norm2_w likewise; every shard holds
 * the whole token x and the whole-matrix gammas (pack the whole matrix, then
 * slice the packed rows / byte columns).  Per block:
 *   1. bitnet_ffn_tp_gate_up on every shard: h' [M,Ir] (fp32), the shard's
 *      absmax of h' * n2 (amax2 [M]) and sum of h'^2 (sumsq_h [M], fp64),
 *      and the token's sum of x^2 (sumsq_x [M], fp64; equal on every shard);
 *   2. all-reduce amax2 with MAX and sumsq_h with SUM over the shards;
 *   3. bitnet_ffn_tp_down on every shard: h' * n2 quantised with the
 *      all-reduced absmax (the codes the whole-block quantiser gives these
 *      features), times the shard's down columns: partial integer
 *      accumulators acc [M,H] (int32);
 *   4. all-reduce acc with SUM (exact integers: sharding changes no code or
 *      accumulator);
 *   5. bitnet_ffn_tp_finish: y = bf16((fp32(acc) * (gamma_d / s2)) *
 *      fp32(r1^3 r2)) with r1, r2 from sumsq_x and the all-reduced sumsq_h,
 *      I the whole intermediate width, as bitnet_ffn computes it.
 * Codes and accumulators equal the single-device block's bit for bit; y32
 * differs only through the rounding order of the all-reduced fp64 sum
 * (within 1e-5 relative).  The collectives are the caller's (the Python
 * module tensor_parallel runs them with torch.distributed).
 * Shapes: H % 64 == 0, Ir % 64 == 0; workspace >=
 * bitnet_ffn_tp_workspace_size(M, H, Ir) for steps 1 and 3.
 */
BITNET_API size_t bitnet_ffn_tp_workspace_size(int64_t M, int64_t H, int64_t Ir);
BITNET_API bitnet_status bitnet_ffn_tp_gate_up(const uint16_t* x, int64_t M, int64_t H, int64_t Ir,
                                               const float* norm1_w, const uint8_t* gate,
                                               const float* gamma_gate, const uint8_t* up,
                                               const float* gamma_up, const float* norm2_w,
                                               float* h, float* amax2, double* sumsq_h,
                                               double* sumsq_x, void* workspace,
                                               size_t workspace_bytes, void* stream);
BITNET_API bitnet_status bitnet_ffn_tp_down(const float* h, int64_t M, int64_t H, int64_t Ir,
                                            const float* norm2_w, const uint8_t* down,
                                            const float* amax2, int32_t* acc, void* workspace,
                                            size_t workspace_bytes, void* stream);
BITNET_API bitnet_status bitnet_ffn_tp_finish(const int32_t* acc, int64_t M, int64_t H, int64_t I,
                                              const float* gamma_down, const float* amax2,
                                              const double* sumsq_x, const double* sumsq_h,
                                              float eps, uint16_t* y, float* y_f32, void* stream);

/*
 * Synchronise `stream`, then return and clear the device status word of the
 * current device: BITNET_OK, BITNET_ERR_TIMEOUT (a bounded wait expired; the
 * affected outputs are unspecified) or BITNET_ERR_NONFINITE.  A failing
 * synchronisation returns BITNET_ERR_CUDA.
 */
BITNET_API bitnet_status bitnet_last_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H_ */
