/*
 * wq.h - C ABI of libwq: round-to-nearest group-wise affine INT4 weight quantization
 * and the W4A16 dequant-matmul, for NVIDIA B200 (sm_100a).
 *
 * Definitions followed (page title, section):
 *   "Model Quantization", 1 "Mathematical Mechanics of Quantization": affine
 *      W_q = round(W/S) + Z, W_dequant = S (W_q - Z); one S and Z per group of g = 128.
 *   "DL S067 - Quantization", 1 "The core math": asymmetric
 *      S = (beta - alpha)/(q_max - q_min), Z = round(q_min - alpha/S),
 *      q = clip(round(W/S) + Z, q_min, q_max); symmetric S = max|W|/q_max.
 *   "DL S067 - Quantization", 2 "Per-tensor vs per-channel vs per-group": a group is g
 *      consecutive weights along the input dimension of W [out_features, in_features].
 *   "LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
 *      "The vocabulary": W4A16 = 4-bit weights dequantized to 16 bits inside the kernel,
 *      16-bit matmul (here: bf16 operands, fp32 accumulation), Y = X W^T.
 *
 * Numerics fixed by this library (the pages leave them open):
 *   - alpha = min(0, min w), beta = max(0, max w) over the group (zero is exact);
 *   - S' = binary16 round-half-even of the EXACT (beta - alpha)/15; S' = 0 -> 1.0;
 *   - Z = clip(round-half-even(-alpha/S'), 0, 15) on the exact quotient, stored binary16;
 *   - q = clip(round-half-even(w/S') + Z, 0, 15) on the exact quotient;
 *   - INT4 symmetric per group ("DL S067 - Quantization", section 2, quantize_per_group):
 *     s' = binary16(max|w|/7) (0 -> 1), q = clip(RNE(w/s'), -8, 7), stored in the INT4
 *     layout below as code q + 8 with Z = 8, so dequant and matmul treat both alike;
 *   - INT8 symmetric: s' = binary16(max|w|/127), q = clip(RNE(w/s'), -127, 127).
 *
 * Data layout (row-major, all device memory owned by the caller):
 *   W      [N, K] fp32 or bf16, leading dimension ldw elements (N = out, K = in)
 *   packed [N, K/2] uint8: byte j of row n = q[n][2j] | q[n][2j+1] << 4
 *   S, Z   [N, K/g] binary16 bit patterns (uint16), contiguous
 *   X      [M, K] bf16, leading dimension ldx; Y [M, N] bf16, leading dimension ldy
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless stated, in
 *     memory of the CURRENT device (cudaSetDevice) or managed memory; any other pointer
 *     (host memory, pinned or not, or another device's memory) is rejected with
 *     WQ_ERR_DEVICE before anything is launched. The library allocates no device memory;
 *     a small device status word and the kernels' code are module globals.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream) on the current device.
 *   - Argument errors are returned synchronously and launch nothing. A failed launch
 *     returns WQ_ERR_CUDA. Data-dependent errors (non-finite weights, scale overflow,
 *     codes > 15, a bounded wait that timed out) are recorded in the device status word
 *     and returned by wq_get_status(); outputs of such a call are unspecified.
 *   - Thread-safe for distinct streams; calls on one stream are ordered.
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WQ_VERSION 100 /* 0.1.0 */

typedef enum wq_status {
  WQ_OK = 0,
  WQ_ERR_NULL = 1,        /* a required pointer is NULL                          */
  WQ_ERR_SHAPE = 2,       /* sizes <= 0, K % g != 0, ld too small, alpha outside  */
                          /* [0, 1], ...                                          */
  WQ_ERR_ALIGN = 3,       /* a pointer or leading dimension breaks 16-B alignment */
  WQ_ERR_DTYPE = 4,       /* dtype not supported by this call                    */
  WQ_ERR_UNSUPPORTED = 5, /* parameter combination not implemented               */
  WQ_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed                */
  WQ_ERR_NONFINITE = 7,   /* device: NaN/inf weight or binary16 scale overflow   */
  WQ_ERR_TIMEOUT = 8,     /* device: a bounded barrier wait gave up              */
  WQ_ERR_RANGE = 9,       /* device: a code given to wq_pack_int4 exceeds 15, or */
                          /* a factor s_j given to wq_quantize_rtn_scaled is not */
                          /* finite and > 0                                       */
  WQ_ERR_NODEVICE = 10,   /* no CUDA device, or it is not sm_100                 */
  WQ_ERR_DEVICE = 11      /* a pointer is not memory of the current device      */
} wq_status;

typedef enum wq_dtype { WQ_F32 = 0, WQ_BF16 = 1, WQ_F16 = 2, WQ_U8 = 3, WQ_I8 = 4 } wq_dtype;

/* Quantization parameters, named after the usual config keys (w_bit, q_group_size,
 * zero_point). Supported: {4, g, 1} (asymmetric) and {4, g, 0} (symmetric, stored with
 * Z = 8) with g a multiple of 32 that divides K (g = K is per output channel), and
 * {8, K, 0} (INT8 symmetric per channel). */
typedef struct wq_qparams {
  int32_t w_bit;      /* 4 or 8                                      */
  int32_t group;      /* g: weights per scale along K                 */
  int32_t zero_point; /* 1 = asymmetric [0, 15]; 0 = symmetric        */
                      /*   (INT4: [-8, 7], stored as q + 8 with Z = 8) */
} wq_qparams;

/* Library version (WQ_VERSION) and a static description of a status code. */
int32_t wq_version(void);
const char* wq_status_string(wq_status status);

/* Round-to-nearest quantization of W [N, K] ("DL S067 - Quantization", sections 1-2).
 *   W       fp32 or bf16 (w_dtype), row stride ldw >= K elements; base and row stride
 *           16-byte aligned.
 *   params  NULL means {4, 128, 1}.
 *   INT4 ({4, g, 1} or {4, g, 0}): packed [N, K/2] uint8, S and Z [N, K/g] binary16
 *           (symmetric: every Z is 8.0 and codes lie in [0, 15] as q + 8).
 *   INT8 ({8, K, 0}): packed receives int8 codes [N, K]; S [N] binary16; Z must be NULL.
 * Non-finite weights or a scale above the binary16 range set WQ_ERR_NONFINITE in the
 * device status word. Requires K % 32 == 0. */
wq_status wq_quantize_rtn_g128(const void* W, wq_dtype w_dtype, int64_t N, int64_t K,
                               int64_t ldw, const wq_qparams* params, uint8_t* packed,
                               uint16_t* S, uint16_t* Z, void* stream);

/* Per-tensor asymmetric INT4 (one S, Z for all of W; same page, section 2). Two passes:
 * a min/max reduction into the caller's `workspace` (device memory of at least
 * wq_quantize_per_tensor_workspace_bytes(N, K) bytes, 16-byte aligned, no initial
 * contents required), then the codes. S and Z each receive one binary16 value. */
size_t wq_quantize_per_tensor_workspace_bytes(int64_t N, int64_t K);
wq_status wq_quantize_rtn_per_tensor(const void* W, wq_dtype w_dtype, int64_t N,
                                     int64_t K, int64_t ldw, uint8_t* packed, uint16_t* S,
                                     uint16_t* Z, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Per-tensor asymmetric INT4 like wq_quantize_rtn_per_tensor, for callers that cannot
 * allocate device memory (no workspace argument; nothing is allocated). The pages have no
 * counterpart: this is a deployment variant. The grid-wide min/max goes to a fixed 32 KB
 * array inside the library (4096 (min, max) slots; 8 are used per SM, so a device with
 * more than 512 SMs gets WQ_ERR_UNSUPPORTED). The array exists once per device for as
 * long as the library is loaded, and all calls on a device share it, so calls that
 * overlap on the GPU race with one another. The first call on each device looks up the
 * array's device address; make it before any stream capture. Outputs as for
 * wq_quantize_rtn_per_tensor. */
wq_status wq_quantize_rtn_per_tensor_noalloc(const void* W, wq_dtype w_dtype, int64_t N,
                                             int64_t K, int64_t ldw, uint8_t* packed,
                                             uint16_t* S, uint16_t* Z, void* stream);

/* Pack 4-bit codes two per byte (the storage of "INT4 weights + FP16 scales/zero-points",
 * "Model Quantization", section 4): codes [N, K] uint8 in [0, 15] -> packed [N, K/2].
 * A code above 15 sets WQ_ERR_RANGE in the status word. Requires K % 32 == 0. */
wq_status wq_pack_int4(const uint8_t* codes, int64_t N, int64_t K, uint8_t* packed,
                       void* stream);

/* Dequantize W_hat = S' (q - Z) ("Model Quantization", section 1) into out [N, K]:
 * WQ_F32 is exact; WQ_BF16 is its round-half-even to bfloat16. group = g as above, or
 * 0 for per-tensor (S, Z hold one value). Requires K % 32 == 0. */
wq_status wq_dequant(const uint8_t* packed, const uint16_t* S, const uint16_t* Z,
                     int64_t N, int64_t K, int32_t group, void* out, wq_dtype out_dtype,
                     void* stream);

/* W4A16 matmul Y = X W_hat^T ("LLM Weight Quantization ...", "The vocabulary"):
 *   X [M, K] bf16 (ldx), packed/S/Z as produced above with group g (0 = per-tensor),
 *   Y [M, N] bf16 (ldy), fp32 accumulation.
 * Kernel choice by M:
 *   - 9 <= M <= 64 with g = 128 (K % 128 == 0), and 3 <= M <= 8 where the decode kernels
 *     below would pass over the weights more than once (rows too long for blocks of M
 *     tokens): the skinny tensor-core kernel, one pass
 *     over the weights for all tokens. tcgen05 kind::f16 multiplies the centred codes
 *     q - Z (exact in bf16) with the activations as stored, every product exact in fp32 and
 *     summed in fp32 per group of 128 k, and S' is applied per group in fp32, so the
 *     product is with the exact S'(q - Z). K is split over a thread-block cluster whose
 *     partial rows are summed in a fixed order (deterministic).
 *   - otherwise M <= 32: decode kernels, for M > 8 in passes over blocks of at most 8 tokens
 *     (when some block size needs at most 8 passes; else the tensor-core GEMM). The packed rows
 *     stream through shared memory (bulk copies or TMA boxes) or registers, codes are
 *     decoded in registers (into warp-level bf16 MMAs for g = 128 and N % 16 == 0, else
 *     packed fp32 FMAs), and S' and Z are applied per group in fp32: the product is with
 *     the exact S'(q - Z). The result is deterministic (fixed reduction order). M = 1 with
 *     K > 32768 stays on a decode kernel only where a streaming one takes the shape (g = 128,
 *     K % 128 == 0, N % 32 == 0 or N % 16 == 0, 16-byte aligned X, S, Z, and X plus one
 *     tile's S' and Z within shared memory); otherwise it runs on the tensor-core GEMM.
 *   - larger M: the tcgen05/TMEM tensor-core GEMM, which dequantizes each weight tile to
 *     bf16 in tensor memory (so W_hat is rounded to bfloat16 there, then multiplied
 *     exactly with fp32 accumulation).
 * Requirements: K % 32 == 0; g a multiple of 32 dividing K, or 0; X 16-byte aligned and
 * ldx % 8 == 0; packed 16-byte aligned; S, Z, Y 2-byte aligned. On the tensor-core path
 * also K % 64 == 0 (else WQ_ERR_SHAPE), Y 16-byte aligned and ldy % 8 == 0 (else
 * WQ_ERR_ALIGN). A launch may start before the previous kernel on the stream ends
 * (programmatic dependent launch); it reads its inputs only after that kernel completes
 * (before that it may only issue L2 prefetch hints for the weights, which cannot return
 * stale data). */
wq_status wq_w4a16_gemm(const uint16_t* X, int64_t M, int64_t ldx, const uint8_t* packed,
                        const uint16_t* S, const uint16_t* Z, int64_t N, int64_t K,
                        int32_t group, uint16_t* Y, int64_t ldy, void* stream);

/* W8A16 matmul with INT8 symmetric per-channel weights: codes int8 [N, K], S [N]
 * binary16; Y = X (s' q)^T, fp32 accumulation, bf16 out. 3 <= M <= 64 with K % 128 == 0
 * runs on the skinny tensor-core kernel (tcgen05 kind::i8 on the s8 codes as stored and
 * each token's activations of a group as exact integers x 2^s below 2^22 in three signed
 * bytes, s from the group's largest exponent: exact within 2^14 of the group's largest |x|,
 * else off by at most 2^-23 of it; s' applied to the finished row), one pass over the
 * weights; M <= 2 (and other M <= 8) on CUDA cores with the exact s' q; larger
 * M on the tensor-core GEMM (s' q rounded to bf16). Same requirements as wq_w4a16_gemm. */
wq_status wq_w8a16_gemm(const uint16_t* X, int64_t M, int64_t ldx, const int8_t* codes,
                        const uint16_t* S, int64_t N, int64_t K, uint16_t* Y, int64_t ldy,
                        void* stream);

/* ---- Per-input-channel scale folding ("LLM Weight Quantization ...", sections
 * "Granularity and outliers" (SmoothQuant) and "GPTQ vs AWQ: two ways to choose what error
 * to keep" (AWQ); "DL S067 - Quantization", section 5 "AWQ intuition"). A factor s_j > 0
 * per input channel j multiplies weight column j before round-to-nearest and divides
 * activation column j, so that (X / s)(W diag(s))^T = X W^T. At serve time the folded
 * codes run on wq_w4a16_gemm unchanged, with activations X / s: either produced by the
 * previous layer (1/s folded into its weights, as the AWQ section suggests) or by
 * wq_scale_activations below. s is float32 [K], device memory. */

/* Per-column statistic of A [rows, cols] (fp32 or bf16, row stride lda elements):
 *   WQ_STAT_ABSMAX   out[j] = max_i |A_ij| (exact; a NaN propagates);
 *   WQ_STAT_ABSMEAN  out[j] = mean_i |A_ij|: float64 sums, the quotient by rows rounded once
 *                    to float32 (exact whenever the column's sum fits 53 bits).
 * The factor formulas below take these: max |X_j| over calibration tokens and max |W_j|
 * over output rows (SmoothQuant), mean |X_j| (AWQ). The result is deterministic.
 * Requires rows >= 1 (else WQ_ERR_SHAPE; cols == 0 is a no-op), cols % 8 == 0, lda >= cols,
 * A and lda * element size 16-byte aligned, out [cols] float32. */
typedef enum wq_stat { WQ_STAT_ABSMAX = 0, WQ_STAT_ABSMEAN = 1 } wq_stat;
wq_status wq_channel_stat(const void* A, wq_dtype dtype, int64_t rows, int64_t cols,
                          int64_t lda, int32_t stat, float* out, void* stream);

/* SmoothQuant factors s_j = xmax_j^alpha / wmax_j^(1 - alpha) ("Granularity and outliers";
 * alpha = 0.5 there), computed in float64 and rounded to float32; s_j = 1 where xmax_j or
 * wmax_j is not > 0. xmax, wmax, s: float32 [K]. alpha in [0, 1], else WQ_ERR_SHAPE. */
wq_status wq_smooth_scales(const float* xmax, const float* wmax, int64_t K, float alpha,
                           float* s, void* stream);

/* AWQ factors for one exponent alpha ("GPTQ vs AWQ ..."): p_j = a_j^alpha over the channels
 * with a_j > 0 (a = mean |X_j| on calibration data), s_j = p_j / sqrt(max p * min p) so that
 * the factors are centred on 1; s_j = 1 where a_j is not > 0. float64 arithmetic, float32
 * result. alpha in [0, 1], else WQ_ERR_SHAPE. One CTA (K is one layer's input width). */
wq_status wq_awq_scales(const float* a_mag, int64_t K, float alpha, float* s, void* stream);

/* Round-to-nearest INT4 of the folded weights W diag(s): w'_nk = w_nk * s_k rounded once to
 * float32, then exactly the steps and outputs of wq_quantize_rtn_g128 for {4, g, 1} or
 * {4, g, 0} (params NULL = {4, 128, 1}; g a multiple of 32 dividing K). A factor that is not
 * finite and > 0 sets WQ_ERR_RANGE in the status word (its column is folded as 0); a folded
 * weight that is not finite, or a scale overflow, WQ_ERR_NONFINITE. W as for wq_quantize_rtn_g128; s float32 [K],
 * 16-byte aligned. The dequantized codes approximate W diag(s): multiply by the activations
 * X / s (or divide the dequantized column by s_k) to approximate W. */
wq_status wq_quantize_rtn_scaled(const void* W, wq_dtype w_dtype, int64_t N, int64_t K,
                                 int64_t ldw, const float* s, const wq_qparams* params,
                                 uint8_t* packed, uint16_t* S, uint16_t* Z, void* stream);

/* Xs = X / s per column: each bf16 x_mk divided by s_k in float32 (round-to-nearest), the
 * quotient rounded to bfloat16 (ties to even). X, Xs [M, K] bf16 with row strides ldx, ldxs
 * (multiples of 8, 16-byte aligned bases); s float32 [K], 16-byte aligned; K % 8 == 0.
 * Xs may be X itself (in place) when ldxs == ldx; other overlaps are undefined. No check of
 * s: a zero or non-finite factor gives the IEEE quotient. */
wq_status wq_scale_activations(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                               const float* s, uint16_t* Xs, int64_t ldxs, void* stream);

/* GPTQ ("LLM Weight Quantization ...", "GPTQ vs AWQ: two ways to choose what error to keep";
 * "DL S067 - Quantization", section 4): quantize W [N, K] one input column at a time, moving
 * each column's rounding error onto the columns not yet quantized through the inverse of the
 * dampened Hessian H = X^T X + damp * mean(diag H) * I of the calibration activations
 * X [T, K] (bf16, row stride ldx), and dropping the finished column from the inverse
 * (Optimal Brain Surgeon update). The grid is fixed before the sweep: S' and Z of every
 * group are those of wq_quantize_rtn_g128 on the original W ({4, g, 1} or {4, g, 0};
 * params NULL = {4, 128, 1}); only the codes differ. The output format is the same, for the
 * unchanged matmul kernels. The Hessian, its inverse (Gauss-Jordan, no pivoting) and the
 * sweep run in float64; one CTA sweeps one row. Requirements: K % 64 == 0, K <= 8192,
 * T >= 1, 0 <= damp (the page's toy uses 0.01); W as for wq_quantize_rtn_g128; X 2-byte
 * aligned; workspace of at least wq_gptq_workspace_bytes(N, K) bytes (8 K^2 + 32 K),
 * 16-byte aligned, no initial contents. A Hessian that is not positive definite (for
 * example damp = 0 with fewer calibration rows than K) or a non-finite weight sets
 * WQ_ERR_NONFINITE in the status word. Offline: 2K launches of O(K^2) each plus the sweep
 * (measured 17 ms for 1024 x 1024 with 256 calibration rows, 0.56 s for 4096 x 4096 with
 * 512). */
size_t wq_gptq_workspace_bytes(int64_t N, int64_t K);
wq_status wq_quantize_gptq(const void* W, wq_dtype w_dtype, int64_t N, int64_t K, int64_t ldw,
                           const uint16_t* X, int64_t T, int64_t ldx, double damp,
                           const wq_qparams* params, uint8_t* packed, uint16_t* S, uint16_t* Z,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Synchronize `stream`, then return and clear the current device's status word:
 * WQ_OK, or the first of WQ_ERR_NONFINITE / WQ_ERR_RANGE / WQ_ERR_TIMEOUT recorded by a
 * kernel since the last call; WQ_ERR_CUDA if the synchronization itself failed. */
wq_status wq_get_status(void* stream);

/* Self-test of failure detection: launches one CTA whose single mbarrier wait (on a barrier
 * nothing arrives at) is bounded by limit_ns nanoseconds, with the same bounded wait the
 * pipelined kernels use (spin != 0: the spinning form, else the suspending one). The wait
 * gives up, records WQ_ERR_TIMEOUT in the device status word and the kernel returns; the
 * next wq_get_status() reports it and clears it, and the context stays usable. No fault, trap
 * or unbounded wait is involved. limit_ns in [1e3, 1e9], else WQ_ERR_SHAPE. */
wq_status wq_selftest_bounded_wait(uint64_t limit_ns, int32_t spin, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
