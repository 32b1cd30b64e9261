/*
 * w8a8.h -- C ABI of the B200 (sm_100a) W8A8 quantized linear layer.
 *
 * The layer is the one described by the PDMIX glossary entry ("PDMIX
 * 阶段间混合量化算法 量化术语百科词条") and the PDMIX Parameter Configuration
 * Workflow Guide: INT8 activations quantized per token (dynamic, symmetric)
 * during Prefill and per tensor (static, asymmetric, calibrated offline)
 * during Decode, against ONE per-output-channel symmetric INT8 weight shared
 * by both phases; plus, as a second mode, the vector-wise quantization with
 * mixed-precision outlier decomposition of the LLM.int8() paper summary
 * (blog.rainlin.top/posts/llm-int8).
 *
 * Notation: X is the activation [M, K] (tokens x in-features), W the weight
 * [K, N] as on the pages (out = X W). The library keeps the quantized weight
 * as Wq [N, K] int8 with K contiguous ("K-major"), so both GEMM operands are
 * read along K.
 *
 * Conventions shared by every call:
 *   - Pointers named as device memory must be device pointers to memory the
 *     caller allocated and owns; the library allocates nothing.
 *   - Each compute call is asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and returns a w8a8_status. Arguments are
 *     checked on the host before any launch; a call that returns an error
 *     launched nothing (except W8A8_ERR_CUDA, which reports the launch error).
 *   - bf16 tensors are passed as `const void*` holding __nv_bfloat16 values.
 *   - Matrix base pointers must be 16-byte aligned; leading dimensions are in
 *     elements and must keep every row 16-byte aligned.
 *   - K must be a positive multiple of 16 and at most 65536 (so every
 *     corrected int32 accumulator is exact); M and N are arbitrary >= 0
 *     (M == 0 or N == 0 returns W8A8_OK without launching).
 *   - Nothing prints; nothing throws across the ABI. The only state the
 *     library keeps is a per-device cache of device properties and one
 *     per-device 32-bit device status word (see w8a8_check_device_error).
 *   - Calls on the same stream are ordered; calls on different streams that
 *     share output buffers are the caller's race.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t w8a8_status;
#define W8A8_OK 0
#define W8A8_ERR_INVALID_ARG 1        /* null pointer, negative size, bad enum */
#define W8A8_ERR_MISALIGNED 2         /* pointer or leading dimension breaks 16-byte rows */
#define W8A8_ERR_UNSUPPORTED_SHAPE 3  /* e.g. K not a multiple of 16, K > 65536 */
#define W8A8_ERR_UNSUPPORTED_DTYPE 4  /* dtype not accepted by this call */
#define W8A8_ERR_CUDA 5               /* a CUDA runtime/driver call or launch failed */
#define W8A8_ERR_DEVICE_TIMEOUT 6     /* a bounded device-side wait ran out (device status) */
#define W8A8_ERR_OUTLIER_OVERFLOW 7   /* more outlier columns than `cap` (device status) */
#define W8A8_ERR_NOT_IMPLEMENTED 8
#define W8A8_ERR_WORKSPACE 9          /* workspace missing or smaller than the query says */
#define W8A8_ERR_NO_DEVICE 10         /* no usable sm_100 device is current */

typedef int32_t w8a8_dtype;
#define W8A8_BF16 0
#define W8A8_FP32 1
#define W8A8_I32 2  /* GEMM output only: the corrected integer accumulator acc - Z*colsum[n] */

/* Human-readable name of a status code (static string; never NULL). */
const char *w8a8_status_string(w8a8_status status);

/*
 * Weight quantization, once at load time.
 * Source: PDMIX configuration guide, Step 2 YAML and Step 3 row qconfig.weight.*
 * (int8, per_channel, symmetric, minmax); PDMIX glossary §2.1 and §2.4 (one
 * quantized weight shared by Prefill and Decode); LLM.int8() summary step (1)
 * (C_w is the absmax of each column of W) and step (2) (W * 127 / C_w); its
 * limitations paragraph (INT8 weights are re-quantized from 16-bit at load).
 *
 * For every output channel n: a = max_k |W[k, n]|, s_w[n] = a / 127,
 * Wq[n, k] = clamp(rne(W[k, n] * (127 / a)), -127, 127) (0, with s_w[n] = 0, when a == 0 or
 * when 127 / a overflows fp32, a below 127/FLT_MAX ~ 3.7e-37), and
 * colsum[n] = sum_k Wq[n, k] (used by the zero-point correction).
 *   W       device, [K, N] row-major, row stride ldw elements; bf16 or fp32 (w_dtype)
 *   Wq      device, [N, K] int8, dense (row stride K), written
 *   s_w     device, [N] fp32, written
 *   colsum  device, [N] int32, written
 * Errors: INVALID_ARG (null, ldw < N), MISALIGNED (W not aligned to its
 * element size, or Wq not 8-byte aligned), UNSUPPORTED_SHAPE (K), UNSUPPORTED_DTYPE.
 */
w8a8_status w8a8_quant_weight_per_channel(const void *W, w8a8_dtype w_dtype, int64_t K, int64_t N,
                                          int64_t ldw, int8_t *Wq, float *s_w, int32_t *colsum,
                                          void *stream);

/*
 * Offline MinMax calibration of the Decode per-tensor static parameters.
 * Source: PDMIX glossary §2.3 eq. Q_decode (S_tensor and Z_tensor computed
 * offline; [Qmin, Qmax] = [-128, 127]); PDMIX configuration guide §3 and
 * Step 3 rows qconfig.act.symmetric / qconfig.act.method (asymmetric, exported
 * zero point, MinMax observer).
 * Reading of the pages: the observed range is widened to contain 0,
 * lo = min(0, min X), hi = max(0, max X); then S = (hi - lo) / 255,
 * r = 255 / (hi - lo), Z = clamp(-128 - rne(lo * r), -128, 127); an all-zero
 * input, or a range so small that 255 / (hi - lo) overflows fp32, gives
 * S = r = 1, Z = 0, so r is always finite.
 *   Xcal  device, [T, K] row-major, row stride ldx; bf16 or fp32 (x_dtype)
 *   S, r  device, one fp32 each, written;  Z  device, one int32, written
 * K here is any positive count (no multiple-of-16 rule). T*K must be > 0.
 */
w8a8_status w8a8_calibrate_static(const void *Xcal, w8a8_dtype x_dtype, int64_t T, int64_t K,
                                  int64_t ldx, float *S, float *r, int32_t *Z, void *stream);

/*
 * Prefill activation quantization: per token (row), dynamic, symmetric.
 * Source: PDMIX glossary §2.3 eq. Q_prefill (S_token computed online per
 * token); PDMIX configuration guide §3 (Prefill uses per-token symmetric
 * quantization, so Z_token = 0); LLM.int8() summary §一.1 absmax equation.
 * For each row m: a = max_k |X[m, k]|, S_x[m] = a / 127,
 * Xq[m, k] = clamp(rne(X[m, k] * (127 / a)), -127, 127); a row with a == 0, or
 * with a so small that 127 / a overflows fp32 (a below 127/FLT_MAX ~ 3.7e-37),
 * is quantized as zero: S_x[m] = 0 and all codes 0.
 *   X    device bf16 [M, K], row stride ldx (>= K, multiple of 8)
 *   Xq   device int8 [M, K], dense, written
 *   S_x  device fp32 [M], written
 */
w8a8_status w8a8_quant_per_token(const void *X, int64_t M, int64_t K, int64_t ldx, int8_t *Xq,
                                 float *S_x, void *stream);

/*
 * Decode activation quantization with static per-tensor parameters.
 * Source: PDMIX glossary §2.3 eq. Q_decode; the saturation it implies for
 * out-of-range tokens is the risk named in §2.4.
 * Xq[m, k] = clamp(rne(X[m, k] * r) + Z, -128, 127), r and Z from
 * w8a8_calibrate_static (device scalars, read by the kernel). Z is an int8
 * zero point, in [-128, 127] as w8a8_calibrate_static writes it; the result
 * for a Z outside that range is unspecified (the kernel cannot check a
 * device scalar without a synchronisation). r is finite (w8a8_calibrate_static
 * never writes an infinite one); for an infinite r the codes are unspecified.
 *   X   device bf16 [M, K], row stride ldx;  Xq device int8 [M, K] dense, written
 */
w8a8_status w8a8_quant_per_tensor(const void *X, int64_t M, int64_t K, int64_t ldx, const float *r,
                                  const int32_t *Z, int8_t *Xq, void *stream);

/*
 * Static per-tensor dequantization, the inverse of w8a8_quant_per_tensor:
 *   out[m, k] = S * (float)(Xq[m, k] - Z)     (one fp32 product; q - Z is exact)
 * rounded to bf16 (RNE) for W8A8_BF16, or stored as fp32 for W8A8_FP32.
 * This is the read side of an INT8 KV cache kept in the Decode scheme: K and
 * V quantized once with w8a8_calibrate_static's S, r, Z and
 * w8a8_quant_per_tensor, and expanded by this call where attention needs
 * them (attention itself is not part of this library).
 * Source: PDMIX glossary §2.3 (q = round(x / S) + Z, so x ~ S (q - Z)) and
 * §3 (KVCache Quant, the companion of PDMIX); PDMIX configuration guide (the
 * W8A8C8 combination). No page fixes a separate scheme for the cache, so the
 * Decode scheme is taken.
 *   Xq   device int8 [M, K], row stride ldq bytes (a multiple of 16)
 *   S, Z device scalars (fp32, int32), as from w8a8_calibrate_static
 *        (Z in [-128, 127]; outside it the result is unspecified)
 *   out  device [M, K] dense, 16-byte aligned, written
 */
w8a8_status w8a8_dequant_per_tensor(const int8_t *Xq, int64_t M, int64_t K, int64_t ldq, const float *S,
                                    const int32_t *Z, void *out, w8a8_dtype out_dtype, void *stream);

/*
 * INT8 x INT8 -> INT32 GEMM with the dequant epilogue fused in.
 * Source: LLM.int8() summary steps (3)-(4) (INT32 accumulation; rescale by
 * the outer product of the row and column constants) and §一.2 four-term
 * zero-point expansion, which with a symmetric weight (zp_b = 0) leaves the
 * correction -Z * colsum[n]; PDMIX glossary §2.3 (q = round(x / S) + Z).
 * Per element, in this order (fp32, round to nearest even):
 *   acc = sum_k Xq[m, k] * Wq[n, k]              (int32, exact)
 *   c   = acc - Z * colsum[n]                    (when Z != NULL)
 *   y   = fmaf((float) c, S_x[m] * s_w[n], bias ? bias[n] : 0)
 *   out[m, n] = y as bf16 (RNE) or fp32; W8A8_I32 writes c itself.
 *   Xq      device int8 [M, K] dense;  Wq device int8 [N, K] dense
 *   S_x     device fp32: [M] if s_x_per_row != 0, else one scalar (the
 *           per-tensor S of the Decode phase)
 *   Z       device int32 scalar or NULL (symmetric: no correction)
 *   colsum  device int32 [N]; required when Z != NULL
 *   s_w     device fp32 [N];  bias device fp32 [N] or NULL
 *   out     device [M, N] dense, out_dtype W8A8_BF16, W8A8_FP32 or W8A8_I32
 *   workspace/workspace_bytes: accepted for compatibility with
 *           w8a8_linear_static and not used by this call (NULL/0 allowed).
 * M <= 64 (Decode-shaped) runs a weight-streaming kernel: one cluster of up to
 * 8 CTAs per 128 output channels splits K, and the partial int32 sums are
 * added in distributed shared memory, so the call keeps no state in device
 * memory between calls and calls on different streams may overlap.
 * Every GEMM kernel of this call (Decode-shaped or not) uses programmatic
 * dependent launch: it may start while the previous kernel on the stream is
 * still running, and it loads its first weight tiles at once. Everything
 * else (Xq, S_x, Z, colsum, s_w, bias, out) is touched only after the
 * previous kernel has completed. So Wq, a constant weight, must not be
 * written by a kernel that lets its dependents launch early
 * (griddepcontrol.launch_dependents) and immediately precedes this call; no
 * kernel of this library that writes Wq does so.
 */
w8a8_status w8a8_gemm_dequant(const int8_t *Xq, const float *S_x, int32_t s_x_per_row,
                              const int32_t *Z, const int8_t *Wq, const float *s_w,
                              const int32_t *colsum, const float *bias, int64_t M, int64_t N,
                              int64_t K, void *out, w8a8_dtype out_dtype, void *workspace,
                              size_t workspace_bytes, void *stream);

/* Bytes of device workspace w8a8_linear_static needs for this shape: 0 when
 * it runs as one kernel (M <= 16, or M <= 32 with N <= 4096: the GEMM kernel
 * quantizes the activation itself), else M*K bytes rounded up to 256 for the
 * statically quantized activation (no zero-fill needed; every byte read is
 * written by the same call). Calls that overlap on the GPU must not share a
 * workspace. */
size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * Decode linear in one call: static per-tensor quantization of bf16 X, then
 * the GEMM with the zero-point corrected epilogue. Same result as
 * w8a8_quant_per_tensor followed by w8a8_gemm_dequant with s_x_per_row = 0.
 * For M <= 16, and for M <= 32 with N <= 4096, it is ONE kernel: the
 * weight-streaming GEMM loads each bf16 activation k-block and quantizes it in
 * shared memory before its MMAs read it, and no workspace is used (NULL
 * allowed). Other shapes quantize into the workspace with a separate kernel
 * first (every 128-channel tile of the fused kernel re-quantizes the whole
 * activation, which costs more than it saves there), then run the
 * Decode-shaped GEMM for M <= 64 and the tile GEMM beyond. All of these
 * kernels use programmatic dependent launch (they stream their first weight
 * tiles while the previous kernel finishes); the rule on writing Wq given for
 * w8a8_gemm_dequant applies.
 * Source: PDMIX glossary §2.2 (Decode has few tokens and is latency bound, so
 * a per-step quantization launch would be visible overhead) and §2.3 eq.
 * Q_decode; the hardware-acceleration chapter's note that decode is memory
 * bandwidth bound and that runtimes fuse small operations into one kernel.
 *   X            device bf16 [M, K], row stride ldx
 *   S, r, Z      device scalars from w8a8_calibrate_static
 *   Wq, s_w, colsum, bias, out, out_dtype: as in w8a8_gemm_dequant
 *   workspace    device, >= w8a8_gemm_workspace_size(M, N, K) bytes, 16-byte
 *                aligned (NULL allowed when that size is 0)
 */
w8a8_status w8a8_linear_static(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                               const float *r, const int32_t *Z, const int8_t *Wq,
                               const float *s_w, const int32_t *colsum, const float *bias,
                               int64_t N, void *out, w8a8_dtype out_dtype, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * Decode linear whose result is handed to the next linear already quantized:
 * w8a8_linear_static with a bf16 result, then that result quantized with the
 * NEXT linear's static per-tensor parameters, in one call and with no bf16
 * output written:
 *   Xq_out[m, n] = clamp(rne(float(bf16(y[m, n])) * r_out) + Z_out, -128, 127)
 * where y is the fp32 value of w8a8_linear_static's formula. The result is
 * identical to w8a8_linear_static (out_dtype W8A8_BF16) followed by
 * w8a8_quant_per_tensor(out, r_out, Z_out). The code is taken from the
 * bf16-rounded value so that fusing changes no result.
 * Source: PDMIX glossary §2.3 eq. Q_decode (the static scale and zero point
 * of the next linear are known before the step runs) and §2.2 (Decode is
 * latency bound, so the standalone quantization launch of each step is
 * overhead); the hardware-acceleration chapter's note that runtimes fuse
 * small operations into one kernel. No page fuses the two; this is a
 * deployment entry point of this library.
 *   X, S, r, Z, Wq, s_w, colsum, bias, workspace: as in w8a8_linear_static
 *   r_out, Z_out  device scalars of the next linear (w8a8_calibrate_static)
 *   Xq_out        device int8 [M, N] dense, 16-byte aligned, written
 * M <= 64 only (the Decode-shaped kernels); larger M returns
 * W8A8_ERR_UNSUPPORTED_SHAPE without launching anything. r_out and Z_out are
 * read after the previous kernel on the stream has completed (the rule on
 * writing Wq of w8a8_gemm_dequant applies).
 */
w8a8_status w8a8_linear_static_requant(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                                       const float *r, const int32_t *Z, const int8_t *Wq,
                                       const float *s_w, const int32_t *colsum, const float *bias,
                                       int64_t N, const float *r_out, const int32_t *Z_out, int8_t *Xq_out,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * w8a8_gemm_dequant whose result is handed to the next linear already
 * quantized: for int8 codes in (for example the output of
 * w8a8_linear_static_requant), int8 codes of the next linear out, so that a
 * chain of Decode linears passes no bf16 tensor between them.
 *   Xq_out[m, n] = clamp(rne(float(bf16(y[m, n])) * r_out) + Z_out, -128, 127)
 * with y the fp32 value of w8a8_gemm_dequant's formula: identical to
 * w8a8_gemm_dequant (W8A8_BF16) followed by w8a8_quant_per_tensor(out,
 * r_out, Z_out). Source and readings as for w8a8_linear_static_requant.
 *   Xq, S_x, s_x_per_row, Z, Wq, s_w, colsum, bias: as in w8a8_gemm_dequant
 *   r_out, Z_out  device scalars of the next linear
 *   Xq_out        device int8 [M, N] dense, 16-byte aligned, written
 * M <= 64 only (the Decode-shaped kernel); larger M returns
 * W8A8_ERR_UNSUPPORTED_SHAPE. Programmatic dependent launch as in
 * w8a8_gemm_dequant; r_out and Z_out are read after the previous kernel.
 */
w8a8_status w8a8_gemm_requant(const int8_t *Xq, const float *S_x, int32_t s_x_per_row, const int32_t *Z,
                              const int8_t *Wq, const float *s_w, const int32_t *colsum, const float *bias,
                              int64_t M, int64_t N, int64_t K, const float *r_out, const int32_t *Z_out,
                              int8_t *Xq_out, void *stream);

/*
 * w8a8_linear_static without a workspace argument: the same computation and
 * result as w8a8_linear_static (same arguments, same checks), for callers
 * that cannot allocate device memory when they run a Decode step -- a
 * plug-in inside a runtime that owns every byte of device memory and hands
 * none out, or a latency-critical step that cannot take the device-wide
 * synchronization a cudaMalloc / cudaFree may cause. No counterpart on the
 * pages: this is a deployment entry point of this library.
 * It always computes in two kernels -- the static quantization into a
 * scratch, then the Decode-shaped GEMM -- where w8a8_linear_static fuses both
 * for some shapes; the results are identical. The scratch (the quantized
 * activation) is one fixed device array inside the library, 524,288 bytes
 * (32 tokens x 16384), held by every GPU that loads the library until the
 * process exits. It serves M <= 32, N <= 32768 and K <= 16384; larger shapes
 * return W8A8_ERR_UNSUPPORTED_SHAPE without launching anything. The call
 * allocates nothing (no cudaMalloc, no allocating library routine).
 * The first call on a device also sets up that device (looks up the array's
 * device address with cudaGetSymbolAddress and zero-fills it once,
 * synchronously): make that first call before any stream capture. All calls
 * on a device share the one array, which keeps the last call's contents
 * (every byte a call reads is written earlier by the same call), so calls
 * that overlap on the GPU (different streams) race: serialize them.
 */
w8a8_status w8a8_linear_static_noalloc(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                                       const float *r, const int32_t *Z, const int8_t *Wq,
                                       const float *s_w, const int32_t *colsum, const float *bias,
                                       int64_t N, void *out, w8a8_dtype out_dtype, void *stream);

/*
 * LLM.int8() outlier split with vector-wise row quantization.
 * Source: LLM.int8() summary, architecture figure: 16-bit decomposition step
 * (1) (pick the columns of X whose magnitude exceeds the threshold, with the
 * matching rows of W) and 8-bit vector-wise steps (1)-(2) (row constant C_x,
 * X * 127 / C_x); mixed-precision decomposition steps 1-2 (threshold 6.0).
 * Readings: a column is an outlier when any |X[m, k]| > threshold (strict);
 * its entries become 0 in Xq and do not enter the row scale; outlier indices
 * are reported in ascending order.
 *   X            device bf16 [M, K], row stride ldx
 *   Xq           device int8 [M, K] dense, written (outlier columns = 0)
 *   S_x          device fp32 [M], written: absmax over normal columns / 127
 *                (0, with all of the row's codes 0, where that absmax is 0 or
 *                so small that 127 / absmax overflows fp32)
 *   outlier_idx  device int32 [cap], written: first min(n, cap) indices
 *   n_out        device int32 scalar, written: the number n of outlier columns
 *   Xo           device bf16 [M, cap] dense, written: Xo[m, j] = X[m, idx[j]]
 *                for j < min(n, cap)
 *   workspace    device, >= int8_outlier_split_workspace_size(K) bytes, 4-byte
 *                aligned (a K-bit column bitmap; the call clears it itself)
 * cap is in [0, 4096]. n > cap sets W8A8_ERR_OUTLIER_OVERFLOW in the device
 * status word; the outputs then describe only the first cap outliers (the
 * others are still zeroed in Xq, so the result would be wrong: check it).
 * M == 0 writes nothing.
 */
w8a8_status int8_outlier_split(const void *X, int64_t M, int64_t K, int64_t ldx, float threshold,
                               int32_t cap, int8_t *Xq, float *S_x, int32_t *outlier_idx,
                               int32_t *n_out, void *Xo, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Bytes of device workspace int8_outlier_split needs for K columns. */
size_t int8_outlier_split_workspace_size(int64_t K);

/*
 * LLM.int8() mixed-precision decomposition GEMM: the vector-wise INT8 product
 * plus the 16-bit product of the outlier columns, summed in the epilogue.
 * Source: LLM.int8() summary, architecture figure steps (3)-(4) and the
 * 16-bit decomposition step (2); the mixed-precision decomposition formula
 * Y = X_outlier W_outlier (16-bit) + Q(X_normal) Q(W_normal) (INT8).
 * Reading: the 16-bit side path takes bf16 inputs with fp32 accumulation,
 * side[m, n] = fmaf chain over j ascending of Xo[m, j] * W[idx[j], n] from 0;
 * Wq / s_w are the load-time per-channel weight over ALL K rows (its outlier
 * rows meet zeros in Xq). Per element:
 *   y = fmaf((float) acc, S_x[m] * s_w[n], side[m, n] + (bias ? bias[n] : 0))
 *   Xq, S_x, Xo, outlier_idx, n_out, cap: as written by int8_outlier_split
 *           (n_out is read on the device; min(n_out, cap) columns are used)
 *   Wq, s_w   device, from w8a8_quant_weight_per_channel of W
 *   W         device bf16 [K, N], row stride ldw: the unquantized weight
 *   bias      device fp32 [N] or NULL;  out device [M, N], bf16 or fp32
 * Cost: the side product runs on the CUDA cores, n_used fmaf per output
 * element; the first 16 outlier rows of W are staged per tile in shared
 * memory, later ones are read from global memory. This is the faster of the
 * two mixed GEMMs up to 16 outlier columns; beyond that use
 * int8_mixed_decomp_gemm_tc, whose cost barely grows with the count.
 */
w8a8_status int8_mixed_decomp_gemm(const int8_t *Xq, const float *S_x, const void *Xo,
                                   const int32_t *outlier_idx, const int32_t *n_out, int32_t cap,
                                   const int8_t *Wq, const float *s_w, const void *W, int64_t ldw,
                                   const float *bias, int64_t M, int64_t N, int64_t K, void *out,
                                   w8a8_dtype out_dtype, void *stream);

/*
 * int8_mixed_decomp_gemm with the 16-bit side product on the tensor cores:
 * the same arguments, checks and formula, except that
 *   side[m, n] = sum_{j < n_used} Xo[m, j] * W[idx[j], n]
 * is formed by bf16 x bf16 -> fp32 tensor-core MMAs (tcgen05.mma kind::f16)
 * in the hardware's summation order instead of the ascending fmaf chain.
 * The products are exact in fp32, so side differs from the chain only by
 * fp32 rounding of the sum: |side - side_chain| <= 2 n_used 2^-23
 * sum_j |Xo[m, j] W[idx[j], n]|; y then follows the same fixed-order epilogue
 * (y = fmaf((float) acc, S_x[m] * s_w[n], side + bias[n])). Built for heavy
 * outlier loads: its cost grows with ceil(n_used / 64) MMA k-blocks on the
 * tensor pipe rather than with n_used fmaf per output element.
 * Source: LLM.int8() summary, 16-bit decomposition step (2) (X_F16 W_F16 for
 * the outlier columns, then summed with the dequantized INT8 product) and
 * the mixed-precision decomposition formula Y. Reading: the pages' FP16 side
 * GEMM is taken as bf16 inputs with fp32 accumulation, as in
 * int8_mixed_decomp_gemm.
 *   workspace  device, >= int8_mixed_decomp_gemm_tc_workspace_size(M, N, cap)
 *              bytes, 16-byte aligned: the side operands, zero-padded to
 *              whole blocks of 64 outlier columns, written by the call (no
 *              initial contents needed; calls that overlap on the GPU must
 *              not share it).
 * Any M; Xo and W 16-byte aligned; the columns of Xo at or past n_used are
 * not read. Errors as int8_mixed_decomp_gemm, plus W8A8_ERR_WORKSPACE.
 */
w8a8_status int8_mixed_decomp_gemm_tc(const int8_t *Xq, const float *S_x, const void *Xo,
                                      const int32_t *outlier_idx, const int32_t *n_out, int32_t cap,
                                      const int8_t *Wq, const float *s_w, const void *W, int64_t ldw,
                                      const float *bias, int64_t M, int64_t N, int64_t K, void *out,
                                      w8a8_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Bytes of device workspace int8_mixed_decomp_gemm_tc needs: (M + N) rows of
 * cap rounded up to a multiple of 64 bf16 values (0 for a bad shape). */
size_t int8_mixed_decomp_gemm_tc_workspace_size(int64_t M, int64_t N, int32_t cap);

/*
 * Device status word. Kernels record device-side failures (a bounded wait
 * that ran out, an outlier count above cap) in one 32-bit word per device;
 * the first failure sticks. This call synchronizes `stream`, copies the word
 * into *device_status (W8A8_OK when nothing failed) and clears it. Returns
 * W8A8_ERR_CUDA when the synchronization itself failed.
 */
w8a8_status w8a8_check_device_error(void *stream, w8a8_status *device_status);

/*
 * Self-test of the bounded-wait path: launches one kernel that waits on a
 * barrier nothing will ever complete, with a limit of limit_ns nanoseconds
 * (1 ms .. 10 s). The wait gives up, records W8A8_ERR_DEVICE_TIMEOUT in the
 * device status word and the kernel returns; the device stays usable.
 * No counterpart on the pages: this exercises the failure path every
 * pipelined kernel here uses.
 */
w8a8_status w8a8_debug_wait_timeout_selftest(uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
