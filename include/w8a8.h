/*
 * w8a8.h -- C ABI of the B200 (sm_100a) W8A8 SmoothQuant linear path.
 *
 * The path is the INT8 W8A8 linear layer of a Llama-3-class decoder: per-token symmetric
 * dynamic activation quantization (fused with an RMSNorm whose gamma carries the SmoothQuant
 * factors, or with SiLU(gate)*up), an int8 x int8 -> int32 GEMM against per-output-channel
 * int8 weights, and a dequantization epilogue to bf16. Page citations are by page title and
 * section:
 *   [W8A8]  "INT8 W8A8 quantization of Llama 3.1 8B with SmoothQuant and GPTQ" (arc-codex)
 *   [PTQ]   "INT8 Post-Training Quantization for LLM Inference on NVIDIA GPUs" (devtechtools)
 *   [SERVE] "W8A8 Llama 3.1 8B: accuracy and serving results" (Red Hat developers)
 *   [INFENG] "05 Quantization AWQ GPTQ FP8" (inference-engineering notes)
 *   [AUTOGPTQ] "Optimizing Llama 3 Inference Speed Using INT8 Quantization via AutoGPTQ"
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; row-major, contiguous.
 *     The library allocates no device memory in any call; it keeps one small device status
 *     word per device (see w8a8_device_status) and nothing else.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream). Host-detectable
 *     errors are returned before anything is launched; a launch failure returns
 *     W8A8_ERR_CUDA. Device-side problems (a bounded wait that ran out) are reported by
 *     w8a8_device_status().
 *   - bf16 values are raw 16-bit patterns (w8a8_bf16). fp32 arithmetic is IEEE binary32 with
 *     round-to-nearest-even, including division and square root.
 *   - Base pointers of vectors read or written 16 bytes at a time must be 16-byte aligned
 *     (stated per argument); otherwise W8A8_ERR_ALIGNMENT.
 *   - Inputs must be finite; results for NaN or Inf inputs are unspecified.
 *   - Calls are thread-safe; the only mutable host state is a once-per-process init.
 *   - There is no CPU fallback: without a B200-class device a call returns
 *     W8A8_ERR_NO_DEVICE.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W8A8_API __attribute__((visibility("default")))
#else
#define W8A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *w8a8_stream_t; /* identical to cudaStream_t / CUstream */
typedef uint16_t w8a8_bf16;                /* raw bf16 bit pattern */

enum w8a8_status {
    W8A8_OK = 0,
    W8A8_ERR_INVALID_ARG = -1,       /* null pointer, non-positive size, aliasing */
    W8A8_ERR_ALIGNMENT = -2,         /* a base pointer is not 16-byte aligned */
    W8A8_ERR_UNSUPPORTED_SHAPE = -3, /* K or N not a supported multiple, or too large */
    W8A8_ERR_WORKSPACE = -4,         /* workspace missing or smaller than required */
    W8A8_ERR_CUDA = -5,              /* a CUDA runtime/driver call failed */
    W8A8_ERR_TIMEOUT = -6,           /* a device-side bounded wait ran out */
    W8A8_ERR_NO_DEVICE = -7,         /* no sm_100 device is current */
    W8A8_ERR_NUMERIC = -8            /* a matrix that must be positive definite is not */
};

/*
 * Per-token dynamic symmetric quantization of activations [W8A8 "Why activation
 * quantization is hard"; PTQ "1. Min-Max Calibration"], optionally with the SmoothQuant
 * factors folded into X (X' = X diag(1/s), [W8A8 "How the SmoothQuant smoothing factor is
 * computed"]):
 *   y[m,j]   = float(x[m,j]) * smooth_inv[j]          (or float(x[m,j]) if smooth_inv == NULL)
 *   s_tok[m] = max_j |y[m,j]| / 127
 *   q[m,j]   = clamp(round_half_even(y[m,j] / s_tok[m]), -127, 127)
 *   an all-zero row gives s_tok = 0 and q = 0.
 * x: bf16 [M,K], 16-byte aligned. smooth_inv: fp32 [K] or NULL, 16-byte aligned.
 * q: int8 [M,K], 16-byte aligned, must not overlap x. s_tok: fp32 [M].
 * Requires M >= 1, K >= 16, K % 16 == 0, K <= 32768.
 * Also serves the offline per-output-channel weight quantization [W8A8 "The problem with
 * naive quantization"]: with x = W [N,K] and smooth_inv = s (the factors themselves) it
 * yields the round-to-nearest int8 weights of diag(s)-smoothed W and their scales s_ch.
 */
W8A8_API int w8a8_quantize_rows(const w8a8_bf16 *x, const float *smooth_inv, int64_t M, int64_t K,
                       int8_t *q, float *s_tok, w8a8_stream_t stream);

/*
 * Static per-tensor symmetric quantization of activations [PTQ "1. Min-Max Calibration"]:
 * one scale for every token, fixed offline from a calibration batch as
 * scale = max(|min|, |max|) / 127, so no per-token range is measured at run time:
 *   y[m,j]   = float(x[m,j]) * smooth_inv[j]          (or float(x[m,j]) if smooth_inv == NULL)
 *   q[m,j]   = clamp(round_half_even(y[m,j] / scale), -127, 127)   (values beyond the
 *              calibrated range saturate at +-127)
 *   s_tok[m] = scale  (when s_tok is not NULL, so w8a8_gemm_dequant can consume it as is)
 * scale: finite and > 0, else W8A8_ERR_INVALID_ARG. Layout, alignment and shape rules as
 * for w8a8_quantize_rows; s_tok may be NULL.
 */
W8A8_API int w8a8_quantize_rows_static(const w8a8_bf16 *x, const float *smooth_inv, float scale,
                                       int64_t M, int64_t K, int8_t *q, float *s_tok,
                                       w8a8_stream_t stream);

/*
 * Smoothed RMSNorm fused with per-token quantization [W8A8 "How SmoothQuant prevents
 * outliers in activation tensors": RMSNorm divides by the RMS, then multiplies by gamma;
 * SmoothQuant divides gamma by s]:
 *   h[m,j]   = bf16(float(x[m,j]) + float(residual[m,j]))  if residual != NULL, written to h_out
 *              float(x[m,j])                                otherwise
 *   ms[m]    = float( (sum_j double(h[m,j]^2)) / K )      (binary64 sum, any order)
 *   rstd[m]  = 1 / sqrt(ms[m] + eps)                       (binary32)
 *   y[m,j]   = (h[m,j] * rstd[m]) * gamma_smoothed[j]      (binary32, in this order)
 *   then s_tok, q from y exactly as in w8a8_quantize_rows.
 * x, residual, h_out: bf16 [M,K], 16-byte aligned; residual and h_out are both NULL or both
 * non-NULL (h_out may alias residual, not x). gamma_smoothed: fp32 [K] (gamma / s), 16-byte
 * aligned. q: int8 [M,K], 16-byte aligned. s_tok: fp32 [M].
 * Requires M >= 1, K >= 16, K % 16 == 0, K <= 32768, eps >= 0.
 */
W8A8_API int w8a8_smooth_rmsnorm_quant(const w8a8_bf16 *x, const w8a8_bf16 *residual, w8a8_bf16 *h_out,
                              const float *gamma_smoothed, float eps, int64_t M, int64_t K,
                              int8_t *q, float *s_tok, w8a8_stream_t stream);

/*
 * SiLU(gate) * up fused with per-token requantization, the input of a Llama MLP's down
 * projection (not on the pages; the decoder-block workload's MLP):
 *   g = float(gate_up[m, j]), u = float(gate_up[m, I + j])
 *   a[m,j] = (g / (1 + w8a8_exp(-g))) * u                  (binary32)
 *   then s_tok, q from a exactly as in w8a8_quantize_rows.
 * w8a8_exp is a fixed binary32 exp: Cody-Waite reduction x = k ln2 + r with
 * k = rint(x * RN(1/ln2)), r = fma(-k, ln2_hi, x) then fma(-k, ln2_lo, r) (ln2_hi = ln2 to 16
 * significant bits, ln2_lo = RN(ln2 - ln2_hi)), the degree-7 Taylor polynomial of e^r with
 * coefficients RN(1/i!) by Horner's rule in fmaf, times 2^(k/2) then 2^(k - k/2) (k/2
 * truncated); x > 89 gives +inf and x < -104 gives +0.
 * gate_up: bf16 [M, 2I] ([gate | up] halves), 16-byte aligned. q: int8 [M, I], 16-byte
 * aligned. s_tok: fp32 [M]. Requires M >= 1, I >= 16, I % 16 == 0, I <= 32768.
 */
W8A8_API int w8a8_silu_mul_quant(const w8a8_bf16 *gate_up, int64_t M, int64_t I, int8_t *q,
                        float *s_tok, w8a8_stream_t stream);

/*
 * Bytes of device workspace w8a8_gemm_dequant needs for this shape (0 if none). The
 * workspace must be zero-filled before its first use; every call that returns W8A8_OK
 * leaves it ready for the next one (its flag words zero again), so one buffer serves any
 * number of calls issued in order on one stream. Calls that may run concurrently need
 * separate workspaces.
 */
W8A8_API size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * INT8 tensor-core GEMM with the fused dequantization epilogue [W8A8 "How we compressed the
 * model" (INT8 tensor cores), "Why activation quantization is hard" (one scale per token,
 * applied and reversed after accumulation); SERVE "Inter-token latency (ITL)" (multiply,
 * then convert back to BF16)]:
 *   acc[m,n] = sum_k int32(xq[m,k]) * int32(wq[n,k])        (exact int32)
 *   y[m,n]   = bf16( (float(acc[m,n]) * s_tok[m]) * s_ch[n] )  (binary32 RN, then RN to bf16)
 * xq: int8 [M,K] (K contiguous), 16-byte aligned. wq: int8 [N,K] (K contiguous, i.e. the
 * weight in nn.Linear layout), 16-byte aligned. s_tok: fp32 [M]. s_ch: fp32 [N], 16-byte
 * aligned. y: bf16 [M,N], 16-byte aligned. acc_out: int32 [M,N] or NULL; when given, the
 * raw accumulators are written too (a check mode; it adds 4 bytes of traffic per output).
 * workspace/workspace_bytes: see w8a8_gemm_workspace_size (may be NULL/0 when it returns 0).
 * Requires M >= 1, N >= 8, N % 8 == 0, K >= 16, K % 16 == 0, K <= 133144 (so that
 * 127 * 127 * K fits in int32), M, N <= 2^31 - 1.
 * Small M (at most 64 tokens by default, up to 256 on request) runs a swap-AB kernel that
 * streams the weight: split-K over thread-block clusters (partials summed in distributed
 * shared memory) when the weight has few 128-channel blocks, persistent stream-K over all SMs
 * otherwise; larger M runs a persistent tile kernel (256 x 256 tiles on CTA pairs, or 128-row
 * tiles), which splits the tiles' k-blocks evenly over the CTA pairs (stream-K: a tile shared
 * by several pairs is finished by the one holding its first k-blocks, after adding the
 * others' int32 partials from the workspace) when there are few, long tiles (at most one per
 * two CTA pairs, K >= 8192). All give identical results.
 */
W8A8_API int w8a8_gemm_dequant(const int8_t *xq, const float *s_tok, const int8_t *wq,
                      const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                      int32_t *acc_out, void *workspace, size_t workspace_bytes,
                      w8a8_stream_t stream);

/*
 * The same GEMM with the kernel chosen by the caller, for tests and tuning:
 * variant 0 = automatic (as w8a8_gemm_dequant), 1 = persistent tile kernel, 2 = swap-AB
 * stream-K kernel, 3 = swap-AB cluster split-K kernel (2 and 3: M <= 1024; beyond 256 tokens
 * the tokens are taken 256 at a time, each channel block once per such tile). ctas:
 * variant 2 = persistent CTAs sharing the weight stream (0 = one per SM, at most one per SM);
 * variant 3 = cluster size, the number of K splits per 128-channel block (0 = automatic,
 * at most 8, fewer if the clusters would not all fit on the GPU at once); variant 1 with
 * tile_n 512 = CTA pairs of the stream-K schedule (0 = whole tiles; at most one pair per two
 * SMs, and at most three pairs per tile so that a split tile has at most three later pieces).
 * tile_n (variant 1) = 0 automatic, 128 (128 x 128 output tiles), 256 (128 x 256) or 512
 * (256 x 256). The workspace needed is w8a8_gemm_workspace_size_ex() of the same arguments
 * (variant 2, and variant 1 on the stream-K schedule, use one).
 */
W8A8_API int w8a8_gemm_dequant_ex(const int8_t *xq, const float *s_tok, const int8_t *wq,
                         const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                         int32_t *acc_out, void *workspace, size_t workspace_bytes,
                         int variant, int ctas, int tile_n, w8a8_stream_t stream);
W8A8_API size_t w8a8_gemm_workspace_size_ex(int64_t M, int64_t N, int64_t K, int variant, int ctas,
                                   int tile_n);

/*
 * Small-M GEMM for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for callers of this library
 * that hold no device allocator of their own, or must not use one at the moment they call:
 * a plugin or hook run inside another runtime's launch path, code working within a fixed,
 * pre-planned memory budget, or code running while a stream is being captured. For them
 * cudaMalloc would synchronize the device, fail, or break the budget, so they cannot
 * provide the zero-filled workspace that w8a8_gemm_dequant's stream-K kernel needs.
 *
 * Computes exactly what w8a8_gemm_dequant computes, always with its small-M swap-AB kernels
 * (M <= 256), and allocates nothing. Only the stream-K kernel, used when the weight has many
 * 128-channel blocks, needs scratch; it is a file-scope static device array of
 * W8A8_NOALLOC_SCRATCH_BYTES (8 MiB) inside the library; every GPU on which the library is
 * loaded holds that array until the process exits. The caller still owns and passes every
 * input and output. Arguments and requirements are those of w8a8_gemm_dequant without
 * acc_out and workspace.
 *   - Returns W8A8_ERR_WORKSPACE when this shape's scratch exceeds
 *     W8A8_NOALLOC_SCRATCH_BYTES: 4 KiB of flags plus 512 bytes per token (M rounded up to
 *     a multiple of 4) of partial sums per CTA (one CTA per SM), needed only when a CTA's
 *     share of the weight stream ends inside a 128-channel block. So on a 148-SM B200
 *     M <= 108 always fits. W8A8_ERR_UNSUPPORTED_SHAPE for M > 256.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - Each call that needs the scratch clears its 4 KiB of flag words (cudaMemsetAsync on
 *     `stream`) before its kernel runs, so flags left raised by an earlier call whose wait
 *     ran out cannot leak into it; the partial sums need no clearing (each is written
 *     before its flag is raised).
 *   - All calls on a device share the one array and it keeps the last call's contents:
 *     calls whose kernels can overlap on the GPU (different streams without ordering
 *     between them) race on it and give wrong results. Serialize them.
 */
#define W8A8_NOALLOC_SCRATCH_BYTES (8u << 20)
W8A8_API int w8a8_gemm_dequant_noalloc(const int8_t *xq, const float *s_tok, const int8_t *wq,
                                       const float *s_ch, int64_t M, int64_t N, int64_t K,
                                       w8a8_bf16 *y, w8a8_stream_t stream);

/*
 * The gate|up projection of a Llama MLP fused with SiLU(gate)*up [SiLU*up is not on the
 * pages; it is the decoder block's MLP]: the INT8 GEMM of w8a8_gemm_dequant whose epilogue
 * forms a = silu(g) * u instead of storing the [M, 2I] gate|up output, followed by the
 * per-token quantization of a. Results are bit for bit those of w8a8_gemm_dequant followed by
 * w8a8_silu_mul_quant on the plain weight:
 *   g, u     = the bf16 outputs of w8a8_gemm_dequant for gate channel j and up channel j
 *   a[m,j]   = (g / (1 + exp(-g))) * u in binary32 (exp as in w8a8_silu_mul_quant)
 *   s_out[m] = max_j |a[m,j]| / 127,  q[m,j] = clamp(round_half_even(a[m,j] / s_out[m]), +-127)
 * xq, s_tok: as for w8a8_gemm_dequant (M tokens, K inputs). wq_il: int8 [2I, K], the gate|up
 * weight with its rows interleaved in blocks of 64: rows 128b .. 128b+63 are gate rows
 * 64b .. 64b+63 and rows 128b+64 .. 128b+127 are up rows 64b .. 64b+63 (b < I/64); s_ch_il:
 * fp32 [2I], the channel scales in the same order. I % 64 == 0.
 * a: fp32 [M, I] (written, then read by the quantization; 16-byte aligned). q: int8 [M, I],
 * s_out: fp32 [M]. workspace: w8a8_gemm_silu_quant_workspace_size(M, I, K) bytes (0 when the
 * GEMM's plan needs none), 16-byte aligned: the GEMM's own workspace, with the rules of
 * w8a8_gemm_workspace_size, so one zero-filled buffer serves calls of this entry point and of
 * w8a8_gemm_dequant alike, issued in order on one stream. Other requirements and errors as
 * for w8a8_gemm_dequant (acc_out is not available here).
 */
W8A8_API size_t w8a8_gemm_silu_quant_workspace_size(int64_t M, int64_t I, int64_t K);
W8A8_API int w8a8_gemm_silu_quant(const int8_t *xq, const float *s_tok, const int8_t *wq_il,
                                  const float *s_ch_il, int64_t M, int64_t I, int64_t K,
                                  float *a, int8_t *q, float *s_out, void *workspace,
                                  size_t workspace_bytes, w8a8_stream_t stream);

/*
 * The o projection's GEMM followed by the residual add and the next smoothed RMSNorm with its
 * per-token quantization [W8A8 "How we compressed the model" (the INT8 linear); SERVE
 * "Inter-token latency (ITL)" (the per-layer quantize steps between the GEMMs at decode);
 * W8A8 "How SmoothQuant prevents outliers in activation tensors" (RMSNorm with gamma / s)].
 * It computes exactly what this chain of two calls computes:
 *   y            = w8a8_gemm_dequant(xq, s_tok, wq, s_ch)             bf16 [M, N]
 *   h_out, q, s_out = w8a8_smooth_rmsnorm_quant(y, residual, h_out, gamma_smoothed, eps)
 * i.e. h = bf16(y + residual), then the RMSNorm of h (row length N) with gamma_smoothed, then
 * per-token INT8 codes. Two forms, with identical results:
 *   one_launch = 0 (w8a8_gemm_rmsnorm_quant): the GEMM, then the row kernel, which the
 *     dependent launch starts while the GEMM drains. The faster form on B200 at every size
 *     measured, and the default.
 *   one_launch = 1: at decode sizes (the cluster split-K plan of w8a8_gemm_dequant: at most 64
 *     tokens, N <= 8192, few 128-channel blocks; w8a8_gemm_rmsnorm_quant_one_launch_ok(M, N,
 *     K) returns 1) a single launch: the GEMM's CTAs take a ticket in the workspace once
 *     their outputs are stored, and the last min(M, 64) of them run the row pass over y (read
 *     back through L2). Other shapes return W8A8_ERR_UNSUPPORTED_SHAPE. Measured ~1.2-1.9 us
 *     slower per call than the two launches: the ticket handshake (a release fence, an atomic
 *     and a poll) costs more than the kernel boundary it removes.
 * xq, s_tok, wq, s_ch, y: as for w8a8_gemm_dequant (y is written; it must not alias residual
 * or h_out). residual, h_out: bf16 [M, N], 16-byte aligned; h_out may alias residual.
 * gamma_smoothed: fp32 [N], 16-byte aligned. q: int8 [M, N], 16-byte aligned; s_out: fp32 [M].
 * eps >= 0. N must also satisfy the row rules of w8a8_smooth_rmsnorm_quant (N % 16 == 0,
 * N <= 32768).
 * workspace: w8a8_gemm_rmsnorm_quant_workspace_size(M, N, K) bytes (at least 4 KiB: the
 * GEMM's own workspace with its flag words, two of which, words 1022 and 1023, hold the
 * one-launch form's counters), 16-byte aligned, zero-filled before first use; every completed
 * call leaves the flag words zero again, so one buffer serves this entry point and
 * w8a8_gemm_dequant alike, calls issued in order on one stream. After a call that reported
 * W8A8_ERR_TIMEOUT through w8a8_last_device_status, zero the workspace again.
 * Errors: W8A8_ERR_INVALID_ARG (NULL pointer, eps < 0 or NaN, y aliasing residual or h_out,
 * one_launch not 0 or 1), W8A8_ERR_ALIGNMENT, W8A8_ERR_UNSUPPORTED_SHAPE (as for the two
 * calls, or one_launch = 1 for a shape without the one-launch form), W8A8_ERR_WORKSPACE.
 */
W8A8_API size_t w8a8_gemm_rmsnorm_quant_workspace_size(int64_t M, int64_t N, int64_t K);
W8A8_API int w8a8_gemm_rmsnorm_quant_one_launch_ok(int64_t M, int64_t N, int64_t K);
W8A8_API int w8a8_gemm_rmsnorm_quant(const int8_t *xq, const float *s_tok, const int8_t *wq,
                                     const float *s_ch, int64_t M, int64_t N, int64_t K,
                                     w8a8_bf16 *y, const w8a8_bf16 *residual, w8a8_bf16 *h_out,
                                     const float *gamma_smoothed, float eps, int8_t *q,
                                     float *s_out, void *workspace, size_t workspace_bytes,
                                     w8a8_stream_t stream);
W8A8_API int w8a8_gemm_rmsnorm_quant_ex(const int8_t *xq, const float *s_tok, const int8_t *wq,
                                        const float *s_ch, int64_t M, int64_t N, int64_t K,
                                        w8a8_bf16 *y, const w8a8_bf16 *residual,
                                        w8a8_bf16 *h_out, const float *gamma_smoothed, float eps,
                                        int8_t *q, float *s_out, void *workspace,
                                        size_t workspace_bytes, int one_launch,
                                        w8a8_stream_t stream);

/*
 * ---------------------------------------------------------------- the fused decoder block
 *
 * One Llama decoder block's whole linear path at decode sizes (1 <= M <= 64 tokens) as a single
 * persistent kernel (the fused block path: the row operations and the four GEMMs in one
 * launch, a grid-wide barrier between dependent phases, the weight stream running on across
 * phase boundaries). It computes what this chain of the separate entry points computes:
 *   q1, s1      = w8a8_smooth_rmsnorm_quant(x, gamma1)
 *   qkv_out     = w8a8_gemm_dequant(q1, s1, qkv)
 *   q2, s2      = w8a8_quantize_rows(attn, sinv_o)
 *   o_out       = w8a8_gemm_dequant(q2, s2, o)
 *   q3, s3, h_out = w8a8_smooth_rmsnorm_quant(o_out, gamma2, residual = x)
 *   q4, s4, a_out = w8a8_gemm_silu_quant(q3, s3, gate_up_il)
 *   y_out       = w8a8_gemm_dequant(q4, s4, down)
 * with identical results except that the binary64 sums of squares of the two RMSNorms are
 * added in another order (the method leaves the order free; a row whose mean of squares lies
 * within that order's effect of a binary32 rounding boundary may round to the neighbour).
 * attn stands for the attention output (the o projection's input). Shapes: x, attn, o_out,
 * h_out, y_out bf16 [M, H]; qkv_out bf16 [M, QKV]; a_out fp32 [M, I]; q1..q3 int8 [M, H], q4
 * int8 [M, I], s1..s4 fp32 [M]; gamma1, gamma2, sinv_o fp32 [H] (sinv_o may not be NULL: pass
 * ones for no smoothing); weights int8 [N, K] with fp32 scales [N]: qkv [QKV, H], o [H, H],
 * gate_up_il [2I, H] interleaved as for w8a8_gemm_silu_quant, down [H, I]. Every pointer
 * 16-byte aligned. Requires 1 <= M <= 64, H a multiple of 128 up to 8192, I a multiple of 128
 * up to 32768, QKV a multiple of 8. workspace: w8a8_block_decode_workspace_size() bytes, 256-byte aligned, zero-filled
 * before its first use; each call leaves it ready for the next call in stream order (a call
 * that returned W8A8_ERR_TIMEOUT through w8a8_device_status leaves it to be zero-filled
 * again). Launched as a cooperative grid of one CTA per SM.
 */
typedef struct w8a8_linear {
    const int8_t *wq;  /* int8 [N, K] */
    const float *s_ch; /* fp32 [N] */
} w8a8_linear;

typedef struct w8a8_block_io {
    int64_t M, H, I, QKV;
    float eps;
    const w8a8_bf16 *x, *attn;
    const float *gamma1, *sinv_o, *gamma2;
    w8a8_linear qkv, o, gate_up_il, down;
    w8a8_bf16 *qkv_out, *o_out, *h_out, *y_out;
    float *a_out;
    int8_t *q1, *q2, *q3, *q4;
    float *s1, *s2, *s3, *s4;
} w8a8_block_io;

W8A8_API size_t w8a8_block_decode_workspace_size(int64_t M, int64_t H, int64_t I, int64_t QKV);
W8A8_API int w8a8_block_decode(const w8a8_block_io *io, void *workspace, size_t workspace_bytes,
                               w8a8_stream_t stream);

/*
 * ---------------------------------------------------------------- FP8 (E4M3) variant
 *
 * W8A8 with 8-bit floating-point codes instead of int8, the variant for Hopper and Blackwell
 * GPUs [SERVE "When W8A8 INT8 quantization is a good fit", "What to explore next"; INFENG
 * "Ladder"]. The pages do not fix the encoding; this library uses
 * OCP E4M3 (sign, 4 exponent bits with bias 7, 3 fraction bits; no infinities; largest
 * finite 448; S.1111.111 is NaN) and:
 *   e4m3(v)  = v rounded to nearest E4M3 value, ties to even, saturated to +-448
 *   s        = amax / 448 (binary32), code = e4m3(RN(y / s)); an all-zero row: s = 0, codes +0
 * Codes travel as uint8 bit patterns. Each entry point below is its INT8 namesake with those
 * codes and that scale; arguments, layouts, alignment, shape rules and errors are the same.
 */
W8A8_API int w8a8_quantize_rows_fp8(const w8a8_bf16 *x, const float *smooth_inv, int64_t M,
                                    int64_t K, uint8_t *q, float *s_tok, w8a8_stream_t stream);
W8A8_API int w8a8_smooth_rmsnorm_quant_fp8(const w8a8_bf16 *x, const w8a8_bf16 *residual,
                                           w8a8_bf16 *h_out, const float *gamma_smoothed,
                                           float eps, int64_t M, int64_t K, uint8_t *q,
                                           float *s_tok, w8a8_stream_t stream);
W8A8_API int w8a8_silu_mul_quant_fp8(const w8a8_bf16 *gate_up, int64_t M, int64_t I, uint8_t *q,
                                     float *s_tok, w8a8_stream_t stream);

/*
 * FP8 tensor-core GEMM (tcgen05.mma kind::f8f6f4, E4M3 x E4M3) with the dequantization
 * epilogue:
 *   acc[m,n] = sum_k e4m3(xq[m,k]) * e4m3(wq[n,k])   accumulated in binary32 by the tensor
 *              cores (each product is exact; the order and the rounding of the additions are
 *              the hardware's, so acc differs from the exact sum by at most a few units of
 *              2^-24 times sum_k |products|; split-K partial sums are added in binary32)
 *   y[m,n]   = bf16( (acc[m,n] * s_tok[m]) * s_ch[n] )  (binary32 RN, then RN to bf16)
 * xq: uint8 E4M3 codes [M,K]; wq: uint8 E4M3 codes [N,K] (per-output-channel scales s_ch =
 * max_k |w[n,k]| / 448); acc_out: fp32 [M,N] or NULL (the accumulators, as a check mode).
 * variant, ctas, tile_n, workspace and all other rules as for w8a8_gemm_dequant_ex (the
 * cluster split-K kernel, variant 3, adds the binary32 partials of a cluster in rank order,
 * read from the CTAs' shared memory); the workspace size is w8a8_gemm_fp8_workspace_size() of
 * the same arguments.
 */
W8A8_API size_t w8a8_gemm_fp8_workspace_size(int64_t M, int64_t N, int64_t K, int variant,
                                             int ctas, int tile_n);
W8A8_API int w8a8_gemm_dequant_fp8(const uint8_t *xq, const float *s_tok, const uint8_t *wq,
                                   const float *s_ch, int64_t M, int64_t N, int64_t K,
                                   w8a8_bf16 *y, float *acc_out, void *workspace,
                                   size_t workspace_bytes, int variant, int ctas, int tile_n,
                                   w8a8_stream_t stream);

/*
 * The fused gate|up GEMM + SiLU(gate)*up + per-token quantization of w8a8_gemm_silu_quant
 * with FP8 operands and codes: the same interleaved weight layout and arguments (xq, wq_il
 * E4M3 codes as uint8; q: E4M3 codes [M,I] as uint8, s_out = max_i |a[m,i]| / 448). The
 * epilogue rounds the dequantized gate and up values to bf16 exactly as w8a8_gemm_dequant_fp8
 * stores them and continues as w8a8_silu_mul_quant_fp8, so the result is bit-identical to
 * those two calls whenever the GEMM's binary32 accumulators are the same; that holds for the
 * same kernel plan on the interleaved weight. The plan is the GEMM's automatic one, with
 * stream-K in place of the cluster split-K (it has no SiLU epilogue). Workspace:
 * w8a8_gemm_silu_quant_fp8_workspace_size(M, I, K) bytes, under w8a8_gemm_workspace_size's
 * rules.
 */
W8A8_API size_t w8a8_gemm_silu_quant_fp8_workspace_size(int64_t M, int64_t I, int64_t K);
W8A8_API int w8a8_gemm_silu_quant_fp8(const uint8_t *xq, const float *s_tok,
                                      const uint8_t *wq_il, const float *s_ch_il, int64_t M,
                                      int64_t I, int64_t K, float *a, uint8_t *q, float *s_out,
                                      void *workspace, size_t workspace_bytes,
                                      w8a8_stream_t stream);

/*
 * ---------------------------------------------------------------- GPTQ weights (offline)
 *
 * GPTQ quantization of one linear layer's weight to the int8 + per-channel-scale format of
 * w8a8_gemm_dequant [W8A8 "The solution: How GPTQ improves on naive quantization": after
 * rounding each weight, measure the error and redistribute it over the weights not yet
 * quantized, guided by a Hessian from the calibration activations; AUTOGPTQ "Crucial Config
 * Tips for Performance": the dampening factor]. In binary64 on the device:
 *   W'[n,j] = float(w[n,j]) * smooth[j]   (binary32 product; W' = w if smooth == NULL)
 *   s_ch[n] = max_j |W'[n,j]| / 127       (binary32, as RTN)
 *   H       = (2/T) x^T x; H_jj = 0 (an input channel that is always zero) -> H_jj = 1 and
 *             column j of W' is zeroed; then H_jj += damp * mean_j(H_jj)
 *   U       = the upper Cholesky factor of H^-1 (H^-1 = U^T U)
 *   for j = 0 .. K-1, every row n:  q = clamp(rint(W'[n,j] / s_ch[n]), -127, 127),
 *             e = (W'[n,j] - q s_ch[n]) / U[j][j],  W'[n,k] -= e U[j][k] for k > j
 * The column updates are applied in blocks of 64 and groups of four blocks (the lazy-batch
 * form), so the binary64 sums run in another order than the column-by-column statement; a code can differ from that
 * statement's only where W'/s lies within rounding distance of a half-integer.
 * w: bf16 [N,K] (nn.Linear layout). smooth: fp32 [K] or NULL (SmoothQuant factors s_j).
 * x_cal: fp32 [T,K], the layer's calibration inputs as the layer receives them (X diag(1/s)).
 * damp > 0 (0.01 is GPTQ's usual value). wq: int8 [N,K], 16-byte aligned; s_ch: fp32 [N].
 * u_out: fp64 [K,K] or NULL (U, for checking), 8-byte aligned. workspace:
 * w8a8_gptq_workspace_size(N, K) bytes, 256-byte aligned, any contents (W8A8_ERR_ALIGNMENT
 * otherwise). Requires K % 64 == 0, 64 <= K <= 32768, N >= 1, T >= 1.
 * Unlike the rest of the library this call SYNCHRONIZES `stream` at its end (offline
 * preparation): it returns W8A8_ERR_NUMERIC when H is not positive definite in binary64 (not
 * possible with damp > 0 in exact arithmetic).
 */
W8A8_API size_t w8a8_gptq_workspace_size(int64_t N, int64_t K);
W8A8_API int w8a8_gptq_quantize(const w8a8_bf16 *w, const float *smooth, const float *x_cal,
                                int64_t N, int64_t K, int64_t T, double damp, int8_t *wq,
                                float *s_ch, double *u_out, void *workspace,
                                size_t workspace_bytes, w8a8_stream_t stream);

/*
 * Measurement aid, not part of the W8A8 path (the pages have no counterpart): launches `ctas`
 * CTAs (0 = one per SM), each issuing `iters` back-to-back dense tcgen05.mma kind::i8 of
 * shape 128 x n x 32 (n = 16, 32, 64, 128 or 256) on shared-memory operands into tensor
 * memory. Timing it gives the device's INT8 tensor-core rate at that shape,
 * 2 * 128 * n * 32 * iters * ctas operations. W8A8_ERR_INVALID_ARG for any other n.
 */
W8A8_API int w8a8_probe_i8_mma(long long iters, int n, int ctas, w8a8_stream_t stream);

/*
 * Measurement aid for the GPTQ kernels' roofline (no counterpart on the pages): `ctas` CTAs of
 * 256 threads, each thread running 8 independent chains of `iters` binary64 fused
 * multiply-adds, 2 * 8 * iters * 256 * ctas flops in all; out: fp64 [ctas * 256] (the chains'
 * sums, written so the work is kept). W8A8_ERR_INVALID_ARG for iters < 1, ctas < 1, out NULL.
 */
W8A8_API int w8a8_probe_f64_fma(long long iters, int ctas, double *out, w8a8_stream_t stream);

/*
 * Kernel overlap mode, process-wide (default 1). Results are identical in every mode.
 *   0: each kernel of this library starts after the previous work in its stream completes.
 *   1: programmatic dependent launch: a kernel may launch and run its prologue (barrier
 *      set-up, tensor-memory allocation, descriptor prefetch) while the previous kernel in
 *      the stream is still running; it waits for that kernel to complete before it reads
 *      any input or writes any output.
 *   2: as 1, and the GEMMs also start streaming their int8 weights (wq) before that wait,
 *      so a GEMM's weight traffic overlaps the tail of the kernels before it; likewise the
 *      smoothed RMSNorm reads gamma_smoothed before it. Only valid when no kernel enqueued
 *      on the stream since its last completed synchronization writes wq or gamma_smoothed
 *      -- e.g. weights prepared once and synchronized before serving.
 * Returns the previous mode, or W8A8_ERR_INVALID_ARG for another value. Applies to launches
 * made after the call (a captured CUDA graph keeps the mode it was captured with).
 */
W8A8_API int w8a8_set_overlap(int mode);
W8A8_API int w8a8_get_overlap(void);

/*
 * Device status: synchronizes the current device, then returns W8A8_OK or
 * W8A8_ERR_TIMEOUT if any kernel of this library on it gave up a bounded wait (every
 * mbarrier and cross-CTA flag wait in the kernels is limited, ~2 s) since the last reset.
 * reset != 0 clears the word. Returns W8A8_ERR_CUDA if synchronization fails.
 */
W8A8_API int w8a8_device_status(int reset);

/*
 * Stream status: waits until `stream` has finished the work queued on it so far (not the
 * whole device), then returns W8A8_OK, or W8A8_ERR_TIMEOUT if a kernel of this library on
 * the current device gave up a bounded wait since the device word was last cleared. The word
 * is per device, not per stream: a timeout in a kernel of another stream on the same device
 * shows here too once that kernel has run. It is not cleared here (w8a8_device_status(1)
 * clears it). Returns W8A8_ERR_CUDA if the stream's work failed. [No counterpart on the
 * pages: the failure-detection side of every call above.]
 */
W8A8_API int w8a8_last_device_status(w8a8_stream_t stream);

/*
 * Self-test of the failure path (no counterpart on the pages): launches one small kernel
 * whose two waits -- on an mbarrier and on a global flag that nothing ever sets -- each give
 * up after limit_ns nanoseconds (1e3 <= limit_ns <= 2e9, else W8A8_ERR_INVALID_ARG). The
 * kernel then raises the device status word and returns, so the next w8a8_device_status()
 * reports W8A8_ERR_TIMEOUT while the context stays usable. No fault, trap or hang is involved.
 */
W8A8_API int w8a8_selftest_wait_timeout(unsigned long long limit_ns, w8a8_stream_t stream);

/* Static, human-readable name of a status code. */
W8A8_API const char *w8a8_status_string(int status);

/* ABI version: (major << 16) | minor. */
W8A8_API int w8a8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
