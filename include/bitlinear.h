/*
 * bitlinear.h -- C ABI of the BitNet b1.58 BitLinear forward library for
 * NVIDIA B200 (sm_100a).  Library: libbitlinear.so.
 *
 * The operation (sources, cited by page title and section):
 *   [P1] "QAT与BitNet：1-bit及1.58-bit量化训练解析" (kongchang.com)
 *   [P3] "BitNet b1.58深度解析：三值权重如何重塑大模型推理" (0539edu.com)
 *   [P5] "QAT and BitNet: A Deep Dive into 1-bit and 1.58-bit
 *         Quantization-Aware Training" (kongchang.com/en)
 *
 *   W [N, K] latent weights (row-major, out x in, as an nn.Linear weight);
 *   gamma = mean |W| over the whole matrix            [P3] §3.1, [P5] recipe
 *   W_q = clamp(round(W / (gamma + eps)), -1, 1)      [P3] §3.1, [P5] recipe
 *   packed rows: 2 bits per weight or 5 trits/byte    [P3] §2.3 §6.3, [P5]
 *   s_m = max_k |x[m, k]| (floored at 1e-6);
 *   x_q = clamp(round(x / s_m * 127), -127, 127)      [P3] §3.2 §5.2
 *   acc[m, n] = sum_k W_q[n, k] x_q[m, k]  (INT32)    [P3] §4.2 §3.3
 *   y[m, n] = acc[m, n] * (gamma * s_m / 127)         [P3] §3.2 §5.3, [P5]
 *
 * Around that path: the pre-norm LayerNorm feeding x_q ([P5] recipe step 1),
 * several layers on one input (a block's Q, K, V: [P3] §5.4), the 1-bit
 * variant (alpha = mean W, codes sign(W - alpha), beta = mean |W|, 8 weights
 * per byte: [P5] recipe steps 2 and 4) and the straight-through backward
 * (dx = gamma dy W_q, dW = gamma dy^T x_deq: [P3] §5.3).
 *
 * Exact conventions (where the pages are silent):
 *   - gamma: |w| summed in fp64 in a fixed order (below), divided by N*K in
 *     fp64, rounded to fp32.  Order: elements in row-major order e = n*K + k;
 *     chunk c = elements [8192c, 8192c + 8192); lane l (0..255) of a chunk adds
 *     elements 8192c + 2048i + 8l + j for i = 0..3, j = 0..7, in that order;
 *     the 256 lane sums combine by the stride-halving tree p[l] += p[l + s],
 *     s = 128..1; chunk sums, zero-padded to a power of two P, combine by the
 *     same tree, s = P/2..1.
 *   - d = gamma + eps (fp32); W_q = clamp(rint(w / d), -1, 1) with an IEEE
 *     fp32 quotient and round-half-to-even (a ratio of exactly 0.5 gives 0).
 *   - x_q: fp32 quotient x / s_m, then an fp32 multiply by 127, then
 *     round-half-to-even.
 *   - dequant: c_m = (gamma * s_m) / 127 in fp32, y = (float)acc * c_m; a
 *     bf16 y is that fp32 value rounded to nearest even.
 *   - 2-bit format: digit q + 1 (-1 -> 00, 0 -> 01, +1 -> 10) of weight k in
 *     bits 2*(k % 4) of byte k / 4.  Base-3 format: byte j of a row is
 *     sum_i (q[5j + i] + 1) * 3^i.  Every row is padded to a multiple of 16
 *     bytes with digits of weight 0 (0x55 / 121).  1-bit format: bit k % 8 of
 *     byte k / 8 is 1 for +1 and 0 for -1, pad bits 0.  Row stride =
 *     bitlinear_packed_row_bytes(K, fmt).
 *
 * Conventions of every call:
 *   - Array arguments are DEVICE pointers owned by the caller, aligned to 16
 *     bytes; scalars are host values; `stream` is a cudaStream_t (NULL = the
 *     legacy default stream).  The library allocates no memory and keeps no
 *     state between calls.
 *   - Calls validate their arguments on the host and return an error before
 *     launching anything; on success they only enqueue work on `stream` and
 *     return BL_OK (no host synchronisation).
 *   - Errors found on the device (a code outside {-1, 0, 1} given to
 *     bitlinear_pack, or a wait inside a kernel that ran out of time) set a
 *     sticky flag in the workspace header; bitlinear_device_status() reports
 *     and clears it.
 *   - Inputs must be finite; NaN or Inf inputs give unspecified codes.
 *   - Limits: 1 <= K <= 2^20; N * K <= 2^32; 0 <= M, N < 2^31 (an empty M
 *     or N is a no-op); larger sizes return BL_ERR_INVALID_VALUE (the size
 *     queries return 0).
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_VALUE = 1,       /* a size, dtype, format or pointer is wrong */
  BL_ERR_UNSUPPORTED = 2,         /* valid, but not implemented on this device */
  BL_ERR_MISALIGNED = 3,          /* an array is not 16-byte aligned */
  BL_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the query function's size */
  BL_ERR_CUDA = 5,                /* a CUDA runtime call failed */
  BL_ERR_DEVICE_TIMEOUT = 6,      /* a kernel's bounded wait ran out (device flag) */
  BL_ERR_BAD_CODE = 7,            /* bitlinear_pack met a code outside {-1,0,1} */
  BL_ERR_SCRATCH_LIMIT = 8        /* too large for bitlinear_absmean_noalloc's fixed scratch */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1, BL_I8 = 2, BL_I32 = 3 } bl_dtype;

typedef enum {
  BL_PACK_I2 = 0, /* 2 bits per weight, 4 weights per byte */
  BL_PACK_T5 = 1, /* 5 trits per byte in base 3 (3^5 = 243 <= 256) */
  BL_PACK_B1 = 2  /* 1-bit BitNet: 1 bit per weight, 8 per byte; bit i of byte j
                     is weight 8j + i, 1 for +1 and 0 for -1, pad bits 0 */
} bl_pack;

/* Bytes at the start of every workspace that hold the device status flags.
 * They must be zero before a workspace is first used (bitlinear_workspace_init
 * or cudaMemset); the library keeps them consistent afterwards. */
#define BL_WS_HEADER_BYTES 256

/* Row stride of a packed matrix: ceil(K / per) bytes (per = 4, 5 or 8) rounded up
 * to a multiple of 16.  [P3] §4.1 (70B x 0.25 B = 17.5 GB; 5 per byte ~14 GB).
 * Returns -1 for K < 1 or an unknown format. */
BL_API int64_t bitlinear_packed_row_bytes(int64_t K, int fmt);

/* Workspace bytes needed by bitlinear_quantize_weights for an N x K matrix
 * (the header plus one fp64 partial sum per 8192-element chunk). */
BL_API size_t bitlinear_quantize_weights_workspace_bytes(int64_t N, int64_t K);

/* Workspace bytes needed by bitlinear_forward for these sizes and formats (the
 * header, plus x_q when activations are quantized ahead of the tensor-core
 * path, plus a 2-bit copy of base-3 or 1-bit weights for that path (and of
 * 1-bit rows longer than 4096 bytes for any M), plus the INT32
 * partial sums when a layer with few tokens (5..128) is split along K so
 * that it spreads over every SM; the split depends on the device's SM
 * count, so query on the device that runs the call). */
BL_API size_t bitlinear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int xdt);

/* Zero the status header of a workspace (enqueued on `stream`). */
BL_API bl_status bitlinear_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Absmean ternarization and packing of a latent weight matrix (steps 1-3).
 * [P3] §3.1; [P5] "The Ternary Weight Recipe"; [P3] §2.3 and §6.3 (formats).
 *   W       [N, K] fp32 or bf16 (wdt = BL_F32 | BL_BF16), read twice.
 *   eps     > 0 and finite (the pages use 1e-5).
 *   fmt     BL_PACK_I2 | BL_PACK_T5.
 *   packed  [N, bitlinear_packed_row_bytes(K, fmt)] uint8 output, or NULL.
 *   codes   [N, K] int8 output in {-1, 0, 1}, or NULL.
 *   gamma   [1] fp32 device output (stays on the device: no host sync).
 *   ws      workspace of at least bitlinear_quantize_weights_workspace_bytes.
 * At least one of packed / codes must be given. */
BL_API bl_status bitlinear_quantize_weights(const void *W, int wdt, int64_t N, int64_t K, float eps,
                                     int fmt, uint8_t *packed, int8_t *codes, float *gamma,
                                     void *ws, size_t ws_bytes, void *stream);

/* Absmean scale alone (step 1): gamma = mean |W| in the fixed fp64 order,
 * written to the device.  [P3] §3.1; [P5] "The Ternary Weight Recipe" (step
 * 1); [P3] §6.2 suggests watching gamma during training.
 *   W      [N, K] fp32 or bf16.   gamma  [1] fp32 device output.
 *   ws     at least bitlinear_quantize_weights_workspace_bytes(N, K); a
 *          workspace serves one call at a time (its header counts the chunks
 *          that are done). */
BL_API bl_status bitlinear_absmean(const void *W, int wdt, int64_t N, int64_t K, float *gamma,
                                   void *ws, size_t ws_bytes, void *stream);

/* The absmean scale (step 1, the same result as bitlinear_absmean) for
 * callers that cannot allocate device memory at the time they need it: for
 * example code whose device memory belongs to another runtime or pool that
 * hands out no raw buffers, or a service that reserves all its memory at
 * start-up and may not call cudaMalloc / cudaFree (which can synchronize the
 * device) afterwards.  The pages have no counterpart; this is a library
 * convenience.
 *   W      [N, K] fp32 or bf16, 16-byte aligned;  gamma [1] fp32 device output.
 *   Limit  N * K <= 2^28 elements (32768 chunks of 8192); larger sizes return
 *          BL_ERR_SCRATCH_LIMIT without launching anything.
 * The partial sums live in a 256 KiB device array owned by the library (held
 * on every GPU that loads it, until the process exits); nothing is allocated.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and keeps it, so make that first call
 * before any stream capture.  The kept address belongs to the device context
 * of that first call: after cudaDeviceReset it is stale, so a process that
 * resets a device must not call this entry point on it again.  Every call
 * shares the one array and resets its counter: calls whose kernels overlap on
 * the GPU (different streams, or different host threads) race and must be
 * serialized by the caller. */
BL_API bl_status bitlinear_absmean_noalloc(const void *W, int wdt, int64_t N, int64_t K, float *gamma,
                                           void *stream);

/* Ternarize and pack with a gamma that is already on the device (step 2-3 only;
 * for instance a gamma reduced across ranks).  [P3] §3.1 and [P5] "The
 * Ternary Weight Recipe" (W_q = clamp(round(W / (gamma + eps)), -1, 1));
 * [P3] §2.3 and §6.3 (formats).  Same arrays as above; `gamma` is an input
 * here. */
BL_API bl_status bitlinear_ternarize_pack(const void *W, int wdt, int64_t N, int64_t K,
                                   const float *gamma, float eps, int fmt, uint8_t *packed,
                                   int8_t *codes, void *stream);

/* 1-bit BitNet weights (the 1-bit variant of steps 1-3).  [P5] "The BitLinear
 * Recipe" steps 2 and 4: alpha = mean of the weights, a weight above alpha
 * becomes +1 and any other -1 (a weight equal to alpha gives -1, a reading:
 * the pages do not say), beta = mean |W| rescales the output.  alpha and beta
 * are fp64 sums in the same fixed order as gamma's (for alpha the terms are
 * w), divided by N K and rounded to fp32; beta equals the gamma of
 * bitlinear_absmean.  The forward then takes fmt = BL_PACK_B1 with beta in
 * place of gamma.
 *   W       [N, K] fp32 or bf16.
 *   packed  [N, bitlinear_packed_row_bytes(K, BL_PACK_B1)] uint8 output, or NULL.
 *   codes   [N, K] int8 output in {-1, +1}, or NULL (not both NULL).
 *   beta, alpha  [1] fp32 device outputs.
 *   ws      at least bitlinear_binarize_weights_workspace_bytes(N, K) (two
 *           fp64 partial sums per 8192-element chunk). */
BL_API size_t bitlinear_binarize_weights_workspace_bytes(int64_t N, int64_t K);
BL_API bl_status bitlinear_binarize_weights(const void *W, int wdt, int64_t N, int64_t K, uint8_t *packed,
                                         int8_t *codes, float *beta, float *alpha, void *ws, size_t ws_bytes,
                                         void *stream);

/* Pack int8 codes in {-1, 0, 1} (step 3).  [P3] §2.3, §6.3.
 *   codes  [N, K] int8; packed [N, row_bytes] uint8 output.
 *   ws     at least BL_WS_HEADER_BYTES; a code outside {-1, 0, 1} is packed
 *          as weight 0 and sets BL_ERR_BAD_CODE in the workspace flag.
 * With fmt = BL_PACK_B1 the codes must be -1 or +1; any other code packs as -1
 * and sets BL_ERR_BAD_CODE. */
BL_API bl_status bitlinear_pack(const int8_t *codes, int64_t N, int64_t K, int fmt, uint8_t *packed,
                         void *ws, size_t ws_bytes, void *stream);

/* Per-token absmax INT8 quantization (step 4).  [P3] §3.2, §5.2.
 *   x      [M, K] fp32 or bf16;  xq [M, K] int8 output;  scale [M] fp32 output. */
BL_API bl_status bitlinear_quantize_acts(const void *x, int xdt, int64_t M, int64_t K, int8_t *xq,
                                  float *scale, void *stream);

/* Pre-norm + step 4: LayerNorm of each token, then per-token absmax INT8.
 * [P5] "The BitLinear Recipe" step 1 (the input is quantized with absmax
 * scaling after LayerNorm); [P3] §5.5 (LayerNorm kept in high precision,
 * bf16 activations between layers).  Computes, for each token (row of x):
 * mu and the biased variance as fp64 sums in a fixed order (element k goes to
 * lane k mod 256, each lane adds its elements in turn, the 256 lane sums
 * combine by the stride-halving tree s = 128, ..., 1), r = 1 / sqrt(var + eps),
 * y = ((x - mu) r) ln_w + ln_b in fp64, rounded to fp32 and then to bf16, and
 * the INT8 codes of the bf16 y exactly as bitlinear_quantize_acts does.
 *   x      [M, K] fp32 or bf16 (16-byte aligned); ln_w, ln_b [K] fp32.
 *   eps    > 0 (PyTorch's LayerNorm default is 1e-5).
 *   y      [M, K] bf16 bits output of the LayerNorm, or NULL.
 *   xq     [M, K] int8 output;  scale [M] fp32 output.
 * Feeds bitlinear_forward with xdt = BL_I8. */
BL_API bl_status bitlinear_layernorm_quantize_acts(const void *x, int xdt, const float *ln_w, const float *ln_b,
                                                float eps, int64_t M, int64_t K, uint16_t *y, int8_t *xq,
                                                float *scale, void *stream);

/* BitLinear forward, y = dequant(x_q . W_q^T) (steps 4-6).
 * [P3] §4.2 (add / subtract / skip), §3.3 (INT32 accumulation), §5.3.
 *   packed  [N, row_bytes] from bitlinear_quantize_weights / bitlinear_pack
 *           (fmt BL_PACK_I2 | BL_PACK_T5), or from bitlinear_binarize_weights
 *           (fmt BL_PACK_B1: weights in {-1, +1}).
 *   gamma   [1] fp32 device pointer (beta for BL_PACK_B1).
 *   x       [M, K]: fp32 or bf16 (quantized inside; `scale` [M] is written),
 *           or int8 x_q (xdt = BL_I8; `scale` [M] is read).
 *   y       [M, N]: ydt = BL_F32 | BL_BF16, or BL_I32 for the raw INT32
 *           accumulators (no dequantization).
 *   ws      at least bitlinear_forward_workspace_bytes(M, N, K, fmt, xdt). */
BL_API bl_status bitlinear_forward(const uint8_t *packed, int fmt, const float *gamma, int64_t N,
                            int64_t K, const void *x, int xdt, float *scale, int64_t M, void *y,
                            int ydt, void *ws, size_t ws_bytes, void *stream);

/* Several BitLinear layers that share their input, in one call (for example
 * a block's Q, K and V projections).  [P3] §5.4 replaces the attention's Q, K,
 * V and output projections by BitLinear layers of the same input size; each
 * keeps its own gamma.  Row group g (group_rows[g] rows, at most
 * BL_MAX_ROW_GROUPS groups) is a weight matrix; its packed rows follow those of
 * group g - 1 in `packed`, gammas[g] is its gamma, and its outputs are the
 * columns sum(group_rows[0..g-1]) .. + group_rows[g] - 1 of y [M, sum of
 * group_rows].  The result equals bitlinear_forward per group: for at most 4
 * tokens one GEMV launch covers every group; otherwise the tokens are
 * quantized once and each group's tensor-core product writes its columns.
 *   gammas      [ngroups] fp32 device array.
 *   group_rows  [ngroups] host array, each >= 1.
 *   ws          at least bitlinear_forward_grouped_workspace_bytes(...). */
#define BL_MAX_ROW_GROUPS 8
BL_API size_t bitlinear_forward_grouped_workspace_bytes(int64_t M, int64_t ngroups, const int64_t *group_rows,
                                                     int64_t K, int fmt, int xdt);
BL_API bl_status bitlinear_forward_grouped(const uint8_t *packed, int fmt, const float *gammas, int64_t ngroups,
                                        const int64_t *group_rows, int64_t K, const void *x, int xdt,
                                        float *scale, int64_t M, void *y, int ydt, void *ws, size_t ws_bytes,
                                        void *stream);

/* STE backward of the BitLinear layer (the training side).  [P3] §5.3 (the
 * layer's F.linear(x_deq, W_eff) * gamma with W_eff = W_ternary + W -
 * W.detach(): the quantizer is the identity in the backward pass); [P5] "How
 * Gradients Flow: Fake Quantization and STE".  Both quantizers pass the
 * gradient straight through and gamma is a constant of the step, so for an
 * upstream gradient dy [M, N] (fp32 or bf16):
 *   dx [M, K] = gamma * dy . W_q        (bitlinear_backward_dx)
 *   dW [N, K] = gamma * dy^T . x_deq    (bitlinear_backward_dw),
 *   x_deq[m, k] = x_q[m, k] * s_m / 127 (the forward's codes and scales).
 * Both are fp64 sums in a fixed order rounded once to fp32: dx adds the rows
 * in chunks of 64 (each chunk from 0.0 in row order; chunk sums from 0.0 in
 * chunk order) then multiplies by gamma; dW adds (dy x_q) (s_m / 127) from
 * 0.0 in token order then multiplies by gamma.  A CUDA-core path for few
 * tokens: dx reads the packed weights once per two tokens.
 *   packed, fmt, gamma  as for bitlinear_forward (gamma: beta for BL_PACK_B1).
 *   dx    [M, K] fp32 output;  dw [N, K] fp32 output (16-byte aligned).
 *   ws    at least bitlinear_backward_dx_workspace_bytes(M, N, K, fmt). */
BL_API size_t bitlinear_backward_dx_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt);
BL_API bl_status bitlinear_backward_dx(const uint8_t *packed, int fmt, const float *gamma, int64_t N, int64_t K,
                                    const void *dy, int dydt, int64_t M, float *dx, void *ws, size_t ws_bytes,
                                    void *stream);
BL_API bl_status bitlinear_backward_dw(const void *dy, int dydt, const int8_t *xq, const float *scale,
                                    const float *gamma, int64_t M, int64_t N, int64_t K, float *dw,
                                    void *stream);

/* Failure-detection self test: launches the tensor-core kernel with its data
 * producer switched off and a wait limit of about a millisecond, so that its
 * bounded waits run out; the kernel then records BL_ERR_DEVICE_TIMEOUT in the
 * workspace flag, frees what it holds and exits (no memory is read or written
 * besides the flag).  Read the result with bitlinear_device_status.  The pages
 * have no counterpart; this tests the error path of every wait.
 *   ws  at least BL_WS_HEADER_BYTES + 8192 bytes. */
BL_API bl_status bitlinear_selftest_wait_timeout(void *ws, size_t ws_bytes, void *stream);

/* Synchronize `stream`, then read and clear the workspace's device flags.
 * Returns BL_OK, BL_ERR_DEVICE_TIMEOUT, BL_ERR_BAD_CODE or BL_ERR_CUDA. */
BL_API bl_status bitlinear_device_status(void *ws, void *stream);

/* A static description of a status code. */
BL_API const char *bitlinear_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
BL_API int bitlinear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
