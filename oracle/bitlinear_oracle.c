/*
 * bitlinear_oracle.c -- plain, slow, single-threaded CPU oracle for the
 * BitNet b1.58 BitLinear forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check of the graft entry
 * point and the CPU-baseline leg of bench.py use it.  It shares no code,
 * header, table or constant with the CUDA library; it is built by gcc without
 * fast-math (IEEE single/double, round-to-nearest-even, no FMA contraction).
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "QAT与BitNet：1-bit及1.58-bit量化训练解析" (kongchang.com)
 *   [P3] "BitNet b1.58深度解析：三值权重如何重塑大模型推理" (0539edu.com)
 *   [P5] "QAT and BitNet: A Deep Dive into 1-bit and 1.58-bit
 *         Quantization-Aware Training" (kongchang.com/en)
 *
 * What the pages leave open is fixed here by the plainest reading; every such
 * reading is listed next to the function that takes it.
 *
 * Parity pins: every function below is pinned by a CPU test against the
 * pages' worked examples, closed forms, exact arithmetic or brute force; none
 * is "parity unpinned".
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs single-precision float evaluation (FLT_EVAL_METHOD == 0)"
#endif

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_I8 2
#define ORC_I32 3

#define ORC_PACK_I2 0 /* 2 bits per weight, 4 weights per byte */
#define ORC_PACK_T5 1 /* 5 trits per byte, base 3 */
#define ORC_PACK_B1 2 /* 1 bit per weight, 8 weights per byte (1-bit BitNet) */

/* ------------------------------------------------------------------------ */
/* dtype helpers                                                            */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN -> quiet NaN). */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static float load_f(const void *p, int dt, int64_t i) {
  if (dt == ORC_F32) return ((const float *)p)[i];
  return orc_bf16_to_f32(((const uint16_t *)p)[i]);
}

/* ------------------------------------------------------------------------ */
/* Step 1: absmean scale gamma = mean(|W|) over the whole weight matrix.     */
/* [P1]/[P5] "The Ternary Weight Recipe" (gamma = w.abs().mean());           */
/* [P3] §3.1 (gamma = mean(|W|), one per weight matrix).                     */
/*                                                                          */
/* Reading (pages silent on summation order): the sum of |w| is taken in     */
/* fp64 in this fixed order, so that every implementation reaches the same  */
/* bits:                                                                    */
/*   - elements in row-major order e = n*K + k, T = N*K;                    */
/*   - chunk c holds e in [c*8192, (c+1)*8192);                             */
/*   - in chunk c, lane l (0..255) adds, in this order, the elements        */
/*     c*8192 + 2048*i + 8*l + j for i = 0..3, j = 0..7 (those below T),    */
/*     starting from 0.0;                                                   */
/*   - lane sums combine by the stride-halving tree p[l] += p[l+s],          */
/*     s = 128, 64, ..., 1; p[0] is the chunk sum;                          */
/*   - chunk sums, padded with 0.0 up to the next power of two P, combine   */
/*     by the same tree with s = P/2, ..., 1.                               */
/* gamma64 = S / T, and gamma is gamma64 rounded to fp32.                    */
/* ------------------------------------------------------------------------ */

#define ORC_CHUNK 8192
#define ORC_LANES 256

/* absval = 1: the terms are |w|; absval = 0: the terms are w (the signed  */
/* sum of the 1-bit variant below takes the same order).                    */
static double chunk_sum(const void *W, int dt, int64_t T, int64_t c,
                        int absval) {
  double p[ORC_LANES];
  for (int l = 0; l < ORC_LANES; ++l) {
    double acc = 0.0;
    for (int i = 0; i < 4; ++i)
      for (int j = 0; j < 8; ++j) {
        int64_t e = c * ORC_CHUNK + 2048 * (int64_t)i + 8 * (int64_t)l + j;
        if (e < T) {
          float w = load_f(W, dt, e);
          acc += (double)(absval ? fabsf(w) : w);
        }
      }
    p[l] = acc;
  }
  for (int s = ORC_LANES / 2; s >= 1; s /= 2)
    for (int l = 0; l < s; ++l) p[l] += p[l + s];
  return p[0];
}

static double fixed_order_sum(const void *W, int dt, int64_t N, int64_t K,
                              int absval) {
  int64_t T = N * K;
  if (T <= 0) return 0.0;
  int64_t C = (T + ORC_CHUNK - 1) / ORC_CHUNK;
  int64_t P = 1;
  while (P < C) P *= 2;
  double *q = (double *)calloc((size_t)P, sizeof(double));
  if (!q) return NAN;
  for (int64_t c = 0; c < C; ++c) q[c] = chunk_sum(W, dt, T, c, absval);
  for (int64_t s = P / 2; s >= 1; s /= 2)
    for (int64_t c = 0; c < s; ++c) q[c] += q[c + s];
  double S = q[0];
  free(q);
  return S;
}

double orc_absmean_sum(const void *W, int dt, int64_t N, int64_t K) {
  return fixed_order_sum(W, dt, N, K, 1);
}

double orc_signed_sum(const void *W, int dt, int64_t N, int64_t K) {
  return fixed_order_sum(W, dt, N, K, 0);
}

float orc_gamma(const void *W, int dt, int64_t N, int64_t K) {
  double S = orc_absmean_sum(W, dt, N, K);
  double g = S / (double)(N * K);
  return (float)g;
}

/* ------------------------------------------------------------------------ */
/* Step 2: ternarize, W_q = clamp(round(W / (gamma + eps)), -1, 1).          */
/* [P1]/[P5] "The Ternary Weight Recipe" (ternary_weights, eps = 1e-5);      */
/* [P3] §3.1 (W_norm = W / gamma, round, clamp to [-1, 1]).                  */
/* Readings: d = gamma + eps is one fp32 add; the division is one IEEE fp32  */
/* division; round is half-to-even (torch.round), so a ratio of exactly 0.5 */
/* goes to 0, which agrees with the page's "|w| <= gamma/2 -> 0".            */
/* ------------------------------------------------------------------------ */

void orc_ternarize(const void *W, int dt, int64_t N, int64_t K, float gamma,
                   float eps, int8_t *codes) {
  float d = gamma + eps;
  for (int64_t e = 0; e < N * K; ++e) {
    float r = load_f(W, dt, e) / d;
    float q = nearbyintf(r);
    if (q > 1.0f) q = 1.0f;
    if (q < -1.0f) q = -1.0f;
    codes[e] = (int8_t)q;
  }
}

/* ------------------------------------------------------------------------ */
/* Step 3: packing.                                                         */
/* [P1]/[P5] "Why Is It Called 1.58 Bits?" (2 bits per weight; five trits   */
/* per byte, 3^5 = 243 <= 256); [P3] §2.3 and §6.3 (codes "00, 01, 10",     */
/* four weights per byte; five per byte by table lookup or bit operations). */
/* Readings: code = q + 1 (-1 -> 00, 0 -> 01, +1 -> 10), first weight in    */
/* the least significant bits; base 3 byte = sum (q_i + 1) * 3^i with the   */
/* first weight least significant; each row is padded to a multiple of 16  */
/* bytes with digits that encode weight 0 (a whole pad byte is 0x55 in the  */
/* 2-bit format, 121 in base 3).                                            */
/* ------------------------------------------------------------------------ */

/* The 1-bit format (ORC_PACK_B1) follows the same byte order: bit i of     */
/* byte j holds weight 8 j + i, 1 for +1 and 0 for -1; pad bits are 0 (the  */
/* pages give 8 weights per byte and no bit order, so this is a reading).   */

static int per_byte(int fmt) {
  return fmt == ORC_PACK_I2 ? 4 : (fmt == ORC_PACK_T5 ? 5 : 8);
}

int64_t orc_packed_row_bytes(int64_t K, int fmt) {
  int64_t per = per_byte(fmt);
  int64_t used = (K + per - 1) / per;
  return (used + 15) / 16 * 16;
}

/* returns 0, or -1 if a code is outside {-1, 0, 1} ({-1, 1} for 1 bit) */
int orc_pack(const int8_t *codes, int64_t N, int64_t K, int fmt,
             uint8_t *packed) {
  int per = per_byte(fmt);
  int64_t rb = orc_packed_row_bytes(K, fmt);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < rb; ++j) {
      unsigned byte = 0, pow3 = 1;
      for (int i = 0; i < per; ++i) {
        int64_t k = j * per + i;
        int q = 0;
        if (k < K) {
          q = codes[n * K + k];
          if (q < -1 || q > 1) return -1;
          if (fmt == ORC_PACK_B1 && q == 0) return -1;
        }
        if (fmt == ORC_PACK_B1) {
          if (q > 0) byte |= 1u << i;
          continue;
        }
        unsigned digit = (unsigned)(q + 1);
        if (fmt == ORC_PACK_I2)
          byte |= digit << (2 * i);
        else
          byte += digit * pow3;
        pow3 *= 3;
      }
      packed[n * rb + j] = (uint8_t)byte;
    }
  return 0;
}

/* Inverse of orc_pack.  Returns 0, -1 for an invalid code (2-bit code 11 or
 * a base-3 byte >= 243), -2 for a padding digit that is not weight 0. */
int orc_unpack(const uint8_t *packed, int64_t N, int64_t K, int fmt,
               int8_t *codes) {
  int per = per_byte(fmt);
  int64_t rb = orc_packed_row_bytes(K, fmt);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < rb; ++j) {
      unsigned byte = packed[n * rb + j];
      if (fmt == ORC_PACK_T5 && byte >= 243) return -1;
      for (int i = 0; i < per; ++i) {
        unsigned digit;
        if (fmt == ORC_PACK_B1) {
          unsigned bit = (byte >> i) & 1u;
          int64_t kb = j * per + i;
          if (kb < K)
            codes[n * K + kb] = (int8_t)(bit ? 1 : -1);
          else if (bit != 0)
            return -2;
          continue;
        }
        if (fmt == ORC_PACK_I2) {
          digit = (byte >> (2 * i)) & 3u;
          if (digit == 3) return -1;
        } else {
          digit = byte % 3;
          byte /= 3;
        }
        int64_t k = j * per + i;
        if (k < K)
          codes[n * K + k] = (int8_t)((int)digit - 1);
        else if (digit != 1)
          return -2;
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 4: per-token absmax INT8 activation quantization.                   */
/* [P3] §3.2 (scale = max|x| per token; x_q = clamp(round(x/scale*127),      */
/* -127, 127)) and §5.2 (activation_quantize_int8 floors the scale at 1e-6). */
/* Readings: a token is one row of x over K; s = max(max|x|, 1e-6); the     */
/* quotient x/s is one fp32 division, then one fp32 multiply by 127, then  */
/* round half-to-even; the range is symmetric, -128 never occurs.           */
/* ------------------------------------------------------------------------ */

void orc_act_quant(const void *x, int dt, int64_t M, int64_t K, int8_t *xq,
                   float *scale) {
  for (int64_t m = 0; m < M; ++m) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(load_f(x, dt, m * K + k));
      if (a > amax) amax = a;
    }
    float s = amax > 1e-6f ? amax : 1e-6f;
    scale[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      float t = load_f(x, dt, m * K + k) / s;
      t = t * 127.0f;
      float q = nearbyintf(t);
      if (q > 127.0f) q = 127.0f;
      if (q < -127.0f) q = -127.0f;
      xq[m * K + k] = (int8_t)q;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Step 5: ternary x INT8 matrix product with INT32 accumulation,            */
/* acc[m][n] = sum_k W_q[n][k] * x_q[m][k]  (y = x W^T as in F.linear).      */
/* [P3] §4.2 (y_i = sum_j w_ij x_j: add for +1, subtract for -1, skip 0);   */
/* [P3] §3.3 (INT32 accumulator).                                           */
/* ------------------------------------------------------------------------ */

void orc_matmul_i32(const int8_t *codes, const int8_t *xq, int64_t M,
                    int64_t N, int64_t K, int32_t *acc) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int32_t s = 0;
      for (int64_t k = 0; k < K; ++k)
        s += (int32_t)codes[n * K + k] * (int32_t)xq[m * K + k];
      acc[m * N + n] = s;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 6: dequantize, y = acc * gamma * s_m / 127.                          */
/* [P1]/[P5] "The BitLinear Recipe" step 4 (rescale by both factors);        */
/* [P3] §3.2 (x is x_q * scale / 127) and §5.3 (output multiplied by gamma). */
/* Readings: the weight factor is gamma itself (not gamma + eps); the order */
/* is c_m = (gamma * s_m) / 127 in fp32, then y = (float)acc * c_m; a bf16  */
/* output is that fp32 value rounded to nearest even.                       */
/* ------------------------------------------------------------------------ */

void orc_dequant(const int32_t *acc, float gamma, const float *scale,
                 int64_t M, int64_t N, void *y, int ydt) {
  for (int64_t m = 0; m < M; ++m) {
    float c = (gamma * scale[m]) / 127.0f;
    for (int64_t n = 0; n < N; ++n) {
      int64_t i = m * N + n;
      float v = (float)acc[i] * c;
      if (ydt == ORC_F32)
        ((float *)y)[i] = v;
      else if (ydt == ORC_BF16)
        ((uint16_t *)y)[i] = orc_f32_to_bf16(v);
      else
        ((int32_t *)y)[i] = acc[i];
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Whole forward: unpack, quantize activations (or take x_q and its scales  */
/* as given when xdt is ORC_I8), multiply, dequantize.  The same arguments  */
/* as the library's forward entry point.  Returns 0, or the unpack status. */
/* ------------------------------------------------------------------------ */

int orc_forward(const uint8_t *packed, int fmt, float gamma, int64_t N,
                int64_t K, const void *x, int xdt, float *scale, int64_t M,
                void *y, int ydt) {
  int8_t *codes = (int8_t *)malloc((size_t)(N * K));
  int8_t *xq = (int8_t *)malloc((size_t)(M * K));
  int32_t *acc = (int32_t *)malloc((size_t)(M * N) * sizeof(int32_t));
  int rc = -3;
  if (!codes || !xq || !acc) goto out;
  rc = orc_unpack(packed, N, K, fmt, codes);
  if (rc != 0) goto out;
  if (xdt == ORC_I8)
    memcpy(xq, x, (size_t)(M * K));
  else
    orc_act_quant(x, xdt, M, K, xq, scale);
  orc_matmul_i32(codes, xq, M, N, K, acc);
  orc_dequant(acc, gamma, scale, M, N, y, ydt);
out:
  free(codes);
  free(xq);
  free(acc);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* 1-bit BitNet weights, used to reproduce the pages' five-weight example.   */
/* [P1]/[P5] "The BitLinear Recipe" step 2 (alpha = mean of the weights,    */
/* above alpha -> +1, below -> -1) and step 4 (beta = mean |W|); "A         */
/* Five-Weight Example".                                                    */
/* Reading: a weight equal to alpha maps to -1 (the pages do not say);      */
/* beta is the uncentred mean |w| (the example's 0.57 requires it).         */
/* ------------------------------------------------------------------------ */

void orc_onebit(const float *w, int64_t n, int8_t *b, float *alpha,
                float *beta) {
  double s = 0.0, sa = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    s += (double)w[i];
    sa += (double)fabsf(w[i]);
  }
  float a = (float)(s / (double)n);
  *alpha = a;
  *beta = (float)(sa / (double)n);
  for (int64_t i = 0; i < n; ++i) b[i] = (int8_t)(w[i] > a ? 1 : -1);
}

/* ------------------------------------------------------------------------ */
/* 1-bit BitNet weights for a whole matrix (the 1-bit variant of steps 1-2). */
/* [P1]/[P5] "The BitLinear Recipe" step 2 (alpha = mean of the weights;    */
/* a weight above alpha becomes +1, one below -1) and step 4 (beta = mean   */
/* |W| rescales the output, in place of gamma).                             */
/* Readings: alpha and beta are fp64 sums in the fixed order of step 1 (for */
/* alpha the terms are w, for beta |w|), divided by N K and rounded to fp32; */
/* beta is therefore gamma.  A weight equal to alpha maps to -1 (the pages  */
/* do not say); w > alpha in fp32 is the sign of w - alpha, since the fp32  */
/* difference of two distinct floats is never 0.  The forward is then steps */
/* 4-6 unchanged with codes in {-1, +1} and beta as the weight factor.      */
/* ------------------------------------------------------------------------ */

void orc_binarize_weights(const void *W, int dt, int64_t N, int64_t K,
                          float *alpha, float *beta, int8_t *codes) {
  double S = orc_signed_sum(W, dt, N, K);
  float a = (float)(S / (double)(N * K));
  *alpha = a;
  *beta = orc_gamma(W, dt, N, K);
  if (codes != NULL)
    for (int64_t e = 0; e < N * K; ++e)
      codes[e] = (int8_t)(load_f(W, dt, e) > a ? 1 : -1);
}

/* ------------------------------------------------------------------------ */
/* STE backward of the BitLinear layer (the training side).                 */
/* [P3] §5.3 (BitLinear: out = F.linear(x_deq, W_eff) * gamma with W_eff =  */
/* W_ternary + W - W.detach(), the straight-through estimator taking the    */
/* quantizer as the identity in the backward pass); [P1]/[P5] "How          */
/* Gradients Flow: Fake Quantization and STE" (forward with the quantized   */
/* values, backward as if rounding were the identity).                     */
/* Readings: both quantizers pass the gradient straight through and gamma  */
/* is a constant of the step (no gradient through mean |W|), so for an     */
/* upstream gradient dy [M, N]:                                             */
/*   dx[m][k] = gamma * sum_n dy[m][n] * W_q[n][k]                          */
/*   dW[n][k] = gamma * sum_m dy[m][n] * x_deq[m][k],                       */
/*              x_deq[m][k] = x_q[m][k] * s_m / 127 (the forward's codes).  */
/* dx: the pages fix no summation order, so none is taken: S is the exact   */
/* real sum of the terms +dy, -dy or nothing (add / subtract / skip),       */
/* rounded once to fp64 (nearest, ties to even); dx = fp32(gamma * S) with  */
/* the product in fp64.  Any summation order gives the same S.             */
/* dW: c_m = s_m / 127, each term is (dy[m][n] * x_q[m][k]) * c_m, added    */
/* from 0.0 in token order (the plain order of the sum) into T;            */
/* dW = fp32(gamma * T).  Gradients are finite.                            */
/* ------------------------------------------------------------------------ */

/* Exact sum of fp32 values.  Every finite fp32 value is an integer multiple */
/* of 2^-149 (the smallest subnormal) and below 2^128, i.e. an integer below */
/* 2^277 in that unit; 2^31 terms stay below 2^308.  The integer is held as  */
/* ORC_XLIMBS little-endian base-2^32 digits in int64 slots, so a digit may   */
/* run ahead of its carries for 2^29 additions (each adds less than 2^32).   */
#define ORC_XLIMBS 10
typedef struct {
  int64_t d[ORC_XLIMBS];
  int64_t adds;
} orc_xsum;

static void xsum_normalize(orc_xsum *a) {
  for (int i = 0; i + 1 < ORC_XLIMBS; ++i) {
    int64_t low = a->d[i] & (int64_t)0xffffffff;
    int64_t carry = (a->d[i] - low) / ((int64_t)1 << 32); /* exact: floor */
    a->d[i] = low;
    a->d[i + 1] += carry;
  }
  a->adds = 0;
}

/* a += sign * v exactly (sign = +1 or -1). */
static void xsum_add(orc_xsum *a, float v, int sign) {
  uint32_t u;
  memcpy(&u, &v, sizeof u);
  uint32_t e = (u >> 23) & 0xffu, f = u & 0x7fffffu;
  uint64_t mant = e ? (f | 0x800000u) : f;
  int shift = e ? (int)e - 1 : 0; /* value = mant * 2^(shift - 149) */
  if (u >> 31) sign = -sign;
  uint64_t t = mant << (shift & 31);
  int i = shift >> 5;
  int64_t lo = (int64_t)(t & 0xffffffffu), hi = (int64_t)(t >> 32);
  a->d[i] += sign * lo;
  a->d[i + 1] += sign * hi;
  if (++a->adds == ((int64_t)1 << 29)) xsum_normalize(a);
}

/* The exact sum rounded once to fp64 (nearest, ties to even). */
static double xsum_round(orc_xsum *a) {
  xsum_normalize(a);
  double sign = 1.0;
  uint32_t mag[ORC_XLIMBS];
  if (a->d[ORC_XLIMBS - 1] < 0) { /* magnitude = 0 - a, digit by digit */
    sign = -1.0;
    int64_t borrow = 0;
    for (int i = 0; i < ORC_XLIMBS; ++i) {
      int64_t v = -a->d[i] - borrow;
      borrow = v < 0;
      mag[i] = (uint32_t)(v + (borrow ? ((int64_t)1 << 32) : 0));
    }
  } else {
    for (int i = 0; i < ORC_XLIMBS; ++i) mag[i] = (uint32_t)a->d[i];
  }
  int top = -1; /* index of the highest set bit */
  for (int i = ORC_XLIMBS - 1; i >= 0 && top < 0; --i)
    if (mag[i])
      for (int b = 31; b >= 0; --b)
        if ((mag[i] >> b) & 1u) { top = 32 * i + b; break; }
  if (top < 0) return 0.0;
#define XBIT(n) ((mag[(n) >> 5] >> ((n) & 31)) & 1u)
  if (top <= 52) { /* fits in the fp64 significand: exact */
    uint64_t v = 0;
    for (int n = top; n >= 0; --n) v = (v << 1) | XBIT(n);
    return sign * ldexp((double)v, -149);
  }
  uint64_t sig = 0;
  for (int n = top; n >= top - 52; --n) sig = (sig << 1) | XBIT(n);
  int round_bit = (int)XBIT(top - 53), sticky = 0;
  for (int n = top - 54; n >= 0 && !sticky; --n) sticky = (int)XBIT(n);
#undef XBIT
  int exp = top - 52 - 149;
  if (round_bit && (sticky || (sig & 1u))) {
    ++sig;
    if (sig == ((uint64_t)1 << 53)) { sig >>= 1; ++exp; }
  }
  return sign * ldexp((double)sig, exp);
}

void orc_backward_dx(const int8_t *codes, int64_t N, int64_t K,
                     const void *dy, int dydt, int64_t M, float gamma,
                     float *dx) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      orc_xsum acc;
      memset(&acc, 0, sizeof acc);
      for (int64_t n = 0; n < N; ++n) {
        int q = codes[n * K + k];
        if (q == 1)
          xsum_add(&acc, load_f(dy, dydt, m * N + n), +1);
        else if (q == -1)
          xsum_add(&acc, load_f(dy, dydt, m * N + n), -1);
      }
      double S = xsum_round(&acc);
      dx[m * K + k] = (float)((double)gamma * S);
    }
}

void orc_backward_dw(const void *dy, int dydt, const int8_t *xq,
                     const float *scale, float gamma, int64_t M, int64_t N,
                     int64_t K, float *dw) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      double T = 0.0;
      for (int64_t m = 0; m < M; ++m) {
        double c = (double)scale[m] / 127.0;
        double t = (double)load_f(dy, dydt, m * N + n) * (double)xq[m * K + k];
        T += t * c;
      }
      dw[n * K + k] = (float)((double)gamma * T);
    }
}

/* ------------------------------------------------------------------------ */
/* Pre-norm + step 4: LayerNorm of each token, then per-token absmax INT8.  */
/* [P5] "The BitLinear Recipe" step 1 (the input is quantized with absmax   */
/* scaling after LayerNorm, whose output has a stable scale); [P3] §5.5    */
/* (the training configuration keeps LayerNorm in high precision, bf16 for */
/* the activations between layers).                                       */
/* Readings: LayerNorm over a token's K values with elementwise fp32      */
/* weight g and bias b and eps added to the (biased) variance; the mean    */
/* and the variance are sums in fp64 in a fixed order -- lane l in         */
/* [0, 256) adds the elements l, l + 256, l + 512, ... of the token in turn */
/* from 0.0, and the 256 lane sums combine by the stride-halving tree      */
/* p[l] += p[l + s], s = 128, ..., 1 (lanes with no element hold 0.0) --   */
/* mu = S1 / K, var = S2 / K with S2 the sum of (x - mu)^2 in that order,  */
/* r = 1 / sqrt(var + eps) (fp64, correctly rounded); y = ((x - mu) r) g + b */
/* in fp64, one rounding per operation, then rounded to fp32 and to bf16;  */
/* the bf16 y is then quantized exactly as orc_act_quant does.             */
/* ------------------------------------------------------------------------ */

static double token_tree_sum(const double *lane_sum) {
  double p[256];
  for (int l = 0; l < 256; ++l) p[l] = lane_sum[l];
  for (int s = 128; s >= 1; s >>= 1)
    for (int l = 0; l < s; ++l) p[l] = p[l] + p[l + s];
  return p[0];
}

void orc_layernorm(const void *x, int dt, const float *g, const float *b, float eps, int64_t M,
                   int64_t K, uint16_t *y) {
  double lane[256];
  for (int64_t m = 0; m < M; ++m) {
    for (int l = 0; l < 256; ++l) {
      double acc = 0.0;
      for (int64_t k = l; k < K; k += 256) acc = acc + (double)load_f(x, dt, m * K + k);
      lane[l] = acc;
    }
    const double mu = token_tree_sum(lane) / (double)K;
    for (int l = 0; l < 256; ++l) {
      double acc = 0.0;
      for (int64_t k = l; k < K; k += 256) {
        const double d = (double)load_f(x, dt, m * K + k) - mu;
        acc = acc + d * d;
      }
      lane[l] = acc;
    }
    const double var = token_tree_sum(lane) / (double)K;
    const double r = 1.0 / sqrt(var + (double)eps);
    for (int64_t k = 0; k < K; ++k) {
      const double v = (((double)load_f(x, dt, m * K + k) - mu) * r) * (double)g[k] + (double)b[k];
      y[m * K + k] = orc_f32_to_bf16((float)v);
    }
  }
}

void orc_layernorm_quant(const void *x, int dt, const float *g, const float *b, float eps,
                         int64_t M, int64_t K, uint16_t *y, int8_t *xq, float *scale) {
  orc_layernorm(x, dt, g, b, eps, M, K, y);
  orc_act_quant(y, ORC_BF16, M, K, xq, scale);
}
