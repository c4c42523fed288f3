// bl_gemv.cu -- decode GEMV for a few tokens: y = dequant(x_q . W_q^T).
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §4.2: with weights in
// {-1, 0, +1} the product is add / subtract / skip, and decode is bound by
// moving the weights (§1, §4.1).  This kernel streams each packed row once
// with 128-bit coalesced loads and does the add / subtract / skip with integer
// dot-product instructions on INT8 activations:
//   2-bit:  sum_k (d_k - 1) x_k = sum_k d_k x_k - sum_k x_k, d_k in {0,1,2} the
//           stored digits; four dp4a per 32-bit word take the digits with
//           masks, against activations stored in shared memory in the matching
//           interleaved order; sum_k x_k is reduced once per token.
//   base 3: a 256-entry shared table maps a byte to its five signed weights
//           (entries 243..255, invalid bytes, hold zeros); two dp4a per byte.
// The per-token activation quantization (absmax INT8, "§3.2") is done in each
// CTA's prologue while the first packed loads are in flight; INT32 partial
// sums meet by warp reduction; the dequantization y = acc * (gamma s / 127)
// ("§5.3") is fused into the store.
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kGemvThreads = 768;  // one CTA per SM: the token prologue runs once per SM
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvDepth = 6;  // row-block items whose loads are in flight per warp

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Activation bytes per token in shared memory for one packed row of rowbytes.
__host__ __device__ inline int64_t gemv_x_bytes(int fmt, int64_t rowbytes) {
  return fmt == BL_PACK_I2 ? rowbytes * 4 : rowbytes * 8;
}

// dp4a with unsigned bytes in a and signed bytes in b.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <int XDT>
__device__ __forceinline__ float load_x(const void* x, int64_t i) {
  if constexpr (XDT == BL_I8) {
    return static_cast<float>(static_cast<const int8_t*>(x)[i]);
  } else {
    return load_elem<XDT>(x, i);
  }
}

// Shared activation layout (per token), chosen so that the 32 lanes of a warp,
// which work on 32 consecutive 16-byte segments s of a row, read consecutive
// shared words (no bank conflicts):
//   2-bit:  segment s, packed word w (0..3): 16 bytes at ((w * segs) + s) * 16,
//           byte 4j + b = x[64 s + 16 w + 4 b + j]  (the digit order of the word)
//   base 3: segment s, packed byte wb = 4 w + b: 8 bytes at ((wb * segs) + s) * 8,
//           {x[5 p], .., x[5 p + 3]} and {x[5 p + 4], 0, 0, 0}, p = 16 s + wb
__device__ __forceinline__ uint32_t x_slot(int fmt, uint32_t k, uint32_t segs) {  // k < 2^20
  if (fmt == BL_PACK_I2) {
    const uint32_t g = k >> 4, r = k & 15;            // packed word g, digit r
    const uint32_t s = g >> 2, w = g & 3, j = r & 3, b = r >> 2;
    return ((w * segs) + s) * 16 + 4 * j + b;
  } else {
    const uint32_t p = k / 5, i = k - 5 * p;          // packed byte p, digit i
    const uint32_t s = p >> 4, wb = p & 15;
    return ((wb * segs) + s) * 8 + (i < 4 ? i : 4);
  }
}

template <int FMT, int MT, int XDT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                void* __restrict__ y, int ydt, int write_scale) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int64_t xb = gemv_x_bytes(FMT, rowbytes);
  uint8_t* xs = smem;                                     // [MT][xb]
  uint2* lut = reinterpret_cast<uint2*>(smem + MT * xb);  // base 3 only
  __shared__ float red_f[MT][kGemvWarps];
  __shared__ int red_i[MT][kGemvWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t segs = static_cast<uint32_t>(rowbytes >> 4);
  const uint32_t nb = (segs + 31) >> 5;  // 32-segment blocks per row
  const int64_t TW = static_cast<int64_t>(gridDim.x) * kGemvWarps;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kGemvWarps + warp;
  const int64_t nrows = r0 < N ? (N - 1 - r0) / TW + 1 : 0;

  // The warp's items are (row r0 + ri TW, 32-segment block blk), in order;
  // the lane's segment of an item is 32 blk + lane.  Two cursors walk them:
  // one for the loads in flight, one for the item being reduced.
  int64_t l_ri = 0;
  uint32_t l_blk = 0;
  const uint8_t* l_row = packed + r0 * rowbytes;
  auto load_next = [&](uint4& dst) {
    const uint32_t s = 32 * l_blk + lane;
    if (s < segs) dst = ld_stream(reinterpret_cast<const uint4*>(l_row) + s);
    if (++l_blk == nb) {
      l_blk = 0;
      ++l_ri;
      l_row += TW * rowbytes;
    }
  };

  // 1. the first kGemvDepth items' loads go out before the prologue
  uint4 buf[kGemvDepth];
#pragma unroll
  for (int d = 0; d < kGemvDepth; ++d) {
    buf[d] = make_uint4(0, 0, 0, 0);
    if (l_ri < nrows) load_next(buf[d]);
  }

  // 2. prologue: zero the activation area, per-token absmax, then scatter the
  //    INT8 codes into the layout above.
  {
    uint4* z = reinterpret_cast<uint4*>(xs);
    for (int64_t i = threadIdx.x; i < MT * xb / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  }
  if constexpr (FMT == BL_PACK_T5) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      uint32_t lo = 0, hi = 0;
      if (b < 243) {
        int v = b;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const uint32_t w = static_cast<uint8_t>(static_cast<int8_t>(v % 3 - 1));
          v /= 3;
          if (i < 4) lo |= w << (8 * i);
          else hi = w;
        }
      }
      lut[b] = make_uint2(lo, hi);
    }
  }
  const bool vec = (K % 8) == 0;
  float s_tok[MT];
  if constexpr (XDT != BL_I8) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float amax = 0.0f;
      if (vec) {
        for (int64_t v = threadIdx.x; v < K / 8; v += blockDim.x) {
          float e[8];
          load8_aligned<XDT>(x, m * K + 8 * v, e);
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[j]));
        }
      } else {
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(load_x<XDT>(x, m * K + k)));
      }
      amax = warp_maxf(amax);
      if (lane == 0) red_f[m][warp] = amax;
    }
  }
  __syncthreads();  // zeroed activations, table and per-warp maxima are visible
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if constexpr (XDT != BL_I8) {
      float a = red_f[m][0];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, red_f[m][w]);
      s_tok[m] = fmaxf(a, 1e-6f);
    } else {
      s_tok[m] = __ldg(scale + m);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int part = 0;
    uint8_t* xm = xs + m * xb;
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok[m]);
    if (vec) {
      for (int64_t v = threadIdx.x; v < K / 8; v += blockDim.x) {
        int q[8];
        if constexpr (XDT == BL_I8) {
          const uint2 raw = __ldg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + 8 * v));
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
        } else {
          float e[8];
          load8_aligned<XDT>(x, m * K + 8 * v, e);
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = quant_act_fast(e[j], s_tok[m], c127);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          xm[x_slot(FMT, static_cast<uint32_t>(8 * v + j), segs)] = static_cast<uint8_t>(q[j]);
          part += q[j];
        }
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const int q = (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[m * K + k])
                                     : quant_act_fast(load_x<XDT>(x, m * K + k), s_tok[m], c127);
        xm[x_slot(FMT, static_cast<uint32_t>(k), segs)] = static_cast<uint8_t>(q);
        part += q;
      }
    }
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0) red_i[m][warp] = part;
  }
  __syncthreads();  // activations and per-warp sums are visible
  const float g = __ldg(gamma);
  float cfac[MT];
  int corr[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) t += red_i[m][w];
    corr[m] = (FMT == BL_PACK_I2) ? t : 0;  // 2-bit digits are q + 1: subtract sum x once
    cfac[m] = dequant_factor(g, s_tok[m]);
    if (XDT != BL_I8 && write_scale && blockIdx.x == 0 && threadIdx.x == 0) scale[m] = s_tok[m];
  }

  // 3. stream the items, kGemvDepth loads always in flight.  2-bit: the digit
  //    of weight position j of each byte is taken in place, w & (3 << 2j), so
  //    each byte holds d 4^j; accumulator j collects 4^j sum d x, and the
  //    factor comes off exactly at the end of the row.
  int acc[MT], acc1[MT], acc2[MT], acc3[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = acc1[m] = acc2[m] = acc3[m] = 0;
  int64_t c_ri = 0;
  uint32_t c_blk = 0;
  while (c_ri < nrows) {
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d) {
      if (c_ri >= nrows) break;
      const uint4 cur = buf[d];
      if (l_ri < nrows) load_next(buf[d]);
      const uint32_t s = 32 * c_blk + lane;
      if (s < segs) {
        const uint32_t wd[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          if constexpr (FMT == BL_PACK_I2 && MT == 1) {
            const uint32_t c0 = wd[w] & 0x03030303u, c1 = wd[w] & 0x0c0c0c0cu;
            const uint32_t c2 = wd[w] & 0x30303030u, c3 = wd[w] & 0xc0c0c0c0u;
            const uint4 X = *reinterpret_cast<const uint4*>(xs + ((w * segs) + s) * 16);
            acc[0] = dp4a_us(c0, X.x, acc[0]);
            acc1[0] = dp4a_us(c1, X.y, acc1[0]);
            acc2[0] = dp4a_us(c2, X.z, acc2[0]);
            acc3[0] = dp4a_us(c3, X.w, acc3[0]);
          } else if constexpr (FMT == BL_PACK_I2) {  // several tokens: digits shifted down once
            const uint32_t c0 = wd[w] & 0x03030303u, c1 = (wd[w] >> 2) & 0x03030303u;
            const uint32_t c2 = (wd[w] >> 4) & 0x03030303u, c3 = (wd[w] >> 6) & 0x03030303u;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const uint4 X = *reinterpret_cast<const uint4*>(xs + m * xb + ((w * segs) + s) * 16);
              acc[m] = __dp4a(static_cast<int>(c0), static_cast<int>(X.x), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c1), static_cast<int>(X.y), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c2), static_cast<int>(X.z), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c3), static_cast<int>(X.w), acc[m]);
            }
          } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const uint2 Lw = lut[(wd[w] >> (8 * b)) & 0xffu];
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const uint2 X = *reinterpret_cast<const uint2*>(xs + m * xb + (((4 * w + b) * segs) + s) * 8);
                acc[m] = __dp4a(static_cast<int>(Lw.x), static_cast<int>(X.x), acc[m]);
                acc[m] = __dp4a(static_cast<int>(Lw.y), static_cast<int>(X.y), acc[m]);
              }
            }
          }
        }
      }
      if (c_blk == nb - 1) {  // the row is complete: reduce, dequantize, store
        const int64_t r = r0 + c_ri * TW;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int lane_sum = acc[m] + (acc1[m] >> 2) + (acc2[m] >> 4) + (acc3[m] >> 6);
          const int a = __reduce_add_sync(0xffffffffu, lane_sum) - corr[m];
          acc[m] = acc1[m] = acc2[m] = acc3[m] = 0;
          if (lane == 0) {
            const int64_t o = m * N + r;
            if (ydt == BL_I32)
              static_cast<int32_t*>(y)[o] = a;
            else if (ydt == BL_F32)
              static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cfac[m]);
            else
              static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cfac[m]));
          }
        }
        c_blk = 0;
        ++c_ri;
      } else {
        ++c_blk;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
int gemv_max_tokens(int fmt, int64_t rowbytes) {
  const int64_t xb = gemv_x_bytes(fmt, rowbytes);
  const int64_t budget = kGemvSmemBudget - (fmt == BL_PACK_T5 ? 256 * 8 : 0);
  int64_t mt = budget / xb;
  if (mt > kGemvMaxTokens) mt = kGemvMaxTokens;
  return static_cast<int>(mt);
}

template <int FMT, int MT, int XDT>
static cudaError_t launch_gemv_t(const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                 int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                 int write_scale, cudaStream_t st) {
  auto kern = gemv_kernel<FMT, MT, XDT>;
  const size_t smem = static_cast<size_t>(MT * gemv_x_bytes(FMT, rowbytes)) + (FMT == BL_PACK_T5 ? 256 * 8 : 0);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGemvSmemBudget));
  if (e != cudaSuccess) return e;
  const int sms = device_sms();
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t need = (N + kGemvWarps - 1) / kGemvWarps;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  kern<<<static_cast<unsigned>(grid), kGemvThreads, smem, st>>>(packed, rowbytes, gamma, N, K, x, scale,
                                                                 y, ydt, write_scale);
  return cudaGetLastError();
}

template <int FMT, int XDT>
static cudaError_t launch_gemv_mt(int mt, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, cudaStream_t st) {
  switch (mt) {
    case 1: return launch_gemv_t<FMT, 1, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, st);
    case 2: return launch_gemv_t<FMT, 2, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, st);
    case 3: return launch_gemv_t<FMT, 3, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, st);
    default: return launch_gemv_t<FMT, 4, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, st);
  }
}

// Runs the GEMV over all M tokens in groups that fit in shared memory.
cudaError_t launch_gemv(const uint8_t* packed, int fmt, const float* gamma, int64_t N, int64_t K,
                        const void* x, int xdt, float* scale, int64_t M, void* y, int ydt,
                        cudaStream_t st) {
  const int64_t rowbytes = (fmt == BL_PACK_I2) ? ((K + 3) / 4 + 15) / 16 * 16 : ((K + 4) / 5 + 15) / 16 * 16;
  const int mt_max = gemv_max_tokens(fmt, rowbytes);
  if (mt_max < 1) return cudaErrorInvalidValue;
  const int esz = (xdt == BL_F32) ? 4 : (xdt == BL_BF16 ? 2 : 1);
  const int ysz = (ydt == BL_BF16) ? 2 : 4;
  for (int64_t m0 = 0; m0 < M; m0 += mt_max) {
    const int mt = static_cast<int>((M - m0) < mt_max ? (M - m0) : mt_max);
    const void* xm = static_cast<const uint8_t*>(x) + m0 * K * esz;
    float* sm = scale + m0;
    void* ym = static_cast<uint8_t*>(y) + m0 * N * ysz;
    cudaError_t e;
    if (fmt == BL_PACK_I2) {
      if (xdt == BL_F32) e = launch_gemv_mt<BL_PACK_I2, BL_F32>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, st);
      else if (xdt == BL_BF16) e = launch_gemv_mt<BL_PACK_I2, BL_BF16>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, st);
      else e = launch_gemv_mt<BL_PACK_I2, BL_I8>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, st);
    } else {
      if (xdt == BL_F32) e = launch_gemv_mt<BL_PACK_T5, BL_F32>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, st);
      else if (xdt == BL_BF16) e = launch_gemv_mt<BL_PACK_T5, BL_BF16>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, st);
      else e = launch_gemv_mt<BL_PACK_T5, BL_I8>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, st);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bl
