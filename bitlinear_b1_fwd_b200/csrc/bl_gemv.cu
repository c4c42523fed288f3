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

constexpr int kGemvThreads = 512;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvU = 4;  // 16-byte segments per lane per pass

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

template <int XDT>
__device__ __forceinline__ float load_x(const void* x, int64_t i) {
  if constexpr (XDT == BL_I8) {
    return static_cast<float>(static_cast<const int8_t*>(x)[i]);
  } else {
    return load_elem<XDT>(x, i);
  }
}

template <int FMT, int MT, int XDT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                void* __restrict__ y, int ydt, int write_scale) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int64_t xb = gemv_x_bytes(FMT, rowbytes);
  uint8_t* xs = smem;                                           // [MT][xb]
  uint2* lut = reinterpret_cast<uint2*>(smem + MT * xb);        // base 3 only
  __shared__ float red_f[kGemvWarps][MT];
  __shared__ int red_i[kGemvWarps][MT];
  __shared__ float s_tok[MT];
  __shared__ int sum_tok[MT];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t segs = rowbytes >> 4;
  const int64_t TW = static_cast<int64_t>(gridDim.x) * kGemvWarps;
  int64_t r = static_cast<int64_t>(blockIdx.x) * kGemvWarps + warp;

  // 1. first packed loads of this warp's first row go out before the prologue.
  uint4 pre[kGemvU];
  if (r < N) {
    const uint4* rp = reinterpret_cast<const uint4*>(packed + r * rowbytes);
#pragma unroll
    for (int u = 0; u < kGemvU; ++u) {
      const int64_t s = lane + 32 * u;
      if (s < segs) pre[u] = ld_stream(rp + s);
    }
  }

  // 2. prologue: quantize the MT tokens into shared memory.
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
  // one "group" = the activations of one packed 32-bit word: 16 weights (2-bit)
  // or 20 weights (base 3)
  constexpr int GW = (FMT == BL_PACK_I2) ? 16 : 20;
  const int64_t groups = rowbytes / 4;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float s;
    if constexpr (XDT != BL_I8) {
      float amax = 0.0f;
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
        amax = fmaxf(amax, fabsf(load_x<XDT>(x, m * K + k)));
      amax = warp_maxf(amax);
      if (lane == 0) red_f[warp][m] = amax;
      __syncthreads();
      if (threadIdx.x == 0) {
        float a = red_f[0][m];
        for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, red_f[w][m]);
        s_tok[m] = fmaxf(a, 1e-6f);
      }
      __syncthreads();
      s = s_tok[m];
    } else {
      s = 0.0f;
    }
    int part = 0;
    for (int64_t g = threadIdx.x; g < groups; g += blockDim.x) {
      int q[GW];
#pragma unroll
      for (int i = 0; i < GW; ++i) {
        const int64_t k = g * GW + i;
        if (k < K) {
          if constexpr (XDT == BL_I8)
            q[i] = static_cast<const int8_t*>(x)[m * K + k];
          else
            q[i] = quant_act(load_x<XDT>(x, m * K + k), s);
        } else {
          q[i] = 0;
        }
        part += q[i];
      }
      if constexpr (FMT == BL_PACK_I2) {
        // word j holds x[16g + j + 4b] in byte b
        uint32_t w4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w4[j] = (static_cast<uint32_t>(q[j] & 0xff)) | (static_cast<uint32_t>(q[j + 4] & 0xff) << 8) |
                  (static_cast<uint32_t>(q[j + 8] & 0xff) << 16) |
                  (static_cast<uint32_t>(q[j + 12] & 0xff) << 24);
        reinterpret_cast<uint4*>(xs + m * xb)[g] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      } else {
        // byte j of the word: {x[5j..5j+3]} and {x[5j+4], 0, 0, 0}
        uint2* dst = reinterpret_cast<uint2*>(xs + m * xb) + 4 * g;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int* qq = q + 5 * b;
          const uint32_t lo = (static_cast<uint32_t>(qq[0] & 0xff)) | (static_cast<uint32_t>(qq[1] & 0xff) << 8) |
                              (static_cast<uint32_t>(qq[2] & 0xff) << 16) |
                              (static_cast<uint32_t>(qq[3] & 0xff) << 24);
          dst[b] = make_uint2(lo, static_cast<uint32_t>(qq[4] & 0xff));
        }
      }
    }
    if constexpr (FMT == BL_PACK_I2) {
      part = __reduce_add_sync(0xffffffffu, part);
      if (lane == 0) red_i[warp][m] = part;
    }
    if constexpr (XDT == BL_I8) {
      if (threadIdx.x == 0) s_tok[m] = scale[m];
    }
  }
  __syncthreads();
  if (threadIdx.x < MT) {
    const int m = threadIdx.x;
    if constexpr (FMT == BL_PACK_I2) {
      int t = 0;
      for (int w = 0; w < kGemvWarps; ++w) t += red_i[w][m];
      sum_tok[m] = t;
    } else {
      sum_tok[m] = 0;
    }
    if (XDT != BL_I8 && write_scale && blockIdx.x == 0) scale[m] = s_tok[m];
  }
  __syncthreads();

  const float g = __ldg(gamma);
  float cfac[MT];
  int corr[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    cfac[m] = dequant_factor(g, s_tok[m]);
    corr[m] = sum_tok[m];
  }

  // 3. rows: warp-per-row, lanes stride over the row's 16-byte segments.
  bool first = true;
  for (; r < N; r += TW) {
    const uint4* rp = reinterpret_cast<const uint4*>(packed + r * rowbytes);
    int acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
    for (int64_t s0 = 0; s0 < segs; s0 += 32 * kGemvU) {
      uint4 buf[kGemvU];
      if (first && s0 == 0) {
#pragma unroll
        for (int u = 0; u < kGemvU; ++u) buf[u] = pre[u];
      } else {
#pragma unroll
        for (int u = 0; u < kGemvU; ++u) {
          const int64_t s = s0 + lane + 32 * u;
          if (s < segs) buf[u] = ld_stream(rp + s);
        }
      }
#pragma unroll
      for (int u = 0; u < kGemvU; ++u) {
        const int64_t s = s0 + lane + 32 * u;
        if (s >= segs) break;
        const uint32_t wd[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          if constexpr (FMT == BL_PACK_I2) {
            const uint32_t c0 = wd[w] & 0x03030303u, c1 = (wd[w] >> 2) & 0x03030303u;
            const uint32_t c2 = (wd[w] >> 4) & 0x03030303u, c3 = (wd[w] >> 6) & 0x03030303u;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const uint4 X = reinterpret_cast<const uint4*>(xs + m * xb)[4 * s + w];
              acc[m] = __dp4a(static_cast<int>(c0), static_cast<int>(X.x), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c1), static_cast<int>(X.y), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c2), static_cast<int>(X.z), acc[m]);
              acc[m] = __dp4a(static_cast<int>(c3), static_cast<int>(X.w), acc[m]);
            }
          } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const uint2 L = lut[(wd[w] >> (8 * b)) & 0xffu];
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const uint2 X = reinterpret_cast<const uint2*>(xs + m * xb)[16 * s + 4 * w + b];
                acc[m] = __dp4a(static_cast<int>(L.x), static_cast<int>(X.x), acc[m]);
                acc[m] = __dp4a(static_cast<int>(L.y), static_cast<int>(X.y), acc[m]);
              }
            }
          }
        }
      }
    }
    first = false;
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = __reduce_add_sync(0xffffffffu, acc[m]);
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int a = acc[m] - corr[m];
        const int64_t o = m * N + r;
        if (ydt == BL_I32)
          static_cast<int32_t*>(y)[o] = a;
        else if (ydt == BL_F32)
          static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cfac[m]);
        else
          static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cfac[m]));
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
