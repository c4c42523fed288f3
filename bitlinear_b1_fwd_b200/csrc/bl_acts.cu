// bl_acts.cu -- per-token absmax INT8 activation quantization.
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §3.2 and §5.2: each token
// (one row of x over K) is scaled by its own max |x| (floored at 1e-6) and
// x_q = clamp(round(x / s * 127), -127, 127).  One CTA per token: a max
// reduction (warp shuffles, then across warps) and a second pass that writes
// the INT8 codes, 8 per thread-iteration, with 16-byte loads when K allows.
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kActThreads = 256;

template <int XDT>
__global__ void __launch_bounds__(kActThreads)
    act_quant_kernel(const void* __restrict__ x, int64_t M, int64_t K, int8_t* __restrict__ xq,
                     float* __restrict__ scale, bool vec) {
  __shared__ float red[kActThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const int64_t base = m * K;
    float amax = 0.0f;
    if (vec) {
      for (int64_t v = threadIdx.x; v < K / 8; v += blockDim.x) {
        float e[8];
        load8_aligned<XDT>(x, base + 8 * v, e);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[j]));
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(load_elem<XDT>(x, base + k)));
    }
    amax = warp_maxf(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float a = red[0];
#pragma unroll
    for (int w = 1; w < kActThreads / 32; ++w) a = fmaxf(a, red[w]);
    const float s = fmaxf(a, 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    if (vec) {
      for (int64_t v = threadIdx.x; v < K / 8; v += blockDim.x) {
        float e[8];
        load8_aligned<XDT>(x, base + 8 * v, e);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          lo |= static_cast<uint32_t>(quant_act_fast(e[j], s, c127) & 0xff) << (8 * j);
          hi |= static_cast<uint32_t>(quant_act_fast(e[j + 4], s, c127) & 0xff) << (8 * j);
        }
        *reinterpret_cast<uint2*>(xq + base + 8 * v) = make_uint2(lo, hi);
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
        xq[base + k] = static_cast<int8_t>(quant_act_fast(load_elem<XDT>(x, base + k), s, c127));
    }
    if (threadIdx.x == 0) scale[m] = s;
    __syncthreads();  // red[] is reused by the next token
  }
}

cudaError_t launch_act_quant(const void* x, int xdt, int64_t M, int64_t K, int8_t* xq, float* scale,
                             cudaStream_t st) {
  const int sms = device_sms();
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(M < cap ? M : cap);
  const bool vec = (K % 8) == 0;
  if (xdt == BL_F32)
    act_quant_kernel<BL_F32><<<grid, kActThreads, 0, st>>>(x, M, K, xq, scale, vec);
  else
    act_quant_kernel<BL_BF16><<<grid, kActThreads, 0, st>>>(x, M, K, xq, scale, vec);
  return cudaGetLastError();
}

}  // namespace bl
