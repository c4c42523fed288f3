// bl_acts.cu -- per-token absmax INT8 activation quantization.
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §3.2 and §5.2: each token
// (one row of x over K) is scaled by its own max |x| (floored at 1e-6) and
// x_q = clamp(round(x / s * 127), -127, 127).  One warp per token: a max
// reduction (warp shuffles) and a second pass that writes
// the INT8 codes, 8 per lane-iteration, with 16-byte loads when K allows.
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kActThreads = 256;

// One warp per token: the absmax over the row (16-byte loads, warp shuffles),
// then a second pass over the same row (mostly L1 hits) that writes the codes,
// 8 per lane-iteration.  No shared memory, no block barriers.
template <int XDT>
__global__ void __launch_bounds__(kActThreads)
    act_quant_kernel(const void* __restrict__ x, int64_t M, int64_t K, int8_t* __restrict__ xq,
                     float* __restrict__ scale, bool vec) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t tw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t m = gw; m < M; m += tw) {
    const int64_t base = m * K;
    float amax = 0.0f;
    if (vec) {
#pragma unroll 4
      for (int64_t v = lane; v < K / 8; v += 32) {
        float e[8];
        load8_aligned<XDT>(x, base + 8 * v, e);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[j]));
      }
    } else {
      for (int64_t k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(load_elem<XDT>(x, base + k)));
    }
    amax = warp_maxf(amax);
    const float s = fmaxf(amax, 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    if (vec) {
#pragma unroll 4
      for (int64_t v = lane; v < K / 8; v += 32) {
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
      for (int64_t k = lane; k < K; k += 32)
        xq[base + k] = static_cast<int8_t>(quant_act_fast(load_elem<XDT>(x, base + k), s, c127));
    }
    if (lane == 0) scale[m] = s;
  }
}

cudaError_t launch_act_quant(const void* x, int xdt, int64_t M, int64_t K, int8_t* xq, float* scale,
                             cudaStream_t st) {
  const int64_t warps_per_cta = kActThreads / 32;
  const int64_t need = (M + warps_per_cta - 1) / warps_per_cta;
  const int64_t cap = static_cast<int64_t>(device_sms()) * (2048 / kActThreads);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  const bool vec = (K % 8) == 0;
  if (xdt == BL_F32)
    act_quant_kernel<BL_F32><<<grid, kActThreads, 0, st>>>(x, M, K, xq, scale, vec);
  else
    act_quant_kernel<BL_BF16><<<grid, kActThreads, 0, st>>>(x, M, K, xq, scale, vec);
  return cudaGetLastError();
}

}  // namespace bl
