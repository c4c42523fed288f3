// bl_acts.cu -- per-token absmax INT8 activation quantization.
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §3.2 and §5.2: each token
// (one row of x over K) is scaled by its own max |x| (floored at 1e-6) and
// x_q = clamp(round(x / s * 127), -127, 127).  Rows of up to 32 K (bf16) or
// 16 K (fp32) elements with K % 8 (bf16) or K % 4 (fp32) == 0: one CTA per
// token, read once into registers.  Other rows: one CTA per token, two
// passes whose loads go out kActBatch at a time.
#include <type_traits>

#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kActThreads = 256;
constexpr int kActBatch = 4;  // 16-byte loads in flight per lane in the two-pass kernel

__device__ __forceinline__ uint32_t pack_codes4(const int* q) {
  return __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
}

__device__ __forceinline__ uint2 codes8(const float* e, float s, float c127) {
  int q[8];
  quant_act_fast_n<8>(e, s, c127, q);
  return make_uint2(pack_codes4(q), pack_codes4(q + 4));
}

__device__ __forceinline__ void bf16x8(const uint4 r, float* e) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    e[2 * i] = __uint_as_float(w[i] << 16);
    e[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Rows with K % 8 == 0 (bf16) or K % 4 == 0 (fp32) and at most T NV 16-byte
// words: one CTA of T threads per token, read once.  Thread t issues its NV
// loads (words t, t + T, ...) together; the absmax meets across the CTA (warp
// shuffles, one barrier) and the codes come from registers.  Rows of up to
// 8192 bf16 elements take 128-thread CTAs, many per SM, each at its own
// phase, keeping loads in flight while others compute; longer rows (up to
// 32768 bf16 elements) take 512-thread CTAs, so that even a few tokens spread
// over as many threads as their words.
constexpr int kActRowThreads = 128;
constexpr int kActLongRowThreads = 512;

template <int XDT, int NV, int T = kActRowThreads>
__global__ void __launch_bounds__(T)
    act_quant_row_kernel(const void* __restrict__ x, int64_t M, int64_t K, int8_t* __restrict__ xq,
                         float* __restrict__ scale) {
  pdl_enter(x, xq, scale);
  constexpr int kActRowThreads = T;  // this instance's CTA size
  constexpr int EPW = (XDT == BL_F32) ? 4 : 8;  // elements per 16-byte word
  __shared__ float red[kActRowThreads / 32];
  const int t = threadIdx.x, lane = t & 31;
  const int nv = static_cast<int>(K / EPW);
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + m * K * (16 / EPW));
    uint4 r[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = t + kActRowThreads * i;
      r[i] = v < nv ? __ldcg(row + v) : make_uint4(0, 0, 0, 0);
    }
    auto elems = [&](int i, float* e) {
      if constexpr (XDT == BL_F32) {
        e[0] = __uint_as_float(r[i].x); e[1] = __uint_as_float(r[i].y);
        e[2] = __uint_as_float(r[i].z); e[3] = __uint_as_float(r[i].w);
      } else {
        bf16x8(r[i], e);
      }
    };
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float e[8];
      elems(i, e);
#pragma unroll
      for (int j = 0; j < EPW; ++j) amax = fmaxf(amax, fabsf(e[j]));
    }
    amax = warp_maxf(amax);
    if (lane == 0) red[t >> 5] = amax;
    __syncthreads();
    float a = red[0];
#pragma unroll
    for (int w = 1; w < kActRowThreads / 32; ++w) a = fmaxf(a, red[w]);
    __syncthreads();  // red is free for the next token
    const float s = fmaxf(a, 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    int8_t* out = xq + m * K;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = t + kActRowThreads * i;
      if (v < nv) {
        float e[8];
        elems(i, e);
        if constexpr (XDT == BL_F32) {
          int q[4];
          quant_act_fast_n<4>(e, s, c127, q);
          reinterpret_cast<uint32_t*>(out)[v] = pack_codes4(q);
        } else {
          reinterpret_cast<uint2*>(out)[v] = codes8(e, s, c127);
        }
      }
    }
    if (t == 0) scale[m] = s;
  }
}

// Any row: one CTA of kActThreads per token, the absmax pass and the code
// pass over the row, kActBatch 16-byte loads per thread in flight.
template <int XDT>
__global__ void __launch_bounds__(kActThreads)
    act_quant_kernel(const void* __restrict__ x, int64_t M, int64_t K, int8_t* __restrict__ xq,
                     float* __restrict__ scale, bool vec) {
  pdl_enter(x, xq, scale);
  __shared__ float red[kActThreads / 32];
  const int t = threadIdx.x, lane = t & 31;
  constexpr int T = kActThreads;
  const int64_t nv = K / 8;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const int64_t base = m * K;
    float amax = 0.0f;
    if (vec) {
      for (int64_t v0 = t; v0 < nv; v0 += T * kActBatch) {
        float e[kActBatch][8];
#pragma unroll
        for (int b = 0; b < kActBatch; ++b) {
          const int64_t v = v0 + T * b;
          if (v < nv) {
            load8_aligned<XDT>(x, base + 8 * v, e[b]);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) e[b][j] = 0.0f;
          }
        }
#pragma unroll
        for (int b = 0; b < kActBatch; ++b)
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[b][j]));
      }
    } else {
      for (int64_t k = t; k < K; k += T) amax = fmaxf(amax, fabsf(load_elem<XDT>(x, base + k)));
    }
    amax = warp_maxf(amax);
    if (lane == 0) red[t >> 5] = amax;
    __syncthreads();
    float a = red[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) a = fmaxf(a, red[w]);
    __syncthreads();  // red is free for the next token
    const float s = fmaxf(a, 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    if (vec) {
      for (int64_t v0 = t; v0 < nv; v0 += T * kActBatch) {
        float e[kActBatch][8];
#pragma unroll
        for (int b = 0; b < kActBatch; ++b) {
          const int64_t v = v0 + T * b;
          if (v < nv) load8_aligned<XDT>(x, base + 8 * v, e[b]);
        }
#pragma unroll
        for (int b = 0; b < kActBatch; ++b) {
          const int64_t v = v0 + T * b;
          if (v < nv) *reinterpret_cast<uint2*>(xq + base + 8 * v) = codes8(e[b], s, c127);
        }
      }
    } else {
      for (int64_t k = t; k < K; k += T)
        xq[base + k] = static_cast<int8_t>(quant_act_fast(load_elem<XDT>(x, base + k), s, c127));
    }
    if (t == 0) scale[m] = s;
  }
}

// Pre-norm + step 4: LayerNorm of each token, then per-token absmax INT8
// ([P5] "The BitLinear Recipe" step 1: the input is quantized after
// LayerNorm; [P3] §5.5: LayerNorm kept in high precision, bf16 activations).
// One CTA of kLnThreads per token.  The mean and the variance are fp64 sums
// in a fixed order: thread l adds the elements l, l + 256, ... in turn from
// 0.0, and the 256 partial sums combine by the stride-halving tree p[l] +=
// p[l + s], s = 128, ..., 1.  r = 1 / sqrt(var + eps) in fp64; y = ((x - mu) r)
// g + b in fp64 with one rounding per operation, then fp32 and bf16 (RNE).
// The bf16 y is quantized exactly as act_quant_row_kernel does (absmax over
// the token, the division-free exact rounding).  Four passes over the token,
// the later ones from L1/L2.
constexpr int kLnThreads = 256;

template <int XDT>
__global__ void __launch_bounds__(kLnThreads)
    ln_quant_kernel(const void* __restrict__ x, const float* __restrict__ g, const float* __restrict__ b, float eps,
                    int64_t M, int64_t K, uint16_t* __restrict__ y, int8_t* __restrict__ xq,
                    float* __restrict__ scale) {
  pdl_enter(x, g, b, y, xq, scale);
  __shared__ double p[kLnThreads];
  __shared__ float red[kLnThreads / 32];
  const int l = threadIdx.x, lane = l & 31, warp = l >> 5;
  auto tree = [&](double v) -> double {
    p[l] = v;
    __syncthreads();
#pragma unroll
    for (int s = kLnThreads / 2; s >= 1; s >>= 1) {
      if (l < s) p[l] = __dadd_rn(p[l], p[l + s]);
      __syncthreads();
    }
    const double t = p[0];
    __syncthreads();  // p is free for the next sum
    return t;
  };
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const int64_t base = m * K;
    double a = 0.0;
    for (int64_t k = l; k < K; k += kLnThreads) a = __dadd_rn(a, static_cast<double>(load_elem<XDT>(x, base + k)));
    const double mu = __ddiv_rn(tree(a), static_cast<double>(K));
    a = 0.0;
    for (int64_t k = l; k < K; k += kLnThreads) {
      const double d = __dsub_rn(static_cast<double>(load_elem<XDT>(x, base + k)), mu);
      a = __dadd_rn(a, __dmul_rn(d, d));
    }
    const double var = __ddiv_rn(tree(a), static_cast<double>(K));
    const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps))));
    auto yk = [&](int64_t k) -> __nv_bfloat16 {
      const double d = __dsub_rn(static_cast<double>(load_elem<XDT>(x, base + k)), mu);
      const double v = __dadd_rn(__dmul_rn(__dmul_rn(d, r), static_cast<double>(__ldcg(g + k))),
                                 static_cast<double>(__ldcg(b + k)));
      return __float2bfloat16_rn(__double2float_rn(v));
    };
    float amax = 0.0f;
    for (int64_t k = l; k < K; k += kLnThreads) {
      const __nv_bfloat16 v = yk(k);
      amax = fmaxf(amax, fabsf(__bfloat162float(v)));
      if (y != nullptr) y[base + k] = __bfloat16_as_ushort(v);
    }
    amax = warp_maxf(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float am = red[0];
#pragma unroll
    for (int w = 1; w < kLnThreads / 32; ++w) am = fmaxf(am, red[w]);
    __syncthreads();  // red is free for the next token
    const float s = fmaxf(am, 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    for (int64_t k = l; k < K; k += kLnThreads)
      xq[base + k] = static_cast<int8_t>(quant_act_fast(__bfloat162float(yk(k)), s, c127));
    if (l == 0) scale[m] = s;
  }
}


// The same LayerNorm + INT8 with the token held in registers (K even and
// ceil(K / 256) <= NI).  R18's lane l is a set of elements, not a thread:
// here thread t of a 128-thread CTA computes lanes 2t and 2t + 1, loading
// the element pairs (2t + 256 i, 2t + 1 + 256 i) with one 4-byte (bf16) or
// 8-byte (fp32) load each, and adds each lane's elements in R18's order.  A
// tree of the 256 lane sums takes one shared-memory write and one barrier:
// every warp then reads the eight sums of its lane's subtree and adds them in
// the tree's order (levels 128, 64, 32), and levels 16..1 run by shuffles --
// each warp computes the same total, so no broadcast is needed.
// The conversions to and from fp64 run on the SM's narrow conversion pipe, so
// each is done once: the token's elements are converted once and kept in
// registers as fp64 for the three passes, g and b are converted once per CTA
// into shared memory (fp64), and the next token's elements
// are loaded while this one is normalised.  y is kept as bf16 pairs for the
// absmax and the codes.
constexpr int kLnRegThreads = 128;

template <int XDT, int NI>
__global__ void __launch_bounds__(kLnRegThreads, NI > 13 ? 3 : 4)
    ln_quant_reg_kernel(const void* __restrict__ x, const float* __restrict__ g, const float* __restrict__ b,
                        float eps, int64_t M, int64_t K, uint16_t* __restrict__ y, int8_t* __restrict__ xq,
                        float* __restrict__ scale) {
  pdl_enter(x, g, b, y, xq, scale);
  extern __shared__ __align__(16) double gbs[];  // [2][K]: g then b in fp64 (a thread reads 16-byte pairs)
  __shared__ __align__(16) double p1[256];
  __shared__ __align__(16) double p2[256];
  __shared__ uint32_t red[kLnRegThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  double* gd = gbs;
  double* bd = gbs + K;
  for (int64_t k = t; k < K; k += kLnRegThreads) {
    gd[k] = static_cast<double>(__ldcg(g + k));
    bd[k] = static_cast<double>(__ldcg(b + k));
  }
  // the tree of the 256 lane sums held in p, R18's order
  auto tree = [&](const double* p) -> double {
    const int L = lane;
    const double q0 = __dadd_rn(p[L], p[L + 128]), q1 = __dadd_rn(p[L + 64], p[L + 192]);
    const double q2 = __dadd_rn(p[L + 32], p[L + 160]), q3 = __dadd_rn(p[L + 96], p[L + 224]);
    double v = __dadd_rn(__dadd_rn(q0, q1), __dadd_rn(q2, q3));
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v = __dadd_rn(v, __shfl_down_sync(0xffffffffu, v, s));
    return __shfl_sync(0xffffffffu, v, 0);
  };
  // the element pair i of lanes (2t, 2t + 1) as two floats
  constexpr bool kF32 = XDT == BL_F32;
  using Pair = typename std::conditional<kF32, float2, uint32_t>::type;
  auto lo = [](const Pair& v) -> float {
    if constexpr (kF32) return v.x; else return __uint_as_float(v << 16);
  };
  auto hi = [](const Pair& v) -> float {
    if constexpr (kF32) return v.y; else return __uint_as_float(v & 0xffff0000u);
  };
  auto load_token = [&](int64_t m, Pair (&xr)[NI]) {
    const int64_t base = m * K;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int64_t k = 2 * t + 256 * i;
      if constexpr (kF32) {
        xr[i] = (m < M && k < K) ? __ldcg(reinterpret_cast<const float2*>(static_cast<const float*>(x) + base + k))
                                 : make_float2(0.0f, 0.0f);
      } else {
        xr[i] = (m < M && k < K)
                    ? __ldcg(reinterpret_cast<const unsigned int*>(static_cast<const uint16_t*>(x) + base + k))
                    : 0u;
      }
    }
  };
  const double dK = static_cast<double>(K);
  Pair xr[NI];  // the token's raw pairs; loaded one token ahead
  load_token(blockIdx.x, xr);
  __syncthreads();  // gb is complete
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const int64_t base = m * K;
    double xa[NI], xb[NI];  // lanes 2t and 2t + 1 in fp64 (0 past K)
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      xa[i] = static_cast<double>(lo(xr[i]));
      xb[i] = static_cast<double>(hi(xr[i]));
    }
    load_token(m + gridDim.x, xr);  // in flight during the three passes
    // mean: each lane's elements in turn from 0.0
    double sa = 0.0, sb = 0.0;
#pragma unroll
    for (int i = 0; i < NI; ++i)
      if (2 * t + 256 * i < K) {
        sa = __dadd_rn(sa, xa[i]);
        sb = __dadd_rn(sb, xb[i]);
      }
    reinterpret_cast<double2*>(p1)[t] = make_double2(sa, sb);
    __syncthreads();
    const double mu = __ddiv_rn(tree(p1), dK);
    // variance: (x - mu)^2 in the same order; x - mu kept for y
    sa = sb = 0.0;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      xa[i] = __dsub_rn(xa[i], mu);
      xb[i] = __dsub_rn(xb[i], mu);
      if (2 * t + 256 * i < K) {
        sa = __dadd_rn(sa, __dmul_rn(xa[i], xa[i]));
        sb = __dadd_rn(sb, __dmul_rn(xb[i], xb[i]));
      }
    }
    reinterpret_cast<double2*>(p2)[t] = make_double2(sa, sb);
    __syncthreads();
    const double var = __ddiv_rn(tree(p2), dK);
    const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps))));
    // y = ((x - mu) r) g + b, fp64 -> fp32 -> bf16 (RNE, the pair in one
    // conversion), stored and kept (bf16 pairs); the absmax on the magnitude
    // bits of the pairs (finite values order like unsigned integers)
    uint32_t yr[NI];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int64_t k = 2 * t + 256 * i;
      yr[i] = 0u;
      if (k < K) {
        const double2 gg = *reinterpret_cast<const double2*>(gd + k);
        const double2 bb = *reinterpret_cast<const double2*>(bd + k);
        const double va = __dadd_rn(__dmul_rn(__dmul_rn(xa[i], r), gg.x), bb.x);
        const double vb = __dadd_rn(__dmul_rn(__dmul_rn(xb[i], r), gg.y), bb.y);
        const __nv_bfloat162 h = __floats2bfloat162_rn(__double2float_rn(va), __double2float_rn(vb));
        yr[i] = *reinterpret_cast<const uint32_t*>(&h);
        if (y != nullptr) *reinterpret_cast<uint32_t*>(y + base + k) = yr[i];
        mx = __vmaxu2(mx, yr[i] & 0x7fff7fffu);
      }
    }
    mx = __reduce_max_sync(0xffffffffu, max(mx & 0xffffu, mx >> 16) << 16);  // fp32 bits
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    uint32_t am = red[0];
#pragma unroll
    for (int w = 1; w < kLnRegThreads / 32; ++w) am = max(am, red[w]);
    const float s = fmaxf(__uint_as_float(am), 1e-6f);
    const float c127 = __fdiv_rn(127.0f, s);
    // the codes by quant_act_fast's division-free rule, element pairs through
    // the paired fp32 unit: t_a = y c127, rint(t_a) from the adder (the code
    // in the low byte of the sum's bits), t_a - rint(t_a) exact by one fma;
    // one margin test per thread, the exact quotient only near a tie
    const float2 c2 = make_float2(c127, c127), mg = make_float2(12582912.0f, 12582912.0f);
    const float2 nmg = make_float2(-12582912.0f, -12582912.0f), m1 = make_float2(-1.0f, -1.0f);
    uint32_t qw[NI];
    float worst = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const float2 ta = __fmul2_rn(make_float2(__uint_as_float(yr[i] << 16), __uint_as_float(yr[i] & 0xffff0000u)), c2);
      const float2 r2 = __fadd2_rn(ta, mg);
      const float2 d = __ffma2_rn(__fadd2_rn(r2, nmg), m1, ta);
      worst = fmaxf(worst, fmaxf(fabsf(d.x), fabsf(d.y)));
      qw[i] = __byte_perm(__float_as_uint(r2.x), __float_as_uint(r2.y), 0x0040);
    }
    if (!(worst < 0.49993896484375f)) {  // rare: some element is near a tie
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const float e2[2] = {__uint_as_float(yr[i] << 16), __uint_as_float(yr[i] & 0xffff0000u)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float ta = __fmul_rn(e2[h], c127);
          if (!(fabsf(__fsub_rn(ta, rintf(ta))) < 0.49993896484375f)) {
            const uint32_t q = static_cast<uint8_t>(quant_act_slow(e2[h], s));
            qw[i] = h == 0 ? ((qw[i] & 0xff00u) | q) : ((qw[i] & 0x00ffu) | (q << 8));
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int64_t k = 2 * t + 256 * i;
      if (k < K) *reinterpret_cast<uint16_t*>(xq + base + k) = static_cast<uint16_t>(qw[i]);
    }
    if (t == 0) scale[m] = s;
    // red, p1 and p2 are free for the next token once every warp is past here
    __syncthreads();
  }
}

template <int XDT, int NI>
static cudaError_t launch_ln_quant_reg(const void* x, const float* g, const float* b, float eps, int64_t M, int64_t K,
                                       uint16_t* y, int8_t* xq, float* scale, cudaStream_t st) {
  int per_sm = 1;
  auto kern = ln_quant_reg_kernel<XDT, NI>;
  const size_t smem = static_cast<size_t>(2 * K) * sizeof(double);
  // the 4 KB of static shared memory plus the dynamic part can pass the 48 KB
  // default well before the dynamic part alone does: opt in early
  if (smem > 32 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLnRegThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
  const unsigned grid = static_cast<unsigned>(M < cap ? M : cap);
  const cudaError_t e = launch_pdl(kern, grid, kLnRegThreads, smem, st, x, g, b, eps, M, K, y, xq, scale);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_ln_quant(const void* x, int xdt, const float* g, const float* b, float eps, int64_t M, int64_t K,
                            uint16_t* y, int8_t* xq, float* scale, cudaStream_t st) {
  // the register form: K even (vector loads and stores of element pairs), the
  // token in registers, g and b 8-byte aligned (float2 loads), y 4-byte and
  // x_q 2-byte aligned (pair stores)
  const bool pairs = (K % 2) == 0 && (reinterpret_cast<uintptr_t>(g) & 7) == 0 &&
                     (reinterpret_cast<uintptr_t>(b) & 7) == 0 && (reinterpret_cast<uintptr_t>(y) & 3) == 0 &&
                     (reinterpret_cast<uintptr_t>(xq) & 1) == 0;
  if (pairs && K <= 256 * 8)
    return xdt == BL_F32 ? launch_ln_quant_reg<BL_F32, 8>(x, g, b, eps, M, K, y, xq, scale, st)
                         : launch_ln_quant_reg<BL_BF16, 8>(x, g, b, eps, M, K, y, xq, scale, st);
  if (pairs && K <= 256 * 13)  // the 3B hidden size, 3200, without idle registers
    return xdt == BL_F32 ? launch_ln_quant_reg<BL_F32, 13>(x, g, b, eps, M, K, y, xq, scale, st)
                         : launch_ln_quant_reg<BL_BF16, 13>(x, g, b, eps, M, K, y, xq, scale, st);
  if (pairs && K <= 256 * 16)
    return xdt == BL_F32 ? launch_ln_quant_reg<BL_F32, 16>(x, g, b, eps, M, K, y, xq, scale, st)
                         : launch_ln_quant_reg<BL_BF16, 16>(x, g, b, eps, M, K, y, xq, scale, st);

  int per_sm = 1;
  const void* kp = xdt == BL_F32 ? reinterpret_cast<const void*>(ln_quant_kernel<BL_F32>)
                                 : reinterpret_cast<const void*>(ln_quant_kernel<BL_BF16>);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kp, kLnThreads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
  const unsigned grid = static_cast<unsigned>(M < cap ? M : cap);
  cudaError_t e = (xdt == BL_F32)
                      ? launch_pdl(ln_quant_kernel<BL_F32>, grid, kLnThreads, 0, st, x, g, b, eps, M, K, y, xq, scale)
                      : launch_pdl(ln_quant_kernel<BL_BF16>, grid, kLnThreads, 0, st, x, g, b, eps, M, K, y, xq, scale);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* x, int xdt, int64_t M, int64_t K, int8_t* xq, float* scale,
                             cudaStream_t st) {
  const int64_t need = M;  // one CTA per token
  auto grid_for = [&](const void* kern) -> unsigned {
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kActThreads, 0) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
    return static_cast<unsigned>(need < cap ? need : cap);
  };
  const bool vec = (K % 8) == 0;
  const int epw = (xdt == BL_F32) ? 4 : 8;
  const int64_t nv = K / epw;
  if ((K % epw) == 0 && nv <= kActRowThreads * 8) {
    int per_sm = 1;
#define BL_AQ(XDT, NV)                                                                                  \
  if (nv <= kActRowThreads * (NV)) {                                                                    \
    auto kern = act_quant_row_kernel<XDT, NV>;                                                          \
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kActRowThreads, 0) != cudaSuccess || \
        per_sm < 1)                                                                                     \
      per_sm = 1;                                                                                       \
    const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;                                    \
    { const cudaError_t le_ = launch_pdl(kern, static_cast<unsigned>(M < cap ? M : cap), kActRowThreads, 0, st, x, M, K, xq, scale); if (le_ != cudaSuccess) return le_; }      \
    return cudaGetLastError();                                                                          \
  }
    if (xdt == BL_F32) {
      BL_AQ(BL_F32, 2)
      BL_AQ(BL_F32, 4)
      BL_AQ(BL_F32, 8)
    } else {
      BL_AQ(BL_BF16, 2)
      BL_AQ(BL_BF16, 4)
      BL_AQ(BL_BF16, 8)
    }
#undef BL_AQ
  }
  if ((K % epw) == 0 && nv <= kActLongRowThreads * 8) {
    int per_sm = 1;
#define BL_AQL(XDT, NV)                                                                                      \
  if (nv <= kActLongRowThreads * (NV)) {                                                                     \
    auto kern = act_quant_row_kernel<XDT, NV, kActLongRowThreads>;                                           \
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kActLongRowThreads, 0) != cudaSuccess || \
        per_sm < 1)                                                                                          \
      per_sm = 1;                                                                                            \
    const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;                                         \
    const cudaError_t le_ = launch_pdl(kern, static_cast<unsigned>(M < cap ? M : cap), kActLongRowThreads, 0, \
                                       st, x, M, K, xq, scale);                                              \
    if (le_ != cudaSuccess) return le_;                                                                      \
    return cudaGetLastError();                                                                               \
  }
    if (xdt == BL_F32) {
      BL_AQL(BL_F32, 4)
      BL_AQL(BL_F32, 8)
    } else {
      BL_AQL(BL_BF16, 4)
      BL_AQL(BL_BF16, 8)
    }
#undef BL_AQL
  }
  if (xdt == BL_F32)
    { const cudaError_t le_ = launch_pdl(act_quant_kernel<BL_F32>, grid_for(reinterpret_cast<const void*>(act_quant_kernel<BL_F32>)), kActThreads, 0, st, x, M, K, xq, scale, vec); if (le_ != cudaSuccess) return le_; }
  else
    { const cudaError_t le_ = launch_pdl(act_quant_kernel<BL_BF16>, grid_for(reinterpret_cast<const void*>(act_quant_kernel<BL_BF16>)), kActThreads, 0, st, x, M, K, xq, scale, vec); if (le_ != cudaSuccess) return le_; }
  return cudaGetLastError();
}

}  // namespace bl
