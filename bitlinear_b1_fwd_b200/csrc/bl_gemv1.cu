// bl_gemv1.cu -- one-token decode GEMV on 2-bit weights: y = dequant(x_q . W_q^T).
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §4.1: at one token the
// layer is bound by moving its weights; §4.2: with weights in {-1, 0, +1}
// the product is add / subtract / skip.  Here the add / subtract / skip runs
// as dp4a on the stored digits d = q + 1 against INT8 activation codes
// (sum q x = sum d x - sum x), the per-token absmax INT8 quantization (§3.2)
// runs in every CTA, and the dequantization y = acc * (gamma s / 127) (§5.3)
// is fused into the store.
//
// Layout of the work.  A CTA owns a contiguous run of rows (N shared out as
// evenly as the grid allows), i.e. one contiguous byte range of the packed
// matrix.  With segs 16-byte segments per row (64 weights each) and
// R = floor(threads / segs), thread t < R segs keeps column c = t mod segs:
// the 64 activation codes of segment c sit in its registers for the whole
// kernel, and in its i-th step it reads the segment t + i R segs of the
// CTA's range, i.e. column c of row t / segs + i R.  So every step of the CTA
// reads one contiguous block of R rows, every load is a 16-byte coalesced
// load, and no activation byte is read from shared memory per weight.  The
// lanes of a warp that share a row (a warp spans at most two rows when a row
// has 32 segments or more) add their parts with one segmented warp reduction
// and one shared atomic per row.
//
// Early start.  A CTA uses at most half of an SM (512 threads, 64 registers
// each, a few KB of shared memory), so the CTAs of the next launch in the
// stream are resident while this one runs (programmatic dependent launch: the
// trigger follows the wait).  Before its wait a CTA moves the first bytes of
// its rows into L2 with bulk prefetches, which return no data (L2 is the
// point of coherence, so the loads after the wait still see whatever the
// previous kernel writes).  After the wait it reads the token, quantizes it
// and streams its rows with D 16-byte loads in flight per thread.
#include "bl_common.cuh"
#include "bl_gemv.cuh"
#include "bl_kernels.h"

#ifndef BL_G1_PREFETCH
#define BL_G1_PREFETCH 65536  // bytes of each CTA's rows prefetched into L2 before the wait
#endif

namespace bl {

constexpr int kG1MaxThreads = 512;
constexpr int64_t kG1MaxSmem = 96 * 1024;  // two CTAs (of consecutive launches) per SM

// Shared memory: the raw token (K elements), its codes (64 per segment) and
// the CTA's row sums.
__host__ __device__ inline int64_t gemv1_smem_bytes(int64_t rowbytes, int64_t K, int xsize, int64_t rows_per_cta) {
  return (K * xsize + 15) / 16 * 16 + rowbytes * 4 + 4 * rows_per_cta;
}

// 16-byte words of raw activations per 16 elements.
template <int XDT>
constexpr int g1_xwords() {
  return XDT == BL_F32 ? 4 : (XDT == BL_BF16 ? 2 : 1);
}

constexpr int kG1Depth = 6;  // 16-byte weight loads in flight per thread

// 16-byte copy global -> shared without registers (L2 only).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// sum over the 64 weights of a segment of d x, d the stored digit: the mask
// w & (3 << 2j) leaves digit j of every byte in place (4^j d), so accumulator
// j collects 4^j sum d x and the factor comes off exactly with a shift.
// X[w] byte 4j + b holds the code of weight 16 w + 4 b + j of the segment.
__device__ __forceinline__ int dot_seg_i2(const uint4 wv, const uint4 (&X)[4]) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    a0 = dp4a_us(wd[w] & 0x03030303u, X[w].x, a0);
    a1 = dp4a_us(wd[w] & 0x0c0c0c0cu, X[w].y, a1);
    a2 = dp4a_us(wd[w] & 0x30303030u, X[w].z, a2);
    a3 = dp4a_us(wd[w] & 0xc0c0c0c0u, X[w].w, a3);
  }
  return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
}

// XC: 16-element chunks of the token per thread (the chunks of segment c are
// 4c .. 4c + 3; chunk g of thread t is t + T u, u < XC).
template <int XDT, int XC>
__global__ void __launch_bounds__(kG1MaxThreads, 2)
    gemv1_i2_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                    int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                    void* __restrict__ y, int ydt, int write_scale, const RowGroups rg, int R) {
  constexpr int D = kG1Depth;
  constexpr int kXW = g1_xwords<XDT>();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t red[kG1MaxThreads / 32];
  __shared__ float sh_gam[kMaxRowGroups];
  __shared__ int64_t sh_end[kMaxRowGroups];
  __shared__ float sh_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = blockDim.x;
  const int segs = static_cast<int>(rowbytes >> 4);
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));
  const bool active = tid < R * segs;
  const int r0 = active ? tid / segs : 0;  // this thread's first row (of the CTA's rows)
  const int c = active ? tid - r0 * segs : 0;
  // rows of this thread: r0, r0 + R, ... below nrows
  const int nr = (active && r0 < nrows) ? (nrows - r0 + R - 1) / R : 0;
  const uint32_t step = static_cast<uint32_t>(R * rowbytes);  // bytes between a thread's rows (<= 8 KB)
  const int kch = static_cast<int>(K >> 4);  // chunks holding weights (K % 16 == 0)
  const int nch = 4 * segs;                  // chunks of the packed rows (the last ones are padding)
  uint8_t* xraw = smem;                                             // [K] raw token
  uint8_t* xs = smem + (K * kXW + 15) / 16 * 16;                    // [4][segs] 16-byte code slots
  int* rsum = reinterpret_cast<int*>(xs + rowbytes * 4);           // [nrows]

  // 0. before the wait: the first bytes of the CTA's rows into L2
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < BL_G1_PREFETCH ? bytes : BL_G1_PREFETCH);
  }
  for (int i = tid; i < nrows; i += T) rsum[i] = 0;
#pragma unroll
  for (int i = 0; i < kMaxRowGroups; ++i)
    if (tid == i) sh_end[i] = rg.end[i];
  pdl_wait(packed, gamma, x, scale, y);
  pdl_launch_dependents();

  // 1. the token into shared memory, and the first D rows of this thread
  //    into registers, all in flight together
#pragma unroll
  for (int u = 0; u < XC; ++u) {
    const int g = tid + T * u;
    if (g < kch)
#pragma unroll
      for (int i = 0; i < kXW; ++i)
        cp_async16(xraw + (static_cast<int64_t>(g) * kXW + i) * 16,
                   static_cast<const uint8_t*>(x) + (static_cast<int64_t>(g) * kXW + i) * 16);
  }
  const uint8_t* lp = packed + row0 * rowbytes + static_cast<int64_t>(tid) * 16;  // next load
  uint4 buf[D];
#pragma unroll
  for (int j = 0; j < D; ++j) {
    buf[j] = make_uint4(0, 0, 0, 0);
    if (j < nr) buf[j] = ld_stream(reinterpret_cast<const uint4*>(lp));
    lp += step;
  }
  if (tid < rg.n) sh_gam[tid] = __ldcg(gamma + tid);
  if (XDT == BL_I8 && tid == 0) sh_s = __ldcg(scale);
  cp_async_wait_all();
  __syncthreads();  // the raw token, zeroed row sums, gammas and the given scale are visible

  // 2. per-token absmax (fmaxf, so a NaN is ignored; the result is a
  //    non-negative float, whose bits order like unsigned integers)
  float s;
  if constexpr (XDT != BL_I8) {
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < kch)
#pragma unroll
        for (int i = 0; i < kXW; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(xraw + (static_cast<int64_t>(g) * kXW + i) * 16);
          if constexpr (XDT == BL_F32) {
            amax = fmaxf(fmaxf(amax, fabsf(__uint_as_float(v.x))), fabsf(__uint_as_float(v.y)));
            amax = fmaxf(fmaxf(amax, fabsf(__uint_as_float(v.z))), fabsf(__uint_as_float(v.w)));
          } else {
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              amax = fmaxf(amax, fabsf(__uint_as_float(wv[h] << 16)));
              amax = fmaxf(amax, fabsf(__uint_as_float(wv[h] & 0xffff0000u)));
            }
          }
        }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint32_t mm = 0;
    for (int w = 0; w < (T >> 5); ++w) mm = max(mm, red[w]);
    s = fmaxf(__uint_as_float(mm), 1e-6f);
  } else {
    s = sh_s;
  }

  // 3. the codes, written in the slot layout of the packed words
  {
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s);
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < nch) {
        uint32_t P[4] = {0u, 0u, 0u, 0u};  // padding chunks (past K): code 0
        if (g < kch) {
          const uint8_t* src = xraw + static_cast<int64_t>(g) * kXW * 16;
          if constexpr (XDT == BL_I8) {
            const uint4 v = *reinterpret_cast<const uint4*>(src);
            P[0] = v.x;
            P[1] = v.y;
            P[2] = v.z;
            P[3] = v.w;
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // eight elements at a time
              float e[8];
              if constexpr (XDT == BL_F32) {
                const uint4 v0 = *reinterpret_cast<const uint4*>(src + 32 * h);
                const uint4 v1 = *reinterpret_cast<const uint4*>(src + 32 * h + 16);
                e[0] = __uint_as_float(v0.x); e[1] = __uint_as_float(v0.y);
                e[2] = __uint_as_float(v0.z); e[3] = __uint_as_float(v0.w);
                e[4] = __uint_as_float(v1.x); e[5] = __uint_as_float(v1.y);
                e[6] = __uint_as_float(v1.z); e[7] = __uint_as_float(v1.w);
              } else {
                const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * h);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  e[2 * k] = __uint_as_float(wv[k] << 16);
                  e[2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
                }
              }
              int q[8];
              quant_act_fast_n<8>(e, s, c127, q);
              P[2 * h] = pack4(q);
              P[2 * h + 1] = pack4(q + 4);
            }
          }
        }
        *reinterpret_cast<uint4*>(xs + (static_cast<int64_t>(g & 3) * segs + (g >> 2)) * 16) =
            i2_slot(P[0], P[1], P[2], P[3]);
      }
    }
  }
  __syncthreads();

  // 4. this thread's 64 codes and their sum (digits are q + 1: the sum is
  //    taken off once per row)
  uint4 X[4];
  int csum = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    X[w] = active ? *reinterpret_cast<const uint4*>(xs + (static_cast<int64_t>(w) * segs + c) * 16)
                  : make_uint4(0, 0, 0, 0);
    csum = __dp4a(static_cast<int>(X[w].x), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].y), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].z), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].w), 0x01010101, csum);
  }
  // lanes with the same first row share a row at every step
  const uint32_t gmask = __match_any_sync(0xffffffffu, active ? r0 : -1 - lane);
  const bool leader = (__ffs(gmask) - 1) == lane;

  // 5. the stream: consume the oldest load, refill its slot D rows ahead (the
  //    lanes of a group take the same branches: same rows)
  int* rs = rsum + r0;
  for (int k0 = 0; k0 < nr; k0 += D) {
#pragma unroll
    for (int j = 0; j < D; ++j) {
      if (k0 + j < nr) {
        const uint4 wv = buf[j];
        if (k0 + j + D < nr) buf[j] = ld_stream(reinterpret_cast<const uint4*>(lp));
        lp += step;
        const int v = __reduce_add_sync(gmask, dot_seg_i2(wv, X) - csum);
        if (leader) atomicAdd(rs, v);
        rs += R;
      }
    }
  }
  __syncthreads();  // every row sum is complete

  // 6. dequantize and store the CTA's outputs (coalesced)
  const float cf1 = dequant_factor(sh_gam[0], s);
  for (int r = tid; r < nrows; r += T) {
    const int a = rsum[r];
    const int64_t n = row0 + r;
    float cf = cf1;
    if (rg.n > 1) {  // the row's group: the first g with n < end[g]
      int gi = 0;
      while (gi + 1 < rg.n && n >= sh_end[gi]) ++gi;
      cf = dequant_factor(sh_gam[gi], s);
    }
    if (ydt == BL_I32)
      static_cast<int32_t*>(y)[n] = a;
    else if (ydt == BL_F32)
      static_cast<float*>(y)[n] = __fmul_rn(__int2float_rn(a), cf);
    else
      static_cast<__nv_bfloat16*>(y)[n] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cf));
  }
  if (XDT != BL_I8 && write_scale && b == 0 && tid == 0) scale[0] = s;
}

// Launch geometry: R rows per step, threads rounded up to whole warps, and
// the token chunks per thread (1, 2 or 4).
struct Gemv1Geom {
  int R, threads, xc;
  int64_t grid, rows_per_cta, smem;
};

static bool gemv1_geom(int64_t N, int64_t K, int64_t rowbytes, int xdt, Gemv1Geom* g) {
  const int64_t segs = rowbytes / 16;
  if (K % 16 != 0 || segs < 1 || segs > kG1MaxThreads) return false;
  const int64_t sms = device_sms();
  g->grid = N < sms ? N : sms;
  g->rows_per_cta = (N + g->grid - 1) / g->grid;
  const int xsize = xdt == BL_F32 ? 4 : (xdt == BL_BF16 ? 2 : 1);
  g->smem = gemv1_smem_bytes(rowbytes, K, xsize, g->rows_per_cta);
  if (g->smem > kG1MaxSmem) return false;
  int64_t R = kG1MaxThreads / segs;
  if (R > g->rows_per_cta) R = g->rows_per_cta;
  g->R = static_cast<int>(R);
  g->threads = static_cast<int>((R * segs + 31) / 32 * 32);
  const int64_t per = (4 * segs + g->threads - 1) / g->threads;
  g->xc = per <= 1 ? 1 : (per <= 2 ? 2 : 4);
  return true;
}

bool gemv1_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt) {
  Gemv1Geom g;
  return gemv1_geom(N, K, rowbytes, xdt, &g);
}

template <int XDT, int XC>
static cudaError_t launch_gemv1_t(const Gemv1Geom& g, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, cudaStream_t st) {
  auto kern = gemv1_i2_kernel<XDT, XC>;
  const size_t smem = static_cast<size_t>(g.smem);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_pdl(kern, static_cast<unsigned>(g.grid), static_cast<unsigned>(g.threads), smem, st,
                                   packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, g.R);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int XDT>
static cudaError_t launch_gemv1_x(const Gemv1Geom& g, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, cudaStream_t st) {
  if (g.xc == 1) return launch_gemv1_t<XDT, 1>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  if (g.xc == 2) return launch_gemv1_t<XDT, 2>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  return launch_gemv1_t<XDT, 4>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
}

cudaError_t launch_gemv1(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                         const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg,
                         cudaStream_t st) {
  Gemv1Geom g;
  if (!gemv1_geom(N, K, rowbytes, xdt, &g)) return cudaErrorInvalidValue;
  if (xdt == BL_F32) return launch_gemv1_x<BL_F32>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 1, rg, st);
  if (xdt == BL_BF16) return launch_gemv1_x<BL_BF16>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 1, rg, st);
  return launch_gemv1_x<BL_I8>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 0, rg, st);
}

}  // namespace bl
