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
#include "bl_sm100.cuh"

#ifndef BL_G1_PREFETCH
#define BL_G1_PREFETCH 65536  // bytes of each CTA's rows prefetched into L2 before the wait
#endif
#ifndef BL_G1_PREFETCH2
#define BL_G1_PREFETCH2 0  // bytes prefetched into L2 after the wait, while the token is quantized
#endif

namespace bl {

#ifndef BL_G1_MAXT
#define BL_G1_MAXT 512
#endif
#ifndef BL_G1_MAXSMEM
#define BL_G1_MAXSMEM (110 * 1024)
#endif
constexpr int kG1MaxThreads = BL_G1_MAXT;
constexpr int64_t kG1MaxSmem = BL_G1_MAXSMEM;  // two CTAs (of consecutive launches) per SM

// 16-byte words of raw activations per 16 elements.
template <int XDT>
constexpr int g1_xwords() {
  return XDT == BL_F32 ? 4 : (XDT == BL_BF16 ? 2 : 1);
}

// Stages of a thread's row ring: rows copied ahead into shared memory by
// cp.async (no registers held, and no per-warp limit on loads in flight).
constexpr int kG1StagesMax = 8;
constexpr long long kG1WaitCycles = 1ll << 30;  // bound of the token wait (~0.5 s)

// 16-byte copy global -> shared (at a shared-window address) without
// registers, through L2 only.
__device__ __forceinline__ void cp_async16_s(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void red_add_s(uint32_t a, int v) {
  asm volatile("red.shared.add.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bytes of the token region: the raw token, and later its codes in the slot
// layout (4 x 16 bytes per segment), whichever is larger.
__host__ __device__ inline int64_t g1_xregion(int64_t K, int xwords, int64_t rowbytes) {
  const int64_t raw = K * xwords;  // xwords 16-byte words per 16 elements: K * xwords bytes
  return ((raw > rowbytes * 4 ? raw : rowbytes * 4) + 15) / 16 * 16;
}

// a0 + sum over the 64 weights of a segment of d x, d the stored digit: the mask
// w & (3 << 2j) leaves digit j of every byte in place (4^j d), so accumulator
// j collects 4^j sum d x and the factor comes off exactly with a shift.
// X[w] byte 4j + b holds the code of weight 16 w + 4 b + j of the segment.
__device__ __forceinline__ int dot_seg_i2(const uint4 wv, const uint4 (&X)[4], int a0) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  int a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    a0 = dp4a_us(wd[w] & 0x03030303u, X[w].x, a0);
    a1 = dp4a_us(wd[w] & 0x0c0c0c0cu, X[w].y, a1);
    a2 = dp4a_us(wd[w] & 0x30303030u, X[w].z, a2);
    a3 = dp4a_us(wd[w] & 0xc0c0c0c0u, X[w].w, a3);
  }
  return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
}

// The INT8 codes of 16 activations e[0..15] against scale s (c127 =
// fl(127 / s)), returned as the 16-byte slot of their packed word (byte
// 4j + b = code of element 4b + j), or with SLOT false in element order.  Each code is rint(fl(fl(e / s) 127)),
// taken division-free as in quant_act_fast: t_a = fl(e c127) is within 2^-14
// of t, so rint(t_a) = rint(t) unless t_a lies within 2^-14 of a
// half-integer.  rint(t_a) comes from the adder (t_a + 1.5 * 2^23 rounds to
// nearest even and leaves the code in the low byte of the sum's bits, two's
// complement, |code| <= 127), the margin is checked once per eight elements
// on the largest |t_a - rint(t_a)| (an exact difference), and only a group
// with an element that close to a tie takes the exact quotient.
template <bool SLOT = true>
__device__ __forceinline__ uint4 g1_codes16(const float (&e)[16], float s, float c127) {
  // element pairs through the paired fp32 unit (each lane rounds to nearest
  // as the scalar operation does); ta - rint(ta) = fma(rint(ta), -1, ta) is
  // exact, so one rounding of an exact value
  const float2 c2 = make_float2(c127, c127), mg = make_float2(12582912.0f, 12582912.0f);
  const float2 nmg = make_float2(-12582912.0f, -12582912.0f), m1 = make_float2(-1.0f, -1.0f);
  uint32_t r[16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float worst = 0.0f;
#pragma unroll
    for (int j = 8 * h; j < 8 * h + 8; j += 2) {
      const float2 ta = __fmul2_rn(make_float2(e[j], e[j + 1]), c2);
      const float2 r2 = __fadd2_rn(ta, mg);
      const float2 d = __ffma2_rn(__fadd2_rn(r2, nmg), m1, ta);
      worst = fmaxf(worst, fmaxf(fabsf(d.x), fabsf(d.y)));
      r[j] = __float_as_uint(r2.x);
      r[j + 1] = __float_as_uint(r2.y);
    }
    if (!(worst < 0.49993896484375f)) {  // rare: some element is near a tie
#pragma unroll
      for (int j = 8 * h; j < 8 * h + 8; ++j) {
        const float ta = __fmul_rn(e[j], c127);
        if (!(fabsf(__fsub_rn(ta, rintf(ta))) < 0.49993896484375f))
          r[j] = static_cast<uint32_t>(quant_act_slow(e[j], s));
      }
    }
  }
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (SLOT)  // byte 4j + b = code of element 4b + j
      w[j] = __byte_perm(__byte_perm(r[j], r[4 + j], 0x0040), __byte_perm(r[8 + j], r[12 + j], 0x0040), 0x5410);
    else  // linear: byte 4j + b = code of element 4j + b
      w[j] = __byte_perm(__byte_perm(r[4 * j], r[4 * j + 1], 0x0040), __byte_perm(r[4 * j + 2], r[4 * j + 3], 0x0040),
                         0x5410);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// XC: 16-element chunks of the token per thread (the chunks of segment c are
// 4c .. 4c + 3; chunk g of thread t is t + T u, u < XC).  S: stages of the
// thread's row ring.  ALIGNED: segs % 32 == 0, so every warp lies in one row.
template <int XDT, int XC, int S, bool ALIGNED>
__global__ void __launch_bounds__(kG1MaxThreads, 1024 / kG1MaxThreads)
    gemv1_i2_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                    int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                    void* __restrict__ y, int ydt, int write_scale, const RowGroups rg, int R, int lpr, void* ws) {
  constexpr int kXW = g1_xwords<XDT>();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t red[kG1MaxThreads / 32];
  __shared__ float sh_gam[kMaxRowGroups];
  __shared__ int64_t sh_end[kMaxRowGroups];
  __shared__ float sh_s;
  __shared__ __align__(8) uint64_t xbar;  // completion of the token's bulk copy

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = blockDim.x;
  const int segs = static_cast<int>(rowbytes >> 4);
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));
  // lpr lanes per row (segs, or segs rounded up to whole warps so that every
  // warp lies in one row); lane c < segs of a row holds column c
  // (the idle lanes of a row take part in every step with zero codes and no
  // copies, so all lanes of a warp run the same steps)
  const int r0_raw = tid / lpr, c_raw = tid - r0_raw * lpr;
  const bool row_ok = r0_raw < R;
  const bool col_ok = row_ok && c_raw < segs;
  const int r0 = row_ok ? r0_raw : 0;  // this thread's first row (of the CTA's rows)
  const int c = col_ok ? c_raw : 0;
  // rows of this thread: r0, r0 + R, ... below nrows
  const int nr = (row_ok && r0 < nrows) ? (nrows - r0 + R - 1) / R : 0;
  const uint32_t step = static_cast<uint32_t>(R * rowbytes);  // bytes between a thread's rows (<= 8 KB)
  const int kch = static_cast<int>(K >> 4);  // chunks holding weights (K % 16 == 0)
  const int nch = 4 * segs;                  // chunks of the packed rows (the last ones are padding)
  const uint32_t xbytes = static_cast<uint32_t>(K * kXW);  // raw token bytes (a multiple of 16)
  // shared memory: the token region (first the raw token, then its codes in
  // the slot layout [4][segs] x 16 bytes), the row ring [S][T] x 16 bytes,
  // the row sums [nrows]
  const int64_t xreg = g1_xregion(K, kXW, rowbytes);
  uint8_t* xbuf = smem;
  const uint32_t ring_s = smem_u32(smem + xreg) + 16u * tid;       // slot 0 of this thread
  const uint32_t tstride = 16u * T;                                 // bytes between its slots
  int* rsum = reinterpret_cast<int*>(smem + xreg + static_cast<int64_t>(S) * T * 16);

  // 0. before the wait: the first bytes of the CTA's rows into L2, the row
  //    sums zeroed, the token barrier set up
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < BL_G1_PREFETCH ? bytes : BL_G1_PREFETCH);
  }
  for (int i = tid; i < nrows; i += T) rsum[i] = 0;
#pragma unroll
  for (int i = 0; i < kMaxRowGroups; ++i)
    if (tid == i) sh_end[i] = rg.end[i];
  if (tid == 0) {
    mbar_init(&xbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait(packed, gamma, x, scale, y);
  pdl_launch_dependents();

  // 1. while the token is read and quantized the memory system would idle:
  //    the next part of the CTA's rows moves into L2 meanwhile
  if (BL_G1_PREFETCH2 > 0) {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    const int64_t lo = bytes < BL_G1_PREFETCH ? bytes : BL_G1_PREFETCH;
    const int64_t hi = bytes < lo + BL_G1_PREFETCH2 ? bytes : lo + BL_G1_PREFETCH2;
    if (hi > lo) l2_prefetch_bulk(packed + row0 * rowbytes + lo, hi - lo);
  }
  // 1. the token by one bulk copy; the rows follow once it has landed (row
  //    copies issued alongside slow the token's copy several fold, and the
  //    token is on the critical path while the rows have the whole
  //    quantization to arrive)
  if (tid == 0) {
    mbar_expect_tx(&xbar, xbytes);
    bulk_load(xbuf, x, xbytes, &xbar);
  }
  if (tid < rg.n) sh_gam[tid] = __ldcg(gamma + tid);
  if (XDT == BL_I8 && tid == 0) sh_s = __ldcg(scale);
  // every thread waits (bounded) for the token; if any gives up, the CTA
  // records the timeout, lets the copy land (bounded) and leaves
  const bool got = wait_drain(&xbar, 0, kG1WaitCycles);
  if (__syncthreads_or(!got)) {  // also: zeroed row sums, gammas and the given scale are visible
    if (tid == 0) {
      set_flag(ws, kFlagTimeout, 0x601);
      wait_drain(&xbar, 0, kG1WaitCycles);
    }
    return;
  }
  // the thread's first S - 1 rows (one cp.async group each, empty past its rows)
  const uint8_t* gp = packed + (row0 + r0) * rowbytes + static_cast<int64_t>(c) * 16;  // next row to copy
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (col_ok && j < nr) cp_async16_s(ring_s + j * tstride, gp);
    cp_async_commit();
    gp += step;
  }

  // 2. per-token absmax.  The inputs are finite, so the magnitude bits
  //    (sign cleared) order like unsigned integers: the maximum is taken on
  //    them, two bf16 values per 32-bit word at a time.
  float s;
  if constexpr (XDT != BL_I8) {
    uint32_t mx = 0;  // fp32: magnitude bits; bf16: two 16-bit magnitudes
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < kch)
#pragma unroll
        for (int i = 0; i < kXW; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(g) * kXW + i) * 16);
          if constexpr (XDT == BL_F32) {
            const uint32_t a = max(v.x & 0x7fffffffu, v.y & 0x7fffffffu);
            const uint32_t b2 = max(v.z & 0x7fffffffu, v.w & 0x7fffffffu);
            mx = max(mx, max(a, b2));
          } else {
            const uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
            const uint32_t b2 = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
            mx = __vmaxu2(mx, __vmaxu2(a, b2));
          }
        }
    }
    if constexpr (XDT == BL_BF16) mx = max(mx & 0xffffu, mx >> 16) << 16;  // as fp32 bits
    const uint32_t m = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint32_t mm = 0;
    for (int w = 0; w < (T >> 5); ++w) mm = max(mm, red[w]);
    s = fmaxf(__uint_as_float(mm), 1e-6f);
  } else {
    s = sh_s;
  }

  // 3. the codes of the thread's chunks (from the raw token), then, once every
  //    thread has read its raw chunks, written over the token region in the
  //    slot layout of the packed words
  {
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s);
    uint4 slot[XC];
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      uint32_t P[4] = {0u, 0u, 0u, 0u};  // padding chunks (past K): code 0
      if (g < kch) {
        const uint8_t* src = xbuf + static_cast<int64_t>(g) * kXW * 16;
        if constexpr (XDT == BL_I8) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          P[0] = v.x;
          P[1] = v.y;
          P[2] = v.z;
          P[3] = v.w;
        } else {
          float e[16];
          if constexpr (XDT == BL_F32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              e[4 * i] = __uint_as_float(v.x); e[4 * i + 1] = __uint_as_float(v.y);
              e[4 * i + 2] = __uint_as_float(v.z); e[4 * i + 3] = __uint_as_float(v.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                e[8 * i + 2 * k] = __uint_as_float(wv[k] << 16);
                e[8 * i + 2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
              }
            }
          }
          slot[u] = g1_codes16(e, s, c127);
          continue;
        }
      }
      slot[u] = i2_slot(P[0], P[1], P[2], P[3]);
    }
    __syncthreads();  // every raw chunk has been read
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < nch) *reinterpret_cast<uint4*>(xbuf + (static_cast<int64_t>(g & 3) * segs + (g >> 2)) * 16) = slot[u];
    }
  }
  __syncthreads();

  // 4. this thread's 64 codes and their sum (digits are q + 1: the sum is
  //    taken off once per row, as the starting value of the row's sum)
  uint4 X[4];
  int csum = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    X[w] = col_ok ? *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(w) * segs + c) * 16)
                  : make_uint4(0, 0, 0, 0);
    csum = __dp4a(static_cast<int>(X[w].x), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].y), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].z), 0x01010101, csum);
    csum = __dp4a(static_cast<int>(X[w].w), 0x01010101, csum);
  }
  const int init = -csum;
  // lanes with the same first row share a row at every step
  const uint32_t gmask = ALIGNED ? 0xffffffffu : __match_any_sync(0xffffffffu, row_ok ? r0_raw : -1 - lane);
  const bool leader = ALIGNED ? lane == 0 : (__ffs(gmask) - 1) == lane;
  uint32_t rs = smem_u32(rsum + r0);    // this thread's next row sum
  const uint32_t rstep = 4u * R;

  // 5. the stream: copy row k + S - 1 into the slot freed by row k - 1, wait
  //    for row k, consume it (the lanes of a group take the same branches:
  //    same rows); each thread reads back only its own slots.  Blocks of S
  //    rows with no guard while every refill is a row of the thread, then
  //    the rest one by one.
  auto consume = [&](const uint4 wv) {
    int v = dot_seg_i2(wv, X, init);
    v = __reduce_add_sync(gmask, v);
    if (leader) red_add_s(rs, v);
    rs += rstep;
  };
  int k = 0;
  for (; k < nr - 2 * S + 2; k += S) {
#pragma unroll
    for (int j = 0; j < S; ++j) {
      if (col_ok) cp_async16_s(ring_s + ((j + S - 1) % S) * tstride, gp);
      cp_async_commit();
      gp += step;
      cp_async_wait<S - 1>();
      consume(lds128(ring_s + j * tstride));
    }
  }
  for (; k < nr; ++k) {
    if (col_ok && k + S - 1 < nr) cp_async16_s(ring_s + ((k + S - 1) % S) * tstride, gp);
    cp_async_commit();
    gp += step;
    cp_async_wait<S - 1>();
    consume(lds128(ring_s + (k % S) * tstride));
  }
  cp_async_wait<0>();
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

// ---------------------------------------------------------------------------
// One token on base-3 rows (5 weights per byte: digit j of byte b is
// floor(b / 3^j) mod 3, the stored digit q + 1), in the layout of
// gemv1_i2_kernel: a 16-byte segment holds 80 weights, thread t keeps the 80
// activation codes of its column c in registers (xlo[p]: the codes of digits
// 0..3 of byte p; xhi[j] byte i: the code of digit 4 of byte 4j + i) and
// reads segment t + i R segs of its CTA's range at step i, so the rows of a
// step are one contiguous block and the lanes of a row are used as densely
// as in the 2-bit kernel.  A byte is decoded by one 4-byte shared lookup in
// the lane's own copy of a 256-entry table (copy L in bank L: a warp's
// lookups never conflict): byte j of the entry is digit j (j < 4) and bits
// 2..3 of byte 0 hold digit 4.  Per packed word: four lookups, four dp4a on
// the masked entries against xlo, and one dp4a on the gathered fifth digits
// (4 d4 in each byte) against xhi, whose factor 4 comes off at the end.  The
// table depends on nothing the previous kernel writes, so it is filled before
// the dependency wait.  Bytes 243..255 are not produced by the packer; they
// decode as five zero weights.  The token's codes are written in element
// order over the raw token (80 per segment, 0 past K).
// ---------------------------------------------------------------------------
constexpr int kT1LutBytes = 256 * 32 * 4;

__host__ __device__ inline int64_t g1t5_xregion(int64_t K, int xwords, int64_t rowbytes) {
  const int64_t raw = K * xwords;     // the raw token: xwords 16-byte words per 16 elements
  const int64_t codes = rowbytes * 5;  // 80 codes per 16-byte segment
  return ((raw > codes ? raw : codes) + 15) / 16 * 16;
}

// a0 + sum over the 80 weights of a base-3 segment of d x (d the stored digit)
__device__ __forceinline__ int dot_seg_t5(const uint4 wv, const uint32_t (&xlo)[16], const uint32_t (&xhi)[4],
                                          uint32_t lut_l, int a0) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  int v = a0, vh = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t L[4];
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
      const uint32_t a = lut_l + (__byte_perm(wd[w], 0, 0x4440 + bb) << 7);  // entry e of copy L: 128 e + 4 L
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(L[bb]) : "r"(a) : "memory");
    }
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) v = dp4a_us(L[bb] & 0x03030303u, xlo[4 * w + bb], v);
    const uint32_t H =
        __byte_perm(__byte_perm(L[0], L[1], 0x0040), __byte_perm(L[2], L[3], 0x0040), 0x5410) & 0x0c0c0c0cu;
    vh = dp4a_us(H, xhi[w], vh);
  }
  return v + (vh >> 2);
}

template <int XDT, int XC, int S, bool ALIGNED>
__global__ void __launch_bounds__(kG1MaxThreads, 1024 / kG1MaxThreads)
    gemv1_t5_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                    int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                    void* __restrict__ y, int ydt, int write_scale, const RowGroups rg, int R, int lpr, void* ws) {
  constexpr int kXW = g1_xwords<XDT>();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t red[kG1MaxThreads / 32];
  __shared__ float sh_gam[kMaxRowGroups];
  __shared__ int64_t sh_end[kMaxRowGroups];
  __shared__ float sh_s;
  __shared__ __align__(8) uint64_t xbar;  // completion of the token's bulk copy

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = blockDim.x;
  const int segs = static_cast<int>(rowbytes >> 4);
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));
  const int r0_raw = tid / lpr, c_raw = tid - r0_raw * lpr;
  const bool row_ok = r0_raw < R;
  const bool col_ok = row_ok && c_raw < segs;
  const int r0 = row_ok ? r0_raw : 0;
  const int c = col_ok ? c_raw : 0;
  const int nr = (row_ok && r0 < nrows) ? (nrows - r0 + R - 1) / R : 0;
  const uint32_t step = static_cast<uint32_t>(R * rowbytes);
  const int kch = static_cast<int>(K >> 4);  // 16-element chunks of the token (K % 16 == 0)
  const int nch = 5 * segs;                  // 16-code chunks of the codes region (0 past K)
  const uint32_t xbytes = static_cast<uint32_t>(K * kXW);
  // shared memory: the table [256][32] x 4 bytes, the token region (the raw
  // token, then its codes), the row ring [S][T] x 16 bytes, the row sums
  const int64_t xreg = g1t5_xregion(K, kXW, rowbytes);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  uint8_t* xbuf = smem + kT1LutBytes;
  const uint32_t ring_s = smem_u32(xbuf + xreg) + 16u * tid;
  const uint32_t tstride = 16u * T;
  int* rsum = reinterpret_cast<int*>(xbuf + xreg + static_cast<int64_t>(S) * T * 16);

  // 0. before the wait: the first bytes of the CTA's rows into L2, the
  //    table, the row sums zeroed, the token barrier set up
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < BL_G1_PREFETCH ? bytes : BL_G1_PREFETCH);
  }
  for (int i = tid; i < 256 * 32; i += T) {
    const int e = i >> 5;
    uint32_t d[5] = {1, 1, 1, 1, 1};  // bytes past 242: five zero weights
    if (e < 243) {
      int v = e;
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        d[j] = static_cast<uint32_t>(v % 3);
        v /= 3;
      }
    }
    lut[i] = (d[0] | (d[4] << 2)) | (d[1] << 8) | (d[2] << 16) | (d[3] << 24);
  }
  for (int i = tid; i < nrows; i += T) rsum[i] = 0;
#pragma unroll
  for (int i = 0; i < kMaxRowGroups; ++i)
    if (tid == i) sh_end[i] = rg.end[i];
  if (tid == 0) {
    mbar_init(&xbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait(packed, gamma, x, scale, y);
  pdl_launch_dependents();

  // 1. the token by one bulk copy (bounded wait: on expiry the CTA records the
  //    timeout, lets the copy land and leaves)
  if (tid == 0) {
    mbar_expect_tx(&xbar, xbytes);
    bulk_load(xbuf, x, xbytes, &xbar);
  }
  if (tid < rg.n) sh_gam[tid] = __ldcg(gamma + tid);
  if (XDT == BL_I8 && tid == 0) sh_s = __ldcg(scale);
  const bool got = wait_drain(&xbar, 0, kG1WaitCycles);
  if (__syncthreads_or(!got)) {
    if (tid == 0) {
      set_flag(ws, kFlagTimeout, 0x602);
      wait_drain(&xbar, 0, kG1WaitCycles);
    }
    return;
  }
  const uint8_t* gp = packed + (row0 + r0) * rowbytes + static_cast<int64_t>(c) * 16;
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (col_ok && j < nr) cp_async16_s(ring_s + j * tstride, gp);
    cp_async_commit();
    gp += step;
  }

  // 2. per-token absmax on the magnitude bits (finite inputs)
  float s;
  if constexpr (XDT != BL_I8) {
    uint32_t mx = 0;
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < kch)
#pragma unroll
        for (int i = 0; i < kXW; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(g) * kXW + i) * 16);
          if constexpr (XDT == BL_F32) {
            const uint32_t a = max(v.x & 0x7fffffffu, v.y & 0x7fffffffu);
            const uint32_t b2 = max(v.z & 0x7fffffffu, v.w & 0x7fffffffu);
            mx = max(mx, max(a, b2));
          } else {
            const uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
            const uint32_t b2 = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
            mx = __vmaxu2(mx, __vmaxu2(a, b2));
          }
        }
    }
    if constexpr (XDT == BL_BF16) mx = max(mx & 0xffffu, mx >> 16) << 16;
    const uint32_t m = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint32_t mm = 0;
    for (int w = 0; w < (T >> 5); ++w) mm = max(mm, red[w]);
    s = fmaxf(__uint_as_float(mm), 1e-6f);
  } else {
    s = sh_s;
  }

  // 3. the codes of the thread's chunks in element order, written over the
  //    raw token once every thread has read its raw chunks
  {
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s);
    uint4 cw[XC];
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      cw[u] = make_uint4(0u, 0u, 0u, 0u);  // padding chunks (past K): code 0
      if (g < kch) {
        const uint8_t* src = xbuf + static_cast<int64_t>(g) * kXW * 16;
        if constexpr (XDT == BL_I8) {
          cw[u] = *reinterpret_cast<const uint4*>(src);
        } else {
          float e[16];
          if constexpr (XDT == BL_F32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              e[4 * i] = __uint_as_float(v.x); e[4 * i + 1] = __uint_as_float(v.y);
              e[4 * i + 2] = __uint_as_float(v.z); e[4 * i + 3] = __uint_as_float(v.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                e[8 * i + 2 * k] = __uint_as_float(wv[k] << 16);
                e[8 * i + 2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
              }
            }
          }
          cw[u] = g1_codes16<false>(e, s, c127);
        }
      }
    }
    __syncthreads();  // every raw chunk has been read
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < nch) *reinterpret_cast<uint4*>(xbuf + static_cast<int64_t>(g) * 16) = cw[u];
    }
  }
  __syncthreads();

  // 4. this thread's 80 codes (xlo / xhi) and their sum (digits are q + 1:
  //    the sum is taken off once per row, as the row sum's starting value)
  uint32_t xlo[16], xhi[4];
  int csum = 0;
  {
    uint32_t w[20];
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const uint4 t = col_ok ? *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(c) * 5 + i) * 16)
                             : make_uint4(0u, 0u, 0u, 0u);
      w[4 * i] = t.x;
      w[4 * i + 1] = t.y;
      w[4 * i + 2] = t.z;
      w[4 * i + 3] = t.w;
    }
#pragma unroll
    for (int i = 0; i < 20; ++i) csum = __dp4a(static_cast<int>(w[i]), 0x01010101, csum);
#pragma unroll
    for (int p = 0; p < 16; ++p) {  // codes 5p .. 5p + 3 of the segment
      const int o = 5 * p;
      xlo[p] = __byte_perm(w[o >> 2], w[(o >> 2) + 1], 0x3210 + 0x1111 * (o & 3));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // code 5p + 4 of bytes p = 4j .. 4j + 3
      uint32_t h = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 20 * j + 5 * i + 4;
        h |= ((w[t >> 2] >> (8 * (t & 3))) & 0xffu) << (8 * i);
      }
      xhi[j] = h;
    }
  }
  const int init = -csum;
  const uint32_t gmask = ALIGNED ? 0xffffffffu : __match_any_sync(0xffffffffu, row_ok ? r0_raw : -1 - lane);
  const bool leader = ALIGNED ? lane == 0 : (__ffs(gmask) - 1) == lane;
  uint32_t rs = smem_u32(rsum + r0);
  const uint32_t rstep = 4u * R;
  const uint32_t lut_l = smem_u32(lut) + 4u * lane;  // this lane's table copy

  // 5. the stream, as in gemv1_i2_kernel
  auto consume = [&](const uint4 wv) {
    int v = dot_seg_t5(wv, xlo, xhi, lut_l, init);
    v = __reduce_add_sync(gmask, v);
    if (leader) red_add_s(rs, v);
    rs += rstep;
  };
  int k = 0;
  for (; k < nr - 2 * S + 2; k += S) {
#pragma unroll
    for (int j = 0; j < S; ++j) {
      if (col_ok) cp_async16_s(ring_s + ((j + S - 1) % S) * tstride, gp);
      cp_async_commit();
      gp += step;
      cp_async_wait<S - 1>();
      consume(lds128(ring_s + j * tstride));
    }
  }
  for (; k < nr; ++k) {
    if (col_ok && k + S - 1 < nr) cp_async16_s(ring_s + ((k + S - 1) % S) * tstride, gp);
    cp_async_commit();
    gp += step;
    cp_async_wait<S - 1>();
    consume(lds128(ring_s + (k % S) * tstride));
  }
  cp_async_wait<0>();
  __syncthreads();

  // 6. dequantize and store the CTA's outputs (coalesced)
  const float cf1 = dequant_factor(sh_gam[0], s);
  for (int r = tid; r < nrows; r += T) {
    const int a = rsum[r];
    const int64_t n = row0 + r;
    float cf = cf1;
    if (rg.n > 1) {
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

// ---------------------------------------------------------------------------
// One token on 1-bit rows (the 1-bit variant: bit i of byte j of a packed
// 32-bit word is weight 8 j + i of its 32, set = +1, clear = -1), in the same
// column-stationary layout: a 16-byte segment holds 128 weights and thread t
// keeps the 128 activation codes of its column in registers in the bit-plane
// layout X[w][i] (byte j = the code of weight 32 w + 8 j + i), so a mask of
// bit i of every byte and one dp4a collect the sum of the codes over the +1
// weights of plane i, and the product is 2 S - X with X the sum of the
// token's codes.  The codes
// are written in element order over the raw token (128 per segment, 0 past
// K).
// ---------------------------------------------------------------------------
__host__ __device__ inline int64_t g1b1_xregion(int64_t K, int xwords, int64_t rowbytes) {
  const int64_t raw = K * xwords;      // the raw token
  const int64_t codes = rowbytes * 8;  // 128 codes per 16-byte segment
  return ((raw > codes ? raw : codes) + 15) / 16 * 16;
}

// a0 + 2 S over the 128 weights of a 1-bit segment, S the sum of the codes of
// its +1 weights.  Plane i = 2 m + k is masked in (w >> 2m) at bit k, so two
// accumulators (factors 1 and 2) hold every plane.
__device__ __forceinline__ int dot_seg_b1(const uint4 wv, const uint32_t (&X)[4][8], int a0) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  int a_even = 0, a_odd = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t v = wd[w] >> (2 * m);
      a_even = dp4a_us(v & 0x01010101u, X[w][2 * m], a_even);
      a_odd = dp4a_us(v & 0x02020202u, X[w][2 * m + 1], a_odd);
    }
  return a0 + 2 * (a_even + (a_odd >> 1));
}

template <int XDT, int XC, int S, bool ALIGNED>
__global__ void __launch_bounds__(kG1MaxThreads, 1024 / kG1MaxThreads)
    gemv1_b1_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                    int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                    void* __restrict__ y, int ydt, int write_scale, const RowGroups rg, int R, int lpr, void* ws) {
  constexpr int kXW = g1_xwords<XDT>();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t red[kG1MaxThreads / 32];
  __shared__ float sh_gam[kMaxRowGroups];
  __shared__ int64_t sh_end[kMaxRowGroups];
  __shared__ float sh_s;
  __shared__ __align__(8) uint64_t xbar;  // completion of the token's bulk copy

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = blockDim.x;
  const int segs = static_cast<int>(rowbytes >> 4);
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));
  const int r0_raw = tid / lpr, c_raw = tid - r0_raw * lpr;
  const bool row_ok = r0_raw < R;
  const bool col_ok = row_ok && c_raw < segs;
  const int r0 = row_ok ? r0_raw : 0;
  const int c = col_ok ? c_raw : 0;
  const int nr = (row_ok && r0 < nrows) ? (nrows - r0 + R - 1) / R : 0;
  const uint32_t step = static_cast<uint32_t>(R * rowbytes);
  const int kch = static_cast<int>(K >> 4);  // 16-element chunks of the token (K % 16 == 0)
  const int nch = 8 * segs;                  // 16-code chunks of the codes region (0 past K)
  const uint32_t xbytes = static_cast<uint32_t>(K * kXW);
  // shared memory: the token region (the raw token, then its codes), the row
  // ring [S][T] x 16 bytes, the row sums
  const int64_t xreg = g1b1_xregion(K, kXW, rowbytes);
  uint8_t* xbuf = smem;
  const uint32_t ring_s = smem_u32(xbuf + xreg) + 16u * tid;
  const uint32_t tstride = 16u * T;
  int* rsum = reinterpret_cast<int*>(xbuf + xreg + static_cast<int64_t>(S) * T * 16);

  // 0. before the wait: the first bytes of the CTA's rows into L2, the row
  //    sums zeroed, the token barrier set up
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < BL_G1_PREFETCH ? bytes : BL_G1_PREFETCH);
  }
  for (int i = tid; i < nrows; i += T) rsum[i] = 0;
#pragma unroll
  for (int i = 0; i < kMaxRowGroups; ++i)
    if (tid == i) sh_end[i] = rg.end[i];
  if (tid == 0) {
    mbar_init(&xbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait(packed, gamma, x, scale, y);
  pdl_launch_dependents();

  // 1. the token by one bulk copy (bounded wait: on expiry the CTA records the
  //    timeout, lets the copy land and leaves)
  if (tid == 0) {
    mbar_expect_tx(&xbar, xbytes);
    bulk_load(xbuf, x, xbytes, &xbar);
  }
  if (tid < rg.n) sh_gam[tid] = __ldcg(gamma + tid);
  if (XDT == BL_I8 && tid == 0) sh_s = __ldcg(scale);
  const bool got = wait_drain(&xbar, 0, kG1WaitCycles);
  if (__syncthreads_or(!got)) {
    if (tid == 0) {
      set_flag(ws, kFlagTimeout, 0x603);
      wait_drain(&xbar, 0, kG1WaitCycles);
    }
    return;
  }
  const uint8_t* gp = packed + (row0 + r0) * rowbytes + static_cast<int64_t>(c) * 16;
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (col_ok && j < nr) cp_async16_s(ring_s + j * tstride, gp);
    cp_async_commit();
    gp += step;
  }

  // 2. per-token absmax on the magnitude bits (finite inputs)
  float s;
  if constexpr (XDT != BL_I8) {
    uint32_t mx = 0;
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < kch)
#pragma unroll
        for (int i = 0; i < kXW; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(g) * kXW + i) * 16);
          if constexpr (XDT == BL_F32) {
            const uint32_t a = max(v.x & 0x7fffffffu, v.y & 0x7fffffffu);
            const uint32_t b2 = max(v.z & 0x7fffffffu, v.w & 0x7fffffffu);
            mx = max(mx, max(a, b2));
          } else {
            const uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
            const uint32_t b2 = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
            mx = __vmaxu2(mx, __vmaxu2(a, b2));
          }
        }
    }
    if constexpr (XDT == BL_BF16) mx = max(mx & 0xffffu, mx >> 16) << 16;
    const uint32_t m = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint32_t mm = 0;
    for (int w = 0; w < (T >> 5); ++w) mm = max(mm, red[w]);
    s = fmaxf(__uint_as_float(mm), 1e-6f);
  } else {
    s = sh_s;
  }

  // 3. the codes of the thread's chunks in element order, written over the
  //    raw token once every thread has read its raw chunks
  {
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s);
    uint4 cw[XC];
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      cw[u] = make_uint4(0u, 0u, 0u, 0u);  // padding chunks (past K): code 0
      if (g < kch) {
        const uint8_t* src = xbuf + static_cast<int64_t>(g) * kXW * 16;
        if constexpr (XDT == BL_I8) {
          cw[u] = *reinterpret_cast<const uint4*>(src);
        } else {
          float e[16];
          if constexpr (XDT == BL_F32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              e[4 * i] = __uint_as_float(v.x); e[4 * i + 1] = __uint_as_float(v.y);
              e[4 * i + 2] = __uint_as_float(v.z); e[4 * i + 3] = __uint_as_float(v.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                e[8 * i + 2 * k] = __uint_as_float(wv[k] << 16);
                e[8 * i + 2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
              }
            }
          }
          cw[u] = g1_codes16<false>(e, s, c127);
        }
      }
    }
    __syncthreads();  // every raw chunk has been read
#pragma unroll
    for (int u = 0; u < XC; ++u) {
      const int g = tid + T * u;
      if (g < nch) *reinterpret_cast<uint4*>(xbuf + static_cast<int64_t>(g) * 16) = cw[u];
    }
  }
  __syncthreads();

  // 4. this thread's 128 codes in the bit-plane layout and their sum (the
  //    product is 2 S - X, S the sum over the +1 weights: X is taken off once
  //    per row, as the row sum's starting value)
  uint32_t X[4][8];
  int csum = 0;
  {
    uint32_t lw[32];  // lw[m]: codes 4m .. 4m + 3 of the segment
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 t = col_ok ? *reinterpret_cast<const uint4*>(xbuf + (static_cast<int64_t>(c) * 8 + i) * 16)
                             : make_uint4(0u, 0u, 0u, 0u);
      lw[4 * i] = t.x;
      lw[4 * i + 1] = t.y;
      lw[4 * i + 2] = t.z;
      lw[4 * i + 3] = t.w;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) csum = __dp4a(static_cast<int>(lw[i]), 0x01010101, csum);
    // X[w][i] byte j = code of weight 32 w + 8 j + i = byte (i & 3) of
    // lw[8 w + 2 j + (i >> 2)]
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int o = 8 * w + (i >> 2);
        const uint32_t sel = static_cast<uint32_t>(i & 3) | (static_cast<uint32_t>(4 + (i & 3)) << 4);
        X[w][i] = __byte_perm(__byte_perm(lw[o], lw[o + 2], sel), __byte_perm(lw[o + 4], lw[o + 6], sel), 0x5410);
      }
  }
  const int init = -csum;
  const uint32_t gmask = ALIGNED ? 0xffffffffu : __match_any_sync(0xffffffffu, row_ok ? r0_raw : -1 - lane);
  const bool leader = ALIGNED ? lane == 0 : (__ffs(gmask) - 1) == lane;
  uint32_t rs = smem_u32(rsum + r0);
  const uint32_t rstep = 4u * R;

  // 5. the stream, as in gemv1_i2_kernel
  auto consume = [&](const uint4 wv) {
    int v = dot_seg_b1(wv, X, init);
    v = __reduce_add_sync(gmask, v);
    if (leader) red_add_s(rs, v);
    rs += rstep;
  };
  int k = 0;
  for (; k < nr - 2 * S + 2; k += S) {
#pragma unroll
    for (int j = 0; j < S; ++j) {
      if (col_ok) cp_async16_s(ring_s + ((j + S - 1) % S) * tstride, gp);
      cp_async_commit();
      gp += step;
      cp_async_wait<S - 1>();
      consume(lds128(ring_s + j * tstride));
    }
  }
  for (; k < nr; ++k) {
    if (col_ok && k + S - 1 < nr) cp_async16_s(ring_s + ((k + S - 1) % S) * tstride, gp);
    cp_async_commit();
    gp += step;
    cp_async_wait<S - 1>();
    consume(lds128(ring_s + (k % S) * tstride));
  }
  cp_async_wait<0>();
  __syncthreads();

  // 6. dequantize and store the CTA's outputs (coalesced)
  const float cf1 = dequant_factor(sh_gam[0], s);
  for (int r = tid; r < nrows; r += T) {
    const int a = rsum[r];
    const int64_t n = row0 + r;
    float cf = cf1;
    if (rg.n > 1) {
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
  int R, lpr, threads, xc, stages;
  int64_t grid, rows_per_cta, smem;
};

static bool gemv1_geom(int64_t N, int64_t K, int64_t rowbytes, int xdt, Gemv1Geom* g, int fmt = BL_PACK_I2) {
  const int64_t segs = rowbytes / 16;
  if (K % 16 != 0 || segs < 1 || segs > kG1MaxThreads) return false;
  const int64_t sms = device_sms();
  g->grid = N < sms ? N : sms;
  g->rows_per_cta = (N + g->grid - 1) / g->grid;
  // rows of at least 32 segments take whole warps (the lanes past the row's
  // end idle), so that every warp lies in one row and sums with a full mask
  const int64_t lpr = segs >= 32 ? (segs + 31) / 32 * 32 : segs;
  if (lpr > kG1MaxThreads) return false;
  int64_t R = kG1MaxThreads / lpr;
  if (R > g->rows_per_cta) R = g->rows_per_cta;
  g->R = static_cast<int>(R);
  g->lpr = static_cast<int>(lpr);
  g->threads = static_cast<int>((R * lpr + 31) / 32 * 32);
  // 16-byte chunks of the codes: 4 per 2-bit segment (64 codes), 5 per base-3
  // segment (80 codes), 8 per 1-bit segment (128 codes)
  const int cps = fmt == BL_PACK_T5 ? 5 : (fmt == BL_PACK_B1 ? 8 : 4);
  const int64_t per = (cps * segs + g->threads - 1) / g->threads;
  if (per > 4) return false;
  // 1-bit rows needing more than two chunks per thread (K above 16384) ran
  // slower here than in the lean kernel (70B down-projection: 17.5 against
  // 16.0 us), so they stay there
  if (fmt == BL_PACK_B1 && per > 2) return false;
  g->xc = per <= 1 ? 1 : (per <= 2 ? 2 : 4);
  const int xwords = xdt == BL_F32 ? 4 : (xdt == BL_BF16 ? 2 : 1);
  const int64_t xreg = fmt == BL_PACK_T5   ? kT1LutBytes + g1t5_xregion(K, xwords, rowbytes)
                       : fmt == BL_PACK_B1 ? g1b1_xregion(K, xwords, rowbytes)
                                           : g1_xregion(K, xwords, rowbytes);
  const int64_t fixed = xreg + 4 * g->rows_per_cta;
  for (int st : {kG1StagesMax, 6}) {  // the deepest ring that keeps two CTAs per SM
    // (the 1-bit kernel's 32 code registers leave room for 6 stages only)
    if (fmt == BL_PACK_B1 && st > 6) continue;
    g->stages = st;
    g->smem = fixed + int64_t{16} * st * g->threads;
    if (g->smem <= kG1MaxSmem) return true;
  }
  return false;
}

bool gemv1_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt) {
  Gemv1Geom g;
  return gemv1_geom(N, K, rowbytes, xdt, &g);
}

bool gemv1_t5_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt) {
  Gemv1Geom g;
  return gemv1_geom(N, K, rowbytes, xdt, &g, BL_PACK_T5);
}

bool gemv1_b1_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt) {
  Gemv1Geom g;
  return gemv1_geom(N, K, rowbytes, xdt, &g, BL_PACK_B1);
}

template <int FMT, int XDT, int XC, int S>
static cudaError_t launch_gemv1_t(const Gemv1Geom& g, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, void* ws, cudaStream_t st) {
  const bool al = g.lpr % 32 == 0;
  auto pick = [al]() {
    if constexpr (FMT == BL_PACK_T5)
      return al ? gemv1_t5_kernel<XDT, XC, S, true> : gemv1_t5_kernel<XDT, XC, S, false>;
    else if constexpr (FMT == BL_PACK_B1)
      return al ? gemv1_b1_kernel<XDT, XC, S, true> : gemv1_b1_kernel<XDT, XC, S, false>;
    else
      return al ? gemv1_i2_kernel<XDT, XC, S, true> : gemv1_i2_kernel<XDT, XC, S, false>;
  };
  auto kern = pick();
  const size_t smem = static_cast<size_t>(g.smem);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_pdl(kern, static_cast<unsigned>(g.grid), static_cast<unsigned>(g.threads), smem, st,
                                   packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, g.R, g.lpr, ws);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT, int XDT, int XC>
static cudaError_t launch_gemv1_s(const Gemv1Geom& g, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, void* ws, cudaStream_t st) {
  if constexpr (FMT != BL_PACK_B1) {  // the 1-bit kernel runs with 6 stages only
    if (g.stages == kG1StagesMax)
      return launch_gemv1_t<FMT, XDT, XC, kG1StagesMax>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt,
                                                       write_scale, rg, ws, st);
  }
  return launch_gemv1_t<FMT, XDT, XC, 6>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, ws, st);
}

template <int FMT, int XDT>
static cudaError_t launch_gemv1_x(const Gemv1Geom& g, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, void* ws, cudaStream_t st) {
  if (g.xc == 1)
    return launch_gemv1_s<FMT, XDT, 1>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, ws, st);
  if (g.xc == 2)
    return launch_gemv1_s<FMT, XDT, 2>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, ws, st);
  return launch_gemv1_s<FMT, XDT, 4>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, ws, st);
}

template <int FMT>
static cudaError_t launch_gemv1_f(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                                  const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg,
                                  void* ws, cudaStream_t st) {
  Gemv1Geom g;
  if (!gemv1_geom(N, K, rowbytes, xdt, &g, FMT)) return cudaErrorInvalidValue;
  if (xdt == BL_F32)
    return launch_gemv1_x<FMT, BL_F32>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 1, rg, ws, st);
  if (xdt == BL_BF16)
    return launch_gemv1_x<FMT, BL_BF16>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 1, rg, ws, st);
  return launch_gemv1_x<FMT, BL_I8>(g, packed, rowbytes, gamma, N, K, x, scale, y, ydt, 0, rg, ws, st);
}

cudaError_t launch_gemv1(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                         const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                         cudaStream_t st) {
  return launch_gemv1_f<BL_PACK_I2>(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
}

cudaError_t launch_gemv1_t5(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                            const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                            cudaStream_t st) {
  return launch_gemv1_f<BL_PACK_T5>(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
}

cudaError_t launch_gemv1_b1(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                            const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                            cudaStream_t st) {
  return launch_gemv1_f<BL_PACK_B1>(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
}

}  // namespace bl
