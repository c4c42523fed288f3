// bl_backward.cu -- STE backward of the BitLinear layer.
//
// "BitNet b1.58深度解析：三值权重如何重塑大模型推理" §5.3: the layer computes
// F.linear(x_deq, W_eff) * gamma with W_eff = W_ternary + W - W.detach(), the
// straight-through estimator taking each quantizer as the identity in the
// backward pass ("QAT and BitNet: A Deep Dive into 1-bit and 1.58-bit
// Quantization-Aware Training", "How Gradients Flow: Fake Quantization and
// STE").  With gamma a constant of the step and an upstream gradient dy [M, N]:
//   dx[m, k] = gamma * sum_n dy[m, n] W_q[n, k]
//   dW[n, k] = gamma * sum_m dy[m, n] x_q[m, k] s_m / 127
// dx is defined by the exact sum over the rows rounded once to fp64 (no
// order), then gamma * S in fp64 and fp32; this kernel adds in fp64 in an
// order of its own (the two rows of a row pair first, one rounding of
// w_a dy_a + w_b dy_b; then a warp's pairs in order, the tile's warps in
// order, the row blocks in order), so every term passes through far fewer
// than N roundings and the result stays within one fp32 ulp plus
// gamma N 2^-52 sum |W_q dy| of the definition.
// dW: c_m = s_m / 127, terms (dy[m, n] x_q[m, k]) c_m added in fp64 from 0.0
// in token order (the plain order of the sum), then gamma * T, rounded once
// to fp32.
// dx reads the packed 2-bit weights once per pass of up to two tokens in 2-D
// tiles (512 columns x at least 64 rows: about two CTAs per SM, partial sums
// a few percent of the weight bytes); dW writes N K fp32 values (the
// HBM-bound part for few tokens).
#include "bl_common.cuh"
#include "bl_kernels.h"
#include "bl_sm100.cuh"

namespace bl {

constexpr int kDxMinRows = 64;     // rows per row block, at least (the workspace holds ceil(N / 64) blocks)
constexpr int kDxTokens = 2;       // tokens per pass: 16 columns x 2 tokens of fp64 sums per lane
constexpr int kDxWarps = 8;        // warps of a CTA
constexpr int kDxChunkPairs = 64;  // row pairs of one chunk of a row block: 8 per warp
constexpr int kDxTable = 256;      // bytes per row pair: a 16-entry fp64 table per token, at +128 t
constexpr int kDxTablesBytes = 2 * kDxChunkPairs * kDxTable;  // two chunks' tables (double buffer)

template <int DYT>
__device__ __forceinline__ double load_grad(const void* p, int64_t i) {
  return static_cast<double>(load_elem<DYT>(p, i));
}

// The weight of a stored 2-bit digit times g: digit 2 -> +g, 0 -> -g, 1 -> 0
// (3, which no packer writes, also 0).
__device__ __forceinline__ double digit_times(uint32_t d, double g) {
  return d == 2u ? g : (d == 0u ? -g : 0.0);
}

template <int OFF>
__device__ __forceinline__ double lds_f64(uint32_t addr) {
  double v;
  asm volatile("ld.shared.f64 %0, [%1+%2];" : "=d"(v) : "r"(addr), "n"(OFF) : "memory");
  return v;
}

// Partial sums over one tile: CTA (cb, rb) takes the 32 packed words
// 32 cb .. 32 cb + 31 of each row (columns 512 cb .. 512 cb + 511; lane L one
// word, so a warp reads a 128-byte piece of a row) of the rows of row block
// rb, two rows at a time.  For the row pair (a, a + 1) and token m a table of
// 16 fp64 entries holds T[da + 4 db] = w(da) dy[m, a] + w(db) dy[m, a + 1]
// (w the weight of a digit; one rounding), so a lane adds one table entry
// per column and token for two weights: the 4-bit index of each of its 16
// columns comes from the two words by a few mask-and-shift steps, and one
// byte permute puts 8 x the index into the low byte of the table's
// (256-byte aligned) shared address.  A 128-byte table spans the 32 banks
// once, so the lookups of a warp are free of bank conflicts.
// The row block is walked in chunks of 64 row pairs, warp w taking the pairs
// w, w + 8, ... of a chunk; the next chunk's words and gradients are loaded
// while the current chunk is added, and its tables are built into the other
// half of a double buffer.  The warps' sums meet in shared memory in a fixed
// order and go to part[rb][m][k] (fp64).
template <int DYT, int MT>
__global__ void __launch_bounds__(kDxWarps * 32, 2)
    backward_dx_tile_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, int64_t N, int64_t K,
                            const void* __restrict__ dy, int64_t m0, int64_t rows_per_block,
                            double* __restrict__ part) {
  pdl_enter(packed, dy, part);
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float stage[2][MT][2 * kDxChunkPairs];  // a chunk's gradients (0 past the block)
  const uint32_t raw = smem_u32(dsm);
  const uint32_t pad = (256u - (raw & 255u)) & 255u;
  const uint32_t tab_s = raw + pad;  // low byte zero
  double* tab = reinterpret_cast<double*>(dsm + pad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t words = (K + 15) / 16;                // packed 32-bit words holding weights below K
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + lane;  // this lane's word
  const bool live = c < words;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t n1 = n0 + rows_per_block < N ? n0 + rows_per_block : N;
  const int64_t pairs = (n1 - n0 + 1) / 2;
  const int chunks = static_cast<int>((pairs + kDxChunkPairs - 1) / kDxChunkPairs);
  const int64_t stride = rowbytes / 4;
  const uint32_t* col = reinterpret_cast<const uint32_t*>(packed) + c;

  // this warp's words of chunk ch (weight-0 words past the block or K)
  auto load_words = [&](int ch, uint32_t (&wa)[8], uint32_t (&wb)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t a = n0 + 2 * (static_cast<int64_t>(ch) * kDxChunkPairs + warp + 8 * j);
      wa[j] = (live && a < n1) ? __ldcg(col + a * stride) : 0x55555555u;
      wb[j] = (live && a + 1 < n1) ? __ldcg(col + (a + 1) * stride) : 0x55555555u;
    }
  };
  // one gradient of chunk ch per thread (at most 128 MT of them)
  auto load_dy = [&](int ch) -> float {
    const int i = threadIdx.x;
    if (i >= MT * 2 * kDxChunkPairs) return 0.0f;
    const int t = i / (2 * kDxChunkPairs), r = i % (2 * kDxChunkPairs);
    const int64_t n = n0 + static_cast<int64_t>(ch) * 2 * kDxChunkPairs + r;
    return n < n1 ? load_elem<DYT>(dy, (m0 + t) * N + n) : 0.0f;
  };
  auto put_dy = [&](int buf, float v) {
    const int i = threadIdx.x;
    if (i < MT * 2 * kDxChunkPairs) stage[buf][i / (2 * kDxChunkPairs)][i % (2 * kDxChunkPairs)] = v;
  };
  // the tables of a chunk from its staged gradients (16 threads per table:
  // each warp's stores cover two whole tables)
  auto build = [&](int buf) {
    double* tb = tab + buf * (kDxChunkPairs * kDxTable / 8);
    for (int e = threadIdx.x; e < kDxChunkPairs * MT * 16; e += kDxWarps * 32) {
      const int idx = e & 15, pt = e >> 4, p = pt / MT, t = pt % MT;
      const double g0 = static_cast<double>(stage[buf][t][2 * p]);
      const double g1 = static_cast<double>(stage[buf][t][2 * p + 1]);
      tb[p * (kDxTable / 8) + t * 16 + idx] = __dadd_rn(digit_times(idx & 3u, g0), digit_times(idx >> 2, g1));
    }
  };

  double acc[MT][16];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[m][i] = 0.0;

  uint32_t wa[8], wb[8];
  load_words(0, wa, wb);
  put_dy(0, load_dy(0));
  __syncthreads();
  build(0);
  __syncthreads();
  for (int ch = 0; ch < chunks; ++ch) {
    const int buf = ch & 1;
    const bool more = ch + 1 < chunks;
    uint32_t na[8], nb[8];
    float ndy = 0.0f;
    if (more) {  // in flight while this chunk is added
      load_words(ch + 1, na, nb);
      ndy = load_dy(ch + 1);
    }
    const int np = static_cast<int>(pairs - static_cast<int64_t>(ch) * kDxChunkPairs < kDxChunkPairs
                                        ? pairs - static_cast<int64_t>(ch) * kDxChunkPairs
                                        : kDxChunkPairs);
    const uint32_t tbase = tab_s + static_cast<uint32_t>(buf * kDxChunkPairs * kDxTable);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int p = warp + 8 * j;
      if (p < np) {  // uniform over the warp
        const uint32_t base = tbase + static_cast<uint32_t>(p * kDxTable);
        // nibble i of A / B: the index (row a digit | row a + 1 digit << 2) of
        // column 2 i / 2 i + 1
        const uint32_t A = (wa[j] & 0x33333333u) | ((wb[j] << 2) & 0xccccccccu);
        const uint32_t B = ((wa[j] >> 2) & 0x33333333u) | (wb[j] & 0xccccccccu);
        // byte b of e[r]: 8 x the index of column 4 b + r
        const uint32_t e[4] = {(A << 3) & 0x78787878u, (B << 3) & 0x78787878u, (A >> 1) & 0x78787878u,
                               (B >> 1) & 0x78787878u};
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t addr = __byte_perm(e[r], base, 0x7650u | static_cast<uint32_t>(b));
            acc[0][4 * b + r] = __dadd_rn(acc[0][4 * b + r], lds_f64<0>(addr));
            if (MT > 1) acc[MT - 1][4 * b + r] = __dadd_rn(acc[MT - 1][4 * b + r], lds_f64<128>(addr));
          }
      }
    }
    if (more) {
      put_dy(buf ^ 1, ndy);
      __syncthreads();  // the staged gradients are visible
      build(buf ^ 1);   // the other buffer: its last chunk was added before the previous barrier
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        wa[j] = na[j];
        wb[j] = nb[j];
      }
    }
    __syncthreads();  // the next chunk's tables are complete (and this chunk's are read)
  }
  // the warps' sums, transposed through shared memory over the tables (a
  // padded row of 33 per column keeps both the writes and the reads free of
  // bank conflicts)
  double* sh = tab;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 16; ++i) sh[(warp * MT * 16 + m * 16 + i) * 33 + lane] = acc[m][i];
  __syncthreads();
  // output o = (m, lane L, i): column 16 (32 cb + L) + i, the warps added in order
  for (int o = threadIdx.x; o < MT * 32 * 16; o += kDxWarps * 32) {
    const int m = o / 512, L = (o / 16) & 31, i = o & 15;
    const int64_t k = 16 * (static_cast<int64_t>(blockIdx.x) * 32 + L) + i;
    double v = 0.0;
#pragma unroll
    for (int w = 0; w < kDxWarps; ++w) v = __dadd_rn(v, sh[(w * MT * 16 + m * 16 + i) * 33 + L]);
    if (k < K) part[(static_cast<int64_t>(blockIdx.y) * MT + m) * K + k] = v;
  }
}

// dx[m0 + m, k] = fp32(gamma * sum_r part[r][m][k]).  A CTA takes 32
// columns (lane L column 32 blockIdx.x + L, so each read of a partial row is
// coalesced) of token m = blockIdx.y; warp w adds the row blocks
// [w C / 8, (w + 1) C / 8) in order, and the 8 warp sums meet in warp order
// through shared memory (a fixed order: the result is the same on every run).
template <int MT>
__global__ void __launch_bounds__(256)
    backward_dx_reduce_kernel(const double* __restrict__ part, int64_t chunks, int64_t K, const float* __restrict__ gamma,
                              int64_t m0, float* __restrict__ dx) {
  pdl_enter(part, gamma, dx);
  __shared__ double sh[8][32];
  __shared__ double sh_g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) sh_g = static_cast<double>(__ldcg(gamma));
  const int m = blockIdx.y;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  const int64_t r0 = chunks * warp / 8, r1 = chunks * (warp + 1) / 8;
  double S = 0.0;
  if (k < K) {
    const double* p = part + m * K + k;
#pragma unroll 4
    for (int64_t r = r0; r < r1; ++r) S = __dadd_rn(S, __ldcg(p + r * MT * K));
  }
  sh[warp][lane] = S;
  __syncthreads();
  if (warp == 0 && k < K) {
    double t = sh[0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) t = __dadd_rn(t, sh[w][lane]);
    dx[(m0 + m) * K + k] = __double2float_rn(__dmul_rn(sh_g, t));
  }
}

// dW: thread owns four consecutive outputs (n, k0 .. k0 + 3) and adds the M
// tokens in order; c_m = s_m / 127 is computed once per CTA per token block in
// shared memory.  The grid-stride loop runs the same number of iterations in
// every thread of a CTA (the barriers of the token blocks are uniform).
constexpr int kDwTokBlock = 256;

// An int32 of magnitude below 2^31 as fp64 without the conversion unit: the
// double with high word 0x43380000 and low word i + 2^31 is exactly
// 1.5 2^52 + 2^31 + i (the low word counts units of the last place, 1 at
// 2^52), so one exact fp64 subtraction leaves i.
__device__ __forceinline__ double i32_to_f64(int i) {
  return __dsub_rn(__hiloint2double(0x43380000, static_cast<int>(static_cast<uint32_t>(i) ^ 0x80000000u)),
                   6755401588539392.0);
}

template <int DYT>
__global__ void __launch_bounds__(256)
    backward_dw_kernel(const void* __restrict__ dy, const int8_t* __restrict__ xq, const float* __restrict__ scale,
                       const float* __restrict__ gamma, int64_t M, int64_t N, int64_t K, float* __restrict__ dw) {
  pdl_enter(dy, xq, scale, gamma, dw);
  __shared__ double sh_c[kDwTokBlock];
  __shared__ double sh_g;
  if (threadIdx.x == 0) sh_g = static_cast<double>(__ldcg(gamma));
  // N K < 2^32, so the (row, quad) items fit 32-bit index arithmetic
  const uint32_t kq = static_cast<uint32_t>((K + 3) / 4);
  const uint32_t total = static_cast<uint32_t>(N) * kq;
  const bool vec = (K % 4) == 0;
  auto term4 = [&](int64_t m, int64_t n, int64_t k0, double c, double (&T)[4]) {
    const double g = load_grad<DYT>(dy, m * N + n);
    int q[4];
    if (vec) {
      const uint32_t w = __ldcg(reinterpret_cast<const uint32_t*>(xq + m * K + k0));
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = static_cast<int8_t>(w >> (8 * i));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = (k0 + i < K) ? static_cast<int>(__ldcg(xq + m * K + k0 + i)) : 0;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) T[i] = __dadd_rn(T[i], __dmul_rn(__dmul_rn(g, i32_to_f64(q[i])), c));
  };
  auto store4 = [&](int64_t n, int64_t k0, const double (&T)[4], double g) {
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __double2float_rn(__dmul_rn(g, T[i]));
    float* dst = dw + n * K + k0;
    if (vec) {
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (k0 + i < K) dst[i] = o[i];
    }
  };
  // item e = (row nn, quad qq) with e = nn kq + qq; the grid stride S moves it
  // by (S / kq, S mod kq) with one carry, so the loop divides only once
  const uint32_t S = gridDim.x * blockDim.x;
  const uint32_t Sn = S / kq, Sr = S - Sn * kq;
  const uint32_t e0 = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t nn = e0 / kq, qq = e0 - (e0 / kq) * kq;
  auto advance = [&]() {
    nn += Sn;
    qq += Sr;
    if (qq >= kq) {
      qq -= kq;
      ++nn;
    }
  };
  if (M <= kDwTokBlock) {  // every token's factor in shared memory once; no barrier in the loop
    if (threadIdx.x < M) sh_c[threadIdx.x] = __ddiv_rn(static_cast<double>(__ldcg(scale + threadIdx.x)), 127.0);
    __syncthreads();
    const double g = sh_g;
    for (uint32_t e = e0; e < total; e += S, advance()) {
      const int64_t n = nn, k0 = 4 * static_cast<int64_t>(qq);
      double T[4] = {0.0, 0.0, 0.0, 0.0};
      for (int64_t m = 0; m < M; ++m) term4(m, n, k0, sh_c[m], T);
      store4(n, k0, T, g);
    }
    return;
  }
  for (uint32_t base = blockIdx.x * blockDim.x; base < total; base += S, advance()) {
    const uint32_t e = base + threadIdx.x;
    const bool active = e < total;
    const int64_t n = active ? static_cast<int64_t>(nn) : 0;
    const int64_t k0 = active ? 4 * static_cast<int64_t>(qq) : 0;
    double T[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t t0 = 0; t0 < M; t0 += kDwTokBlock) {
      const int64_t tn = (M - t0) < kDwTokBlock ? (M - t0) : kDwTokBlock;
      __syncthreads();  // the previous block's factors have been read
      if (threadIdx.x < tn) sh_c[threadIdx.x] = __ddiv_rn(static_cast<double>(__ldcg(scale + t0 + threadIdx.x)), 127.0);
      __syncthreads();
      if (active)
        for (int64_t j = 0; j < tn; ++j) term4(t0 + j, n, k0, sh_c[j], T);
    }
    if (active) store4(n, k0, T, sh_g);
  }
}

// dW for one token: dW[n, k] depends on row n only through dy[n] and on
// column k only through the code x_q[k], so each row has at most 256
// distinct outputs.  A CTA takes rows n = b, b + G, ...: per row its threads
// first fill a 256-entry table of the outputs for every code (the same fp64
// operations as backward_dw_kernel: T = 0.0 + (dy x_q) c, then gamma T to
// fp32), then write the row by lookups (four codes per 32-bit load, one
// 16-byte store).  Four copies of the table (lane mod 4 picks one) spread a
// warp's lookups over the banks.
constexpr int kDw1Copies = 4;

template <int DYT>
__global__ void __launch_bounds__(256)
    backward_dw1_kernel(const void* __restrict__ dy, const int8_t* __restrict__ xq, const float* __restrict__ scale,
                        const float* __restrict__ gamma, int64_t N, int64_t K, float* __restrict__ dw) {
  pdl_enter(dy, xq, scale, gamma, dw);
  __shared__ float tab[256][kDw1Copies];  // [code + 128][copy]
  const double c = __ddiv_rn(static_cast<double>(__ldcg(scale)), 127.0);
  const double g = static_cast<double>(__ldcg(gamma));
  const int t = threadIdx.x;
  const int copy = t & (kDw1Copies - 1);
  const bool vec = (K % 4) == 0;
  const uint32_t kq = static_cast<uint32_t>((K + 3) / 4);
  const double q_t = i32_to_f64(t - 128);  // this thread's code
  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const double a = load_grad<DYT>(dy, n);
    const float o = __double2float_rn(__dmul_rn(g, __dadd_rn(0.0, __dmul_rn(__dmul_rn(a, q_t), c))));
    __syncthreads();  // the previous row's lookups are done
#pragma unroll
    for (int j = 0; j < kDw1Copies; ++j) tab[t][j] = o;
    __syncthreads();
    float* row = dw + n * K;
    for (uint32_t qd = t; qd < kq; qd += blockDim.x) {
      const int64_t k0 = 4 * static_cast<int64_t>(qd);
      if (vec) {
        const uint32_t w = __ldcg(reinterpret_cast<const uint32_t*>(xq + k0));
        float4 v;
        v.x = tab[(w & 0xffu) ^ 0x80u][copy];
        v.y = tab[((w >> 8) & 0xffu) ^ 0x80u][copy];
        v.z = tab[((w >> 16) & 0xffu) ^ 0x80u][copy];
        v.w = tab[(w >> 24) ^ 0x80u][copy];
        *reinterpret_cast<float4*>(row + k0) = v;
      } else {
        for (int i = 0; i < 4 && k0 + i < K; ++i)
          row[k0 + i] = tab[(static_cast<uint32_t>(static_cast<uint8_t>(xq[k0 + i]))) ^ 0x80u][copy];
      }
    }
  }
}

// ---- host side --------------------------------------------------------------------
int64_t backward_dx_chunks(int64_t N) { return (N + kDxMinRows - 1) / kDxMinRows; }
int backward_dx_tokens_per_pass() { return kDxTokens; }

static unsigned grid_of(int64_t work, int per_sm) {
  const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
  int64_t g = (work + 255) / 256;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<unsigned>(g);
}

template <int DYT, int MT>
static cudaError_t launch_dx_tile(dim3 grid, const uint8_t* packed, int64_t rowbytes, int64_t N, int64_t K,
                                  const void* dy, int64_t m0, int64_t rows, double* part, cudaStream_t st) {
  auto kern = backward_dx_tile_kernel<DYT, MT>;
  const size_t comb = static_cast<size_t>(kDxWarps) * MT * 16 * 33 * sizeof(double);
  const size_t smem = 256 + (comb > static_cast<size_t>(kDxTablesBytes) ? comb : kDxTablesBytes);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, grid, kDxWarps * 32, smem, st, packed, rowbytes, N, K, dy, m0, rows, part);
}

cudaError_t launch_backward_dx(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                               const void* dy, int dydt, int64_t M, float* dx, double* part, cudaStream_t st) {
  // tiles: 512-column blocks x row blocks of at least kDxMinRows rows, about
  // two CTAs per SM (more and smaller row blocks measured slower: each
  // builds its own tables and writes its own partial sums; the row blocks
  // never outnumber backward_dx_chunks(N), which the workspace holds)
  const int64_t words = (K + 15) / 16;
  const int64_t cbs = (words + 31) / 32;
  int64_t rbs = (2 * static_cast<int64_t>(device_sms()) + cbs - 1) / cbs;
  int64_t rows = (N + rbs - 1) / rbs;
  rows = rows < kDxMinRows ? kDxMinRows : (rows + 7) / 8 * 8;
  rbs = (N + rows - 1) / rows;
  const dim3 grid(static_cast<unsigned>(cbs), static_cast<unsigned>(rbs));
  for (int64_t m0 = 0; m0 < M; m0 += kDxTokens) {
    const int mt = (M - m0) < kDxTokens ? static_cast<int>(M - m0) : kDxTokens;
    const dim3 gr(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>(mt));
    cudaError_t e;
    if (dydt == BL_F32)
      e = mt == 2 ? launch_dx_tile<BL_F32, 2>(grid, packed, rowbytes, N, K, dy, m0, rows, part, st)
                  : launch_dx_tile<BL_F32, 1>(grid, packed, rowbytes, N, K, dy, m0, rows, part, st);
    else
      e = mt == 2 ? launch_dx_tile<BL_BF16, 2>(grid, packed, rowbytes, N, K, dy, m0, rows, part, st)
                  : launch_dx_tile<BL_BF16, 1>(grid, packed, rowbytes, N, K, dy, m0, rows, part, st);
    if (e != cudaSuccess) return e;
    e = mt == 2 ? launch_pdl(backward_dx_reduce_kernel<2>, gr, 256, 0, st, part, rbs, K, gamma, m0, dx)
                : launch_pdl(backward_dx_reduce_kernel<1>, gr, 256, 0, st, part, rbs, K, gamma, m0, dx);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_backward_dw(const void* dy, int dydt, const int8_t* xq, const float* scale, const float* gamma,
                               int64_t M, int64_t N, int64_t K, float* dw, cudaStream_t st) {
  if (M == 1) {  // one token: a 256-entry table of outputs per row
    const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
    const unsigned g1 = static_cast<unsigned>(N < cap ? N : cap);
    const cudaError_t e = dydt == BL_F32
                              ? launch_pdl(backward_dw1_kernel<BL_F32>, g1, 256, 0, st, dy, xq, scale, gamma, N, K, dw)
                              : launch_pdl(backward_dw1_kernel<BL_BF16>, g1, 256, 0, st, dy, xq, scale, gamma, N, K, dw);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const unsigned g = grid_of(N * ((K + 3) / 4), 8);
  cudaError_t e = dydt == BL_F32
                      ? launch_pdl(backward_dw_kernel<BL_F32>, g, 256, 0, st, dy, xq, scale, gamma, M, N, K, dw)
                      : launch_pdl(backward_dw_kernel<BL_BF16>, g, 256, 0, st, dy, xq, scale, gamma, M, N, K, dw);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bl
