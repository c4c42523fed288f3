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
// order of its own (+dy for weight +1, -dy for -1, nothing for 0; per tile a
// warp's rows in order, the tile's warps in order, the row blocks in order),
// which stays within one fp32 ulp plus gamma N 2^-52 sum |dy| of the
// definition.
// dW: c_m = s_m / 127, terms (dy[m, n] x_q[m, k]) c_m added in fp64 from 0.0
// in token order (the plain order of the sum), then gamma * T, rounded once
// to fp32.
// dx reads the packed 2-bit weights once per pass of up to two tokens in 2-D
// tiles (512 columns x at least 64 rows: about two CTAs per SM, partial sums
// a few percent of the weight bytes); dW writes N K fp32 values (the
// HBM-bound part for few tokens).
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kDxMinRows = 64;  // rows per row block, at least (the workspace holds ceil(N / 64) blocks)
constexpr int kDxTokens = 2;    // tokens per pass: 16 columns x 2 tokens of fp64 sums per lane
constexpr int kDxWarps = 8;     // warps of a CTA: each takes every 8th row of the row block
constexpr int kDxAhead = 4;     // rows whose words and gradients are loaded ahead of the adds

template <int DYT>
__device__ __forceinline__ double load_grad(const void* p, int64_t i) {
  return static_cast<double>(load_elem<DYT>(p, i));
}

// Partial sums over one tile: CTA (cb, rb) takes the 32 packed words
// 32 cb .. 32 cb + 31 of each row (columns 512 cb .. 512 cb + 511; lane L one
// word, so a warp reads a 128-byte piece of a row) of the rows of row block
// rb; warp w takes every kDxWarps-th row.  A lane adds +dy, -dy or nothing
// (the stored digit 2, 0 or 1) into 16 fp64 sums per token; the warps' sums
// meet in shared memory in a fixed order and go to part[rb][m][k] (fp64).
template <int DYT, int MT>
__global__ void __launch_bounds__(kDxWarps * 32)
    backward_dx_tile_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, int64_t N, int64_t K,
                            const void* __restrict__ dy, int64_t m0, int64_t rows_per_block,
                            double* __restrict__ part) {
  pdl_enter(packed, dy, part);
  extern __shared__ __align__(16) double sh[];  // [kDxWarps][MT * 16][33]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t words = (K + 15) / 16;                // packed 32-bit words holding weights below K
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + lane;  // this lane's word
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t n1 = n0 + rows_per_block < N ? n0 + rows_per_block : N;
  const int64_t stride = rowbytes / 4;
  double acc[MT][16];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[m][i] = 0.0;
  if (c < words) {
    const uint32_t* col = reinterpret_cast<const uint32_t*>(packed) + c;
    for (int64_t nb = n0 + warp; nb < n1; nb += kDxWarps * kDxAhead) {
      uint32_t wv[kDxAhead];
      double gv[kDxAhead][MT];
#pragma unroll
      for (int j = 0; j < kDxAhead; ++j) {
        const int64_t n = nb + static_cast<int64_t>(kDxWarps) * j;
        wv[j] = n < n1 ? __ldcg(col + n * stride) : 0x55555555u;  // past the block: weight 0
#pragma unroll
        for (int m = 0; m < MT; ++m) gv[j][m] = n < n1 ? load_grad<DYT>(dy, (m0 + m) * N + n) : 0.0;
      }
#pragma unroll
      for (int j = 0; j < kDxAhead; ++j) {
        // bit 2i of pos / neg: weight i of the word is +1 / -1 (digit 2 / 0)
        const uint32_t w = wv[j];
        const uint32_t pos = (w >> 1) & ~w & 0x55555555u;
        const uint32_t neg = ~(w | (w >> 1)) & 0x55555555u;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            // two independent one-instruction conditionals (predicated adds,
            // no divergent branch)
            if (pos & (1u << (2 * i))) acc[m][i] = __dadd_rn(acc[m][i], gv[j][m]);
            if (neg & (1u << (2 * i))) acc[m][i] = __dadd_rn(acc[m][i], -gv[j][m]);
          }
        }
      }
    }
  }
  // the warps' sums, transposed through shared memory (a padded row of 33 per
  // column keeps both the writes and the reads free of bank conflicts)
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

template <int DYT>
__global__ void __launch_bounds__(256)
    backward_dw_kernel(const void* __restrict__ dy, const int8_t* __restrict__ xq, const float* __restrict__ scale,
                       const float* __restrict__ gamma, int64_t M, int64_t N, int64_t K, float* __restrict__ dw) {
  pdl_enter(dy, xq, scale, gamma, dw);
  __shared__ double sh_c[kDwTokBlock];
  __shared__ double sh_g;
  if (threadIdx.x == 0) sh_g = static_cast<double>(__ldcg(gamma));
  const int64_t kq = (K + 3) / 4;
  const int64_t total = N * kq;
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
    for (int i = 0; i < 4; ++i) T[i] = __dadd_rn(T[i], __dmul_rn(__dmul_rn(g, static_cast<double>(q[i])), c));
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
  if (M <= kDwTokBlock) {  // every token's factor in shared memory once; no barrier in the loop
    if (threadIdx.x < M) sh_c[threadIdx.x] = __ddiv_rn(static_cast<double>(__ldcg(scale + threadIdx.x)), 127.0);
    __syncthreads();
    const double g = sh_g;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t n = e / kq, k0 = 4 * (e - n * kq);
      double T[4] = {0.0, 0.0, 0.0, 0.0};
      for (int64_t m = 0; m < M; ++m) term4(m, n, k0, sh_c[m], T);
      store4(n, k0, T, g);
    }
    return;
  }
  for (int64_t base = blockIdx.x * static_cast<int64_t>(blockDim.x); base < total;
       base += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = base + threadIdx.x;
    const bool active = e < total;
    const int64_t n = active ? e / kq : 0;
    const int64_t k0 = active ? 4 * (e - n * kq) : 0;
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
  const size_t smem = static_cast<size_t>(kDxWarps) * MT * 16 * 33 * sizeof(double);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, grid, kDxWarps * 32, smem, st, packed, rowbytes, N, K, dy, m0, rows, part);
}

cudaError_t launch_backward_dx(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                               const void* dy, int dydt, int64_t M, float* dx, double* part, cudaStream_t st) {
  // tiles: 512-column blocks x row blocks of at least kDxMinRows rows, about
  // two CTAs per SM (the row blocks never outnumber backward_dx_chunks(N),
  // which the workspace holds)
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
  const unsigned g = grid_of(N * ((K + 3) / 4), 8);
  cudaError_t e = dydt == BL_F32
                      ? launch_pdl(backward_dw_kernel<BL_F32>, g, 256, 0, st, dy, xq, scale, gamma, M, N, K, dw)
                      : launch_pdl(backward_dw_kernel<BL_BF16>, g, 256, 0, st, dy, xq, scale, gamma, M, N, K, dw);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bl
