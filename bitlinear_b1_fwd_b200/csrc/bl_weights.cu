// bl_weights.cu -- weight preparation: absmean scale, ternarization, packing.
//
// Steps 1-3 of the BitNet b1.58 BitLinear ("BitNet b1.58深度解析：三值权重如何
// 重塑大模型推理" §3.1 absmean; "QAT and BitNet: A Deep Dive into 1-bit and
// 1.58-bit Quantization-Aware Training", "The Ternary Weight Recipe" and "Why Is
// It Called 1.58 Bits?").  All three kernels are HBM-bound streams over W.
#include <atomic>

#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {

// ---------------------------------------------------------------------------
// absmean.  The fixed order: in chunk c (elements [8192c, 8192c + 8192)),
// "lane" l = 0..255 adds, in fp64 and in this order, the elements
// 8192c + 2048i + 8l + j for i = 0..3, j = 0..7; the 256 lane sums meet in the
// stride-halving tree p[l] += p[l + s], s = 128..1.
//
// The kernel below gives lane l of a chunk to thread l of a 256-thread CTA;
// for fixed i the CTA reads 2048 consecutive elements, each thread 32
// contiguous bytes.
//
// When all warps of a CTA are done, the CTA takes a ticket; the CTA with the
// last ticket combines the C chunk sums, zero-padded to P = 2^ceil(log2 C), by
// the stride-halving tree s = P/2..1, and writes gamma = fp32(S / T):
//   - the levels s >= 256 act on each residue class mod 256 on its own, as a
//     stride-halving tree over k of q[t + 256k]; that tree equals the pairwise
//     (contiguous) tree over the bit-reversed sequence, which thread t folds
//     with a binary-counter stack (fp64 addition is commutative, so operand
//     order inside a pair does not matter);
//   - the last 8 levels run in shared memory and warp shuffles.
// ---------------------------------------------------------------------------

// The last CTA's combination of the C chunk sums into gamma (see above), by
// the threads of the calling CTA whatever their number; p is a shared array of
// kLanes doubles.  Resets the ticket for the next call on the workspace.
__device__ __forceinline__ void absmean_finish(const double* __restrict__ partials, int64_t C, int lgR, int64_t T,
                                               double* p, WsHeader* __restrict__ hdr, float* __restrict__ gamma) {
  const int64_t R = int64_t{1} << lgR;  // P / 256, or 1 when P <= 256
  for (int l = threadIdx.x; l < kLanes; l += blockDim.x) {
    double st[kFinishMaxLevels + 1];
    for (int64_t i0 = 0; i0 < R; i0 += 8) {
      double vals[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u;
        const int64_t k =
            (lgR == 0) ? 0 : static_cast<int64_t>(__brevll(static_cast<unsigned long long>(i)) >> (64 - lgR));
        const int64_t idx = l + static_cast<int64_t>(kLanes) * k;
        vals[u] = (i < R && idx < C) ? __ldcg(partials + idx) : 0.0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u;
        if (i >= R) break;
        double val = vals[u];
        int64_t jj = i;
        int lvl = 0;
        while (jj & 1) {
          val = __dadd_rn(st[lvl], val);
          jj >>= 1;
          ++lvl;
        }
        st[lvl] = val;
      }
    }
    p[l] = st[lgR];
  }
  __syncthreads();
#pragma unroll
  for (int s = kLanes / 2; s >= 32; s >>= 1) {
    for (int l = threadIdx.x; l < s; l += blockDim.x) p[l] = __dadd_rn(p[l], p[l + s]);
    __syncthreads();
  }
  if (threadIdx.x < 32) {
    double t = p[threadIdx.x];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, s));
    if (threadIdx.x == 0) {
      gamma[0] = __double2float_rn(__ddiv_rn(t, static_cast<double>(T)));
      hdr->ticket = 0u;  // ready for the next call on this workspace
    }
  }
}

// Streaming absmean: persistent CTAs of 256 threads, kAbsCtasPerSm per SM;
// thread l is lane l of the fixed order.  CTA b takes the chunks b, b + G, ...:
// each thread loads its 32 elements of the chunk (the i = 0..3 runs of 8, as
// 16-byte loads straight into registers) and adds them in order; the lane sums
// go to a shared array (two copies, by chunk parity), one barrier, and warp
// (k mod 8) of the CTA takes the chunk's tree (levels 128, 64, 32 in
// registers, 16..1 by shuffles) while the other warps load the next chunk.
// The copy written for chunk k is written again for chunk k + 2 only after the
// barrier of chunk k + 1, which the tree warp of chunk k reaches after its
// reads.  Reads from L2 or HBM straight to registers (no shared staging):
// with 4 CTAs per SM, 128 KB per SM can be in flight.
constexpr int kAbsCtasPerSm = 4;

// With MEAN (the 1-bit variant) the kernel also adds the signed weights in the
// same order, into partials[C + c], and the last CTA writes alpha = fp32(S / T)
// beside gamma (= beta).
template <int WDT, bool MEAN>
__global__ void __launch_bounds__(kLanes, kAbsCtasPerSm)
    absmean_kernel(const void* __restrict__ W, int64_t T, int64_t C, int lgR, double* __restrict__ partials,
                   WsHeader* __restrict__ hdr, float* __restrict__ gamma, float* __restrict__ alpha) {
  pdl_enter(W, partials, hdr, gamma, alpha);
  constexpr int NS = MEAN ? 2 : 1;  // sums per lane
  __shared__ double lsum[2][NS][kLanes];
  __shared__ double p[kLanes];
  __shared__ bool last;
  const int l = threadIdx.x, warp = l >> 5, L = l & 31;
  const int64_t G = gridDim.x;
  int k = 0;
  for (int64_t c = blockIdx.x; c < C; c += G, ++k) {
    const int64_t c0 = c * kChunk;
    float v[4][8];
    if (c0 + kChunk <= T) {
#pragma unroll
      for (int i = 0; i < 4; ++i) load8_aligned<WDT>(W, c0 + 2048 * i + 8 * l, v[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t e0 = c0 + 2048 * i + 8 * l;
#pragma unroll
        for (int j = 0; j < 8; ++j) v[i][j] = (e0 + j < T) ? load_elem<WDT>(W, e0 + j) : 0.0f;
      }
    }
    double acc = 0.0, acc_s = 0.0;  // +0.0 for elements past T leaves the sums unchanged
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc = __dadd_rn(acc, static_cast<double>(fabsf(v[i][j])));
        if constexpr (MEAN) acc_s = __dadd_rn(acc_s, static_cast<double>(v[i][j]));
      }
    lsum[k & 1][0][l] = acc;
    if constexpr (MEAN) lsum[k & 1][NS - 1][l] = acc_s;
    __syncthreads();
    if (warp == (k & 7)) {
#pragma unroll
      for (int z = 0; z < NS; ++z) {
        const double* ls = lsum[k & 1][z];
        double q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) q[u] = ls[L + 32 * u];
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = __dadd_rn(q[u], q[u + 4]);  // level 128
        q[0] = __dadd_rn(q[0], q[2]);                                   // level 64
        q[1] = __dadd_rn(q[1], q[3]);
        double t = __dadd_rn(q[0], q[1]);                               // level 32
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, o));
        if (L == 0) partials[z * C + c] = t;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned ticket = atomicAdd(&hdr->ticket, 1u);
    last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  absmean_finish(partials, C, lgR, T, p, hdr, gamma);
  if constexpr (MEAN) {
    __syncthreads();  // warp 0 has read p
    absmean_finish(partials + C, C, lgR, T, p, hdr, alpha);
  }
}

// ---------------------------------------------------------------------------
// Ternarize and pack.  rint(fl(w / d)) is 0 exactly when the real quotient
// |w| / d <= 1/2 + 2^-25 (fp32 rounds quotients up to that midpoint down to
// 0.5, and rint sends 0.5 to 0).  d * (1/2 + 2^-25) is exact in fp64 (24 x 25
// significant bits), and for fp32 |w| the comparison with it equals the
// comparison with its fp32 round-down.  So code = sign(w) if |w| > thr else 0,
// with thr = RD32(d * (1/2 + 2^-25)): the same codes as the IEEE division,
// with one compare per weight.  Codes past +-1 are clamped by construction.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ternary_threshold(float gamma, float eps) {
  const float d = __fadd_rn(gamma, eps);
  return __double2float_rd(__dmul_rn(static_cast<double>(d), 0.5 + 0x1p-25));
}

__device__ __forceinline__ uint32_t ternary_digit(float w, float thr) {  // q + 1
  return fabsf(w) > thr ? (w > 0.0f ? 2u : 0u) : 1u;
}

// 16 consecutive weights of a row, widened to fp32, with 16-byte loads.
template <int WDT>
__device__ __forceinline__ void load16_aligned(const void* p, int64_t e, float v[16]) {
  load8_aligned<WDT>(p, e, v);
  load8_aligned<WDT>(p, e + 8, v + 8);
}

__device__ __forceinline__ uint32_t codes4_word(const float* v, float thr) {  // 4 int8 codes
  uint32_t u = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) u |= ((ternary_digit(v[i], thr) - 1u) & 0xffu) << (8 * i);
  return u;
}

// One thread writes one 16-byte segment of a packed row: 64 weights (2-bit)
// or 80 weights (base 3).  Weights past K are weight 0 (padding digits).
// Threads walk the segments from the end of W backwards: the latent weights
// were just streamed front to back by the absmean kernel, so the last ones
// read there are the likeliest to still be in L2.
template <int WDT, int FMT>
__global__ void __launch_bounds__(256)
    ternarize_pack_kernel(const void* __restrict__ W, int64_t N, int64_t K,
                          const float* __restrict__ gamma, float eps, uint8_t* __restrict__ packed,
                          int8_t* __restrict__ codes, int64_t rowbytes, bool vec_ok) {
  pdl_enter(W, gamma, packed, codes);
  constexpr int PER = (FMT == BL_PACK_I2) ? 4 : 5;
  constexpr int WPS = 16 * PER;  // weights per segment
  __shared__ float sh_thr;  // gamma once per CTA: a load by every warp hits one L2 line thousands of times
  if (threadIdx.x == 0) sh_thr = ternary_threshold(__ldcg(gamma), eps);
  __syncthreads();
  const float thr = sh_thr;
  const int64_t segs = rowbytes / 16;
  const int64_t total = N * segs;
  for (int64_t it = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; it < total;
       it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t gid = total - 1 - it;
    const int64_t n = gid / segs;
    const int64_t sg = gid - n * segs;
    const int64_t k0 = sg * WPS;
    const int64_t base = n * K + k0;
    uint32_t out[4];
    if (vec_ok && k0 + WPS <= K) {
      float v[WPS];
#pragma unroll
      for (int g = 0; g < WPS / 16; ++g) load16_aligned<WDT>(W, base + 16 * g, v + 16 * g);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t byte = 0;
          if constexpr (FMT == BL_PACK_I2) {
#pragma unroll
            for (int i = 0; i < 4; ++i) byte |= ternary_digit(v[16 * w + 4 * b + i], thr) << (2 * i);
          } else {
#pragma unroll
            for (int i = 4; i >= 0; --i) byte = byte * 3u + ternary_digit(v[20 * w + 5 * b + i], thr);
          }
          word |= byte << (8 * b);
        }
        out[w] = word;
      }
      if (codes != nullptr) {
        int8_t* dst = codes + base;
        if ((K % 16) == 0) {
#pragma unroll
          for (int g = 0; g < WPS / 16; ++g)
            *reinterpret_cast<uint4*>(dst + 16 * g) =
                make_uint4(codes4_word(v + 16 * g, thr), codes4_word(v + 16 * g + 4, thr),
                           codes4_word(v + 16 * g + 8, thr), codes4_word(v + 16 * g + 12, thr));
        } else {
#pragma unroll
          for (int i = 0; i < WPS; ++i) dst[i] = static_cast<int8_t>(static_cast<int>(ternary_digit(v[i], thr)) - 1);
        }
      }
    } else {
      // ragged tail of a row (or unaligned rows): guarded scalar loads
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t byte = 0;
#pragma unroll
          for (int ii = 0; ii < PER; ++ii) {
            const int i = (FMT == BL_PACK_I2) ? ii : PER - 1 - ii;
            const int kk = (FMT == BL_PACK_I2) ? 16 * w + 4 * b + i : 20 * w + 5 * b + i;
            const uint32_t d = (k0 + kk < K) ? ternary_digit(load_elem<WDT>(W, base + kk), thr) : 1u;
            if (codes != nullptr && k0 + kk < K) codes[base + kk] = static_cast<int8_t>(static_cast<int>(d) - 1);
            if constexpr (FMT == BL_PACK_I2)
              byte |= d << (2 * i);
            else
              byte = byte * 3u + d;
          }
          word |= byte << (8 * b);
        }
        out[w] = word;
      }
    }
    if (packed != nullptr)
      *reinterpret_cast<uint4*>(packed + n * rowbytes + sg * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// Flat 2-bit ternarize + pack, for K % 64 == 0.  The row stride is then K / 4
// bytes with no padding, so packed byte p of the matrix holds the weights
// 4p .. 4p + 3 of W in row-major order and the matrix is one stream.  A thread
// turns a group of 16 consecutive weights (16-byte loads straight into
// registers) into 4 packed bytes (one 32-bit store) and, if asked, 16 int8
// codes (one 16-byte store).  It works on 64 bytes of W (two groups of bf16,
// one of fp32) while the loads of the next 64 are in flight (issued ahead in program order: the loads are
// L2-coherent asm loads, which the compiler does not move across the stores
// of the groups before them), and a persistent
// grid of kTernCtasPerSm CTAs per SM walks the groups from the end of W
// backwards (the absmean kernel streamed W front to back, so the last groups it
// read are the likeliest to still be in L2).
constexpr int kTernCtasPerSm = 4;

template <int WDT>
__global__ void __launch_bounds__(256, kTernCtasPerSm)
    ternarize_flat_kernel(const void* __restrict__ W, int64_t T, const float* __restrict__ gamma, float eps,
                          uint8_t* __restrict__ packed, int8_t* __restrict__ codes) {
  pdl_enter(W, gamma, packed, codes);
  const int64_t ng = T / 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // raw 16-byte words of the thread's U groups (64 bytes of W); the next U
  // groups' loads go out before the current ones are turned into codes
  constexpr int RW = (WDT == BL_F32) ? 4 : 2;  // 16-byte words per group
  constexpr int EW = 16 / RW;                   // weights per word
  constexpr int U = (WDT == BL_F32) ? 1 : 2;    // groups per step
  auto fetch = [&](int64_t gi, uint4 (&r)[U][RW]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = ng - 1 - (gi + u * stride);
      const uint4* q = static_cast<const uint4*>(W) + g * RW;  // group g: 16 weights, RW words
#pragma unroll
      for (int i = 0; i < RW; ++i) r[u][i] = g >= 0 ? __ldcg(q + i) : make_uint4(0, 0, 0, 0);
    }
  };
  int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint4 cur[U][RW];
  if (gi < ng) fetch(gi, cur);  // (the first loads go out before the threshold is known)
  __shared__ float sh_thr;      // gamma once per CTA: a load by every warp hits one L2 line thousands of times
  if (threadIdx.x == 0) sh_thr = ternary_threshold(__ldcg(gamma), eps);
  __syncthreads();
  const float thr = sh_thr;
  for (; gi < ng; gi += U * stride) {
    uint4 nxt[U][RW];
    fetch(gi + U * stride, nxt);  // (zeros past the last group)
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = ng - 1 - (gi + u * stride);
      if (g < 0) continue;
      uint32_t word = 0, cw[4];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const uint32_t w[4] = {cur[u][i].x, cur[u][i].y, cur[u][i].z, cur[u][i].w};
        float v[EW];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if constexpr (WDT == BL_F32) {
            v[j] = __uint_as_float(w[j]);
          } else {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
          }
        }
#pragma unroll
        for (int j = 0; j < EW; ++j) word |= ternary_digit(v[j], thr) << (2 * (EW * i + j));
#pragma unroll
        for (int j = 0; j < EW / 4; ++j) cw[EW / 4 * i + j] = codes4_word(v + 4 * j, thr);
      }
      reinterpret_cast<uint32_t*>(packed)[g] = word;
      if (codes != nullptr) reinterpret_cast<uint4*>(codes)[g] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < RW; ++i) cur[u][i] = nxt[u][i];
  }
}

// ---------------------------------------------------------------------------
// 1-bit binarize and pack ("QAT and BitNet: A Deep Dive into 1-bit and
// 1.58-bit Quantization-Aware Training", "The BitLinear Recipe" step 2): a
// weight above alpha is +1, any other -1.  Bit i of byte j of a row holds
// weight 8 j + i (1 for +1); bits past K are 0.  One thread writes one 16-byte
// segment (128 weights) of a packed row, one 32-bit word (32 weights) at a
// time, with 16-byte loads of W when the row allows them; segments are walked
// from the end of W backwards (the scale kernel just streamed W front to back).
// ---------------------------------------------------------------------------
template <int WDT>
__global__ void __launch_bounds__(256)
    binarize_pack_kernel(const void* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ alpha,
                         uint8_t* __restrict__ packed, int8_t* __restrict__ codes, int64_t rowbytes, bool vec_ok) {
  pdl_enter(W, alpha, packed, codes);
  __shared__ float sh_alpha;  // once per CTA
  if (threadIdx.x == 0) sh_alpha = __ldcg(alpha);
  __syncthreads();
  const float a = sh_alpha;
  const int64_t segs = rowbytes / 16;
  const int64_t total = N * segs;
  for (int64_t it = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; it < total;
       it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t gid = total - 1 - it;
    const int64_t n = gid / segs;
    const int64_t sg = gid - n * segs;
    uint32_t out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int64_t k0 = sg * 128 + 32 * w;
      const int64_t base = n * K + k0;
      uint32_t word = 0;
      if (vec_ok && k0 + 32 <= K) {
        float v[32];
#pragma unroll
        for (int g = 0; g < 4; ++g) load8_aligned<WDT>(W, base + 8 * g, v + 8 * g);
#pragma unroll
        for (int i = 0; i < 32; ++i) word |= (v[i] > a ? 1u : 0u) << i;
        if (codes != nullptr) {
          uint32_t cw[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t c = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) c |= (v[4 * j + b] > a ? 0x01u : 0xffu) << (8 * b);
            cw[j] = c;
          }
          if ((K % 16) == 0) {
            uint4* dst = reinterpret_cast<uint4*>(codes + base);
            dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) codes[base + i] = static_cast<int8_t>(v[i] > a ? 1 : -1);
          }
        }
      } else {
        for (int i = 0; i < 32; ++i) {
          if (k0 + i >= K) break;
          const bool plus = load_elem<WDT>(W, base + i) > a;
          word |= (plus ? 1u : 0u) << i;
          if (codes != nullptr) codes[base + i] = static_cast<int8_t>(plus ? 1 : -1);
        }
      }
      out[w] = word;
    }
    if (packed != nullptr)
      *reinterpret_cast<uint4*>(packed + n * rowbytes + sg * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// Pack int8 codes (same segment mapping).  A code outside {-1, 0, 1} packs as
// weight 0 and raises the bad-code flag.
template <int FMT>
__global__ void __launch_bounds__(256)
    pack_kernel(const int8_t* __restrict__ codes, int64_t N, int64_t K, uint8_t* __restrict__ packed,
                int64_t rowbytes, void* ws) {
  pdl_enter(codes, packed, ws);
  constexpr int PER = (FMT == BL_PACK_I2) ? 4 : (FMT == BL_PACK_T5 ? 5 : 8);
  constexpr int WPS = 16 * PER;
  // N segs < 2^32 (N K <= 2^32): 32-bit item indices
  const uint32_t segs = static_cast<uint32_t>(rowbytes / 16);
  const uint32_t total = static_cast<uint32_t>(N) * segs;
  // K % 16 == 0: every 16-code chunk of a segment starts 16-byte aligned and
  // lies wholly inside or past the row, so the segment's codes come in with
  // 16-byte loads (chunks past K read as 0)
  const bool vec = (K & 15) == 0;
  for (uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x; gid < total; gid += gridDim.x * blockDim.x) {
    const uint32_t n32 = gid / segs;
    const int64_t n = n32;
    const int64_t sg = gid - n32 * segs;
    const int64_t k0 = sg * WPS;
    const int8_t* src = codes + n * K + k0;
    uint32_t cw[WPS / 4];
    if (vec) {
#pragma unroll
      for (int j = 0; j < WPS / 16; ++j) {
        const uint4 v = k0 + 16 * j < K ? __ldcg(reinterpret_cast<const uint4*>(src + 16 * j)) : make_uint4(0, 0, 0, 0);
        cw[4 * j] = v.x;
        cw[4 * j + 1] = v.y;
        cw[4 * j + 2] = v.z;
        cw[4 * j + 3] = v.w;
      }
    }
    bool bad = false;
    uint32_t out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        uint32_t byte = 0;
#pragma unroll
        for (int ii = 0; ii < PER; ++ii) {
          const int i = (FMT == BL_PACK_T5) ? PER - 1 - ii : ii;
          const int kk = 4 * PER * w + PER * b + i;
          int c = vec ? static_cast<int>(static_cast<int8_t>(cw[kk >> 2] >> (8 * (kk & 3))))
                      : ((k0 + kk < K) ? static_cast<int>(__ldcg(src + kk)) : 0);
          if constexpr (FMT == BL_PACK_B1) {  // {-1, +1}; pad bits 0
            if (k0 + kk < K && c != 1 && c != -1) bad = true;
            byte |= (c == 1 ? 1u : 0u) << i;
            continue;
          }
          if (c < -1 || c > 1) {
            bad = true;
            c = 0;
          }
          if constexpr (FMT == BL_PACK_I2)
            byte |= static_cast<uint32_t>(c + 1) << (2 * i);
          else
            byte = byte * 3u + static_cast<uint32_t>(c + 1);
        }
        word |= byte << (8 * b);
      }
      out[w] = word;
    }
    *reinterpret_cast<uint4*>(packed + n * rowbytes + sg * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    if (bad) set_flag(ws, kFlagBadCode, 0x100u);
  }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
int device_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

static int grid_for(int64_t work, int threads, int per_sm_ctas) {
  const int sms = device_sms();
  const int64_t need = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sms) * per_sm_ctas;
  return static_cast<int>(need < cap ? (need < 1 ? 1 : need) : cap);
}

cudaError_t launch_absmean(const void* W, int wdt, int64_t N, int64_t K, void* ws, float* gamma,
                           cudaStream_t st, float* alpha) {
  const int64_t T = N * K;
  const int64_t C = (T + kChunk - 1) / kChunk;
  int lgP = 0;
  while ((int64_t{1} << lgP) < C) ++lgP;
  const int lgR = lgP > 8 ? lgP - 8 : 0;  // 256 = kLanes slots in the final tree
  if (lgR > kFinishMaxLevels) return cudaErrorInvalidValue;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  double* partials = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES);
  // persistent streaming grid: kAbsCtasPerSm CTAs per SM (at most one per chunk)
  const int64_t cap = static_cast<int64_t>(device_sms()) * kAbsCtasPerSm;
  const int64_t grid = C < cap ? C : cap;
  const unsigned g = static_cast<unsigned>(grid);
  if (alpha != nullptr) {
    if (wdt == BL_F32)
      return launch_pdl(absmean_kernel<BL_F32, true>, g, kLanes, 0, st, W, T, C, lgR, partials, hdr, gamma, alpha);
    return launch_pdl(absmean_kernel<BL_BF16, true>, g, kLanes, 0, st, W, T, C, lgR, partials, hdr, gamma, alpha);
  }
  if (wdt == BL_F32)
    return launch_pdl(absmean_kernel<BL_F32, false>, g, kLanes, 0, st, W, T, C, lgR, partials, hdr, gamma, alpha);
  return launch_pdl(absmean_kernel<BL_BF16, false>, g, kLanes, 0, st, W, T, C, lgR, partials, hdr, gamma, alpha);
}

cudaError_t launch_ternarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* gamma,
                                  float eps, int fmt, uint8_t* packed, int8_t* codes, int64_t rowbytes, void* ws,
                                  cudaStream_t st) {
  if (fmt == BL_PACK_I2 && (K % 64) == 0 && packed != nullptr) {
    const int64_t T = N * K;
    const int64_t ng = T / 16;
    const int64_t cap = static_cast<int64_t>(device_sms()) * kTernCtasPerSm;
    int64_t grid = (ng + 511) / 512;  // two groups per thread
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (wdt == BL_F32)
      return launch_pdl(ternarize_flat_kernel<BL_F32>, static_cast<unsigned>(grid), 256, 0, st, W, T, gamma, eps,
                        packed, codes);
    return launch_pdl(ternarize_flat_kernel<BL_BF16>, static_cast<unsigned>(grid), 256, 0, st, W, T, gamma, eps,
                      packed, codes);
  }
  const bool vec_ok = (wdt == BL_F32) ? (K % 4 == 0) : (K % 8 == 0);
  const int64_t work = N * (rowbytes / 16);
  const int threads = 256;
  const int grid = grid_for(work, threads, 4);
#define BL_TP(WDT, FMT)                                                                                     \
  return launch_pdl(ternarize_pack_kernel<WDT, FMT>, grid, threads, 0, st, W, N, K, gamma, eps, packed, codes, \
                    rowbytes, vec_ok)
  if (wdt == BL_F32 && fmt == BL_PACK_I2) BL_TP(BL_F32, BL_PACK_I2);
  else if (wdt == BL_F32) BL_TP(BL_F32, BL_PACK_T5);
  else if (fmt == BL_PACK_I2) BL_TP(BL_BF16, BL_PACK_I2);
  else BL_TP(BL_BF16, BL_PACK_T5);
#undef BL_TP
}

cudaError_t launch_pack(const int8_t* codes, int64_t N, int64_t K, int fmt, uint8_t* packed,
                        int64_t rowbytes, void* ws, cudaStream_t st) {
  const int64_t work = N * (rowbytes / 16);
  const int grid = grid_for(work, 256, 8);
  if (fmt == BL_PACK_I2) return launch_pdl(pack_kernel<BL_PACK_I2>, grid, 256, 0, st, codes, N, K, packed, rowbytes, ws);
  if (fmt == BL_PACK_B1) return launch_pdl(pack_kernel<BL_PACK_B1>, grid, 256, 0, st, codes, N, K, packed, rowbytes, ws);
  return launch_pdl(pack_kernel<BL_PACK_T5>, grid, 256, 0, st, codes, N, K, packed, rowbytes, ws);
}

cudaError_t launch_binarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* alpha, uint8_t* packed,
                                 int8_t* codes, int64_t rowbytes, cudaStream_t st) {
  const bool vec_ok = (K % 8) == 0;
  const int64_t work = N * (rowbytes / 16);
  const int grid = grid_for(work, 256, 4);
  if (wdt == BL_F32)
    return launch_pdl(binarize_pack_kernel<BL_F32>, grid, 256, 0, st, W, N, K, alpha, packed, codes, rowbytes, vec_ok);
  return launch_pdl(binarize_pack_kernel<BL_BF16>, grid, 256, 0, st, W, N, K, alpha, packed, codes, rowbytes, vec_ok);
}

}  // namespace bl
