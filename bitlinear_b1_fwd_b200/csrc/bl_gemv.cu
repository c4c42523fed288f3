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
#include "bl_gemv.cuh"
#include "bl_kernels.h"

namespace bl {

constexpr int kGemvThreads = 768;  // one CTA per SM: the token prologue runs once per SM
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvBatch = 4;         // items per load batch; two batches per warp alternate
constexpr int kGemvTileRows = 1024;   // rows whose sums a CTA holds in shared memory at a time


// Activation bytes per token in shared memory for one packed row of rowbytes.
__host__ __device__ inline int64_t gemv_x_bytes(int fmt, int64_t rowbytes) {
  return fmt == BL_PACK_I2 ? rowbytes * 4 : rowbytes * 8;
}

// Dynamic shared memory of one CTA for mt tokens.
__host__ __device__ inline int64_t gemv_smem_bytes(int fmt, int64_t rowbytes, int mt) {
  return mt * gemv_x_bytes(fmt, rowbytes) + int64_t{4} * mt * kGemvTileRows + (fmt == BL_PACK_T5 ? 256 * 8 : 0);
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



// Work split.  CTA b owns the rows [row0, row0 + nrows) (the N rows shared
// out as evenly as the grid allows); they are contiguous in memory, and the CTA
// takes them in tiles of at most kGemvTileRows rows.  A tile is a run of
// S = rows x segs 16-byte segments; its work items are the 32-segment blocks
// of that run (512 bytes each, not aligned to rows), dealt round-robin to the
// warps, so at any time the CTA streams one contiguous window of up to
// 2 kGemvBatch x kGemvWarps blocks (96 KB).  Each warp loads its items in
// batches of kGemvBatch (the loads of a batch are issued together and waited
// for together), two batches alternating: while one is reduced the other is
// in flight.  Lane L
// of an item takes segment 32 j + L; a block covers at most two rows when a
// row has 32 segments or more (any number otherwise).  Each item's INT32 sums
// are reduced per row across the warp and added into the tile's shared row
// sums (integer addition: the order does not matter); after the tile the CTA
// dequantizes the row sums and stores them coalesced.
template <int FMT, int MT, int XDT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                void* __restrict__ y, int ydt, int write_scale, const RowGroups rg) {
  pdl_enter(packed, gamma, x, scale, y);
  extern __shared__ __align__(16) uint8_t smem[];
  const int64_t xb = gemv_x_bytes(FMT, rowbytes);
  uint8_t* xs = smem;                                                 // [MT][xb]
  int* racc = reinterpret_cast<int*>(smem + MT * xb);                 // [MT][kGemvTileRows]
  uint2* lut = reinterpret_cast<uint2*>(racc + MT * kGemvTileRows);   // base 3 only
  __shared__ float red_f[MT][kGemvWarps];
  __shared__ int red_i[MT][kGemvWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t segs = static_cast<uint32_t>(rowbytes >> 4);
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int64_t nrows = per + (b < extra ? 1 : 0);

  // The warp's items in a tile are j = warp + W k.  Two cursors walk them: one
  // for the loads in flight, one for the item being reduced.  (A tile has at
  // most kGemvTileRows x segs < 2^22 segments: 32-bit counts.)
  uint32_t S = 0, nitems = 0, l_j = 0;
  const uint4* tile = nullptr;
  auto start_tile = [&](int64_t t0) {
    const uint32_t nr = static_cast<uint32_t>((nrows - t0) < kGemvTileRows ? (nrows - t0) : kGemvTileRows);
    S = nr * segs;
    nitems = (S + 31) >> 5;
    l_j = warp;
    tile = reinterpret_cast<const uint4*>(packed + (row0 + t0) * rowbytes);
  };
  auto load_next = [&](uint4& dst) {
    const uint32_t g = 32 * l_j + lane;
    if (g < S) dst = ld_stream(tile + g);
    l_j += kGemvWarps;
  };

  auto issue = [&](uint4(&b)[kGemvBatch]) {
#pragma unroll
    for (int d = 0; d < kGemvBatch; ++d)
      if (l_j < nitems) load_next(b[d]);
  };

  // 1. the first tile's first batch goes out before the prologue
  start_tile(0);
  uint4 bufA[kGemvBatch], bufB[kGemvBatch];
#pragma unroll
  for (int d = 0; d < kGemvBatch; ++d) bufA[d] = bufB[d] = make_uint4(0, 0, 0, 0);
  issue(bufA);

  // 2. prologue: per-token absmax, then the INT8 codes in the layout above
  //    gamma (and the scales of int8 tokens) are read once per CTA into
  //    shared memory: a load by every warp sends thousands of requests to one
  //    L2 line
  __shared__ float sh_gs[1 + MT];
  if (threadIdx.x <= MT && (threadIdx.x == 0 || XDT == BL_I8))
    sh_gs[threadIdx.x] = __ldcg(threadIdx.x == 0 ? gamma : scale + (threadIdx.x - 1));
  __shared__ float sh_gam[kMaxRowGroups];  // gamma of each row group
  if (threadIdx.x < rg.n) sh_gam[threadIdx.x] = __ldcg(gamma + threadIdx.x);
  for (int i = threadIdx.x; i < MT * kGemvTileRows; i += blockDim.x) racc[i] = 0;
  if constexpr (FMT == BL_PACK_T5) {
    uint4* z = reinterpret_cast<uint4*>(xs);
    for (int64_t i = threadIdx.x; i < MT * xb / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
      uint32_t lo = 0, hi = 0;
      if (e < 243) {
        int v = e;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const uint32_t w = static_cast<uint8_t>(static_cast<int8_t>(v % 3 - 1));
          v /= 3;
          if (i < 4) lo |= w << (8 * i);
          else hi = w;
        }
      }
      lut[e] = make_uint2(lo, hi);
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
  __syncthreads();  // zeroed sums and activations, table and per-warp maxima are visible
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if constexpr (XDT != BL_I8) {
      float a = red_f[m][0];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, red_f[m][w]);
      s_tok[m] = fmaxf(a, 1e-6f);
    } else {
      s_tok[m] = sh_gs[1 + m];
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int part = 0;
    uint8_t* xm = xs + m * xb;
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok[m]);
    if constexpr (FMT == BL_PACK_I2) {
      // one packed word's 16 codes per step, written as one 16-byte slot
      // (codes past K, under padding digits, are 0)
      for (uint32_t g = threadIdx.x; g < 4 * segs; g += blockDim.x) {
        const int64_t k0 = 16 * static_cast<int64_t>(g);
        const bool full = k0 + 16 <= K && (K % 16) == 0;
        uint32_t P[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // eight codes at a time
          const int64_t kh = k0 + 8 * h;
          int q[8];
          if (full) {
            if constexpr (XDT == BL_I8) {
              const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + kh));
#pragma unroll
              for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
            } else {
              float e[8];
              load8_aligned<XDT>(x, m * K + kh, e);
quant_act_fast_n<8>(e, s_tok[m], c127, q);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int64_t k = kh + j;
              if (k < K)
                q[j] = (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[m * K + k])
                                      : quant_act_fast(load_x<XDT>(x, m * K + k), s_tok[m], c127);
              else
                q[j] = 0;
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) part += q[j];
          P[2 * h] = pack4(q);
          P[2 * h + 1] = pack4(q + 4);
        }
        const uint32_t s = g >> 2, w = g & 3;
        *reinterpret_cast<uint4*>(xm + (w * segs + s) * 16) = i2_slot(P[0], P[1], P[2], P[3]);
      }
    } else if (vec) {
      for (int64_t v = threadIdx.x; v < K / 8; v += blockDim.x) {
        int q[8];
        if constexpr (XDT == BL_I8) {
          const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + 8 * v));
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
        } else {
          float e[8];
          load8_aligned<XDT>(x, m * K + 8 * v, e);
          quant_act_fast_n<8>(e, s_tok[m], c127, q);
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
  const float g = sh_gs[0];
  float cfac[MT];
  int corr[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) t += red_i[m][w];
    corr[m] = (FMT == BL_PACK_I2) ? t : 0;  // 2-bit digits are q + 1: subtract sum x once per row
    cfac[m] = dequant_factor(g, s_tok[m]);
    if (XDT != BL_I8 && write_scale && blockIdx.x == 0 && threadIdx.x == 0) scale[m] = s_tok[m];
  }

  // 3. per tile: stream the items, one batch of loads in flight while the
  //    other is reduced.
  const bool wide = segs >= 32;                            // a block spans at most two rows
  const uint32_t dq = (32u * kGemvWarps) / segs, dr = (32u * kGemvWarps) % segs;  // one step of a warp
  for (int64_t t0 = 0; t0 < nrows; t0 += kGemvTileRows) {
    if (t0 > 0) {
      start_tile(t0);
      issue(bufA);
    }
    const uint32_t nr = S / segs;
    uint32_t c_j = warp;
    uint32_t r0 = (32u * c_j) / segs, s0 = 32u * c_j - r0 * segs;  // row and segment of lane 0
    auto consume = [&](const uint4(&b)[kGemvBatch]) {
#pragma unroll
      for (int d = 0; d < kGemvBatch; ++d) {
        if (c_j >= nitems) break;
        const uint4 cur = b[d];
        const uint32_t g = 32 * c_j + lane;
        uint32_t r, sg;
        if (wide) {
          sg = s0 + lane;
          r = r0;
          if (sg >= segs) {
            sg -= segs;
            ++r;
          }
        } else {
          r = g / segs;
          sg = g - r * segs;
        }
        int v[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) v[m] = 0;
        if (g < S) {
          const uint32_t wd[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            if constexpr (FMT == BL_PACK_I2) {
              const uint32_t c0 = wd[w] & 0x03030303u, c1 = (wd[w] >> 2) & 0x03030303u;
              const uint32_t c2 = (wd[w] >> 4) & 0x03030303u, c3 = (wd[w] >> 6) & 0x03030303u;
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const uint4 X = *reinterpret_cast<const uint4*>(xs + m * xb + ((w * segs) + sg) * 16);
                v[m] = dp4a_us(c0, X.x, v[m]);
                v[m] = dp4a_us(c1, X.y, v[m]);
                v[m] = dp4a_us(c2, X.z, v[m]);
                v[m] = dp4a_us(c3, X.w, v[m]);
              }
            } else {
#pragma unroll
              for (int bb = 0; bb < 4; ++bb) {
                const uint2 Lw = lut[(wd[w] >> (8 * bb)) & 0xffu];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                  const uint2 X = *reinterpret_cast<const uint2*>(xs + m * xb + (((4 * w + bb) * segs) + sg) * 8);
                  v[m] = __dp4a(static_cast<int>(Lw.x), static_cast<int>(X.x), v[m]);
                  v[m] = __dp4a(static_cast<int>(Lw.y), static_cast<int>(X.y), v[m]);
                }
              }
            }
          }
        }
        // per-row sums of the block into the tile's row sums
        if (wide) {
          const uint32_t bnd = segs - s0;  // lanes >= bnd are in row r0 + 1
          const uint32_t lo = bnd >= 32 ? 0xffffffffu : ((1u << bnd) - 1u);
          const uint32_t mask = (static_cast<uint32_t>(lane) < bnd) ? lo : ~lo;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const int t = __reduce_add_sync(mask, v[m]);
            if ((lane == 0 || static_cast<uint32_t>(lane) == bnd) && r < nr) atomicAdd(racc + m * kGemvTileRows + r, t);
          }
        } else {
          const int key = g < S ? static_cast<int>(r) : -1;
          const uint32_t mask = __match_any_sync(0xffffffffu, key);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const int t = __reduce_add_sync(mask, v[m]);
            if (key >= 0 && (__ffs(mask) - 1) == lane) atomicAdd(racc + m * kGemvTileRows + key, t);
          }
        }
        c_j += kGemvWarps;
        r0 += dq;
        s0 += dr;
        if (s0 >= segs) {
          s0 -= segs;
          ++r0;
        }
      }
    };
    while (c_j < nitems) {
      issue(bufB);
      consume(bufA);
      issue(bufA);
      consume(bufB);
    }
    __syncthreads();  // every part of every row of the tile has been added
    for (int r = threadIdx.x; r < static_cast<int>(nr); r += blockDim.x) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int a = racc[m * kGemvTileRows + r] - corr[m];
        racc[m * kGemvTileRows + r] = 0;
        const int64_t o = m * N + row0 + t0 + r;
        const float cf = rg.n == 1 ? cfac[m] : dequant_factor(sh_gam[row_group(rg, row0 + t0 + r)], s_tok[m]);
        if (ydt == BL_I32)
          static_cast<int32_t*>(y)[o] = a;
        else if (ydt == BL_F32)
          static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cf);
        else
          static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cf));
      }
    }
    __syncthreads();  // the row sums are zero again for the next tile
  }
}

// 1-bit activation layout, one-pass prologue: lane pair (2t, 2t + 1) holds the
// 16-code groups e and e + 1 (e even), the two halves of packed word e >> 1
// (P: the group's codes, four per word).  Each lane builds, for the activation
// words i of the word, its two bytes (codes i and 8 + i of its half: bytes 2hb
// and 2hb + 1, hb = e & 1), trades the halves the other lane stores with
// it, and writes the four words of its plane (words 0-3 for hb = 0, 4-7 for
// hb = 1).  Every lane of the warp takes part in the exchange; `valid` only
// gates the store.
template <int kPB>
__device__ __forceinline__ void b1_put_half_t(uint8_t* xm, const uint32_t (&P)[4], uint32_t e, bool valid) {
  // hh[t]: own bytes of words 2t (low half) and 2t + 1 (high half)
  const uint32_t hh[4] = {__byte_perm(P[0], P[2], 0x5140), __byte_perm(P[0], P[2], 0x7362),
                          __byte_perm(P[1], P[3], 0x5140), __byte_perm(P[1], P[3], 0x7362)};
  const uint32_t hb = e & 1u;
  const uint32_t oA = hb ? hh[2] : hh[0], oB = hb ? hh[3] : hh[1];  // kept: this lane's words
  const uint32_t sA = hb ? hh[0] : hh[2], sB = hb ? hh[1] : hh[3];  // sent: the other lane's words
  const uint32_t rA = __shfl_xor_sync(0xffffffffu, sA, 1), rB = __shfl_xor_sync(0xffffffffu, sB, 1);
  const uint32_t loA = hb ? rA : oA, hiA = hb ? oA : rA, loB = hb ? rB : oB, hiB = hb ? oB : rB;
  if (valid) {
    const uint32_t g = e >> 1, s = g >> 2, w = g & 3u;
    *reinterpret_cast<uint4*>(xm + (4 * w + 2 * (s & 1u) + hb) * kPB + (s >> 1) * 16) =
        make_uint4(__byte_perm(loA, hiA, 0x5410), __byte_perm(loA, hiA, 0x7632), __byte_perm(loB, hiB, 0x5410),
                   __byte_perm(loB, hiB, 0x7632));
  }
}

// ---------------------------------------------------------------------------
// 2-bit decode GEMV, lean form (rows of at most 2 kI2Plane bytes).  A work
// item is one 64-segment (1 KB) block of a row; lane L takes the segments
// 64 blk + 2L and 64 blk + 2L + 1 (two 16-byte loads, a warp reads 1 KB
// contiguous).  A block lies in one row (the last block of a row is partial:
// lanes past the row's end load nothing and add 0), so each item ends in one
// warp reduction and one shared atomic into the row sum.  The activations of
// a token sit in 8 planes of kI2Plane bytes, plane 2w + h holding, for the
// segments s with s mod 2 = h, the 16 bytes of packed word w (the digit order
// of the word, as in the general layout) at (s >> 1) * 16: the 32 lanes of a
// warp read 32 consecutive 16-byte slots of a plane (no bank conflicts), and
// the 8 planes of a lane are a compile-time distance apart.  The digits are
// masked in place (w & (3 << 2j)), so accumulator j collects 4^j sum d x and
// the factors come off exactly at the end of the item.  Work split and load
// batching as in gemv_kernel: CTA-owned row ranges, items dealt round-robin
// to the warps, two batches of kI2Batch items alternating.
// ---------------------------------------------------------------------------
constexpr int kI2Plane = 4096;  // bytes per activation plane: segments per row <= 2 kI2Plane / 16
constexpr int kI2Batch = 2;     // items per load batch
constexpr int64_t kI2Prefetch = 65536;  // bytes per CTA prefetched into L2 before the wait

__host__ __device__ inline int64_t gemv_i2_smem_bytes(int mt) {
  return int64_t{8} * kI2Plane * mt + int64_t{4} * mt * kGemvTileRows;
}

// The same kernel serves the 1-bit format (FMT = BL_PACK_B1, rows of at most
// kI2Plane bytes): a 16-byte segment then holds 128 weights, bit i of byte j
// of a packed word being weight 8 j + i of its 32.  The token's codes sit in
// 16 planes of kI2Plane / 2 bytes, plane 4w + 2h + p holding, for the segments
// s with s mod 2 = h, four activation words of packed word w at (s >> 1) * 16:
// word i (i = 4p .. 4p + 3) has in byte j the code of weight 8 j + i, so that
// the mask w & (0x01010101 << i) and one dp4a collect 2^i times the sum of the
// codes over the +1 weights among weights i, 8 + i, 16 + i, 24 + i.  Eight
// accumulators per token, 2^i off exactly at the end of the item; with S the
// sum over the +1 weights and X the sum of the token's codes the product is
// 2 S - X.
template <int FMT, int MT, int XDT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_i2_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                   int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                   void* __restrict__ y, int ydt, int write_scale, const RowGroups rg) {
  constexpr bool kB1 = FMT == BL_PACK_B1;
  constexpr int kNP = kB1 ? 16 : 8;                   // activation planes per token
  constexpr int kPB = kB1 ? kI2Plane / 2 : kI2Plane;  // bytes per plane
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int64_t nrows = per + (b < extra ? 1 : 0);
  // 0. while the previous kernel finishes: the first kI2Prefetch bytes of
  //    this CTA's rows move into L2 (the weights do not depend on it)
  pdl_launch_dependents();
  {
    const int64_t bytes = nrows * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < kI2Prefetch ? bytes : kI2Prefetch);
  }
  pdl_wait(packed, gamma, x, scale, y);
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* xs = smem;                                           // [MT][kNP][kPB]
  int* racc = reinterpret_cast<int*>(smem + MT * 8 * kI2Plane);  // [MT][kGemvTileRows]
  __shared__ float red_f[MT][kGemvWarps];
  __shared__ int red_i[MT][kGemvWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t segs = static_cast<uint32_t>(rowbytes >> 4);
  const uint32_t nb = (segs + 63) >> 6;  // 1 KB blocks per row
  const uint32_t dq = kGemvWarps / nb, dr = kGemvWarps % nb;  // one step of a warp in (row, block)
  const uint32_t s_lane = 2u * lane;                            // first segment of the lane in a block

  // load cursor: item (l_row, l_blk) of the tile, l_row < l_rows
  uint32_t l_row = 0, l_blk = 0, l_rows = 0;
  const uint8_t* tile = packed;
  auto start_tile = [&](int64_t t0) {
    l_rows = static_cast<uint32_t>((nrows - t0) < kGemvTileRows ? (nrows - t0) : kGemvTileRows);
    l_row = warp / nb;
    l_blk = warp % nb;
    tile = packed + (row0 + t0) * rowbytes;
  };
  auto issue = [&](uint4(&bf)[kI2Batch][2]) {
#pragma unroll
    for (int d = 0; d < kI2Batch; ++d) {
      bf[d][0] = bf[d][1] = make_uint4(0, 0, 0, 0);
      if (l_row < l_rows) {
        const uint32_t s = 64u * l_blk + s_lane;
        const uint4* p = reinterpret_cast<const uint4*>(tile + static_cast<int64_t>(l_row) * rowbytes) + s;
        if (s < segs) bf[d][0] = ld_stream(p);
        if (s + 1 < segs) bf[d][1] = ld_stream(p + 1);
        l_blk += dr;
        l_row += dq;
        if (l_blk >= nb) {
          l_blk -= nb;
          ++l_row;
        }
      }
    }
  };

  // 1. one token of bf16 or int8 (K % 16 == 0): each thread's activation loads
  //    go out first and x is read once; the first batch of weights follows
  //    once the codes are written (weight loads issued earlier delay the
  //    activations and stall the prologue's warps at the load instructions).
  //    Otherwise the first batch of weights goes out before the prologue.
  constexpr bool kOnePassType = (MT == 1) && (XDT == BL_BF16 || XDT == BL_I8);
  constexpr int kXW = (XDT == BL_BF16) ? 2 : 1;  // 16-byte words per 16 activations
  const bool one_pass = kOnePassType && (K % 16) == 0;
  uint4 xraw[3][kXW];  // packed words g = tid + 768 u: 4 segs <= 2048 words (rows <= 8 KB)
  // gamma (and the scales of int8 tokens) once per CTA through shared memory,
  // loaded with the activations ahead of the weight stream: a load by every
  // warp sends thousands of requests to one L2 line
  __shared__ float sh_gs[1 + MT];
  if (threadIdx.x <= MT && (threadIdx.x == 0 || XDT == BL_I8))
    sh_gs[threadIdx.x] = __ldcg(threadIdx.x == 0 ? gamma : scale + (threadIdx.x - 1));
  __shared__ float sh_gam[kMaxRowGroups];  // gamma of each row group
  if (threadIdx.x < rg.n) sh_gam[threadIdx.x] = __ldcg(gamma + threadIdx.x);
  if (one_pass) {
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int64_t k0 = 16 * (static_cast<int64_t>(threadIdx.x) + static_cast<int64_t>(kGemvThreads) * u);
#pragma unroll
      for (int i = 0; i < kXW; ++i)
        xraw[u][i] = k0 < K ? __ldcg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + k0 * kXW) + i)
                            : make_uint4(0, 0, 0, 0);
    }
  }
  start_tile(0);
  uint4 bufA[kI2Batch][2], bufB[kI2Batch][2];
  if (!one_pass) issue(bufA);

  // 2. prologue: per-token absmax, then the INT8 codes in the plane layout
  for (int i = threadIdx.x; i < MT * kGemvTileRows; i += blockDim.x) racc[i] = 0;
  float s_tok[MT];
  if (one_pass) {
    // the absmax (bf16) and the codes from the registers loaded above
    auto elem = [&](int u, int jj) -> float {  // bf16 element jj (0..15) of word u
      const uint4 w4 = xraw[u][(jj >> 3) % kXW];
      const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
      const uint32_t wd = wv[(jj >> 1) & 3];
      return __uint_as_float((jj & 1) ? (wd & 0xffff0000u) : (wd << 16));
    };
    if constexpr (XDT == BL_BF16) {
      float amax = 0.0f;
#pragma unroll
      for (int u = 0; u < 3; ++u)
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) amax = fmaxf(amax, fabsf(elem(u, jj)));
      amax = warp_maxf(amax);
      if (lane == 0) red_f[0][warp] = amax;
      __syncthreads();  // zeroed row sums and per-warp maxima are visible
      s_tok[0] = fmaxf(warp_maxf(lane < kGemvWarps ? red_f[0][lane] : 0.0f), 1e-6f);
    } else {
      s_tok[0] = 0.0f;  // int8 tokens: the given scale, read after the barrier below
    }
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok[0]);
    int part = 0;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const uint32_t g = threadIdx.x + kGemvThreads * u;  // 16 codes: 16 g .. 16 g + 15
      if (!kB1 && g >= 4 * segs) break;  // (1-bit: every lane goes on, for the pair exchange)
      uint32_t P[4];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {  // eight codes at a time
        int q[8];
        if constexpr (XDT == BL_I8) {
          const uint4 w4 = xraw[u][0];
          const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) q[jj] = static_cast<int8_t>(wv[2 * hh + (jj >> 2)] >> (8 * (jj & 3)));
        } else {
          float e[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) e[jj] = elem(u, 8 * hh + jj);  // 0 past K: a padding word codes 0
          quant_act_fast_n<8>(e, s_tok[0], c127, q);
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) part += q[jj];
        P[2 * hh] = pack4(q);
        P[2 * hh + 1] = pack4(q + 4);
      }
      if constexpr (kB1) {
        b1_put_half_t<kPB>(xs, P, g, g < 8 * segs);
      } else {
        const uint32_t s = g >> 2, w = g & 3;
        *reinterpret_cast<uint4*>(xs + (2 * w + (s & 1)) * kI2Plane + (s >> 1) * 16) = i2_slot(P[0], P[1], P[2], P[3]);
      }
    }
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0) red_i[0][warp] = part;
    issue(bufA);  // the codes are written: now the first batch of weights
  } else {
    if constexpr (XDT != BL_I8) {
  #pragma unroll
      for (int m = 0; m < MT; ++m) {
        float amax = 0.0f;
        if ((K % 8) == 0) {
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
    __syncthreads();  // zeroed row sums and per-warp maxima are visible
  #pragma unroll
    for (int m = 0; m < MT; ++m) {
      if constexpr (XDT != BL_I8) {
        float a = red_f[m][0];
  #pragma unroll
        for (int w = 1; w < kGemvWarps; ++w) a = fmaxf(a, red_f[m][w]);
        s_tok[m] = fmaxf(a, 1e-6f);
      } else {
        s_tok[m] = 0.0f;  // int8 tokens: the given scale, read after the barrier below
      }
    }
  #pragma unroll
    for (int m = 0; m < MT; ++m) {
      int part = 0;
      uint8_t* xm = xs + m * kNP * kPB;
      const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok[m]);
      if constexpr (kB1) {
        for (uint32_t g = threadIdx.x; g < 4 * segs; g += blockDim.x) {  // one packed word's 32 codes
          const int64_t k0 = 32 * static_cast<int64_t>(g);
          int q[32];
  #pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int64_t kh = k0 + 8 * h;
            if (kh + 8 <= K && (K % 8) == 0) {
              if constexpr (XDT == BL_I8) {
                const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + kh));
  #pragma unroll
                for (int j = 0; j < 8; ++j) q[8 * h + j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
              } else {
                float e[8];
                load8_aligned<XDT>(x, m * K + kh, e);
                quant_act_fast_n<8>(e, s_tok[m], c127, q + 8 * h);
              }
            } else {
  #pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int64_t k = kh + j;
                q[8 * h + j] = k >= K ? 0
                               : (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[m * K + k])
                                                : quant_act_fast(load_x<XDT>(x, m * K + k), s_tok[m], c127);
              }
            }
          }
          uint32_t X[8];
  #pragma unroll
          for (int i = 0; i < 8; ++i) {
            int qq[4] = {q[i], q[8 + i], q[16 + i], q[24 + i]};
            X[i] = pack4(qq);
            part += qq[0] + qq[1] + qq[2] + qq[3];
          }
          const uint32_t s = g >> 2, w = g & 3;
          uint8_t* dst = xm + (4 * w + 2 * (s & 1)) * kPB + (s >> 1) * 16;
          *reinterpret_cast<uint4*>(dst) = make_uint4(X[0], X[1], X[2], X[3]);
          *reinterpret_cast<uint4*>(dst + kPB) = make_uint4(X[4], X[5], X[6], X[7]);
        }
      } else {
      for (uint32_t g = threadIdx.x; g < 4 * segs; g += blockDim.x) {  // one packed word's 16 codes
        const int64_t k0 = 16 * static_cast<int64_t>(g);
        const bool full = k0 + 16 <= K && (K % 16) == 0;
        uint32_t P[4];
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t kh = k0 + 8 * h;
          int q[8];
          if (full) {
            if constexpr (XDT == BL_I8) {
              const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + kh));
  #pragma unroll
              for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
            } else {
              float e[8];
              load8_aligned<XDT>(x, m * K + kh, e);
  quant_act_fast_n<8>(e, s_tok[m], c127, q);
            }
          } else {
  #pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int64_t k = kh + j;
              if (k < K)
                q[j] = (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[m * K + k])
                                      : quant_act_fast(load_x<XDT>(x, m * K + k), s_tok[m], c127);
              else
                q[j] = 0;
            }
          }
  #pragma unroll
          for (int j = 0; j < 8; ++j) part += q[j];
          P[2 * h] = pack4(q);
          P[2 * h + 1] = pack4(q + 4);
        }
        const uint32_t s = g >> 2, w = g & 3;
        *reinterpret_cast<uint4*>(xm + (2 * w + (s & 1)) * kI2Plane + (s >> 1) * 16) = i2_slot(P[0], P[1], P[2], P[3]);
      }
      }
      part = __reduce_add_sync(0xffffffffu, part);
      if (lane == 0) red_i[m][warp] = part;
    }
  }
  __syncthreads();  // activations and per-warp sums are visible
  const float g = sh_gs[0];
  float cfac[MT];
  int corr[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if constexpr (XDT == BL_I8) s_tok[m] = sh_gs[1 + m];
    int t = 0;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) t += red_i[m][w];
    corr[m] = t;  // digits are q + 1: subtract sum x once per row
    cfac[m] = dequant_factor(g, s_tok[m]);
    if (XDT != BL_I8 && write_scale && blockIdx.x == 0 && threadIdx.x == 0) scale[m] = s_tok[m];
  }

  // 3. per tile: one batch of loads in flight while the other is reduced
  const uint8_t* xl = xs + (s_lane >> 1) * 16;  // this lane's slot in block 0 of plane 0
  for (int64_t t0 = 0; t0 < nrows; t0 += kGemvTileRows) {
    if (t0 > 0) {
      start_tile(t0);
      issue(bufA);
    }
    const uint32_t nr = l_rows;
    uint32_t c_row = warp / nb, c_blk = warp % nb;
    auto consume = [&](const uint4(&bf)[kI2Batch][2]) {
#pragma unroll
      for (int d = 0; d < kI2Batch; ++d) {
        if (c_row >= nr) break;
        if constexpr (kB1) {
          int ab[8][MT];
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int m = 0; m < MT; ++m) ab[i][m] = 0;
          const uint8_t* xb = xl + c_blk * 512;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t wd[4] = {bf[d][h].x, bf[d][h].y, bf[d][h].z, bf[d][h].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const uint8_t* xp = xb + (m * kNP + 4 * w + 2 * h) * kPB;
                const uint4 X0 = *reinterpret_cast<const uint4*>(xp);
                const uint4 X1 = *reinterpret_cast<const uint4*>(xp + kPB);
                ab[0][m] = dp4a_us(wd[w] & 0x01010101u, X0.x, ab[0][m]);
                ab[1][m] = dp4a_us(wd[w] & 0x02020202u, X0.y, ab[1][m]);
                ab[2][m] = dp4a_us(wd[w] & 0x04040404u, X0.z, ab[2][m]);
                ab[3][m] = dp4a_us(wd[w] & 0x08080808u, X0.w, ab[3][m]);
                ab[4][m] = dp4a_us(wd[w] & 0x10101010u, X1.x, ab[4][m]);
                ab[5][m] = dp4a_us(wd[w] & 0x20202020u, X1.y, ab[5][m]);
                ab[6][m] = dp4a_us(wd[w] & 0x40404040u, X1.z, ab[6][m]);
                ab[7][m] = dp4a_us(wd[w] & 0x80808080u, X1.w, ab[7][m]);
              }
            }
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int v = ab[0][m];
#pragma unroll
            for (int i = 1; i < 8; ++i) v += ab[i][m] >> i;
            const int t = __reduce_add_sync(0xffffffffu, v);
            if (lane == 0) atomicAdd(racc + m * kGemvTileRows + c_row, t);
          }
        } else {
        int a0[MT], a1[MT], a2[MT], a3[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) a0[m] = a1[m] = a2[m] = a3[m] = 0;
        const uint8_t* xb = xl + c_blk * 512;  // block blk: slots 32 blk .. 32 blk + 31 of each plane
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t wd[4] = {bf[d][h].x, bf[d][h].y, bf[d][h].z, bf[d][h].w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t c0 = wd[w] & 0x03030303u, c1 = wd[w] & 0x0c0c0c0cu;
            const uint32_t c2 = wd[w] & 0x30303030u, c3 = wd[w] & 0xc0c0c0c0u;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const uint4 X = *reinterpret_cast<const uint4*>(xb + (m * 8 + 2 * w + h) * kI2Plane);
              a0[m] = dp4a_us(c0, X.x, a0[m]);
              a1[m] = dp4a_us(c1, X.y, a1[m]);
              a2[m] = dp4a_us(c2, X.z, a2[m]);
              a3[m] = dp4a_us(c3, X.w, a3[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int v = a0[m] + (a1[m] >> 2) + (a2[m] >> 4) + (a3[m] >> 6);
          const int t = __reduce_add_sync(0xffffffffu, v);
          if (lane == 0) atomicAdd(racc + m * kGemvTileRows + c_row, t);
        }
        }
        c_blk += dr;
        c_row += dq;
        if (c_blk >= nb) {
          c_blk -= nb;
          ++c_row;
        }
      }
    };
    const uint32_t first_row = warp / nb;
    if (first_row < nr) {
      for (;;) {
        issue(bufB);
        consume(bufA);
        if (c_row >= nr) break;
        issue(bufA);
        consume(bufB);
        if (c_row >= nr) break;
      }
    }
    __syncthreads();  // every part of every row of the tile has been added
    for (int r = threadIdx.x; r < static_cast<int>(nr); r += blockDim.x) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int a = (kB1 ? 2 : 1) * racc[m * kGemvTileRows + r] - corr[m];
        racc[m * kGemvTileRows + r] = 0;
        const int64_t o = m * N + row0 + t0 + r;
        const float cf = rg.n == 1 ? cfac[m] : dequant_factor(sh_gam[row_group(rg, row0 + t0 + r)], s_tok[m]);
        if (ydt == BL_I32)
          static_cast<int32_t*>(y)[o] = a;
        else if (ydt == BL_F32)
          static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cf);
        else
          static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cf));
      }
    }
    __syncthreads();  // the row sums are zero again for the next tile
  }
}

// ---------------------------------------------------------------------------
// 2-bit decode GEMV for 2..4 tokens, column-stationary.  As in gemv_t5_kernel,
// a row of segs 16-byte segments (64 weights each) is cut into nb columns of
// 32 segments; warp w < nb kc (kc = kMtWarps / nb) keeps column w mod nb and
// takes every kc-th row of its CTA, so lane L holds, for each of the MT tokens,
// the 64 codes of segment 32 c + L in registers (16 words, in the digit order
// of the packed words) for the whole kernel: the weights are read once and no
// token code is read from shared memory per row.  Per row and packed word:
// four digit masks (taken in place), then four dp4a per token into four
// accumulators whose factors 4^j come off exactly at the end of the row, one
// warp reduction and one shared atomic per token.  Digits are q + 1, so the
// sum of each token's codes is subtracted once per row.
// ---------------------------------------------------------------------------
constexpr int kMtThreads = 512;               // 16 warps: 16 MT + load registers per lane
constexpr int kMtWarps = kMtThreads / 32;
constexpr int kMtBatch = 2;                   // rows per load batch; two batches alternate
constexpr int64_t kMtPrefetch = 65536;        // bytes per CTA prefetched into L2 before the wait

__host__ __device__ inline int64_t gemv_mt_smem_bytes(int64_t rowbytes, int mt) {
  return int64_t{4} * rowbytes * mt + int64_t{4} * kGemvTileRows * mt;  // codes | row sums
}

template <int MT, int XDT>
__global__ void __launch_bounds__(kMtThreads, 1)
    gemv_i2_mt_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                      int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                      void* __restrict__ y, int ydt, int write_scale, const RowGroups rg) {
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));  // <= kGemvTileRows (host-checked)
  const uint32_t segs = static_cast<uint32_t>(rowbytes >> 4);
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* xs = smem;                                             // [MT][4][segs][16] codes
  int* racc = reinterpret_cast<int*>(xs + 4 * rowbytes * MT);     // [MT][kGemvTileRows]
  __shared__ float red_f[MT][kMtWarps];
  __shared__ int red_i[MT][kMtWarps];
  __shared__ float sh_gs[1 + MT];
  // 0. while the previous kernel finishes: zeroed row sums and an L2 prefetch
  pdl_launch_dependents();
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < kMtPrefetch ? bytes : kMtPrefetch);
  }
  for (int i = threadIdx.x; i < MT * kGemvTileRows; i += blockDim.x) racc[i] = 0;
  pdl_wait(packed, gamma, x, scale, y);
  if (threadIdx.x <= MT && (threadIdx.x == 0 || XDT == BL_I8))
    sh_gs[threadIdx.x] = __ldcg(threadIdx.x == 0 ? gamma : scale + (threadIdx.x - 1));
  __shared__ float sh_gam[kMaxRowGroups];  // gamma of each row group
  if (threadIdx.x < rg.n) sh_gam[threadIdx.x] = __ldcg(gamma + threadIdx.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nthr = blockDim.x;

  // 1. the tokens' INT8 codes in the general 2-bit layout (packed word w of
  //    segment s: 16 codes at (w segs + s) 16, byte 4 j + b = x[64 s + 16 w + 4 b + j])
  const bool vec = (K % 8) == 0;
  if constexpr (XDT != BL_I8) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float amax = 0.0f;
      if (vec) {
        for (int64_t v = threadIdx.x; v < K / 8; v += nthr) {
          float e[8];
          load8_aligned<XDT>(x, m * K + 8 * v, e);
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[j]));
        }
      } else {
        for (int64_t k = threadIdx.x; k < K; k += nthr) amax = fmaxf(amax, fabsf(load_x<XDT>(x, m * K + k)));
      }
      amax = warp_maxf(amax);
      if (lane == 0) red_f[m][warp] = amax;
    }
  }
  __syncthreads();  // per-warp maxima, zeroed row sums, gamma and the given scales are visible
  float s_tok[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if constexpr (XDT != BL_I8) {
      float a = red_f[m][0];
#pragma unroll
      for (int w = 1; w < kMtWarps; ++w) a = fmaxf(a, red_f[m][w]);
      s_tok[m] = fmaxf(a, 1e-6f);
    } else {
      s_tok[m] = sh_gs[1 + m];
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int part = 0;
    const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok[m]);
    uint8_t* xm = xs + 4 * rowbytes * m;
    for (uint32_t g = threadIdx.x; g < 4 * segs; g += nthr) {  // one packed word's 16 codes
      const int64_t k0 = 16 * static_cast<int64_t>(g);
      uint32_t P[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t kh = k0 + 8 * h;
        int q[8];
        if (vec && kh + 8 <= K) {
          if constexpr (XDT == BL_I8) {
            const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + m * K + kh));
#pragma unroll
            for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
          } else {
            float e[8];
            load8_aligned<XDT>(x, m * K + kh, e);
            quant_act_fast_n<8>(e, s_tok[m], c127, q);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int64_t k = kh + j;
            q[j] = (k >= K) ? 0
                   : (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[m * K + k])
                                    : quant_act_fast(load_x<XDT>(x, m * K + k), s_tok[m], c127);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) part += q[j];
        P[2 * h] = pack4(q);
        P[2 * h + 1] = pack4(q + 4);
      }
      const uint32_t s = g >> 2, w = g & 3;
      *reinterpret_cast<uint4*>(xm + (w * segs + s) * 16) = i2_slot(P[0], P[1], P[2], P[3]);
    }
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0) red_i[m][warp] = part;
  }
  __syncthreads();  // the codes and per-warp sums are visible
  int corr[MT];
  float cfac[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kMtWarps; ++w) t += red_i[m][w];
    corr[m] = t;
    cfac[m] = dequant_factor(sh_gs[0], s_tok[m]);
    if (XDT != BL_I8 && write_scale && blockIdx.x == 0 && threadIdx.x == 0) scale[m] = s_tok[m];
  }

  // 2. this lane's codes: segment s = 32 c + lane of the warp's column
  const int nb = static_cast<int>((segs + 31) >> 5);
  const int kc = kMtWarps / nb;
  const int c = warp % nb, j0 = warp / nb;
  const uint32_t s = 32u * c + lane;
  const bool active = warp < nb * kc;
  const bool mine = active && s < segs;  // lanes past the row's end load nothing and add 0
  uint4 X[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int w = 0; w < 4; ++w)
      X[m][w] = mine ? *reinterpret_cast<const uint4*>(xs + 4 * rowbytes * m + (w * segs + s) * 16)
                     : make_uint4(0, 0, 0, 0);

  // 3. the warp's rows j0, j0 + kc, ...: kMtBatch loads in flight per batch,
  //    two batches alternating
  const int nmine = (active && j0 < nrows) ? (nrows - 1 - j0) / kc + 1 : 0;
  const uint8_t* src = packed + (row0 + j0) * rowbytes + 16 * static_cast<int64_t>(s);
  const int64_t step = static_cast<int64_t>(kc) * rowbytes;
  int issued = 0, done = 0;
  uint4 bufA[kMtBatch], bufB[kMtBatch];
  auto issue = [&](uint4(&bf)[kMtBatch]) {
#pragma unroll
    for (int d = 0; d < kMtBatch; ++d) {
      bf[d] = make_uint4(0, 0, 0, 0);
      if (mine && issued + d < nmine) bf[d] = ld_stream(reinterpret_cast<const uint4*>(src + (issued + d) * step));
    }
    issued += kMtBatch;
  };
  auto consume = [&](const uint4(&bf)[kMtBatch]) {
#pragma unroll
    for (int d = 0; d < kMtBatch; ++d) {
      if (done + d >= nmine) break;  // (uniform across the warp)
      const uint32_t wd[4] = {bf[d].x, bf[d].y, bf[d].z, bf[d].w};
      int a0[MT], a1[MT], a2[MT], a3[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) a0[m] = a1[m] = a2[m] = a3[m] = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t c0 = wd[w] & 0x03030303u, c1 = wd[w] & 0x0c0c0c0cu;
        const uint32_t c2 = wd[w] & 0x30303030u, c3 = wd[w] & 0xc0c0c0c0u;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          a0[m] = dp4a_us(c0, X[m][w].x, a0[m]);
          a1[m] = dp4a_us(c1, X[m][w].y, a1[m]);
          a2[m] = dp4a_us(c2, X[m][w].z, a2[m]);
          a3[m] = dp4a_us(c3, X[m][w].w, a3[m]);
        }
      }
      const int r = j0 + (done + d) * kc;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int t = __reduce_add_sync(0xffffffffu, a0[m] + (a1[m] >> 2) + (a2[m] >> 4) + (a3[m] >> 6));
        if (lane == 0) atomicAdd(racc + m * kGemvTileRows + r, t);
      }
    }
    done += kMtBatch;
  };
  if (nmine > 0) {
    issue(bufA);
    for (;;) {
      issue(bufB);
      consume(bufA);
      if (done >= nmine) break;
      issue(bufA);
      consume(bufB);
      if (done >= nmine) break;
    }
  }
  __syncthreads();  // every part of every row has been added
  for (int r = threadIdx.x; r < nrows; r += nthr) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int a = racc[m * kGemvTileRows + r] - corr[m];
      const int64_t o = m * N + row0 + r;
      const float cf = rg.n == 1 ? cfac[m] : dequant_factor(sh_gam[row_group(rg, row0 + r)], s_tok[m]);
      if (ydt == BL_I32)
        static_cast<int32_t*>(y)[o] = a;
      else if (ydt == BL_F32)
        static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cf);
      else
        static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cf));
    }
  }
}

// ---------------------------------------------------------------------------
// Base-3 decode GEMV for one token, column-stationary.  A row of segs 16-byte
// segments (80 weights each) is cut into nb = ceil(segs / 32) columns of 32
// segments; warp w < nb kc (kc = kGemvWarps / nb) keeps column c = w mod nb
// and takes the rows j, j + kc, ... of its CTA (j = w / nb), so lane L holds
// the 80 activation codes of segment 32 c + L in registers for the whole
// kernel: xlo[p] = the codes of digits 0..3 of packed byte p of the segment,
// xhi[j] byte i = the code of digit 4 of packed byte 4 j + i.  At any time the
// CTA's warps read kc whole rows, one contiguous window.  A packed byte b is
// decoded by one 4-byte shared lookup: byte j of the entry is the digit
// d_j = floor(b / 3^j) mod 3 (j < 4) and bits 2..3 of byte 0 hold d_4.  The
// table has one copy per lane (copy L in bank L), so a warp's 32 lookups are
// one conflict-free shared access whatever the bytes.  Per packed word: four
// lookups, four dp4a on the masked entries (digits 0..3 against xlo) and one
// dp4a on the gathered d_4 (4 d_4 in each byte, against xhi; the factor 4 is
// taken off at the end).  Digits are q + 1, so sum q x = sum d x - sum x with
// the sum of the token's codes subtracted once per row.  Bytes 243..255 are
// not produced by the packer; they decode as five zero weights.
// ---------------------------------------------------------------------------
constexpr int kT5Batch = 4;                 // rows per load batch; two batches alternate
constexpr int kT5LutBytes = 256 * 32 * 4;   // 32 copies of 256 4-byte entries
constexpr int64_t kT5Prefetch = 65536;      // bytes per CTA prefetched into L2 before the wait

__host__ __device__ inline int64_t gemv_t5_smem_bytes(int64_t rowbytes) {
  return kT5LutBytes + (rowbytes / 16) * 80 + int64_t{4} * kGemvTileRows;
}

template <int XDT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_t5_kernel(const uint8_t* __restrict__ packed, int64_t rowbytes, const float* __restrict__ gamma,
                   int64_t N, int64_t K, const void* __restrict__ x, float* __restrict__ scale,
                   void* __restrict__ y, int ydt, int write_scale, const RowGroups rg) {
  const int64_t G = gridDim.x, b = blockIdx.x;
  const int64_t per = N / G, extra = N % G;
  const int64_t row0 = b * per + (b < extra ? b : extra);
  const int nrows = static_cast<int>(per + (b < extra ? 1 : 0));  // <= kGemvTileRows (host-checked)
  // 0. while the previous kernel finishes: the table, the zeroed row sums and
  //    an L2 prefetch of the first kT5Prefetch bytes of this CTA's rows
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);           // [256][32]
  int8_t* xq = reinterpret_cast<int8_t*>(smem + kT5LutBytes);   // [segs * 80] codes, 0 past K
  const uint32_t segs = static_cast<uint32_t>(rowbytes >> 4);
  int* racc = reinterpret_cast<int*>(xq + segs * 80);           // [kGemvTileRows]
  __shared__ float red_f[kGemvWarps];
  __shared__ int red_i[kGemvWarps];
  __shared__ float sh_gs[2];
  {
    const int64_t bytes = static_cast<int64_t>(nrows) * rowbytes;
    l2_prefetch_bulk(packed + row0 * rowbytes, bytes < kT5Prefetch ? bytes : kT5Prefetch);
  }
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
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
  for (int i = threadIdx.x; i < kGemvTileRows; i += blockDim.x) racc[i] = 0;
  pdl_wait(packed, gamma, x, scale, y);
  if (threadIdx.x == 0) sh_gs[0] = __ldcg(gamma);
  if (XDT == BL_I8 && threadIdx.x == 1) sh_gs[1] = __ldcg(scale);
  __shared__ float sh_gam[kMaxRowGroups];  // gamma of each row group
  if (threadIdx.x < rg.n) sh_gam[threadIdx.x] = __ldcg(gamma + threadIdx.x);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nthr = blockDim.x;

  // 1. the token's INT8 codes: per-token absmax (fp32 / bf16) or the given
  //    scale (int8); codes past K are 0
  const uint32_t nq8 = segs * 10;  // groups of eight codes in shared memory
  const bool vec = (K % 8) == 0;
  if constexpr (XDT != BL_I8) {
    float amax = 0.0f;
    if (vec) {
      for (int64_t v = threadIdx.x; v < K / 8; v += nthr) {
        float e[8];
        load8_aligned<XDT>(x, 8 * v, e);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(e[j]));
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += nthr) amax = fmaxf(amax, fabsf(load_x<XDT>(x, k)));
    }
    amax = warp_maxf(amax);
    if (lane == 0) red_f[warp] = amax;
  }
  __syncthreads();  // per-warp maxima, the table and the zeroed row sums are visible
  float s_tok;
  if constexpr (XDT != BL_I8) {
    s_tok = fmaxf(warp_maxf(lane < kGemvWarps ? red_f[lane] : 0.0f), 1e-6f);
  } else {
    s_tok = sh_gs[1];
  }
  const float c127 = (XDT == BL_I8) ? 0.0f : __fdiv_rn(127.0f, s_tok);
  int part = 0;
  for (uint32_t v = threadIdx.x; v < nq8; v += nthr) {
    const int64_t k0 = 8 * static_cast<int64_t>(v);
    int q[8];
    if (vec && k0 + 8 <= K) {
      if constexpr (XDT == BL_I8) {
        const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(static_cast<const int8_t*>(x) + k0));
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = static_cast<int8_t>((j < 4 ? raw.x : raw.y) >> (8 * (j & 3)));
      } else {
        float e[8];
        load8_aligned<XDT>(x, k0, e);
        quant_act_fast_n<8>(e, s_tok, c127, q);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t k = k0 + j;
        q[j] = (k >= K) ? 0
               : (XDT == BL_I8) ? static_cast<int>(static_cast<const int8_t*>(x)[k])
                                : quant_act_fast(load_x<XDT>(x, k), s_tok, c127);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) part += q[j];
    *reinterpret_cast<uint2*>(xq + k0) = make_uint2(pack4(q), pack4(q + 4));
  }
  part = __reduce_add_sync(0xffffffffu, part);
  if (lane == 0) red_i[warp] = part;
  __syncthreads();  // the codes, per-warp sums, gamma and the given scale are visible
  const int corr = __reduce_add_sync(0xffffffffu, lane < kGemvWarps ? red_i[lane] : 0);
  const float cfac = dequant_factor(sh_gs[0], s_tok);
  if (XDT != BL_I8 && write_scale && blockIdx.x == 0 && threadIdx.x == 0) scale[0] = s_tok;

  // 2. this lane's activations: segment s = 32 c + lane of the warp's column
  const int nb = static_cast<int>((segs + 31) >> 5);
  const int kc = kGemvWarps / nb;
  const int c = warp % nb, j0 = warp / nb;
  const uint32_t s = 32u * c + lane;
  const bool active = warp < nb * kc;
  const bool mine = active && s < segs;  // lanes past the row's end load nothing and add 0
  uint32_t xlo[16], xhi[4];
  {
    uint32_t w[20];
    if (mine) {
      const uint4* xp = reinterpret_cast<const uint4*>(xq + 80 * s);
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const uint4 t = xp[i];
        w[4 * i] = t.x;
        w[4 * i + 1] = t.y;
        w[4 * i + 2] = t.z;
        w[4 * i + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 20; ++i) w[i] = 0;
    }
#pragma unroll
    for (int p = 0; p < 16; ++p) {  // codes 5p .. 5p + 3 of the segment
      const int o = 5 * p;
      xlo[p] = __byte_perm(w[o >> 2], w[(o >> 2) + 1], 0x3210 + 0x1111 * (o & 3));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // code 5p + 4 of packed bytes p = 4j .. 4j + 3
      uint32_t h = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 20 * j + 5 * i + 4;
        h |= ((w[t >> 2] >> (8 * (t & 3))) & 0xffu) << (8 * i);
      }
      xhi[j] = h;
    }
  }

  // 3. the warp's rows j0, j0 + kc, ...: kT5Batch loads in flight per batch,
  //    two batches alternating
  const uint32_t* lut_l = lut + lane;  // this lane's copy: entry e at lut_l[32 e]
  const int nmine = (active && j0 < nrows) ? (nrows - 1 - j0) / kc + 1 : 0;
  const uint8_t* src = packed + (row0 + j0) * rowbytes + 16 * static_cast<int64_t>(s);
  const int64_t step = static_cast<int64_t>(kc) * rowbytes;
  int issued = 0, done = 0;
  uint4 bufA[kT5Batch], bufB[kT5Batch];
  auto issue = [&](uint4(&bf)[kT5Batch]) {
#pragma unroll
    for (int d = 0; d < kT5Batch; ++d) {
      bf[d] = make_uint4(0, 0, 0, 0);
      if (mine && issued + d < nmine) bf[d] = ld_stream(reinterpret_cast<const uint4*>(src + (issued + d) * step));
    }
    issued += kT5Batch;
  };
  auto consume = [&](const uint4(&bf)[kT5Batch]) {
#pragma unroll
    for (int d = 0; d < kT5Batch; ++d) {
      if (done + d >= nmine) break;  // (uniform across the warp)
      const uint32_t wd[4] = {bf[d].x, bf[d].y, bf[d].z, bf[d].w};
      int v = 0, vh = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t L[4];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) L[bb] = lut_l[32 * __byte_perm(wd[w], 0, 0x4440 + bb)];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) v = dp4a_us(L[bb] & 0x03030303u, xlo[4 * w + bb], v);
        const uint32_t H =
            __byte_perm(__byte_perm(L[0], L[1], 0x0040), __byte_perm(L[2], L[3], 0x0040), 0x5410) & 0x0c0c0c0cu;
        vh = dp4a_us(H, xhi[w], vh);
      }
      const int t = __reduce_add_sync(0xffffffffu, v + (vh >> 2));  // vh is 4 sum d_4 x: exact
      if (lane == 0) atomicAdd(racc + j0 + (done + d) * kc, t);
    }
    done += kT5Batch;
  };
  if (nmine > 0) {
    issue(bufA);
    for (;;) {
      issue(bufB);
      consume(bufA);
      if (done >= nmine) break;
      issue(bufA);
      consume(bufB);
      if (done >= nmine) break;
    }
  }
  __syncthreads();  // every part of every row has been added
  for (int r = threadIdx.x; r < nrows; r += nthr) {
    const int a = racc[r] - corr;
    const int64_t o = row0 + r;
    const float cf = rg.n == 1 ? cfac : dequant_factor(sh_gam[row_group(rg, o)], s_tok);
    if (ydt == BL_I32)
      static_cast<int32_t*>(y)[o] = a;
    else if (ydt == BL_F32)
      static_cast<float*>(y)[o] = __fmul_rn(__int2float_rn(a), cf);
    else
      static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(__fmul_rn(__int2float_rn(a), cf));
  }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
int gemv_max_tokens(int fmt, int64_t rowbytes) {
  int mt = kGemvMaxTokens;
  while (mt > 0 && gemv_smem_bytes(fmt, rowbytes, mt) > kGemvSmemBudget) --mt;
  return mt;
}

template <int FMT, int MT, int XDT>
static cudaError_t launch_gemv_t(const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                 int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                 int write_scale, const RowGroups& rg, cudaStream_t st) {
  auto kern = gemv_kernel<FMT, MT, XDT>;
  const size_t smem = static_cast<size_t>(gemv_smem_bytes(FMT, rowbytes, MT));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGemvSmemBudget));
  if (e != cudaSuccess) return e;
  const int sms = device_sms();
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t need = N;  // every CTA owns at least one row
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  { const cudaError_t le_ = launch_pdl(kern, static_cast<unsigned>(grid), kGemvThreads, smem, st, packed, rowbytes, gamma, N, K, x, scale,
                                                                 y, ydt, write_scale, rg); if (le_ != cudaSuccess) return le_; }
  return cudaGetLastError();
}

template <int FMT, int MT, int XDT>
static cudaError_t launch_gemv_i2_t(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N,
                                    int64_t K, const void* x, float* scale, void* y, int ydt, int write_scale,
                                    const RowGroups& rg, cudaStream_t st) {
  auto kern = gemv_i2_kernel<FMT, MT, XDT>;
  const size_t smem = static_cast<size_t>(gemv_i2_smem_bytes(MT));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t sms = device_sms();
  const int64_t grid = N < sms ? N : sms;  // every CTA owns at least one row
  { const cudaError_t le_ = launch_pdl(kern, static_cast<unsigned>(grid), kGemvThreads, smem, st, packed, rowbytes, gamma, N, K, x, scale, y, ydt,
                                                                 write_scale, rg); if (le_ != cudaSuccess) return le_; }
  return cudaGetLastError();
}

template <int FMT, int XDT>
static cudaError_t launch_gemv_i2_mt(int mt, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                     int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                     int write_scale, const RowGroups& rg, cudaStream_t st) {
  switch (mt) {
    case 1: return launch_gemv_i2_t<FMT, 1, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    case 2: return launch_gemv_i2_t<FMT, 2, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    case 3: return launch_gemv_i2_t<FMT, 3, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    default: return launch_gemv_i2_t<FMT, 4, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  }
}

template <int XDT>
static cudaError_t launch_gemv_lean(int fmt, int mt, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                    int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                    int write_scale, const RowGroups& rg, cudaStream_t st) {
  if (fmt == BL_PACK_B1)
    return launch_gemv_i2_mt<BL_PACK_B1, XDT>(mt, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  return launch_gemv_i2_mt<BL_PACK_I2, XDT>(mt, packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
}

// The multi-token column-stationary kernel: 2-bit rows of at most
// 32 kMtWarps segments and at most kGemvTileRows rows per CTA.
static bool gemv_mt_fits(int64_t rowbytes, int64_t N, int mt) {
  const int64_t sms = device_sms();
  const int64_t grid = N < sms ? N : sms;
  return rowbytes / 16 <= 32 * kMtWarps && (N + grid - 1) / grid <= kGemvTileRows &&
         gemv_mt_smem_bytes(rowbytes, mt) <= kGemvSmemBudget;
}

template <int MT, int XDT>
static cudaError_t launch_gemv_mt_cs(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N,
                                     int64_t K, const void* x, float* scale, void* y, int ydt, int write_scale,
                                     const RowGroups& rg, cudaStream_t st) {
  auto kern = gemv_i2_mt_kernel<MT, XDT>;
  const size_t smem = static_cast<size_t>(gemv_mt_smem_bytes(rowbytes, MT));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t sms = device_sms();
  const int64_t grid = N < sms ? N : sms;  // every CTA owns at least one row
  e = launch_pdl(kern, static_cast<unsigned>(grid), kMtThreads, smem, st, packed, rowbytes, gamma, N, K, x, scale, y,
                 ydt, write_scale, rg);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int XDT>
static cudaError_t launch_gemv_mt_cs_n(int mt, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                       int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                       int write_scale, const RowGroups& rg, cudaStream_t st) {
  switch (mt) {
    case 2: return launch_gemv_mt_cs<2, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    case 3: return launch_gemv_mt_cs<3, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    default: return launch_gemv_mt_cs<4, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  }
}

// The base-3 column-stationary kernel: rows of at most 32 kGemvWarps
// segments and at most kGemvTileRows rows per CTA.
static bool gemv_t5_fits(int64_t rowbytes, int64_t N) {
  const int64_t sms = device_sms();
  const int64_t grid = N < sms ? N : sms;
  return rowbytes / 16 <= 32 * kGemvWarps && (N + grid - 1) / grid <= kGemvTileRows &&
         gemv_t5_smem_bytes(rowbytes) <= kGemvSmemBudget;
}

template <int XDT>
static cudaError_t launch_gemv_t5_t(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N,
                                    int64_t K, const void* x, float* scale, void* y, int ydt, int write_scale,
                                    const RowGroups& rg, cudaStream_t st) {
  auto kern = gemv_t5_kernel<XDT>;
  const size_t smem = static_cast<size_t>(gemv_t5_smem_bytes(rowbytes));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t sms = device_sms();
  const int64_t grid = N < sms ? N : sms;  // every CTA owns at least one row
  e = launch_pdl(kern, static_cast<unsigned>(grid), kGemvThreads, smem, st, packed, rowbytes, gamma, N, K, x, scale,
                 y, ydt, write_scale, rg);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT, int XDT>
static cudaError_t launch_gemv_mt(int mt, const uint8_t* packed, int64_t rowbytes, const float* gamma,
                                  int64_t N, int64_t K, const void* x, float* scale, void* y, int ydt,
                                  int write_scale, const RowGroups& rg, cudaStream_t st) {
  switch (mt) {
    case 1: return launch_gemv_t<FMT, 1, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    case 2: return launch_gemv_t<FMT, 2, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    case 3: return launch_gemv_t<FMT, 3, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
    default: return launch_gemv_t<FMT, 4, XDT>(packed, rowbytes, gamma, N, K, x, scale, y, ydt, write_scale, rg, st);
  }
}

// Runs the GEMV over all M tokens in groups that fit in shared memory.
cudaError_t launch_gemv(const uint8_t* packed, int fmt, const float* gamma, int64_t N, int64_t K,
                        const void* x, int xdt, float* scale, int64_t M, void* y, int ydt,
                        const RowGroups& rg, void* ws, cudaStream_t st) {
  const int per = (fmt == BL_PACK_I2) ? 4 : (fmt == BL_PACK_T5 ? 5 : 8);
  const int64_t rowbytes = ((K + per - 1) / per + 15) / 16 * 16;
  const int mt_max = gemv_max_tokens(fmt, rowbytes);
  if (mt_max < 1) return cudaErrorInvalidValue;
  // 2-bit rows of up to 2 kI2Plane bytes and 1-bit rows of up to kI2Plane
  // bytes take the lean kernel (its shared memory, 8 x kI2Plane bytes per
  // token, fits kGemvMaxTokens tokens within the budget); longer 1-bit rows
  // are not served here (the caller transcodes them to 2 bits)
  const bool lean = (fmt == BL_PACK_I2 && rowbytes <= 2 * kI2Plane) || (fmt == BL_PACK_B1 && rowbytes <= kI2Plane);
  if (fmt == BL_PACK_B1 && !lean) return cudaErrorInvalidValue;
  if (fmt == BL_PACK_I2 && M == 1 && gemv1_fits(N, K, rowbytes, xdt))
    return launch_gemv1(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
  if (fmt == BL_PACK_T5 && M == 1 && gemv1_t5_fits(N, K, rowbytes, xdt))
    return launch_gemv1_t5(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
  if (fmt == BL_PACK_B1 && M == 1 && gemv1_b1_fits(N, K, rowbytes, xdt))
    return launch_gemv1_b1(packed, rowbytes, gamma, N, K, x, xdt, scale, y, ydt, rg, ws, st);
  const int esz = (xdt == BL_F32) ? 4 : (xdt == BL_BF16 ? 2 : 1);
  const int ysz = (ydt == BL_BF16) ? 2 : 4;
  for (int64_t m0 = 0; m0 < M; m0 += mt_max) {
    const int mt = static_cast<int>((M - m0) < mt_max ? (M - m0) : mt_max);
    const void* xm = static_cast<const uint8_t*>(x) + m0 * K * esz;
    float* sm = scale + m0;
    void* ym = static_cast<uint8_t*>(y) + m0 * N * ysz;
    cudaError_t e;
    if (fmt == BL_PACK_I2 && mt >= 2 && mt <= 4 && gemv_mt_fits(rowbytes, N, mt)) {
      if (xdt == BL_F32) e = launch_gemv_mt_cs_n<BL_F32>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else if (xdt == BL_BF16) e = launch_gemv_mt_cs_n<BL_BF16>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else e = launch_gemv_mt_cs_n<BL_I8>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, rg, st);
    } else if (fmt == BL_PACK_T5 && mt == 1 && M == 1 && gemv_t5_fits(rowbytes, N)) {
      if (xdt == BL_F32) e = launch_gemv_t5_t<BL_F32>(packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else if (xdt == BL_BF16) e = launch_gemv_t5_t<BL_BF16>(packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else e = launch_gemv_t5_t<BL_I8>(packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, rg, st);
    } else if (lean) {
      if (xdt == BL_F32) e = launch_gemv_lean<BL_F32>(fmt, mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else if (xdt == BL_BF16) e = launch_gemv_lean<BL_BF16>(fmt, mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else e = launch_gemv_lean<BL_I8>(fmt, mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, rg, st);
    } else if (fmt == BL_PACK_I2) {
      if (xdt == BL_F32) e = launch_gemv_mt<BL_PACK_I2, BL_F32>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else if (xdt == BL_BF16) e = launch_gemv_mt<BL_PACK_I2, BL_BF16>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else e = launch_gemv_mt<BL_PACK_I2, BL_I8>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, rg, st);
    } else {
      if (xdt == BL_F32) e = launch_gemv_mt<BL_PACK_T5, BL_F32>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else if (xdt == BL_BF16) e = launch_gemv_mt<BL_PACK_T5, BL_BF16>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 1, rg, st);
      else e = launch_gemv_mt<BL_PACK_T5, BL_I8>(mt, packed, rowbytes, gamma, N, K, xm, sm, ym, ydt, 0, rg, st);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bl
