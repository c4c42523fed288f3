// bl_weights.cu -- weight preparation: absmean scale, ternarization, packing.
//
// Steps 1-3 of the BitNet b1.58 BitLinear ("BitNet b1.58深度解析：三值权重如何
// 重塑大模型推理" §3.1 absmean; "QAT and BitNet: A Deep Dive into 1-bit and
// 1.58-bit Quantization-Aware Training", "The Ternary Weight Recipe" and "Why Is
// It Called 1.58 Bits?").  All three kernels are HBM-bound streams over W.
#include <atomic>

#include "bl_common.cuh"
#include "bl_kernels.h"
#include "bl_sm100.cuh"

namespace bl {

// ---------------------------------------------------------------------------
// absmean.  The fixed order: in chunk c (elements [8192c, 8192c + 8192)),
// "lane" l = 0..255 adds, in fp64 and in this order, the elements
// 8192c + 2048i + 8l + j for i = 0..3, j = 0..7; the 256 lane sums meet in the
// stride-halving tree p[l] += p[l + s], s = 128..1.
//
// One warp computes one chunk: lane L holds the eight lanes l = L + 32v
// (v = 0..7) in registers, so the tree levels s = 128, 64, 32 pair registers
// of the same thread (v with v + 4, v + 2, v + 1) and only s = 16..1 cross
// lanes (shuffles).  For fixed (i, v) the warp reads 256 consecutive elements
// (1 KB of fp32), each lane 32 contiguous bytes.  Warps stride over the chunks
// (persistent grid), so no CTA waits on another within a chunk.
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

template <int WDT>
__device__ __forceinline__ double chunk_sum_warp(const void* __restrict__ W, int64_t T, int64_t c, int L) {
  double p[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) p[v] = 0.0;
  const int64_t c0 = c * kChunk;
  const bool full = c0 + kChunk <= T;
#pragma unroll
  for (int h = 0; h < 8; ++h) {  // (i, half) = (h / 2, h % 2): lanes v = 4 (h % 2) .. + 3
    const int i = h >> 1, v0 = 4 * (h & 1);
    float x[4][8];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t e0 = c0 + 2048 * i + 256 * (v0 + v) + 8 * L;
      if (full) {
        load8_aligned<WDT>(W, e0, x[v]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[v][j] = (e0 + j < T) ? load_elem<WDT>(W, e0 + j) : 0.0f;
      }
    }
#pragma unroll
    for (int v = 0; v < 4; ++v)
#pragma unroll
      for (int j = 0; j < 8; ++j) p[v0 + v] = __dadd_rn(p[v0 + v], static_cast<double>(fabsf(x[v][j])));
  }
  // lane levels 128, 64, 32: registers of this thread
#pragma unroll
  for (int v = 0; v < 4; ++v) p[v] = __dadd_rn(p[v], p[v + 4]);
  p[0] = __dadd_rn(p[0], p[2]);
  p[1] = __dadd_rn(p[1], p[3]);
  double t = __dadd_rn(p[0], p[1]);
  // lane levels 16..1: across the warp
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, s));
  return t;
}

// The same fixed-order chunk sum, reading a chunk staged in shared memory.
template <int WDT>
__device__ __forceinline__ double chunk_sum_smem(const uint8_t* stage, int L) {
  constexpr int ES = (WDT == BL_F32) ? 4 : 2;
  double p[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) p[v] = 0.0;
#pragma unroll
  for (int hv = 0; hv < 2; ++hv)
#pragma unroll 1
  for (int i = 0; i < 4; ++i) {
    const int v0 = 4 * hv;
    float x[4][8];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint8_t* src = stage + (2048 * i + 256 * (v0 + v) + 8 * L) * ES;
      if constexpr (WDT == BL_F32) {
        const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 16);
        x[v][0] = a.x; x[v][1] = a.y; x[v][2] = a.z; x[v][3] = a.w;
        x[v][4] = b.x; x[v][5] = b.y; x[v][6] = b.z; x[v][7] = b.w;
      } else {
        const uint4 a = *reinterpret_cast<const uint4*>(src);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[v][2 * k] = __uint_as_float(w[k] << 16);
          x[v][2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
      }
    }
#pragma unroll
    for (int v = 0; v < 4; ++v)
#pragma unroll
      for (int j = 0; j < 8; ++j) p[v0 + v] = __dadd_rn(p[v0 + v], static_cast<double>(fabsf(x[v][j])));
  }
#pragma unroll
  for (int v = 0; v < 4; ++v) p[v] = __dadd_rn(p[v], p[v + 4]);
  p[0] = __dadd_rn(p[0], p[2]);
  p[1] = __dadd_rn(p[1], p[3]);
  double t = __dadd_rn(p[0], p[1]);
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, s));
  return t;
}

// Part of the fixed-order chunk sum done by one of four warps: lanes
// l = L + 32 v for v in {sub, sub + 4}, summed in order and combined at tree
// level 128 (v with v + 4), giving p'[sub].
template <int WDT>
__device__ __forceinline__ double chunk_part_smem(const uint8_t* stage, int L, int sub) {
  constexpr int ES = (WDT == BL_F32) ? 4 : 2;
  double p[2] = {0.0, 0.0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int v = sub + 4 * h;
#pragma unroll 2
    for (int i = 0; i < 4; ++i) {
      float x[8];
      const uint8_t* src = stage + (2048 * i + 256 * v + 8 * L) * ES;
      if constexpr (WDT == BL_F32) {
        const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 16);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      } else {
        const uint4 a = *reinterpret_cast<const uint4*>(src);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[2 * k] = __uint_as_float(w[k] << 16);
          x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) p[h] = __dadd_rn(p[h], static_cast<double>(fabsf(x[j])));
    }
  }
  return __dadd_rn(p[0], p[1]);  // level 128
}

// Bulk-staged absmean: one persistent CTA per SM.  A producer thread keeps
// kBulkStages whole chunks in flight with cp.async.bulk (global -> shared);
// consumer warp w owns stage w: it reduces the chunks j = w, w + S, w + 2S, ...
// of its CTA's list from shared memory, in order, and releases the stage.
// (Every waiter of a stage barrier is then at most one phase ahead of it, which
// a parity wait needs: a waiter two phases ahead would see the phase before
// last, of the same parity, and go on early.)  A partial last chunk is read
// directly from global memory.  All waits are bounded; on expiry the timeout
// flag is set and gamma is not meaningful.
constexpr int kBulkStages = 6;
constexpr int kAbsWarpsPerStage = 4;
constexpr int kBulkConsumers = kBulkStages * kAbsWarpsPerStage;
constexpr int kBulkThreads = 32 * (kBulkConsumers + 1);
constexpr long long kBulkWaitCycles = 1ll << 32;
constexpr int kTernConsumers = kBulkStages;  // one consumer warp per stage, as above
constexpr int kTernThreads = 32 * (kTernConsumers + 1);

template <int WDT>
__global__ void __launch_bounds__(kBulkThreads, 1)
    absmean_bulk_kernel(const void* __restrict__ W, int64_t T, int64_t C, int64_t Cfull, int lgR,
                        double* __restrict__ partials, WsHeader* __restrict__ hdr, float* __restrict__ gamma) {
  constexpr uint32_t CB = kChunk * ((WDT == BL_F32) ? 4 : 2);  // bytes per chunk
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBulkStages * CB);
  uint64_t* empty = full + kBulkStages;
  __shared__ int abort_flag;
  __shared__ double p[kLanes];
  __shared__ double xchg[kBulkStages][kAbsWarpsPerStage][32];
  __shared__ bool last;
  const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
  const int64_t G = gridDim.x, b = blockIdx.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  if (warp == kBulkConsumers) {
    if (L == 0) {  // producer
      for (int64_t j = 0; b + j * G < Cfull; ++j) {
        const int s = static_cast<int>(j % kBulkStages);
        const uint32_t ph = static_cast<uint32_t>((j / kBulkStages) & 1);
        if (!wait1(empty + s, ph ^ 1, kBulkWaitCycles, abort_v)) {
          set_flag(hdr, kFlagTimeout, 0x601);
          *abort_v = 1;
          break;
        }
        mbar_expect_tx(full + s, CB);
        bulk_load(smem + s * CB, static_cast<const uint8_t*>(W) + (b + j * G) * CB, CB, full + s);
      }
    }
  } else {
    // consumer group s (warps 4s .. 4s + 3) owns stage s
    const int s = warp / kAbsWarpsPerStage, sub = warp % kAbsWarpsPerStage;
    for (int64_t j = s; b + j * G < Cfull; j += kBulkStages) {
      const uint32_t ph = static_cast<uint32_t>((j / kBulkStages) & 1);
      const bool okw = wait_warp(full + s, ph, kBulkWaitCycles, abort_v);
      if (!okw && L == 0) {
        set_flag(hdr, kFlagTimeout, 0x602);
        *abort_v = 1;
      }
      const double part = okw ? chunk_part_smem<WDT>(smem + s * CB, L, sub) : 0.0;
      xchg[s][sub][L] = part;
      // the four warps of the group meet here and agree whether to go on
      uint32_t ok_all;
      asm volatile(
          "{\n\t.reg .pred pi, po;\n\t"
          "setp.ne.u32 pi, %1, 0;\n\t"
          "bar.red.and.pred po, %2, %3, pi;\n\t"
          "selp.u32 %0, 1, 0, po;\n\t}"
          : "=r"(ok_all)
          : "r"(okw ? 1u : 0u), "r"(1 + s), "n"(32 * kAbsWarpsPerStage)
          : "memory");
      const bool ok = ok_all != 0;
      if (sub == 0) {
        double q0 = xchg[s][0][L], q1 = xchg[s][1][L];
        const double q2 = xchg[s][2][L], q3 = xchg[s][3][L];
        q0 = __dadd_rn(q0, q2);  // level 64
        q1 = __dadd_rn(q1, q3);
        double t = __dadd_rn(q0, q1);  // level 32
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, o));
        if (L == 0) {
          if (ok) partials[b + j * G] = t;
          mbar_arrive(empty + s);  // the whole group has read the stage and the exchange slots
        }
      }
      if (!ok) break;
    }
    if (warp == 0 && Cfull < C && (C - 1) % G == b) {  // the partial last chunk
      const double t = chunk_sum_warp<WDT>(W, T, C - 1, L);
      if (L == 0) partials[C - 1] = t;
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

  // ---- finish: this CTA is the last one; every partial is visible ----
  // (the 256 residue classes are strided over the CTA's threads, whatever
  // their number)
  __threadfence();
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
  constexpr int PER = (FMT == BL_PACK_I2) ? 4 : 5;
  constexpr int WPS = 16 * PER;  // weights per segment
  const float thr = ternary_threshold(__ldg(gamma), eps);
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
// 4p .. 4p + 3 of W in row-major order: each 8192-weight span of W becomes
// 2048 consecutive packed bytes.  One persistent CTA per SM: a producer keeps
// kBulkStages spans in flight with cp.async.bulk, walking the spans from the
// end of W backwards (the absmean kernel streamed W front to back, so the
// last spans it read are the likeliest to still be in L2); consumer warp w owns
// stage w (as in the absmean kernel) and turns each staged span into packed
// bytes (lane L takes weights 4(32a + L)..+3,
// so the 16-byte shared loads of a warp are contiguous), collects them in its
// own shared buffer and writes them with one bulk store.  A partial last span
// is read directly from global memory.
template <int WDT>
__global__ void __launch_bounds__(kTernThreads, 1)
    ternarize_flat_kernel(const void* __restrict__ W, int64_t T, int64_t Sfull, const float* __restrict__ gamma,
                          float eps, uint8_t* __restrict__ packed, int8_t* __restrict__ codes,
                          WsHeader* __restrict__ hdr) {
  constexpr int ES = (WDT == BL_F32) ? 4 : 2;
  constexpr uint32_t CB = kChunk * ES;       // bytes of W per span
  constexpr uint32_t OB = kChunk / 4;        // packed bytes per span
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* outb = smem + kBulkStages * CB;   // [kTernConsumers][OB]
  uint64_t* full = reinterpret_cast<uint64_t*>(outb + kTernConsumers * OB);
  uint64_t* empty = full + kBulkStages;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
  const int64_t G = gridDim.x, b = blockIdx.x;
  const float thr = ternary_threshold(__ldg(gamma), eps);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  if (warp == kTernConsumers) {
    if (L == 0) {  // producer: spans Sfull - 1 - b - jG, j = 0, 1, ...
      for (int64_t j = 0; b + j * G < Sfull; ++j) {
        const int s = static_cast<int>(j % kBulkStages);
        const uint32_t ph = static_cast<uint32_t>((j / kBulkStages) & 1);
        if (!wait1(empty + s, ph ^ 1, kBulkWaitCycles, abort_v)) {
          set_flag(hdr, kFlagTimeout, 0x611);
          *abort_v = 1;
          break;
        }
        const int64_t span = Sfull - 1 - (b + j * G);
        mbar_expect_tx(full + s, CB);
        bulk_load(smem + s * CB, static_cast<const uint8_t*>(W) + span * CB, CB, full + s);
      }
    }
  } else {
    uint8_t* ob = outb + warp * OB;
    for (int64_t j = warp; b + j * G < Sfull; j += kTernConsumers) {
      const int s = static_cast<int>(j % kBulkStages);
      const uint32_t ph = static_cast<uint32_t>((j / kBulkStages) & 1);
      if (!wait_warp(full + s, ph, kBulkWaitCycles, abort_v)) {
        if (L == 0) {
          set_flag(hdr, kFlagTimeout, 0x612);
          *abort_v = 1;
        }
        break;
      }
      const int64_t span = Sfull - 1 - (b + j * G);
      if (j >= kTernConsumers) {  // this warp's previous bulk store has read its buffer
        if (L == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      const uint8_t* st = smem + s * CB;
#pragma unroll 4
      for (int a = 0; a < static_cast<int>(OB / 32); ++a) {
        const int p = 32 * a + L;  // packed byte of the span
        float v[4];
        if constexpr (WDT == BL_F32) {
          const float4 f = *reinterpret_cast<const float4*>(st + 16 * p);
          v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
        } else {
          const uint2 u = *reinterpret_cast<const uint2*>(st + 8 * p);
          v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
          v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
        }
        uint32_t byte = 0, cw = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t d = ternary_digit(v[i], thr);
          byte |= d << (2 * i);
          cw |= ((d - 1u) & 0xffu) << (8 * i);
        }
        ob[p] = static_cast<uint8_t>(byte);
        if (codes != nullptr) reinterpret_cast<uint32_t*>(codes + span * kChunk)[p] = cw;
      }
      __syncwarp();
      if (L == 0) mbar_arrive(empty + s);  // the stage has been read
      fence_proxy_async_smem();            // this lane's bytes are visible to the bulk store
      __syncwarp();
      if (L == 0) {
        bulk_store(packed + span * OB, ob, OB);
        bulk_commit();
      }
    }
    if (L == 0) bulk_wait<0>();
    if (warp == 0 && b == 0 && Sfull * kChunk < T) {  // the partial last span
      const int64_t e0 = Sfull * kChunk, nbytes = (T - e0) / 4;
      for (int64_t p = L; p < nbytes; p += 32) {
        uint32_t byte = 0, cw = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t d = ternary_digit(load_elem<WDT>(W, e0 + 4 * p + i), thr);
          byte |= d << (2 * i);
          cw |= ((d - 1u) & 0xffu) << (8 * i);
        }
        packed[e0 / 4 + p] = static_cast<uint8_t>(byte);
        if (codes != nullptr) *reinterpret_cast<uint32_t*>(codes + e0 + 4 * p) = cw;
      }
    }
  }
}

// Pack int8 codes (same segment mapping).  A code outside {-1, 0, 1} packs as
// weight 0 and raises the bad-code flag.
template <int FMT>
__global__ void __launch_bounds__(256)
    pack_kernel(const int8_t* __restrict__ codes, int64_t N, int64_t K, uint8_t* __restrict__ packed,
                int64_t rowbytes, void* ws) {
  constexpr int PER = (FMT == BL_PACK_I2) ? 4 : 5;
  constexpr int WPS = 16 * PER;
  const int64_t segs = rowbytes / 16;
  const int64_t total = N * segs;
  for (int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; gid < total;
       gid += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = gid / segs;
    const int64_t sg = gid - n * segs;
    const int64_t k0 = sg * WPS;
    const int8_t* src = codes + n * K + k0;
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
          const int i = (FMT == BL_PACK_I2) ? ii : PER - 1 - ii;
          const int kk = (FMT == BL_PACK_I2) ? 16 * w + 4 * b + i : 20 * w + 5 * b + i;
          int c = (k0 + kk < K) ? static_cast<int>(__ldg(src + kk)) : 0;
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
                           cudaStream_t st) {
  const int64_t T = N * K;
  const int64_t C = (T + kChunk - 1) / kChunk;
  int lgP = 0;
  while ((int64_t{1} << lgP) < C) ++lgP;
  const int lgR = lgP > 8 ? lgP - 8 : 0;  // 256 = kLanes slots in the final tree
  if (lgR > kFinishMaxLevels) return cudaErrorInvalidValue;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  double* partials = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES);
  // bulk-staged path: one CTA per SM (at most one per chunk)
  {
    const int64_t Cfull = T / kChunk;
    const int64_t grid = C < device_sms() ? C : device_sms();
    const uint32_t cb = kChunk * (wdt == BL_F32 ? 4 : 2);
    const size_t smem = static_cast<size_t>(kBulkStages) * cb + 16 * kBulkStages;
    cudaError_t e;
    if (wdt == BL_F32) {
      e = cudaFuncSetAttribute(absmean_bulk_kernel<BL_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      absmean_bulk_kernel<BL_F32><<<static_cast<unsigned>(grid), kBulkThreads, smem, st>>>(W, T, C, Cfull, lgR,
                                                                                        partials, hdr, gamma);
    } else {
      e = cudaFuncSetAttribute(absmean_bulk_kernel<BL_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      absmean_bulk_kernel<BL_BF16><<<static_cast<unsigned>(grid), kBulkThreads, smem, st>>>(W, T, C, Cfull, lgR,
                                                                                         partials, hdr, gamma);
    }
    return cudaGetLastError();
  }
}

cudaError_t launch_ternarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* gamma,
                                  float eps, int fmt, uint8_t* packed, int8_t* codes, int64_t rowbytes, void* ws,
                                  cudaStream_t st) {
  if (fmt == BL_PACK_I2 && (K % 64) == 0 && packed != nullptr) {
    const int64_t T = N * K;
    const int64_t Sfull = T / kChunk;
    const int64_t grid = Sfull < 1 ? 1 : (Sfull < device_sms() ? Sfull : device_sms());
    const uint32_t cb = kChunk * (wdt == BL_F32 ? 4 : 2);
    const size_t smem = static_cast<size_t>(kBulkStages) * cb + kTernConsumers * (kChunk / 4) + 16 * kBulkStages;
    cudaError_t e;
    if (wdt == BL_F32) {
      e = cudaFuncSetAttribute(ternarize_flat_kernel<BL_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      ternarize_flat_kernel<BL_F32><<<static_cast<unsigned>(grid), kTernThreads, smem, st>>>(
          W, T, Sfull, gamma, eps, packed, codes, static_cast<WsHeader*>(ws));
    } else {
      e = cudaFuncSetAttribute(ternarize_flat_kernel<BL_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      ternarize_flat_kernel<BL_BF16><<<static_cast<unsigned>(grid), kTernThreads, smem, st>>>(
          W, T, Sfull, gamma, eps, packed, codes, static_cast<WsHeader*>(ws));
    }
    return cudaGetLastError();
  }
  const bool vec_ok = (wdt == BL_F32) ? (K % 4 == 0) : (K % 8 == 0);
  const int64_t work = N * (rowbytes / 16);
  const int threads = 256;
  const int grid = grid_for(work, threads, 4);
#define BL_TP(WDT, FMT)                                                                            \
  ternarize_pack_kernel<WDT, FMT><<<grid, threads, 0, st>>>(W, N, K, gamma, eps, packed, codes, \
                                                            rowbytes, vec_ok)
  if (wdt == BL_F32 && fmt == BL_PACK_I2) BL_TP(BL_F32, BL_PACK_I2);
  else if (wdt == BL_F32) BL_TP(BL_F32, BL_PACK_T5);
  else if (fmt == BL_PACK_I2) BL_TP(BL_BF16, BL_PACK_I2);
  else BL_TP(BL_BF16, BL_PACK_T5);
#undef BL_TP
  return cudaGetLastError();
}

cudaError_t launch_pack(const int8_t* codes, int64_t N, int64_t K, int fmt, uint8_t* packed,
                        int64_t rowbytes, void* ws, cudaStream_t st) {
  const int64_t work = N * (rowbytes / 16);
  const int grid = grid_for(work, 256, 8);
  if (fmt == BL_PACK_I2)
    pack_kernel<BL_PACK_I2><<<grid, 256, 0, st>>>(codes, N, K, packed, rowbytes, ws);
  else
    pack_kernel<BL_PACK_T5><<<grid, 256, 0, st>>>(codes, N, K, packed, rowbytes, ws);
  return cudaGetLastError();
}

}  // namespace bl
