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
// absmean: one CTA per 8192-element chunk.  Lane l adds in fp64 the elements
// 8192c + 2048i + 8l + j (i = 0..3, j = 0..7) in that order, then the 256 lane
// sums meet in the stride-halving tree p[l] += p[l + s], s = 128..1.  Loads are
// 32 bytes per lane per i (fp32) or 16 bytes (bf16), fully coalesced.
//
// The CTA that finishes last (an atomic ticket in the workspace header) then
// combines the C chunk sums, zero-padded to P = 2^ceil(log2 C), by the
// stride-halving tree s = P/2..1, and writes gamma = fp32(S / T):
//   - the levels s >= 256 act on each residue class mod 256 on its own, as a
//     stride-halving tree over k of q[t + 256k]; that tree equals the pairwise
//     (contiguous) tree over the bit-reversed sequence, which thread t folds
//     with a binary-counter stack (fp64 addition is commutative, so operand
//     order inside a pair does not matter);
//   - the last 8 levels run in shared memory and warp shuffles.
// ---------------------------------------------------------------------------
template <int WDT>
__global__ void __launch_bounds__(kLanes) absmean_kernel(const void* __restrict__ W, int64_t T,
                                                         int64_t C, int lgR, double* __restrict__ partials,
                                                         WsHeader* __restrict__ hdr,
                                                         float* __restrict__ gamma) {
  const int64_t c = blockIdx.x;
  const int l = threadIdx.x;
  float v[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t e0 = c * kChunk + 2048 * i + 8 * l;
    if (e0 + 8 <= T) {
      load8_aligned<WDT>(W, e0, v[i]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[i][j] = (e0 + j < T) ? load_elem<WDT>(W, e0 + j) : 0.0f;
    }
  }
  double acc = 0.0;  // adding +0.0 for elements past T leaves the sum unchanged
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc = __dadd_rn(acc, static_cast<double>(fabsf(v[i][j])));

  __shared__ double p[kLanes];
  __shared__ bool last;
  p[l] = acc;
  __syncthreads();
#pragma unroll
  for (int s = kLanes / 2; s >= 32; s >>= 1) {
    if (l < s) p[l] = __dadd_rn(p[l], p[l + s]);
    __syncthreads();
  }
  if (l < 32) {
    double t = p[l];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, s));
    if (l == 0) {
      partials[c] = t;
      __threadfence();
      const unsigned ticket = atomicAdd(&hdr->ticket, 1u);
      last = (ticket == static_cast<unsigned>(C - 1));
    }
  }
  __syncthreads();
  if (!last) return;

  // ---- finish: this CTA is the last one; every partial is visible ----
  __threadfence();
  const int64_t R = int64_t{1} << lgR;  // P / 256, or 1 when P <= 256
  double st[kFinishMaxLevels + 1];
  for (int64_t i0 = 0; i0 < R; i0 += 8) {
    double vals[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // eight independent loads in flight
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
      int64_t j = i;
      int lvl = 0;
      while (j & 1) {
        val = __dadd_rn(st[lvl], val);
        j >>= 1;
        ++lvl;
      }
      st[lvl] = val;
    }
  }
  p[l] = st[lgR];
  __syncthreads();
#pragma unroll
  for (int s = kLanes / 2; s >= 32; s >>= 1) {
    if (l < s) p[l] = __dadd_rn(p[l], p[l + s]);
    __syncthreads();
  }
  if (l < 32) {
    double t = p[l];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) t = __dadd_rn(t, __shfl_down_sync(0xffffffffu, t, s));
    if (l == 0) {
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

__device__ __forceinline__ int ternary_code(float w, float thr) {
  return fabsf(w) > thr ? (w > 0.0f ? 1 : -1) : 0;
}

// One thread writes one 16-byte segment of a packed row: 64 weights (2-bit)
// or 80 weights (base 3).  Weights past K are weight 0 (padding digits).
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
  for (int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; gid < total;
       gid += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = gid / segs;
    const int64_t sg = gid - n * segs;
    const int64_t k0 = sg * WPS;
    const int64_t base = n * K + k0;
    int8_t q[WPS];
    if (vec_ok && k0 + WPS <= K) {
#pragma unroll
      for (int g = 0; g < WPS / 8; ++g) {
        float v[8];
        load8_aligned<WDT>(W, base + 8 * g, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) q[8 * g + j] = static_cast<int8_t>(ternary_code(v[j], thr));
      }
    } else {
#pragma unroll
      for (int i = 0; i < WPS; ++i)
        q[i] = (k0 + i < K) ? static_cast<int8_t>(ternary_code(load_elem<WDT>(W, base + i), thr))
                            : static_cast<int8_t>(0);
    }
    uint32_t out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        uint32_t byte = 0;
        if constexpr (FMT == BL_PACK_I2) {
#pragma unroll
          for (int i = 0; i < 4; ++i) byte |= static_cast<uint32_t>(q[16 * w + 4 * b + i] + 1) << (2 * i);
        } else {
#pragma unroll
          for (int i = 4; i >= 0; --i) byte = byte * 3u + static_cast<uint32_t>(q[20 * w + 5 * b + i] + 1);
        }
        word |= byte << (8 * b);
      }
      out[w] = word;
    }
    if (packed != nullptr)
      *reinterpret_cast<uint4*>(packed + n * rowbytes + sg * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    if (codes != nullptr) {
      int8_t* dst = codes + base;
      if (vec_ok && k0 + WPS <= K && (K % 16) == 0) {
#pragma unroll
        for (int g = 0; g < WPS / 16; ++g) {
          uint32_t u[4];
#pragma unroll
          for (int w = 0; w < 4; ++w)
            u[w] = (static_cast<uint32_t>(static_cast<uint8_t>(q[16 * g + 4 * w]))) |
                   (static_cast<uint32_t>(static_cast<uint8_t>(q[16 * g + 4 * w + 1])) << 8) |
                   (static_cast<uint32_t>(static_cast<uint8_t>(q[16 * g + 4 * w + 2])) << 16) |
                   (static_cast<uint32_t>(static_cast<uint8_t>(q[16 * g + 4 * w + 3])) << 24);
          *reinterpret_cast<uint4*>(dst + 16 * g) = make_uint4(u[0], u[1], u[2], u[3]);
        }
      } else {
        for (int i = 0; i < WPS && k0 + i < K; ++i) dst[i] = q[i];
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
  if (wdt == BL_F32)
    absmean_kernel<BL_F32><<<static_cast<unsigned>(C), kLanes, 0, st>>>(W, T, C, lgR, partials, hdr, gamma);
  else
    absmean_kernel<BL_BF16><<<static_cast<unsigned>(C), kLanes, 0, st>>>(W, T, C, lgR, partials, hdr, gamma);
  return cudaGetLastError();
}

cudaError_t launch_ternarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* gamma,
                                  float eps, int fmt, uint8_t* packed, int8_t* codes, int64_t rowbytes,
                                  cudaStream_t st) {
  const bool vec_ok = (wdt == BL_F32) ? (K % 4 == 0) : (K % 8 == 0);
  const int64_t work = N * (rowbytes / 16);
  const int threads = 256;
  const int grid = grid_for(work, threads, 8);
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
