// bl_gemm_sm100.cu -- prefill GEMM on the 5th-generation tensor cores.
//
// acc[t, n] = sum_k W_q[n, k] x_q[t, k] with INT32 accumulation, then the
// dequantization y = acc * gamma * s_t / 127 in the epilogue ("BitNet b1.58深度
// 解析：三值权重如何重塑大模型推理" §4.2, §3.3, §5.3).  For many tokens the
// product is a dense contraction, so it runs as int8 x int8 -> s32 MMAs:
//
//   - the MMA's M dimension is 128 weight rows and its N dimension is BT
//     tokens (16..256), so one tile expands each packed weight once and reuses
//     it for BT tokens;
//   - per pipeline stage a TMA load brings the x_q tile [BT x 128 B] in the
//     128-byte-swizzled K-major layout the MMA reads, and a second one the
//     packed 2-bit tile [128 rows x 32 B];
//   - four expansion warps turn 2-bit digits into signed int8 weights with a
//     byte-permute lookup and write them in the same swizzled layout;
//   - one thread issues tcgen05.mma.kind::i8 (K = 32 each) into an INT32
//     accumulator in tensor memory, double-buffered across tiles;
//   - four epilogue warps read the accumulator with tcgen05.ld, dequantize
//     and store, overlapping the next tile's main loop.
// The kernels are persistent (one CTA or CTA pair per SM, work strided by the
// grid).  For 5..128 tokens the one-SM kernel keeps a deep ring of TMA stages
// apart from the ring of expanded tiles, and splits each tile's K range when
// there are too few tiles for the SMs (INT32 partial sums, added by a small
// reduction kernel).  Every wait is bounded: on expiry the kernel sets the
// workspace timeout flag, drains what it issued, frees its tensor memory and
// returns.
#include <cuda.h>
#include <cstring>

#include "bl_common.cuh"
#include "bl_kernels.h"
#include "bl_sm100.cuh"

namespace bl {
namespace {

constexpr int kGemmThreads = 384;  // warp 0 TMA, 1 MMA, 4-7 expansion, 8-11 epilogue
constexpr int kBN = 128;  // weight rows per tile = MMA M
constexpr int kBK = 128;  // K per stage = 4 MMAs of K = 32
constexpr uint32_t kPackedStage = kBN * kBK / 4;  // 4096 bytes
constexpr uint32_t kExpStage = kBN * kBK;         // 16384 bytes
constexpr long long kTimeoutCycles = 1ll << 32;   // ~2 s at 1.9 GHz

// ---- tcgen05 ----------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the layout a 128-byte-swizzled TMA load writes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3fffu);  // start address
  d |= static_cast<uint64_t>(1) << 16;                 // leading offset (unused when swizzled K-major)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride offset between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                 // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                 // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::i8: s32 accumulator, signed A and B, both
// K-major, MMA shape M x N.
__host__ __device__ constexpr uint32_t i8_idesc(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

template <int NCOL>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[NCOL]);

template <>
__device__ __forceinline__ void tmem_load<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <>
__device__ __forceinline__ void tmem_load<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 two-bit digits (q + 1) -> 16 signed int8 weights q, in K order.  The
// digits are spread into nibbles, which select bytes of 0x000100FF
// (digit 0 -> 0xFF = -1, 1 -> 0, 2 -> +1, 3 -> 0).
__device__ __forceinline__ uint32_t spread8(uint32_t h) {  // 8 digits in bits 0..15 -> 8 nibbles
  uint32_t x = h & 0xffffu;
  x = (x | (x << 8)) & 0x00ff00ffu;
  x = (x | (x << 4)) & 0x0f0f0f0fu;
  x = (x | (x << 2)) & 0x33333333u;
  return x;
}
__device__ __forceinline__ uint4 expand16(uint32_t w) {
  const uint32_t lo = spread8(w), hi = spread8(w >> 16);
  uint4 o;
  o.x = __byte_perm(0x000100ffu, 0u, lo & 0xffffu);
  o.y = __byte_perm(0x000100ffu, 0u, lo >> 16);
  o.z = __byte_perm(0x000100ffu, 0u, hi & 0xffffu);
  o.w = __byte_perm(0x000100ffu, 0u, hi >> 16);
  return o;
}

// One-SM tiles (5..128 tokens).  A work unit is a tile of 128 weight rows x BT
// tokens over a range of k-blocks (128 K each): with ks > 1 the k-blocks of a
// tile are cut into ks parts (units = tiles x ks, so that a small layer still
// spreads over every SM), each unit writes its INT32 partial sums to
// part[kz][t][n] and splitk_reduce_kernel adds the parts and dequantizes.
// Three rings decouple the streams:
//   - packed tiles of 128 rows x 128 B (four k-blocks: one full 128-byte line
//     per row and TMA request; 128-byte swizzled, so that the expansion's
//     16-byte reads of eight rows hit eight different bank groups), kSP
//     stages, released by the expansion warps;
//   - x_q tiles [BT x 128 B] per k-block, kSX stages, released by the MMAs;
//   - expanded int8 tiles per k-block, kSB stages, released by the MMAs.
// The expansion warps take whole k-blocks in turn (warp v the k-blocks with
// index v mod kExp): one warp's pass over a k-block is a chain of long
// latencies (barrier test, shared loads, stores, proxy fence, arrive), and
// with the k-blocks dealt out several of them are in flight at once (rows
// dealt out instead left one k-block per ~0.5 us).  Each waiter takes its
// stages in order and waits for a stage's release before its data, so with
// kSB >= kExp and kSB + 3 <= 4 kSP no waiter is two phases ahead of a
// barrier.
constexpr size_t kGemmSmemBudget = 227 * 1024;  // dynamic shared memory per CTA
constexpr int kGroup = 4;                                 // k-blocks per packed tile
constexpr uint32_t kPackedTile = kBN * kGroup * kBK / 4;  // 16384 bytes
constexpr int kSXMax = 16;     // x_q ring, at most

template <int BT>
struct GemmCfg {
  static constexpr uint32_t kXStage = BT * 128;
  static constexpr uint32_t kTmemCols = (2 * BT < 32) ? 32 : 2 * BT;
  static constexpr uint32_t kChunk = BT < 32 ? BT : 32;  // accumulator columns per tcgen05.ld
  static constexpr uint32_t kYStage1 = kChunk * 128 * 4;  // output staging (TMA-store epilogue), x2
  static constexpr int kExp = BT <= 32 ? 8 : 4;                  // expansion warps
  static constexpr int kSB = BT <= 32 ? 8 : (BT <= 64 ? 5 : 4);  // expanded-tile ring (>= kExp)
  static constexpr int kSP = BT == 32 ? 3 : 4;                   // packed-tile ring
  static constexpr int kThreads = 32 * (4 + kExp + 4);  // TMA, MMA, 2 idle | expansion | epilogue
  static_assert(kSB >= kExp && kSB + 3 <= 4 * kSP, "ring depths");
  static constexpr size_t kFixed = 1024 + kSB * kExpStage + kSP * kPackedTile + 2 * kYStage1 +
                                   8 * (2 * kSXMax + 2 * kSP + 2 * kSB + 5) + 16 + 2 * 4 * BT;
  static_assert(kFixed + 2 * kXStage <= kGemmSmemBudget, "shared memory");
  static constexpr size_t kFit = (kGemmSmemBudget - kFixed) / kXStage;
  static constexpr int kSX = kFit > kSXMax ? kSXMax : static_cast<int>(kFit);
  static constexpr size_t kSmem = kFixed + kSX * kXStage;
  static_assert(kSX >= 2, "x_q ring");
};

template <int BT>
__global__ void __launch_bounds__(GemmCfg<BT>::kThreads, 1)
    gemm_i2_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_y, int y_tma, const float* __restrict__ gamma,
                   const float* __restrict__ scale, void* __restrict__ y, int ydt, int M, int N, int K, int ldy, int ks,
                   int32_t* __restrict__ part, WsHeader* __restrict__ hdr, long long limit, int skip_producer) {
  pdl_enter(gamma, scale, y, part, hdr);
  using Cfg = GemmCfg<BT>;
  constexpr int SX = Cfg::kSX, SP = Cfg::kSP, SB = Cfg::kSB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* es = base;                              // SB x [128 x 128 B], swizzled (1024-aligned)
  uint8_t* ps = es + SB * kExpStage;               // SP x [128 rows x 128 B] packed
  uint8_t* xs = ps + SP * kPackedTile;             // SX x [BT x 128 B], swizzled
  uint8_t* ystage = xs + SX * Cfg::kXStage;        // 2 x [kChunk tokens x 128 rows] output staging
  uint64_t* xfull = reinterpret_cast<uint64_t*>(ystage + 2 * Cfg::kYStage1);
  uint64_t* xempty = xfull + SX;
  uint64_t* pfull = xempty + SX;
  uint64_t* pempty = pfull + SP;
  uint64_t* expd = pempty + SP;
  uint64_t* emptyB = expd + SB;
  uint64_t* accf = emptyB + SB;  // 2
  uint64_t* acce = accf + 2;     // 2
  uint64_t* drain = acce + 2;    // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* cfac = reinterpret_cast<float*>(tmem_slot + 4);  // [2][BT] dequant factors per accumulator buffer

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = (K + kBK - 1) / kBK;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int t_tiles = (M + BT - 1) / BT;
  const int units = n_tiles * t_tiles * ks;  // ks <= kblocks (host-checked): no unit is empty
  struct Unit {
    int n_t, t_t, kz, kb0, kb1;
  };
  auto unit_of = [&](int u) {
    Unit w;
    w.n_t = u % n_tiles;
    const int r = u / n_tiles;
    w.kz = r % ks;
    w.t_t = r / ks;
    w.kb0 = static_cast<int>((static_cast<int64_t>(w.kz) * kblocks) / ks);
    w.kb1 = static_cast<int>((static_cast<int64_t>(w.kz + 1) * kblocks) / ks);
    return w;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(xfull + s, 1);
      mbar_init(xempty + s, 1);
    }
    for (int s = 0; s < SP; ++s) {
      mbar_init(pfull + s, 1);
      mbar_init(pempty + s, kGroup);  // one arrival per k-block of the tile
    }
    for (int b = 0; b < SB; ++b) {
      mbar_init(expd + b, 1);  // the warp that expanded it
      mbar_init(emptyB + b, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf + a, 1);
      mbar_init(acce + a, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](uint32_t site) {
    set_flag(hdr, kFlagTimeout, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    // per unit: for each group of kGroup k-blocks its packed tile, then the
    // x_q tile of each of its k-blocks
    if (lane == 0 && !skip_producer) {
      int ix = 0, ip = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit w = unit_of(u);
        for (int kb = w.kb0; kb < w.kb1 && ok; ++kb) {
          if ((kb - w.kb0) % kGroup == 0) {
            const int s = ip % SP;
            if (!wait1(pempty + s, ((ip / SP) & 1) ^ 1, limit, abort_flag)) {
              fail(0x203);
              ok = false;
              break;
            }
            mbar_expect_tx(pfull + s, kPackedTile);
            tma_load_2d(ps + s * kPackedTile, &tm_w, pfull + s, kb * (kBK / 4), w.n_t * kBN);
            ++ip;
          }
          const int s = ix % SX;
          if (!wait1(xempty + s, ((ix / SX) & 1) ^ 1, limit, abort_flag)) {
            fail(0x201);
            ok = false;
            break;
          }
          mbar_expect_tx(xfull + s, Cfg::kXStage);
          tma_load_2d(xs + s * Cfg::kXStage, &tm_x, xfull + s, kb * kBK, w.t_t * BT);
          ++ix;
        }
      }
      // copies still in flight land before the CTA leaves (bounded)
      for (int j = (ix > SX ? ix - SX : 0); j < ix; ++j) (void)wait_drain(xfull + (j % SX), (j / SX) & 1, limit);
      for (int j = (ip > SP ? ip - SP : 0); j < ip; ++j) (void)wait_drain(pfull + (j % SP), (j / SP) & 1, limit);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ---------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = i8_idesc(kBN, BT);
      int it = 0, tc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tc) {
        const Unit w = unit_of(u);
        const int a = tc & 1;
        if (!wait1(acce + a, ((tc >> 1) & 1) ^ 1, limit, abort_flag)) {
          fail(0x301);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(a * BT);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % SX, b = it % SB;
          if (!wait1(xfull + s, (it / SX) & 1, limit, abort_flag) || !wait1(expd + b, (it / SB) & 1, limit, abort_flag)) {
            fail(0x302);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(xs + s * Cfg::kXStage), ea = smem_u32(es + b * kExpStage);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8(d, sw128_desc(ea + 32 * k), sw128_desc(xa + 32 * k), idesc, (kb != w.kb0 || k != 0) ? 1u : 0u);
          mma_commit(xempty + s);  // the x_q tile has been read
          mma_commit(emptyB + b);  // the expanded tile has been read
        }
        if (ok) mma_commit(accf + a);
      }
      // every MMA issued above completes before the accumulator memory is freed
      mma_commit(drain);
      (void)wait_drain(drain, 0, limit);
    }
  } else if (warp >= 4 && warp < 4 + Cfg::kExp) {
    // ------------------------------ expansion ----------------------------------
    // warp v expands the k-blocks it with it % kExp == v, whole: lane L the
    // rows L, L + 32, L + 64, L + 96
    const int v = warp - 4;
    int it = 0, ip = 0;  // k-blocks and packed tiles of the CTA so far (every warp counts all)
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const Unit w = unit_of(u);
      const int nk = w.kb1 - w.kb0;
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
        const int i = kb - w.kb0, j = i % kGroup;
        const int gsz = (nk - (i - j)) < kGroup ? (nk - (i - j)) : kGroup;  // k-blocks of this packed tile
        const int tile_ip = ip;
        if (j == gsz - 1) ++ip;
        if (it % Cfg::kExp != v) continue;
        const int sp = tile_ip % SP, b = it % SB;
        if (!wait_warp(emptyB + b, ((it / SB) & 1) ^ 1, limit, abort_flag)) {
          if (lane == 0) fail(0x402);
          ok = false;
          break;
        }
        if (!wait_warp(pfull + sp, (tile_ip / SP) & 1, limit, abort_flag)) {
          if (lane == 0) fail(0x401);
          ok = false;
          break;
        }
        const uint8_t* pt = ps + sp * kPackedTile;
        uint8_t* et_ = es + b * kExpStage;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int r = lane + 32 * rr;
          const uint8_t* prow = pt + (r >> 3) * 1024 + (r & 7) * 128;  // swizzled 128-byte row
          const uint4 p0 = *reinterpret_cast<const uint4*>(prow + (((2 * j) ^ (r & 7)) << 4));
          const uint4 p1 = *reinterpret_cast<const uint4*>(prow + (((2 * j + 1) ^ (r & 7)) << 4));
          const uint32_t wd[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          uint8_t* row = et_ + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = expand16(wd[c]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(expd + b);
          // the last k-block of a short tile also stands for its missing ones
          mbar_arrive_n(pempty + sp, j == gsz - 1 ? static_cast<uint32_t>(kGroup - gsz + 1) : 1u);
        }
      }
    }
  } else if (warp >= 4 + Cfg::kExp) {
    // ------------------------------ epilogue -----------------------------------
    // (ks == 1: dequantize and store, through a shared staging tile and TMA
    // tensor stores when y has a tensor map; ks > 1: the raw INT32 partial
    // sums to part[kz][t][n], coalesced along n)
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int et = threadIdx.x - 32 * (4 + Cfg::kExp);
    const uint32_t esz = (ydt == BL_BF16) ? 2u : 4u;
    const bool use_tma = y_tma != 0 && ks == 1;
    const float g = __ldcg(gamma);
    int tc = 0, chunk = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++tc) {
      const Unit w = unit_of(u);
      const int a = tc & 1;
      const int n = w.n_t * kBN + 32 * q + lane;
      // dequant factor c_t = (gamma s_t) / 127 of each token of the tile, once
      float* cf = cfac + a * BT;
      if (ks == 1)
        for (int j = et; j < BT; j += 128) {
          const int t = w.t_t * BT + j;
          cf[j] = (t < M && ydt != BL_I32) ? dequant_factor(g, __ldcg(scale + t)) : 0.0f;
        }
      const uint32_t ok_w = wait_warp(accf + a, (tc >> 1) & 1, limit, abort_flag) ? 1u : 0u;
      // the four epilogue warps agree (and see each other's factors) before going on
      uint32_t ok_all;
      asm volatile(
          "{\n\t.reg .pred pi, po;\n\t"
          "setp.ne.u32 pi, %1, 0;\n\t"
          "bar.red.and.pred po, 1, 128, pi;\n\t"
          "selp.u32 %0, 1, 0, po;\n\t}"
          : "=r"(ok_all)
          : "r"(ok_w)
          : "memory");
      if (!ok_all) {
        if (!ok_w && lane == 0) fail(0x501);
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int j0 = 0; j0 < BT; j0 += Cfg::kChunk, ++chunk) {
        uint32_t acc[Cfg::kChunk];
        tmem_load<Cfg::kChunk>(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(a * BT + j0),
                               acc);
        const int t0 = w.t_t * BT + j0;
        if (ks > 1) {
          if (n < N) {
#pragma unroll
            for (int j = 0; j < static_cast<int>(Cfg::kChunk); ++j)
              if (t0 + j < M) part[(static_cast<int64_t>(w.kz) * M + t0 + j) * N + n] = static_cast<int32_t>(acc[j]);
          }
        } else if (use_tma) {
          uint8_t* sb = ystage + (chunk & 1) * Cfg::kYStage1;
          if (chunk >= 2) {  // the store issued from this buffer two chunks ago has read it
            if (et == 0) bulk_wait_read<1>();
            asm volatile("bar.sync 2, 128;" ::: "memory");
          }
          uint8_t* col = sb + (32 * q + lane) * esz;  // this lane's row in the staged tile
#pragma unroll
          for (int j = 0; j < static_cast<int>(Cfg::kChunk); ++j) {
            const int v = static_cast<int>(acc[j]);
            if (ydt == BL_I32) {
              *reinterpret_cast<int32_t*>(col + j * 128 * 4) = v;
            } else {
              const float yv = __fmul_rn(__int2float_rn(v), cf[j0 + j]);
              if (ydt == BL_F32)
                *reinterpret_cast<float*>(col + j * 128 * 4) = yv;
              else
                *reinterpret_cast<__nv_bfloat16*>(col + j * 128 * 2) = __float2bfloat16_rn(yv);
            }
          }
          fence_proxy_async_smem();
          asm volatile("bar.sync 2, 128;" ::: "memory");
          if (et == 0 && w.n_t * kBN < N && t0 < M) tma_store_2d(&tm_y, sb, w.n_t * kBN, t0);
          if (et == 0) bulk_commit();
        } else {
#pragma unroll
          for (int j = 0; j < static_cast<int>(Cfg::kChunk); ++j) {
            const int t = t0 + j;
            if (t < M && n < N) {
              const int64_t o = static_cast<int64_t>(t) * ldy + n;
              const int v = static_cast<int>(acc[j]);
              if (ydt == BL_I32) {
                static_cast<int32_t*>(y)[o] = v;
              } else {
                const float yv = __fmul_rn(__int2float_rn(v), cf[j0 + j]);
                if (ydt == BL_F32)
                  static_cast<float*>(y)[o] = yv;
                else
                  static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(yv);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce + a);
    }
    if (use_tma && et == 0) bulk_wait<0>();  // every output store has landed before the CTA leaves
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols)
                 : "memory");
  }
}

// The ks partial sums of each output (exact INT32 addition, any order), then
// the dequantization y = acc * (gamma s_t) / 127 as in the GEMM epilogues.
// Four consecutive outputs per thread when N % 4 == 0.
__global__ void __launch_bounds__(256)
    splitk_reduce_kernel(const int32_t* __restrict__ part, int ks, int M, int N, int ldy, const float* __restrict__ gamma,
                         const float* __restrict__ scale, void* __restrict__ y, int ydt) {
  pdl_enter(part, gamma, scale, y);
  __shared__ float sh_g;  // gamma once per CTA
  if (threadIdx.x == 0) sh_g = __ldcg(gamma);
  __syncthreads();
  const float g = sh_g;
  const int64_t plane = static_cast<int64_t>(M) * N;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  auto emit = [&](int64_t o, int t, int v) {
    if (ydt == BL_I32) {
      static_cast<int32_t*>(y)[o] = v;
    } else {
      const float yv = __fmul_rn(__int2float_rn(v), dequant_factor(g, __ldcg(scale + t)));
      if (ydt == BL_F32)
        static_cast<float*>(y)[o] = yv;
      else
        static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(yv);
    }
  };
  if ((N % 4) == 0) {
    const int64_t n4 = plane / 4;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
      int4 s = __ldcg(reinterpret_cast<const int4*>(part) + i);
      for (int kz = 1; kz < ks; ++kz) {
        const int4 p = __ldcg(reinterpret_cast<const int4*>(part + kz * plane) + i);
        s.x += p.x;
        s.y += p.y;
        s.z += p.z;
        s.w += p.w;
      }
      const int64_t o = 4 * i;
      const int t = static_cast<int>(o / N);
      const int64_t yo = static_cast<int64_t>(t) * ldy + (o - static_cast<int64_t>(t) * N);  // row stride ldy
      emit(yo, t, s.x);
      emit(yo + 1, t, s.y);
      emit(yo + 2, t, s.z);
      emit(yo + 3, t, s.w);
    }
  } else {
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < plane; o += stride) {
      int s = __ldcg(part + o);
      for (int kz = 1; kz < ks; ++kz) s += __ldcg(part + kz * plane + o);
      const int t = static_cast<int>(o / N);
      emit(static_cast<int64_t>(t) * ldy + (o - static_cast<int64_t>(t) * N), t, s);
    }
  }
}

// ---------------------------------------------------------------------------
// Two-SM variant for many tokens.  A cluster of two CTAs computes a tile of
// 256 weight rows x BT tokens with tcgen05.mma.cta_group::2 (M = 256): CTA r
// stages its own 128 weight rows and tokens r BT/2 .. (r+1) BT/2 - 1, so per
// SM the staged bytes per MAC fall to about 2/3 of the one-SM tile: five TMA
// stages and five expanded stages fit (three expanded stages measured 1-3 %
// slower).  Each CTA's accumulator in tensor memory holds its 128 rows x BT
// tokens.  The leader (rank 0) issues the MMAs; the x loads of both CTAs count
// on the leader's barrier, the packed loads on the local one (the expansion
// warps of each CTA wait there), and the expansion and epilogue warps of both
// CTAs report to the leader by remote arrives.  MMA completion is committed to
// the barriers of both CTAs.  Every wait is bounded as in the one-SM kernel.
// ---------------------------------------------------------------------------
constexpr int kStagesA = 5;  // TMA ring: x half + packed tile per stage
constexpr int kStagesB = 5;  // expanded-weight ring
constexpr uint32_t kYStage = 32 * 128 * 4;  // output staging: 32 tokens x 128 rows, up to 4 bytes each

template <int BT>
struct Gemm2Cfg {
  static constexpr uint32_t kXHalf = (BT / 2) * 128;
  static constexpr uint32_t kTmemCols = 2 * BT;  // BT >= 128: a power of two
  static constexpr size_t kSmem = 1024 + kStagesB * kExpStage + kStagesA * (kXHalf + kPackedStage) +
                                  2 * kYStage + 8 * (3 * kStagesA + 2 * kStagesB + 5) + 16 + 2 * 4 * BT;
};

__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on the barrier at this offset in each CTA of `mask` when the MMAs
// issued so far complete
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

template <int BT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_i2_2sm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_y, int y_tma, const float* __restrict__ gamma,
                       const float* __restrict__ scale, void* __restrict__ y, int ydt, int M, int N, int K, int ldy,
                       WsHeader* __restrict__ hdr, long long limit) {
  pdl_enter(gamma, scale, y, hdr);
  using Cfg = Gemm2Cfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* es = base;                              // kStagesB x [128 x 128 B], swizzled
  uint8_t* xs = es + kStagesB * kExpStage;         // kStagesA x [BT/2 x 128 B], swizzled
  uint8_t* ps = xs + kStagesA * Cfg::kXHalf;       // kStagesA x [128 x 32 B]
  uint8_t* ystage = ps + kStagesA * kPackedStage;  // 2 x [32 tokens x 128 rows] output staging
  uint64_t* xfull = reinterpret_cast<uint64_t*>(ystage + 2 * kYStage);  // leader: x of both CTAs
  uint64_t* pfull = xfull + kStagesA;              // local: packed tile
  uint64_t* emptyA = pfull + kStagesA;             // local: MMAs read x, expansion read packed (1 + 4)
  uint64_t* expd = emptyA + kStagesA;              // leader: expansion of both CTAs (8 warps)
  uint64_t* emptyB = expd + kStagesB;              // local: the MMAs read the expanded stage
  uint64_t* accf = emptyB + kStagesB;              // local: accumulator ready (2)
  uint64_t* acce = accf + 2;                       // leader: epilogues of both CTAs done (2)
  uint64_t* drain = acce + 2;                      // leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* cfac = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int kblocks = (K + kBK - 1) / kBK;
  const int n_tiles = (N + 2 * kBN - 1) / (2 * kBN);
  const int t_tiles = (M + BT - 1) / BT;
  const int tiles = n_tiles * t_tiles;
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(xfull + s, 1);
      mbar_init(pfull + s, 1);
      mbar_init(emptyA + s, 1 + 4);
    }
    for (int s = 0; s < kStagesB; ++s) {
      mbar_init(expd + s, 8);
      mbar_init(emptyB + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf + a, 1);
      mbar_init(acce + a, 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](uint32_t site) {
    set_flag(hdr, kFlagTimeout, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += pairs) {
        const int n_t = tile % n_tiles, t_t = tile / n_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStagesA;
          const uint32_t ph = (it / kStagesA) & 1;
          if (!wait1(emptyA + s, ph ^ 1, limit, abort_flag)) {
            fail(0x211);
            ok = false;
            break;
          }
          if (leader) mbar_expect_tx(xfull + s, 2 * Cfg::kXHalf);
          mbar_expect_tx(pfull + s, kPackedStage);
          tma_load_2d_pair(xs + s * Cfg::kXHalf, &tm_x, mapa_shared(smem_u32(xfull + s), 0), kb * kBK,
                           t_t * BT + static_cast<int>(rank) * (BT / 2));
          tma_load_2d(ps + s * kPackedStage, &tm_w, pfull + s, kb * (kBK / 4),
                      n_t * 2 * kBN + static_cast<int>(rank) * kBN);
        }
      }
      for (int j = (it > kStagesA ? it - kStagesA : 0); j < it; ++j)
        (void)wait_drain(pfull + (j % kStagesA), (j / kStagesA) & 1, limit);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader) -------------------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = i8_idesc(2 * kBN, BT);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += pairs, ++tc) {
        const int a = tc & 1;
        if (!wait1(acce + a, ((tc >> 1) & 1) ^ 1, limit, abort_flag)) {
          fail(0x311);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(a * BT);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int sa = it % kStagesA, sb = it % kStagesB;
          const uint32_t pha = (it / kStagesA) & 1, phb = (it / kStagesB) & 1;
          if (!wait1(xfull + sa, pha, limit, abort_flag) || !wait1(expd + sb, phb, limit, abort_flag)) {
            fail(0x312);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(xs + sa * Cfg::kXHalf), ea = smem_u32(es + sb * kExpStage);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8_pair(d, sw128_desc(ea + 32 * k), sw128_desc(xa + 32 * k), idesc, (kb | k) != 0);
          mma_commit_pair(emptyA + sa, 0x3);
          mma_commit_pair(emptyB + sb, 0x3);
        }
        if (ok) mma_commit_pair(accf + a, 0x3);
      }
      mma_commit_pair(drain, 0x1);
      (void)wait_drain(drain, 0, limit);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------ expansion (both CTAs) -----------------------
    const int r = threadIdx.x - 128;
    int it = 0;
    bool ok = true;
    for (int tile = pair; tile < tiles && ok; tile += pairs) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int sa = it % kStagesA, sb = it % kStagesB;
        const uint32_t pha = (it / kStagesA) & 1, phb = (it / kStagesB) & 1;
        if (!wait_warp(pfull + sa, pha, limit, abort_flag) || !wait_warp(emptyB + sb, phb ^ 1, limit, abort_flag)) {
          if (lane == 0) fail(0x411);
          ok = false;
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(ps + sa * kPackedStage + r * 32);
        const uint4 p0 = src[0], p1 = src[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(emptyA + sa);  // the packed tile has been read
        const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        uint8_t* row = es + sb * kExpStage + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = expand16(w[j]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(expd + sb), 0));
      }
    }
  } else if (warp >= 8) {
    // ------------------------------ epilogue (both CTAs) ------------------------
    // Each 32-token chunk of the tile's accumulator is converted into a shared
    // staging buffer laid out as the output tile [32 tokens x 128 rows] and
    // written by one TMA tensor store (the TMA unit clips rows past N and
    // tokens past M); two buffers alternate, a buffer being rewritten only after
    // the store issued from it two chunks before has read it.  Without a tensor
    // map for y (a row of y not a multiple of 16 bytes) the lanes store directly.
    const int q = warp & 3, et = threadIdx.x - 256;
    const uint32_t esz = (ydt == BL_BF16) ? 2u : 4u;
    const float g = __ldcg(gamma);
    int tc = 0, chunk = 0;
    for (int tile = pair; tile < tiles; tile += pairs, ++tc) {
      const int a = tc & 1;
      const int n_t = tile % n_tiles, t_t = tile / n_tiles;
      const int nbase = n_t * 2 * kBN + static_cast<int>(rank) * kBN;
      const int n = nbase + 32 * q + lane;
      float* cf = cfac + a * BT;
      for (int j = et; j < BT; j += 128) {
        const int t = t_t * BT + j;
        cf[j] = (t < M && ydt != BL_I32) ? dequant_factor(g, __ldcg(scale + t)) : 0.0f;
      }
      const uint32_t ok_w = wait_warp(accf + a, (tc >> 1) & 1, limit, abort_flag) ? 1u : 0u;
      uint32_t ok_all;
      asm volatile(
          "{\n\t.reg .pred pi, po;\n\t"
          "setp.ne.u32 pi, %1, 0;\n\t"
          "bar.red.and.pred po, 1, 128, pi;\n\t"
          "selp.u32 %0, 1, 0, po;\n\t}"
          : "=r"(ok_all)
          : "r"(ok_w)
          : "memory");
      if (!ok_all) {
        if (!ok_w && lane == 0) fail(0x511);
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int j0 = 0; j0 < BT; j0 += 32, ++chunk) {
        uint32_t acc[32];
        tmem_load<32>(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(a * BT + j0), acc);
        const int t0 = t_t * BT + j0;
        if (y_tma) {
          uint8_t* sb = ystage + (chunk & 1) * kYStage;
          if (chunk >= 2) {  // the store issued from this buffer two chunks ago has read it
            if (et == 0) bulk_wait_read<1>();
            asm volatile("bar.sync 2, 128;" ::: "memory");
          }
          uint8_t* col = sb + (32 * q + lane) * esz;  // this lane's row in the staged tile
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int v = static_cast<int>(acc[j]);
            if (ydt == BL_I32) {
              *reinterpret_cast<int32_t*>(col + j * 128 * 4) = v;
            } else {
              const float yv = __fmul_rn(__int2float_rn(v), cf[j0 + j]);
              if (ydt == BL_F32)
                *reinterpret_cast<float*>(col + j * 128 * 4) = yv;
              else
                *reinterpret_cast<__nv_bfloat16*>(col + j * 128 * 2) = __float2bfloat16_rn(yv);
            }
          }
          fence_proxy_async_smem();
          asm volatile("bar.sync 2, 128;" ::: "memory");
          if (et == 0 && nbase < N && t0 < M) {
            tma_store_2d(&tm_y, sb, nbase, t0);
          }
          if (et == 0) bulk_commit();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = t0 + j;
            if (t < M && n < N) {
              const int64_t o = static_cast<int64_t>(t) * ldy + n;
              const int v = static_cast<int>(acc[j]);
              if (ydt == BL_I32) {
                static_cast<int32_t*>(y)[o] = v;
              } else {
                const float yv = __fmul_rn(__int2float_rn(v), cf[j0 + j]);
                if (ydt == BL_F32)
                  static_cast<float*>(y)[o] = yv;
                else
                  static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(yv);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(acce + a), 0));
    }
    if (y_tma && et == 0) bulk_wait<0>();  // every output store has landed before the CTA leaves
  }

  __syncthreads();
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols)
                 : "memory");
  }
}

// Base-3 rows re-encoded as 2-bit rows (a base-3 digit is the 2-bit code of
// the same weight), for the tensor-core path.  Item (n, t): the 16 base-3
// bytes 16t .. 16t + 15 of row n (weights 80t .. 80t + 79; bytes past rb5 read
// as padding, 121 = five weight-0 digits) become 160 bits, i.e. five 32-bit
// words at byte 20t of the 2-bit row (words past rb2 are dropped).  A byte's
// five codes come from a 256-entry table of 10-bit entries with one copy per
// lane, so the 32 lookups of a warp are one conflict-free access.
__global__ void __launch_bounds__(256)
    t5_to_i2_kernel(const uint8_t* __restrict__ t5, int64_t N, int64_t K, int64_t rb5, uint8_t* __restrict__ i2,
                    int64_t rb2) {
  pdl_enter(t5, i2);
  __shared__ uint32_t lut[256][32];
  for (int e = threadIdx.x; e < 256 * 32; e += blockDim.x) {
    const int b = e >> 5;
    uint32_t v = static_cast<uint32_t>(b), d = 0x155u;  // bytes 243..255: five weight-0 digits
    if (b < 243) {
      d = 0;
      for (int i = 0; i < 5; ++i) {
        d |= (v % 3) << (2 * i);
        v /= 3;
      }
    }
    lut[b][e & 31] = d;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  // items fit in 32 bits (N K <= 2^32 and an item covers 80 weights): 32-bit
  // index arithmetic, no 64-bit division per item
  const uint32_t per_row = static_cast<uint32_t>((rb2 + 19) / 20);
  const uint32_t words2 = static_cast<uint32_t>(rb2 / 4);
  const uint32_t items = static_cast<uint32_t>(N) * per_row;
  for (uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x; gid < items; gid += gridDim.x * blockDim.x) {
    const uint32_t nn = gid / per_row, t = gid - nn * per_row;
    const int64_t n = nn;
    const uint4 v = 16 * static_cast<int64_t>(t) < rb5 ? __ldcg(reinterpret_cast<const uint4*>(t5 + n * rb5 + 16 * t))
                                 : make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[6] = {0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t d = lut[(wd[i >> 2] >> (8 * (i & 3))) & 0xffu][lane];
      const int pos = 10 * i, w = pos >> 5, sh = pos & 31;
      out[w] |= d << sh;
      if (sh > 22) out[w + 1] |= d >> (32 - sh);
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(i2 + n * rb2) + 5 * t;
#pragma unroll
    for (int j = 0; j < 5; ++j)
      if (5 * t + j < words2) dst[j] = out[j];
  }
  (void)K;  // the padding digits past K are weight-0 codes in both formats
}

// 1-bit -> 2-bit transcoding (for the tensor-core path, and for decode rows
// too long for the 1-bit GEMV): one thread writes one 16-byte segment (64
// weights) of a 2-bit row from 8 bytes of the 1-bit row.  A set bit (+1) is
// digit 2, a clear bit (-1) digit 0; weights past K are digit 1 (weight 0).
__device__ __forceinline__ uint32_t spread16_to_2bit(uint32_t h) {  // bit i -> bit 2i
  uint32_t x = h & 0xffffu;
  x = (x | (x << 8)) & 0x00ff00ffu;
  x = (x | (x << 4)) & 0x0f0f0f0fu;
  x = (x | (x << 2)) & 0x33333333u;
  x = (x | (x << 1)) & 0x55555555u;
  return x;
}

__global__ void __launch_bounds__(256)
    b1_to_i2_kernel(const uint8_t* __restrict__ b1, int64_t N, int64_t K, int64_t rb1, uint8_t* __restrict__ i2,
                    int64_t rb2) {
  pdl_enter(b1, i2);
  // N segs < 2^32 (N K <= 2^32, a segment covers 64 weights): 32-bit index
  // arithmetic, no 64-bit division per segment
  const uint32_t segs = static_cast<uint32_t>(rb2 / 16);
  const uint32_t items = static_cast<uint32_t>(N) * segs;
  for (uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x; gid < items; gid += gridDim.x * blockDim.x) {
    const uint32_t nn = gid / segs, sg32 = gid - nn * segs;
    const int64_t n = nn, sg = sg32;
    const uint8_t* row = b1 + n * rb1;
    uint32_t out[4];
    // the segment's eight 1-bit bytes in one load (rb1 is a multiple of 16, so
    // they are all in the row or all past it)
    const uint2 raw = 8 * sg < rb1 ? __ldcg(reinterpret_cast<const uint2*>(row + 8 * sg)) : make_uint2(0u, 0u);
#pragma unroll
    for (int w = 0; w < 4; ++w) {  // 16 weights: two bytes of the 1-bit row
      const uint32_t bits = ((w < 2 ? raw.x : raw.y) >> (16 * (w & 1))) & 0xffffu;
      uint32_t d = spread16_to_2bit(bits) << 1;  // +1 -> 10, -1 -> 00
      const int64_t k0 = 64 * sg + 16 * w;
      if (k0 + 16 > K) {
        const int64_t valid = K - k0 < 0 ? 0 : K - k0;  // weights of the word below K
        const uint32_t keep = valid >= 16 ? 0xffffffffu : ((1u << (2 * valid)) - 1u);
        d = (d & keep) | (0x55555555u & ~keep);
      }
      out[w] = d;
    }
    *reinterpret_cast<uint4*>(i2 + n * rb2 + sg * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// ---- host side --------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t stride,
                  uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of y for the TMA-store epilogue: [M x N] of the output type, box
// 128 rows x `tokens` tokens.  False when a row of y is not a multiple of 16
// bytes.
bool encode_y(CUtensorMap* m, void* y, int ydt, int64_t M, int64_t N, int64_t ldy, uint32_t tokens) {
  const uint64_t esz = (ydt == BL_BF16) ? 2 : 4;
  if ((static_cast<uint64_t>(ldy) * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(y) % 16) != 0) return false;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const CUtensorMapDataType dt = ydt == BL_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : ydt == BL_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                 : CU_TENSOR_MAP_DATA_TYPE_INT32;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldy) * esz};
  const cuuint32_t box[2] = {128, tokens};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BT>
cudaError_t launch_gemm_bt(const int8_t* xq, const uint8_t* w, int64_t rb, const float* gamma, const float* scale,
                           void* y, int ydt, int64_t M, int64_t N, int64_t K, int64_t ldy, int ks, int32_t* part, void* ws,
                           long long limit, int skip_producer, cudaStream_t st) {
  CUtensorMap tx, tw;
  if (!encode_2d_u8(&tx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, BT,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tw, w, static_cast<uint64_t>(rb), static_cast<uint64_t>(N), static_cast<uint64_t>(rb),
                    kGroup * kBK / 4, kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  CUtensorMap ty;
  const int y_tma = (ks == 1 && encode_y(&ty, y, ydt, M, N, ldy, GemmCfg<BT>::kChunk)) ? 1 : 0;
  if (!y_tma) memset(&ty, 0, sizeof(ty));
  auto kern = gemm_i2_kernel<BT>;
  const size_t smem = GemmCfg<BT>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = ((N + kBN - 1) / kBN) * ((M + BT - 1) / BT) * ks;
  const int sms = device_sms();
  const unsigned grid = static_cast<unsigned>(units < sms ? units : sms);
  e = launch_pdl(kern, grid, GemmCfg<BT>::kThreads, smem, st, tx, tw, ty, y_tma, gamma, scale, y, ydt, static_cast<int>(M),
                 static_cast<int>(N), static_cast<int>(K), static_cast<int>(ldy), ks, part, static_cast<WsHeader*>(ws), limit,
                 skip_producer);
  if (e != cudaSuccess) return e;
  if (ks > 1) {
    const int64_t work = (N % 4 == 0) ? M * N / 4 : M * N;
    int64_t rgrid = (work + 255) / 256;
    if (rgrid > 8 * sms) rgrid = 8 * sms;
    e = launch_pdl(splitk_reduce_kernel, static_cast<unsigned>(rgrid), 256, 0, st, static_cast<const int32_t*>(part),
                   ks, static_cast<int>(M), static_cast<int>(N), static_cast<int>(ldy), gamma, scale, y, ydt);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <int BT>
cudaError_t launch_gemm_2sm(const int8_t* xq, const uint8_t* w, int64_t rb, const float* gamma, const float* scale,
                            void* y, int ydt, int64_t M, int64_t N, int64_t K, int64_t ldy, void* ws, long long limit,
                            cudaStream_t st) {
  CUtensorMap tx, tw;
  if (!encode_2d_u8(&tx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128,
                    BT / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tw, w, static_cast<uint64_t>(rb), static_cast<uint64_t>(N), static_cast<uint64_t>(rb),
                    kBK / 4, kBN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  CUtensorMap ty;
  const int y_tma = encode_y(&ty, y, ydt, M, N, ldy, 32) ? 1 : 0;
  if (!y_tma) memset(&ty, 0, sizeof(ty));
  auto kern = gemm_i2_2sm_kernel<BT>;
  const size_t smem = Gemm2Cfg<BT>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((N + 2 * kBN - 1) / (2 * kBN)) * ((M + BT - 1) / BT);
  const int64_t pairs_max = device_sms() / 2;
  const int64_t pairs = tiles < pairs_max ? tiles : pairs_max;
  { const cudaError_t le_ = launch_pdl(kern, static_cast<unsigned>(2 * pairs), kGemmThreads, smem, st, tx, tw, ty, y_tma, gamma, scale, y, ydt,
                                                                     static_cast<int>(M), static_cast<int>(N),
                                                                     static_cast<int>(K), static_cast<int>(ldy),
                                                                     static_cast<WsHeader*>(ws),
                                                                     limit); if (le_ != cudaSuccess) return le_; }
  return cudaGetLastError();
}

}  // namespace

int gemm_token_tile(int64_t M) {
  if (M > 128) return 256;
  if (M > 64) return 128;
  if (M > 32) return 64;
  if (M > 16) return 32;
  return 16;
}

// Split of the k-blocks of each one-SM tile: the ks in 1..16 (at most the
// number of k-blocks) with the smallest per-SM makespan in k-blocks, waves x
// (k-blocks per unit + 4), plus 12 for the reduction pass when ks > 1.
int gemm_split_k(int64_t M, int64_t N, int64_t K) {
  if (M > 128) return 1;
  const int64_t bt = gemm_token_tile(M);
  const int64_t tiles = ((N + kBN - 1) / kBN) * ((M + bt - 1) / bt);
  const int64_t kblocks = (K + kBK - 1) / kBK;
  const int64_t sms = device_sms();
  int best = 1;
  int64_t best_cost = -1;
  for (int ks = 1; ks <= 16 && ks <= kblocks; ++ks) {
    const int64_t waves = (tiles * ks + sms - 1) / sms;
    const int64_t cost = waves * ((kblocks + ks - 1) / ks + 4) + (ks > 1 ? 12 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = ks;
    }
  }
  return best;
}

cudaError_t launch_gemm_i2(const int8_t* xq, const uint8_t* w, int64_t rb, const float* gamma, const float* scale,
                           void* y, int ydt, int64_t M, int64_t N, int64_t K, int64_t ldy, int32_t* part, void* ws,
                           long long limit_cycles, int skip_producer, cudaStream_t st) {
  const long long limit = limit_cycles > 0 ? limit_cycles : kTimeoutCycles;
  if (M > 128 && !skip_producer)
    return launch_gemm_2sm<256>(xq, w, rb, gamma, scale, y, ydt, M, N, K, ldy, ws, limit, st);
  const int ks = (part != nullptr && !skip_producer) ? gemm_split_k(M, N, K) : 1;
  switch (gemm_token_tile(M)) {
    case 16: return launch_gemm_bt<16>(xq, w, rb, gamma, scale, y, ydt, M, N, K, ldy, ks, part, ws, limit, skip_producer, st);
    case 32: return launch_gemm_bt<32>(xq, w, rb, gamma, scale, y, ydt, M, N, K, ldy, ks, part, ws, limit, skip_producer, st);
    case 64: return launch_gemm_bt<64>(xq, w, rb, gamma, scale, y, ydt, M, N, K, ldy, ks, part, ws, limit, skip_producer, st);
    default: return launch_gemm_bt<128>(xq, w, rb, gamma, scale, y, ydt, M, N, K, ldy, ks, part, ws, limit, skip_producer, st);
  }
}

cudaError_t launch_b1_to_i2(const uint8_t* b1, int64_t N, int64_t K, int64_t rb1, uint8_t* i2, int64_t rb2,
                            cudaStream_t st) {
  const int64_t work = N * (rb2 / 16);
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  int64_t grid = (work + 255) / 256;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const cudaError_t e = launch_pdl(b1_to_i2_kernel, static_cast<unsigned>(grid), 256, 0, st, b1, N, K, rb1, i2, rb2);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_t5_to_i2(const uint8_t* t5, int64_t N, int64_t K, int64_t rb5, uint8_t* i2, int64_t rb2,
                            cudaStream_t st) {
  const int64_t work = N * ((rb2 + 19) / 20);
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  int64_t grid = (work + 255) / 256;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  { const cudaError_t le_ = launch_pdl(t5_to_i2_kernel, static_cast<unsigned>(grid), 256, 0, st, t5, N, K, rb5, i2, rb2); if (le_ != cudaSuccess) return le_; }
  return cudaGetLastError();
}

}  // namespace bl
