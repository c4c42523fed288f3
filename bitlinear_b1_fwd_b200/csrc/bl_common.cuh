// bl_common.cuh -- helpers shared by the BitLinear kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bitlinear.h"

namespace bl {

// Fixed reduction order of gamma: 8192-element chunks, 256 lanes, groups of 8.
constexpr int kChunk = 8192;
constexpr int kLanes = 256;

// Device flags in the first word of a workspace header.
constexpr uint32_t kFlagTimeout = 1u;
constexpr uint32_t kFlagBadCode = 2u;

struct WsHeader {
  uint32_t flags;   // kFlag* bits, sticky until bitlinear_device_status
  uint32_t site;    // where a bounded wait gave up (kernel-defined code)
  uint32_t ticket;  // absmean: CTAs done so far (back to 0 when a call ends)
  uint32_t reserved[61];
};
static_assert(sizeof(WsHeader) == BL_WS_HEADER_BYTES, "header size");

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Load element i of a float-valued array (fp32 or bf16 bit patterns).
template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i) {
  if constexpr (DT == BL_F32) {
    return __ldcg(static_cast<const float*>(p) + i);
  } else {
    return bf16_bits_to_f32(__ldcg(static_cast<const uint16_t*>(p) + i));
  }
}

// Load 8 consecutive elements starting at element e (e a multiple of 8 and
// the array 16-byte aligned), widened to fp32.
template <int DT>
__device__ __forceinline__ void load8_aligned(const void* p, int64_t e, float v[8]) {
  if constexpr (DT == BL_F32) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + e);
    float4 a = __ldcg(q), b = __ldcg(q + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 a = __ldcg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p) + e));
    uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// Programmatic dependent launch: every kernel of the library lets the next
// kernel in its stream be scheduled as soon as it starts (all of them run as
// one wave of persistent CTAs, so that kernel's CTAs only take SM room this
// grid no longer needs), and waits for the previous kernel to complete (with
// its memory visible) before it reads or writes anything.  Without the launch
// attribute both instructions are no-ops.
// A grid launched this way is alive while its predecessor still writes, so
// nothing it reads may go through the non-coherent read-only path (whose
// contract is data constant for the kernel's whole life): inputs are read
// with L2-coherent loads (ld.global.cg), and the pointers a kernel touches
// are passed through an opaque move issued after the wait, so that no load
// through them is derived from a restrict kernel parameter (which the
// compiler may turn into a read-only-path load) or issued before the wait.
template <typename P>
__device__ __forceinline__ void pdl_after(P& p) {
  uint64_t v;
  asm volatile("mov.b64 %0, %1;" : "=l"(v) : "l"((uint64_t)(p)) : "memory");
  p = (P)(v);
}

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... P>
__device__ __forceinline__ void pdl_wait(P&... ptrs) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  (pdl_after(ptrs), ...);
}

template <typename... P>
__device__ __forceinline__ void pdl_enter(P&... ptrs) {
  pdl_launch_dependents();
  pdl_wait(ptrs...);
}

// Bulk prefetch of [p, p + bytes) into L2 (p 16-byte aligned, bytes a
// multiple of 16), one instruction per 16 KB from threads 0, 1, ...  A
// prefetch returns no data and L2 is the point of coherence, so it may be
// issued before the wait: a later load still sees whatever the previous
// kernel writes there.
__device__ __forceinline__ void l2_prefetch_bulk(const void* p, int64_t bytes) {
  constexpr int64_t kPiece = 16384;
  const int64_t off = static_cast<int64_t>(threadIdx.x) * kPiece;
  if (off < bytes) {
    const uint32_t sz = static_cast<uint32_t>(bytes - off < kPiece ? bytes - off : kPiece);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const uint8_t*>(p) + off), "r"(sz)
                 : "memory");
  }
}

// Per-token INT8 code of x against scale s: rint(fl(fl(x / s) * 127)) clamped
// to [-127, 127]; IEEE quotient, round half to even.
__device__ __forceinline__ int quant_act(float x, float s) {
  float t = __fmul_rn(__fdiv_rn(x, s), 127.0f);
  t = fminf(fmaxf(rintf(t), -127.0f), 127.0f);
  return __float2int_rn(t);
}

// Round to the nearest integer, ties to even, for |t| < 2^22: adding 1.5 * 2^23
// rounds in the adder (round-to-nearest-even) and leaves the integer in the low
// significand bits.  Returns the rounded value as float and as int.
__device__ __forceinline__ float round_magic(float t, int* qi) {
  const float r = __fadd_rn(t, 12582912.0f);
  *qi = static_cast<int>(__float_as_uint(r)) - 0x4b400000;
  return __fsub_rn(r, 12582912.0f);
}

// The same code as quant_act without a division per element, for |x| <= s.
// With c127 = fl(127 / s), t_a = fl(x c127) differs from t = fl(fl(x / s) 127)
// by less than 4.0001 * 2^-24 |t| (two roundings on each side), and
// |t_a| <= 127 (1 + 2^-22), so |t_a - t| < 2^-14: when t_a is farther than
// 2^-14 from every half-integer (|t_a - rint(t_a)| < 1/2 - 2^-14; the
// difference is exact) both round to the same integer, t is not a tie, and
// the code is within [-127, 127] with no clamp; otherwise (rare) the exact
// quotient decides.
static __device__ __noinline__ int quant_act_slow(float x, float s) { return quant_act(x, s); }

__device__ __forceinline__ int quant_act_fast(float x, float s, float c127) {
  const float ta = __fmul_rn(x, c127);
  int qi;
  const float qa = round_magic(ta, &qi);
  if (fabsf(__fsub_rn(ta, qa)) < 0.49993896484375f) return qi;
  return quant_act_slow(x, s);
}

// The codes of N elements (N <= 32) by the rule above, the exact quotient
// taken in one rare branch for the elements near a tie only (so the common
// case evaluates no division).
template <int N>
__device__ __forceinline__ void quant_act_fast_n(const float* e, float s, float c127, int* q) {
  uint32_t near = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float ta = __fmul_rn(e[j], c127);
    const float qa = round_magic(ta, &q[j]);
    if (!(fabsf(__fsub_rn(ta, qa)) < 0.49993896484375f)) near |= 1u << j;
  }
  if (near != 0) {
#pragma unroll
    for (int j = 0; j < N; ++j)
      if ((near >> j) & 1u) q[j] = quant_act_slow(e[j], s);
  }
}

// Dequantization factor c = (gamma * s) / 127 and the dequantized value.
__device__ __forceinline__ float dequant_factor(float gamma, float s) {
  return __fdiv_rn(__fmul_rn(gamma, s), 127.0f);
}

template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_maxf(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void set_flag(void* ws, uint32_t bit, uint32_t site) {
  if (ws == nullptr) return;
  WsHeader* h = static_cast<WsHeader*>(ws);
  atomicOr(&h->flags, bit);
  atomicExch(&h->site, site);
}

}  // namespace bl
