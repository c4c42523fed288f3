// bl_gemv.cuh -- small helpers shared by the decode GEMV kernels.
#pragma once

#include <stdint.h>

namespace bl {

// 16-byte load through L2 only (no L1 allocation): weights stream once, and a
// kernel alive while its predecessor finishes must not read through the
// non-coherent path.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// dp4a with unsigned bytes in a and signed bytes in b.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The four bytes q[0..3] (low byte of each) as one word, q[0] in the low byte.
__device__ __forceinline__ uint32_t pack4(const int* q) {
  return __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
}

// The 2-bit layout's 16-byte slot of the 16 codes q[0..15] of one packed word:
// byte 4j + b = q[4b + j], a 4 x 4 byte transpose of P_b = q[4b .. 4b + 3].
__device__ __forceinline__ uint4 i2_slot(uint32_t P0, uint32_t P1, uint32_t P2, uint32_t P3) {
  const uint32_t t0 = __byte_perm(P0, P1, 0x5140), t1 = __byte_perm(P2, P3, 0x5140);
  const uint32_t t2 = __byte_perm(P0, P1, 0x7362), t3 = __byte_perm(P2, P3, 0x7362);
  return make_uint4(__byte_perm(t0, t1, 0x5410), __byte_perm(t0, t1, 0x7632), __byte_perm(t2, t3, 0x5410),
                    __byte_perm(t2, t3, 0x7632));
}

}  // namespace bl
