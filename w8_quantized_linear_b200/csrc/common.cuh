// Shared device helpers of the BitNest sm_100a kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnest {

constexpr int kGroup = 128;  // columns per weight / activation group

// 16-byte streaming load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ldg_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// d = c + sum_{i<4} ubyte_i(a) * sbyte_i(b)
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// byte permute (PRMT): result byte i = byte sel_i of the 8-byte pair {b:a}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Weight-code offsets of the two models: the planes hold unsigned nibbles,
// draft code = hi - 8, target code = ((hi << 4) | lo) - 136.
template <int MODE>
struct CodeOffset;
template <>
struct CodeOffset<0> {
  static constexpr int value = 8;
};
template <>
struct CodeOffset<1> {
  static constexpr int value = 136;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace bitnest
