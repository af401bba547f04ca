// Shared device helpers of the BitNest sm_100a kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

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

// Programmatic dependent launch: wait for the preceding kernel of the stream
// (no-op when launched without the attribute) / let the next one start.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Programmatic dependent launch is used unless the environment variable
// BITNEST_PDL is "0" (read once per process).
inline bool pdl_enabled() {
  static const int on = [] {
    const char *v = getenv("BITNEST_PDL");
    return (v && v[0] == '0' && v[1] == 0) ? 0 : 1;
  }();
  return on != 0;
}

// Launch `kern` with programmatic stream serialisation allowed when `pdl`.
template <typename Kern, typename... Args>
inline cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              bool pdl, Args... args) {
  pdl = pdl && pdl_enabled();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Symmetric int8 code of one activation (model table row "Activations"):
// q = clamp(rne(x / s), -127, 127), with x / s the correctly rounded fp32
// quotient and s = max|x| / 127 (so |x / s| <= 127.00001).  rs = RN(1 / s).
// The product t = RN(x * rs) lies within 1.6e-5 of the exact quotient and
// RN(x / s) within 3.9e-6 of it; so unless t is within 2^-15 of a
// half-integer both round to the same integer, and only those rare values pay
// for the correctly rounded division.
__device__ __forceinline__ int quant_code(float x, float s, float rs) {
  if (s == 0.0f) return 0;
  const float t = __fmul_rn(x, rs);
  const float frac = t - floorf(t);  // exact: |t| < 2^23
  const int q = fabsf(frac - 0.5f) < 3.0517578125e-05f ? __float2int_rn(__fdiv_rn(x, s))
                                                       : __float2int_rn(t);
  return max(-127, min(127, q));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace bitnest
