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

// Codes of 8 fp16 activations (one 16-byte vector) with scale s and
// rs = RN(1 / s) (rs = 0 when s = 0, which gives zeros), packed
// little-endian (code j in byte j); their sum is added to *sum.  The same
// codes as quant_code, in fewer instructions: t = RN(x * rs) with packed
// f32x2 multiplies; rne(t) by adding and subtracting 1.5 * 2^23 (exact for
// |t| < 2^22; the low byte of t + 1.5 * 2^23 is the two's-complement code);
// and one test of all eight |t - rne(t)| against 1/2 - 2^-15 sends the rare
// vector with a value near a half-integer to quant_code.  |x / s| <= 127.00001
// (s = max|x| / 127) keeps every code in [-127, 127] without a clamp.
__device__ __forceinline__ void f32x2_mul(float &d0, float &d1, float a0, float a1, float b0,
                                          float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void f32x2_add(float &d0, float &d1, float a0, float a1, float b0,
                                          float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void f32x2_sub(float &d0, float &d1, float a0, float a1, float b0,
                                          float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ uint2 quant8(const uint4 v, float s, float rs, int *sum) {
  constexpr float kRound = 12582912.0f;          // 1.5 * 2^23
  constexpr float kTieEdge = 0.499969482421875f;  // 1/2 - 2^-15
  const __half2 *h = reinterpret_cast<const __half2 *>(&v);
  float x[8], t[8], u[8], r[8], d[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    f32x2_mul(t[i], t[i + 1], x[i], x[i + 1], rs, rs);
    f32x2_add(u[i], u[i + 1], t[i], t[i + 1], kRound, kRound);
    f32x2_sub(r[i], r[i + 1], u[i], u[i + 1], kRound, kRound);
    f32x2_sub(d[i], d[i + 1], t[i], t[i + 1], r[i], r[i + 1]);
  }
  bool tie = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) tie |= fabsf(d[i]) > kTieEdge;
  uint32_t ub[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ub[i] = __float_as_uint(u[i]);
  uint32_t w0 = prmt(prmt(ub[0], ub[1], 0x0040), prmt(ub[2], ub[3], 0x0040), 0x5410);
  uint32_t w1 = prmt(prmt(ub[4], ub[5], 0x0040), prmt(ub[6], ub[7], 0x0040), 0x5410);
  if (tie) {  // rare: at least one value within 2^-15 of a half-integer
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i >> 2] |= (uint32_t)(quant_code(x[i], s, rs) & 0xff) << (8 * (i & 3));
    w0 = w[0];
    w1 = w[1];
  }
  *sum = __dp4a((int)w0, 0x01010101, __dp4a((int)w1, 0x01010101, *sum));
  return make_uint2(w0, w1);
}

// max |x| of 8 fp16 activations (compared in fp16: the same maximum)
__device__ __forceinline__ float amax8(const uint4 v) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&v);
  const __half2 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])),
                            __hmax2(__habs2(h[2]), __habs2(h[3])));
  return fmaxf(__low2float(m), __high2float(m));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace bitnest
