// Decode attention over a nested KV cache (BitNest-Llama-3-8B model card,
// model table row "KV cache": nested at runtime, the draft reads KV4, the
// target KV8).  The cache uses the weights' nesting: every K (V) row of one
// token and one KV head (head_dim 128 = one group) is an 8-bit code split
// into a hi and a lo nibble plane with an fp16 scale (packed at runtime with
// bitnest_pack_weights); the draft dequantises (hi - 8) s and reads only the
// hi plane, the target (16 (hi - 8) + (lo - 8)) s / 16 from both.
//
// One new token: head h (of H) attends with KV head h / (H / Hkv) over the T
// cached tokens, softmax(q K^T / sqrt(D)) V.  One CTA per KV head; warp w
// takes tokens w, w + 8, ..; lane i holds columns 4i .. 4i+3 of every row, so
// a K or V row is one 2-byte read per plane per lane.  Each warp keeps an
// online softmax (running maximum, sum and weighted V) for each query head
// of its group; the eight warps are merged through shared memory.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace bitnest {

namespace attn {

constexpr int kD = 128;       // head dimension (one scale group)
constexpr int kWarps = 8;
constexpr int kMaxGroup = 8;  // query heads per KV head

// the 4 dequantised values of this lane's columns in row `row`
template <int MODE>
__device__ __forceinline__ void dequant4(const uint8_t *__restrict__ hi,
                                         const uint8_t *__restrict__ lo,
                                         const uint16_t *__restrict__ scale, int64_t row, int lane,
                                         float (&v)[4]) {
  const float s = __half2float(__ushort_as_half(__ldg(scale + row)));
  const uint32_t h2 = __ldg(reinterpret_cast<const uint16_t *>(hi + row * (kD / 2)) + lane);
  int c[4] = {(int)(h2 & 15u) - 8, (int)((h2 >> 4) & 15u) - 8, (int)((h2 >> 8) & 15u) - 8,
              (int)((h2 >> 12) & 15u) - 8};
  if (MODE) {
    const uint32_t l2 = __ldg(reinterpret_cast<const uint16_t *>(lo + row * (kD / 2)) + lane);
    c[0] = 16 * c[0] + (int)(l2 & 15u) - 8;
    c[1] = 16 * c[1] + (int)((l2 >> 4) & 15u) - 8;
    c[2] = 16 * c[2] + (int)((l2 >> 8) & 15u) - 8;
    c[3] = 16 * c[3] + (int)((l2 >> 12) & 15u) - 8;
  }
  const float f = MODE ? s * 0.0625f : s;  // code * s (/ 16): exact in fp32
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = (float)c[i] * f;
}

template <int MODE, int GQ>
__global__ void __launch_bounds__(kWarps * 32) nested_attention_kernel(
    const uint16_t *__restrict__ q, int Hkv, int T, const uint8_t *__restrict__ k_hi,
    const uint8_t *__restrict__ k_lo, const uint16_t *__restrict__ k_scale,
    const uint8_t *__restrict__ v_hi, const uint8_t *__restrict__ v_lo,
    const uint16_t *__restrict__ v_scale, float *__restrict__ out) {
  const int j = blockIdx.x;  // KV head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  griddep_launch_dependents();
  // this lane's 4 columns of the group's queries, pre-scaled by 1/sqrt(D)
  const float rsd = 1.0f / sqrtf((float)kD);
  float qv[GQ][4];
#pragma unroll
  for (int g = 0; g < GQ; ++g) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(q + (int64_t)(j * GQ + g) * kD) + lane);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
    qv[g][0] = a.x * rsd;
    qv[g][1] = a.y * rsd;
    qv[g][2] = b.x * rsd;
    qv[g][3] = b.y * rsd;
  }
  float m[GQ], l[GQ], acc[GQ][4];
#pragma unroll
  for (int g = 0; g < GQ; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.0f;
  }
  for (int t = warp; t < T; t += kWarps) {
    const int64_t row = (int64_t)t * Hkv + j;
    float kv[4], vv[4];
    dequant4<MODE>(k_hi, k_lo, k_scale, row, lane, kv);
    dequant4<MODE>(v_hi, v_lo, v_scale, row, lane, vv);
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
      float sc = qv[g][0] * kv[0] + qv[g][1] * kv[1] + qv[g][2] * kv[2] + qv[g][3] * kv[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
      const float mn = fmaxf(m[g], sc);
      const float corr = expf(m[g] - mn);  // 0 on the first token (m = -inf)
      const float p = expf(sc - mn);
      l[g] = l[g] * corr + p;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[g][i] = acc[g][i] * corr + p * vv[i];
      m[g] = mn;
    }
  }
  // merge the warps: out = sum_w e^(m_w - M) acc_w / sum_w e^(m_w - M) l_w
  __shared__ float sm[kWarps][kMaxGroup], sl[kWarps][kMaxGroup];
  __shared__ float sacc[kWarps][kMaxGroup][kD];
#pragma unroll
  for (int g = 0; g < GQ; ++g) {
    if (lane == 0) {
      sm[warp][g] = m[g];
      sl[warp][g] = l[g];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sacc[warp][g][4 * lane + i] = acc[g][i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < GQ * kD; e += kWarps * 32) {
    const int g = e / kD, c = e - g * kD;
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[w][g]);
    float num = 0.0f, den = 0.0f;
    for (int w = 0; w < kWarps; ++w) {
      if (sm[w][g] == -INFINITY) continue;  // a warp that saw no token
      const float f = expf(sm[w][g] - M);
      num += f * sacc[w][g][c];
      den += f * sl[w][g];
    }
    out[(int64_t)(j * GQ + g) * kD + c] = num / den;
  }
}

template <int MODE>
cudaError_t launch_mode(const uint16_t *q, int64_t H, int64_t Hkv, int64_t T, const uint8_t *k_hi,
                        const uint8_t *k_lo, const uint16_t *k_scale, const uint8_t *v_hi,
                        const uint8_t *v_lo, const uint16_t *v_scale, float *out,
                        cudaStream_t st) {
  const int gq = (int)(H / Hkv);
  const dim3 grid((unsigned)Hkv), block(kWarps * 32);
#define BITNEST_ATTN_CASE(G)                                                                    \
  case G:                                                                                       \
    return launch_pdl(nested_attention_kernel<MODE, G>, grid, block, 0, st, true, q, (int)Hkv, \
                      (int)T, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale, out);
  switch (gq) {
    BITNEST_ATTN_CASE(1)
    BITNEST_ATTN_CASE(2)
    BITNEST_ATTN_CASE(4)
    BITNEST_ATTN_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef BITNEST_ATTN_CASE
}

}  // namespace attn

bool nested_attention_supported(int64_t H, int64_t Hkv, int64_t D, int64_t T) {
  if (D != attn::kD || Hkv < 1 || H < Hkv || H % Hkv != 0 || T < 1) return false;
  const int64_t g = H / Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return false;
  return Hkv <= 65535 && T <= ((int64_t)1 << 30) && T * Hkv < ((int64_t)1 << 31);
}

cudaError_t launch_nested_attention(int mode, const uint16_t *q, int64_t H, int64_t Hkv,
                                    int64_t T, const uint8_t *k_hi, const uint8_t *k_lo,
                                    const uint16_t *k_scale, const uint8_t *v_hi,
                                    const uint8_t *v_lo, const uint16_t *v_scale, float *out,
                                    cudaStream_t st) {
  cudaError_t e = mode ? attn::launch_mode<1>(q, H, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo,
                                              v_scale, out, st)
                       : attn::launch_mode<0>(q, H, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo,
                                              v_scale, out, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bitnest
