// Plane packing, symmetric int8 activation quantisation and activation group
// sums.  BitNest-Llama-3-8B model card: section "Files" (plane layout) and the
// model table row "Activations" (symmetric int8 per token, per 128-group for
// o_proj).
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace bitnest {

// ---------------------------------------------------------------- packing
// Each thread writes 4 plane bytes from 8 nibbles of one row.
__global__ void pack_kernel(const uint8_t *__restrict__ u, int64_t total_words,
                            uint8_t *__restrict__ plane) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= total_words) return;
  const uint2 v = *reinterpret_cast<const uint2 *>(u + 8 * i);  // columns 8i .. 8i+7
  // t: byte b = u[b] & 15; t | t >> 4 puts u[2j] | u[2j+1] << 4 in byte 2j
  uint32_t a = v.x & 0x0F0F0F0Fu, b = v.y & 0x0F0F0F0Fu;
  a |= a >> 4;
  b |= b >> 4;
  reinterpret_cast<uint32_t *>(plane)[i] = prmt(a, b, 0x6420);
}

cudaError_t launch_pack(const uint8_t *uh, const uint8_t *ul, int64_t N, int64_t K, uint8_t *hi,
                        uint8_t *lo, cudaStream_t st) {
  int64_t words = N * K / 8;
  int threads = 256;
  int64_t blocks = (words + threads - 1) / threads;
  pack_kernel<<<(unsigned)blocks, threads, 0, st>>>(uh, words, hi);
  if (ul && lo) pack_kernel<<<(unsigned)blocks, threads, 0, st>>>(ul, words, lo);
  return cudaGetLastError();
}

// --------------------------------------------------- packer from weights
// BitNest-Llama-3-8B model card, opening paragraph (the high nibble a 4-bit
// model fitted first, the low nibble the closed-form residual back to 8
// bits) and section "Files" (u = q + 8, fp16 scale per 128 columns).  The
// card fits the high nibble by GPTQ; here it is rounded to nearest:
//   s = fp16(max|W| / 7) per row and group, t = W / s (fp32, correctly
//   rounded), q4 = rne(t) (|t| <= 7.007: no clamp needed),
//   ql = clamp(rne(16 (t - q4)), -8, 7), planes u = q + 8; s = 0 for an
//   all-zero group (both nibbles 8).
// One warp per (row, group): lane i holds columns 4i .. 4i+3.
__global__ void __launch_bounds__(256) pack_weights_kernel(const uint16_t *__restrict__ w,
                                                           int64_t N, int64_t K,
                                                           uint8_t *__restrict__ hi,
                                                           uint8_t *__restrict__ lo,
                                                           uint16_t *__restrict__ scale) {
  const int64_t G = K / kGroup;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= N * G) return;  // whole warps leave together
  const int64_t n = wid / G, g = wid - n * G;
  const int64_t k0 = g * kGroup + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2 *>(w + n * K + k0);
  const __half2 h01 = *reinterpret_cast<const __half2 *>(&raw.x);
  const __half2 h23 = *reinterpret_cast<const __half2 *>(&raw.y);
  const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
  const float v[4] = {f01.x, f01.y, f23.x, f23.y};
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half sh = __float2half_rn(__fdiv_rn(amax, 7.0f));
  const float sf = __half2float(sh);
  uint32_t uh[4], ul[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int q4 = 0, ql = 0;
    if (sf != 0.0f) {
      const float t = __fdiv_rn(v[i], sf);
      const float r4 = rintf(t);  // round half to even
      q4 = (int)r4;
      ql = __float2int_rn(__fmul_rn(16.0f, __fsub_rn(t, r4)));
      ql = max(-8, min(7, ql));
    }
    uh[i] = (uint32_t)(q4 + 8);
    ul[i] = (uint32_t)(ql + 8);
  }
  // plane bytes j = k / 2: column 2j in the low nibble, 2j+1 in the high one
  const uint16_t hb = (uint16_t)((uh[0] | (uh[1] << 4)) | ((uh[2] | (uh[3] << 4)) << 8));
  const uint16_t lb = (uint16_t)((ul[0] | (ul[1] << 4)) | ((ul[2] | (ul[3] << 4)) << 8));
  *reinterpret_cast<uint16_t *>(hi + n * (K / 2) + k0 / 2) = hb;
  *reinterpret_cast<uint16_t *>(lo + n * (K / 2) + k0 / 2) = lb;
  if (lane == 0) scale[n * G + g] = __half_as_ushort(sh);
}

cudaError_t launch_pack_weights(const uint16_t *w, int64_t N, int64_t K, uint8_t *hi,
                                uint8_t *lo, uint16_t *scale, cudaStream_t st) {
  const int64_t warps = N * (K / kGroup);
  const int threads = 256;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  pack_weights_kernel<<<(unsigned)blocks, threads, 0, st>>>(w, N, K, hi, lo, scale);
  return cudaGetLastError();
}

// ------------------------------------------------------------ quantiser
// One block per token.  Vector v (8 columns) is handled by thread v % T; a
// group (16 vectors) is 16 consecutive threads of one pass.  With V > 0 every
// thread holds its (at most V) vectors in registers: one read of x, one
// block reduction of max|x|, then the codes.  V == 0 reads x twice (any K).
template <int T, int V>
__global__ void __launch_bounds__(T) quantize_token_kernel(const uint16_t *__restrict__ x,
                                                           int64_t K, int8_t *__restrict__ xq,
                                                           float *__restrict__ xs,
                                                           int32_t *__restrict__ xsum) {
  const int64_t m = blockIdx.x;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + m * K);
  // This block is resident while the preceding kernel runs: ask for the row
  // in L2 now (a hint; the read below comes after the wait).  x may come
  // from the preceding kernel: wait for it, and only then let the next kernel
  // (the layer, which may stream its weights early) start.
  if (threadIdx.x == 0) {
    for (int64_t o = 0; o < K * 2; o += 65536)
      prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(xr) + o,
                       (uint32_t)(K * 2 - o < 65536 ? K * 2 - o : 65536));
  }
  griddep_wait();
  griddep_launch_dependents();
  const int nvec = (int)(K / 8);
  constexpr int R = V > 0 ? V : 1;
  uint4 v[R];
  float amax = 0.0f;
  if (V > 0) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int i = threadIdx.x + j * T;
      v[j] = i < nvec ? __ldg(xr + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < R; ++j) amax = fmaxf(amax, amax8(v[j]));
  } else {
    for (int i = threadIdx.x; i < nvec; i += T) amax = fmaxf(amax, amax8(__ldg(xr + i)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[T / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < T / 32; ++i) amax = fmaxf(amax, red[i]);
  const float s = __fdiv_rn(amax, 127.0f);
  const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
  if (threadIdx.x == 0) xs[m] = s;
  uint2 *qr = reinterpret_cast<uint2 *>(xq + m * K);
  const int G = (int)(K / kGroup);
  // codes of vector i (held in `val`) and the sum of its group
  auto emit = [&](int i, const uint4 &val) {
    int sum = 0;
    if (i < nvec) qr[i] = quant8(val, s, rs, &sum);
    // 16 consecutive threads hold one group (T is a multiple of 16, nvec of 16)
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (xsum && i < nvec && (i & 15) == 0) xsum[m * G + i / 16] = sum;
  };
  if (V > 0) {
#pragma unroll
    for (int j = 0; j < R; ++j) emit(threadIdx.x + j * T, v[j]);
  } else {
    for (int i0 = 0; i0 < nvec; i0 += T) {
      const int i = i0 + threadIdx.x;
      emit(i, i < nvec ? __ldg(xr + i) : make_uint4(0, 0, 0, 0));
    }
  }
}

// act_group = 128: 16 threads per group, one scale per (token, group).
__global__ void __launch_bounds__(256) quantize_group_kernel(const uint16_t *__restrict__ x,
                                                             int64_t M, int64_t K,
                                                             int8_t *__restrict__ xq,
                                                             float *__restrict__ xs,
                                                             int32_t *__restrict__ xsum) {
  const int64_t nvec = M * K / 8;
  const int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // vectors in order
  if (threadIdx.x == 0) {  // this block's slice into L2 before the wait (a hint)
    const int64_t v0 = blockIdx.x * (int64_t)blockDim.x;
    const int64_t n = (nvec - v0 < (int64_t)blockDim.x ? nvec - v0 : (int64_t)blockDim.x);
    prefetch_l2_bulk(reinterpret_cast<const uint4 *>(x) + v0, (uint32_t)(n * 16));
  }
  griddep_wait();
  griddep_launch_dependents();
  const bool ok = v < nvec;  // nvec is a multiple of 16: whole groups share `ok`
  uint4 val = ok ? __ldg(reinterpret_cast<const uint4 *>(x) + v) : make_uint4(0, 0, 0, 0);
  float amax = amax8(val);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  int sum = 0;
  uint2 q = quant8(val, s, s == 0.0f ? 0.0f : __frcp_rn(s), &sum);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (ok) {
    reinterpret_cast<uint2 *>(xq)[v] = q;
    if ((v & 15) == 0) {
      const int64_t grp = v / 16;  // = m * G + g
      xs[grp] = s;
      if (xsum) xsum[grp] = sum;
    }
  }
}

cudaError_t launch_quantize(const uint16_t *x, int64_t M, int64_t K, int act_group, int8_t *xq,
                            float *xs, int32_t *xsum, cudaStream_t st) {
  // programmatic dependent launch: the kernel waits for its predecessor first
  cudaError_t e;
  if (act_group == 0 && K / 8 > 2 * 256 && K / 8 <= 4 * 1024) {
    // long rows (down_proj's K = 14336): 1024 threads, at most 4 vectors each
    constexpr int T = 1024;
    const int64_t per = (K / 8 + T - 1) / T;
    auto kern = per <= 2 ? quantize_token_kernel<T, 2> : quantize_token_kernel<T, 4>;
    e = launch_pdl(kern, dim3((unsigned)M), dim3(T), 0, st, true, x, K, xq, xs, xsum);
  } else if (act_group == 0) {
    constexpr int T = 256;
    const int64_t per = (K / 8 + T - 1) / T;  // vectors per thread
    auto kern = per <= 1 ? quantize_token_kernel<T, 1>
                : per <= 2 ? quantize_token_kernel<T, 2>
                : per <= 4 ? quantize_token_kernel<T, 4>
                : per <= 8 ? quantize_token_kernel<T, 8>
                : per <= 16 ? quantize_token_kernel<T, 16> : quantize_token_kernel<T, 0>;
    e = launch_pdl(kern, dim3((unsigned)M), dim3(T), 0, st, true, x, K, xq, xs, xsum);
  } else {
    const int64_t nvec = M * K / 8;
    const int threads = 256;
    e = launch_pdl(quantize_group_kernel, dim3((unsigned)((nvec + threads - 1) / threads)),
                   dim3(threads), 0, st, true, x, M, K, xq, xs, xsum);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------ activation sums
// One warp per (token, group): 128 bytes, 4 per lane.
__global__ void act_group_sums_kernel(const int8_t *__restrict__ xq, int64_t groups,
                                      int32_t *__restrict__ xsum) {
  const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= groups) return;
  const uint32_t word = reinterpret_cast<const uint32_t *>(xq + w * kGroup)[lane];
  int sum = __dp4a((int)word, 0x01010101, 0);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) xsum[w] = sum;
}

cudaError_t launch_act_group_sums(const int8_t *xq, int64_t M, int64_t K, int32_t *xsum,
                                  cudaStream_t st) {
  const int64_t groups = M * (K / kGroup);
  const int threads = 256;
  const int64_t blocks = (groups * 32 + threads - 1) / threads;
  act_group_sums_kernel<<<(unsigned)blocks, threads, 0, st>>>(xq, groups, xsum);
  return cudaGetLastError();
}

}  // namespace bitnest
