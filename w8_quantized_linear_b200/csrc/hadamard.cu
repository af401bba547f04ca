// Online Hadamard rotation of the down_proj input, fused with its per-token
// int8 quantisation (BitNest-Llama-3-8B model card, model table rows
// "Rotation": R4 online Hadamard on down_proj inputs, and "Activations":
// symmetric int8 per token).
//
// The card ships its R4 matrices; the construction is a reading: x_rot =
// x H / sqrt(K) with H of order K = p (a power of two: Sylvester's matrix)
// or K = 28 p (H = H28 (x) H_p, the order-28 factor outer, H28 from Paley's
// construction I over GF(27)).  x H is evaluated as the Kronecker product
// factorises it: a fast Walsh-Hadamard transform of length p on each of the
// K / p blocks, then each column of the blocks mixed by H28.
//
// One CTA per token.  The row lives in shared memory in fp32 (K <= 32768);
// the rotated row is quantised as the activation quantiser does (s =
// max|x_rot| / 127, codes rne(x_rot / s)) with the group sums of the codes.
//
// Decode sizes of down_proj's K = 28 x 512 (a few tokens): one CTA per token
// leaves the whole rotation to a single SM, so there a cluster of 7 CTAs
// takes each token: CTA r transforms blocks 4 r .. 4 r + 3 and stores them
// into every CTA of the cluster (distributed shared memory), mixes its own 4
// output blocks from the full row, and the 7 partial maxima of |x_rot| meet
// the same way before each CTA quantises its blocks.  The arithmetic is the
// same, in the same order, as the one-CTA kernel's: the codes are identical.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace bitnest {

namespace hd {

constexpr int kThreads = 512;
constexpr int kMaxK = 32768;

// Paley's construction I for q = 27 (q = 3 mod 4): H28 = I + S with
// S = [[0, 1^T], [-1, Q]], Q[a][b] = chi(a - b), chi the quadratic character
// of GF(27).  GF(27) = GF(3)[x] / (x^3 - x - 1); an element a0 + a1 x + a2 x^2
// is the integer a0 + 3 a1 + 9 a2.  Evaluated at compile time: every sign of
// the order-28 mix below is a constant.
__host__ __device__ constexpr int gf27_sub(int a, int b) {
  return (a % 3 - b % 3 + 3) % 3 + 3 * ((a / 3 % 3 - b / 3 % 3 + 3) % 3) +
         9 * ((a / 9 - b / 9 + 3) % 3);
}
__host__ __device__ constexpr int gf27_square(int a) {
  const int d0 = a % 3, d1 = a / 3 % 3, d2 = a / 9;
  // (d0 + d1 x + d2 x^2)^2 with x^3 = x + 1 and x^4 = x^2 + x
  const int c0 = d0 * d0, c1 = 2 * d0 * d1, c2 = 2 * d0 * d2 + d1 * d1, c3 = 2 * d1 * d2,
            c4 = d2 * d2;
  return (c0 + c3) % 3 + 3 * ((c1 + c3 + c4) % 3) + 9 * ((c2 + c4) % 3);
}
__host__ __device__ constexpr bool gf27_is_square(int a) {
  for (int b = 1; b < 27; ++b)
    if (gf27_square(b) == a) return true;
  return false;
}
// H28[i][j] < 0 ?
__host__ __device__ constexpr bool h28_neg(int i, int j) {
  return i == j ? false : i == 0 ? false : j == 0 ? true : !gf27_is_square(gf27_sub(i - 1, j - 1));
}
// The signs as row masks (bit j of row i: H28[i][j] < 0), a constant
// expression wherever it is used.
struct H28Signs {
  uint32_t row[28];
};
__host__ __device__ constexpr H28Signs h28_signs() {
  H28Signs t{};
  for (int i = 0; i < 28; ++i)
    for (int j = 0; j < 28; ++j)
      if (h28_neg(i, j)) t.row[i] |= 1u << j;
  return t;
}

// Length-512 transform of one block by one warp, in registers: lane l holds
// elements 16 l .. 16 l + 15; butterflies of distance 1..8 inside the lane,
// 16..256 across lanes (shuffles).  Reads fp16 from global, writes fp32.
__device__ __forceinline__ void fwht512_warp(const uint16_t *__restrict__ src, float *dst,
                                             int lane) {
  float v[16];
  const uint4 *s4 = reinterpret_cast<const uint4 *>(src + 16 * lane);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint4 raw = __ldg(s4 + q);
    const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      v[8 * q + 2 * i] = f.x;
      v[8 * q + 2 * i + 1] = f.y;
    }
  }
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const bool upper = (lane & d) != 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float w = __shfl_xor_sync(0xffffffffu, v[e], d);
      v[e] = upper ? w - v[e] : v[e] + w;
    }
  }
  float4 *d4 = reinterpret_cast<float4 *>(dst + 16 * lane);
#pragma unroll
  for (int q = 0; q < 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__global__ void __launch_bounds__(kThreads) hadamard_quantize_kernel(
    const uint16_t *__restrict__ x, int K, int lp, float norm, int8_t *__restrict__ xq,
    float *__restrict__ xs, int32_t *__restrict__ xsum) {
  extern __shared__ float sx[];  // [K]
  const int64_t m = blockIdx.x;
  const int p = 1 << lp;  // block length
  const int R = K >> lp;  // 1 or 28 blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  griddep_launch_dependents();
  if (p == 512) {
    // each warp transforms whole blocks in registers
    for (int blk = warp; blk < R; blk += kThreads / 32)
      fwht512_warp(x + m * K + blk * 512, sx + blk * 512, lane);
    __syncthreads();
  } else {
  // fp16 row -> fp32 in shared memory, 8 values per 16-byte load
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + m * K);
  for (int v = threadIdx.x; v < K / 8; v += kThreads) {
    const uint4 raw = __ldg(xr + v);
    const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      sx[8 * v + 2 * i] = f.x;
      sx[8 * v + 2 * i + 1] = f.y;
    }
  }
  __syncthreads();
  // length-p Walsh-Hadamard transform of every block: butterflies
  // (a, a + half) -> (a + b, a - b), half = 1, 2, .., p / 2
  for (int lh = 0; lh < lp; ++lh) {
    const int half = 1 << lh;
    for (int t = threadIdx.x; t < K / 2; t += kThreads) {
      const int lo = ((t >> lh) << (lh + 1)) | (t & (half - 1));  // stays inside its block
      const float a = sx[lo], b = sx[lo + half];
      sx[lo] = a + b;
      sx[lo + half] = a - b;
    }
    __syncthreads();
  }
  }
  // mix the blocks: out[j28][c] = sum_i28 H28[i28][j28] u[i28][c]
  // = sum_i u[i] - 2 sum_{H28[i][j] < 0} u[i]; then 1/sqrt(K)
  if (R == 28) {
    constexpr H28Signs kSigns = h28_signs();  // evaluated by the compiler
    for (int c = threadIdx.x; c < p; c += kThreads) {
      float u[28];
      float total = 0.0f;
#pragma unroll
      for (int i = 0; i < 28; ++i) {
        u[i] = sx[i * p + c];
        total += u[i];
      }
#pragma unroll
      for (int j = 0; j < 28; ++j) {
        float neg = 0.0f;
#pragma unroll
        for (int i = 0; i < 28; ++i)
          if ((kSigns.row[i] >> j) & 1u) neg += u[i];
        sx[j * p + c] = (total - 2.0f * neg) * norm;
      }
    }
  } else {
    for (int k = threadIdx.x; k < K; k += kThreads) sx[k] *= norm;
  }
  __syncthreads();
  // per-token quantisation of the rotated row
  float amax = 0.0f;
  for (int k = threadIdx.x; k < K; k += kThreads) amax = fmaxf(amax, fabsf(sx[k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[kThreads / 32];
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float s = __fdiv_rn(amax, 127.0f);
  const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
  if (threadIdx.x == 0) xs[m] = s;
  // a warp per 128-column group: lane i takes columns 4i .. 4i+3
  const int G = K / kGroup;
  for (int g = warp; g < G; g += kThreads / 32) {
    const float4 v = *reinterpret_cast<const float4 *>(sx + g * kGroup + 4 * lane);
    const int q0 = quant_code(v.x, s, rs), q1 = quant_code(v.y, s, rs);
    const int q2 = quant_code(v.z, s, rs), q3 = quant_code(v.w, s, rs);
    reinterpret_cast<uint32_t *>(xq + m * K + g * kGroup)[lane] =
        (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
        ((uint32_t)(q3 & 0xff) << 24);
    int sum = q0 + q1 + q2 + q3;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (xsum && lane == 0) xsum[m * G + g] = sum;
  }
}

// ----------------------------------------------- cluster kernel (K = 28 x 512)
constexpr int kClusterCtas = 7;                 // CTAs per token
constexpr int kBlocksPerCta = 28 / kClusterCtas;  // 4 blocks of 512
constexpr int kCThreads = 256;
constexpr int kClusterMaxM = 16;                // tokens up to which the cluster kernel is used

__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// distributed shared memory is used only once every CTA of the cluster has
// started: each thread arrives at entry and waits before its first access
__device__ __forceinline__ void cl_arrive() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// 16 bytes to the same shared-memory offset as `p` in CTA `rank` of the cluster
__device__ __forceinline__ void st_cl4(float *p, uint32_t rank, float4 v) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cl1(float *p, uint32_t rank, float v) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

struct ClusterSmem {
  float row[28 * 512];          // the transformed blocks of the whole row
  float out[kBlocksPerCta * 512];  // this CTA's rotated output blocks
  float amax[kClusterCtas];     // the CTAs' maxima of |x_rot|
  float red[kCThreads / 32];
};

__global__ void __launch_bounds__(kCThreads) hadamard_quantize_cluster_kernel(
    const uint16_t *__restrict__ x, float norm, int8_t *__restrict__ xq, float *__restrict__ xs,
    int32_t *__restrict__ xsum) {
  constexpr int K = 28 * 512, p = 512;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ClusterSmem &sh = *reinterpret_cast<ClusterSmem *>(smem_raw);
  const int64_t m = blockIdx.y;
  const uint32_t rank = cl_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b0 = (int)rank * kBlocksPerCta;  // this CTA's blocks
  cl_arrive();
  griddep_wait();
  griddep_launch_dependents();
  // transform this CTA's blocks (one warp each) and store them into every CTA
  if (warp < kBlocksPerCta)
    fwht512_warp(x + m * K + (b0 + warp) * p, sh.out + warp * p, lane);  // staging
  cl_wait();  // every CTA of the cluster has started
  if (warp < kBlocksPerCta) {
    const int blk = b0 + warp;
    const float4 *v4 = reinterpret_cast<const float4 *>(sh.out + warp * p + 16 * lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = v4[q];
      for (int r = 0; r < kClusterCtas; ++r)
        st_cl4(sh.row + blk * p + 16 * lane + 4 * q, (uint32_t)r, v);
    }
  }
  cl_sync();  // every CTA holds the whole transformed row
  // mix: out[j][c] = sum_i H28[i][j] u[i][c] = total - 2 sum_{H28[i][j] < 0} u[i][c],
  // for this CTA's output blocks j = b0 .. b0 + 3, then 1/sqrt(K)
  constexpr H28Signs kSigns = h28_signs();
  float amax = 0.0f;
  for (int c = threadIdx.x; c < p; c += kCThreads) {
    float u[28];
    float total = 0.0f;
#pragma unroll
    for (int i = 0; i < 28; ++i) {
      u[i] = sh.row[i * p + c];
      total += u[i];
    }
#pragma unroll
    for (int jj = 0; jj < kBlocksPerCta; ++jj) {
      const int j = b0 + jj;
      float neg = 0.0f;
#pragma unroll
      for (int i = 0; i < 28; ++i)
        if ((kSigns.row[i] >> j) & 1u) neg += u[i];
      const float o = (total - 2.0f * neg) * norm;
      sh.out[jj * p + c] = o;
      amax = fmaxf(amax, fabsf(o));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) sh.red[warp] = amax;
  __syncthreads();
  if (threadIdx.x < kClusterCtas) {  // this CTA's maximum into slot `rank` of every CTA
    float a = sh.red[0];
#pragma unroll
    for (int w = 1; w < kCThreads / 32; ++w) a = fmaxf(a, sh.red[w]);
    st_cl1(&sh.amax[rank], (uint32_t)threadIdx.x, a);
  }
  cl_sync();
  amax = sh.amax[0];
#pragma unroll
  for (int r = 1; r < kClusterCtas; ++r) amax = fmaxf(amax, sh.amax[r]);
  const float s = __fdiv_rn(amax, 127.0f);
  const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
  if (rank == 0 && threadIdx.x == 0) xs[m] = s;
  // a warp per 128-column group of this CTA's blocks
  constexpr int G = K / kGroup;
  for (int gl = warp; gl < kBlocksPerCta * p / kGroup; gl += kCThreads / 32) {
    const int g = b0 * (p / kGroup) + gl;
    const float4 v = *reinterpret_cast<const float4 *>(sh.out + gl * kGroup + 4 * lane);
    const int q0 = quant_code(v.x, s, rs), q1 = quant_code(v.y, s, rs);
    const int q2 = quant_code(v.z, s, rs), q3 = quant_code(v.w, s, rs);
    reinterpret_cast<uint32_t *>(xq + m * K + g * kGroup)[lane] =
        (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
        ((uint32_t)(q3 & 0xff) << 24);
    int sum = q0 + q1 + q2 + q3;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (xsum && lane == 0) xsum[m * G + g] = sum;
  }
}

// p with K = p or K = 28 p (p a power of two), or 0
int block_length(int64_t K) {
  auto pow2 = [](int64_t v) { return v > 0 && (v & (v - 1)) == 0; };
  if (K % kGroup != 0 || K > kMaxK) return 0;
  if (pow2(K)) return (int)K;
  if (K % 28 == 0 && pow2(K / 28)) return (int)(K / 28);
  return 0;
}

}  // namespace hd

bool hadamard_supported(int64_t K) { return hd::block_length(K) > 0; }

cudaError_t launch_hadamard_quantize(const uint16_t *x, int64_t M, int64_t K, int8_t *xq,
                                     float *xs, int32_t *xsum, cudaStream_t st) {
  const int p = hd::block_length(K);
  if (p == 0 || M > 0x7fffffff) return cudaErrorInvalidValue;
  int lp = 0;
  while ((1 << lp) < p) ++lp;
  const float norm = (float)(1.0 / sqrt((double)K));
  if (K == 28 * 512 && M <= hd::kClusterMaxM) {
    // decode sizes: a cluster of 7 CTAs per token
    auto kern = hd::hadamard_quantize_cluster_kernel;
    constexpr int smem = (int)sizeof(hd::ClusterSmem);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(hd::kClusterCtas, (unsigned)M);
    cfg.blockDim = dim3(hd::kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = hd::kClusterCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, x, norm, xq, xs, xsum);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const size_t smem = (size_t)K * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(hd::hadamard_quantize_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(hd::hadamard_quantize_kernel, dim3((unsigned)M), dim3(hd::kThreads), smem, st,
                 true, x, (int)K, lp, norm, xq, xs, xsum);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bitnest
