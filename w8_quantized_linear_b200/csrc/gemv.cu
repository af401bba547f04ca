// Decode GEMV of the bit-nested linear layer (M <= 8 tokens), CUDA cores.
//
// BitNest-Llama-3-8B model card, section "Files": the draft reads the hi
// plane only (W4 = (hi - 8) * scale), the target reads both planes
// (W8 = (16 (hi - 8) + (lo - 8)) * scale / 16).  Per 128-column group the
// integer sum is formed exactly with dp4a on unsigned operands:
//   draft : S = sum q * hi            - 8   * sum q
//   target: S = sum q * ((hi<<4)|lo)  - 136 * sum q      (16(h-8)+(l-8) = (h<<4|l) - 136)
// and y[m,n] = xscale * sum_g scale[n,g] * S (/16 for the target).
//
// Layout of the work: a warp owns R weight rows at a time and walks K in
// steps of 1024 columns (32 lanes x 16 bytes of a plane = 32 columns per
// lane).  The activations of all M tokens are staged once per CTA in shared
// memory, de-interleaved so that the low nibbles (even columns) and high
// nibbles (odd columns) of a plane word meet their activations without any
// per-row shuffling.
#include "common.cuh"
#include "launch.h"

namespace bitnest {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvSmemLimit = 200 * 1024;

// staged activations (M*K bytes) + one int32 activation sum per 32-column chunk
__host__ __device__ constexpr int64_t gemv_smem_bytes(int64_t M, int64_t K) {
  return M * K + M * (K / 32) * 4;
}

bool gemv_fits(int64_t M, int64_t K) {
  return M >= 1 && M <= 8 && gemv_smem_bytes(M, K) <= kGemvSmemLimit;
}

template <int MODE, int M, int R, int U, bool DEBUG>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const LinearArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int64_t K = a.K, N = a.N;
  const int C = (int)(K / 32);  // 32-column chunks per row
  const int G = (int)(K / kGroup);
  uint4 *xs4 = reinterpret_cast<uint4 *>(smem);                      // [M][2][C]
  int32_t *rsum = reinterpret_cast<int32_t *>(smem + (int64_t)M * K);  // [M][C]

  // ---- stage activations: chunk c of token m -> two 16-byte halves
  for (int item = threadIdx.x; item < M * C; item += kGemvThreads) {
    const int m = item / C, c = item - m * C;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.xq + (int64_t)m * K + 32 * c);
    const uint4 p = __ldg(src), q = __ldg(src + 1);
    // columns 8w..8w+7 are words (2w, 2w+1) of the 32-byte chunk
    const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    uint32_t e[4], o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      e[i] = prmt(w[2 * i], w[2 * i + 1], 0x6420);  // columns 8i + 0,2,4,6
      o[i] = prmt(w[2 * i], w[2 * i + 1], 0x7531);  // columns 8i + 1,3,5,7
    }
    xs4[(m * 2 + 0) * C + c] = make_uint4(e[0], o[0], e[1], o[1]);
    xs4[(m * 2 + 1) * C + c] = make_uint4(e[2], o[2], e[3], o[3]);
    // sum of the chunk's 32 activations: the per-lane offset correction keeps
    // every partial sum an exact integer multiple relation between the models
    int r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) r = __dp4a((int)w[i], 0x01010101, r);
    rsum[m * C + c] = r;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t row_groups = (N + R - 1) / R;
  const int nsteps = (C + 31) / 32;
  constexpr int OFF = CodeOffset<MODE>::value;
  const int64_t row_bytes = K / 2;

  for (int64_t rg = (int64_t)blockIdx.x * kGemvWarps + warp; rg < row_groups;
       rg += (int64_t)gridDim.x * kGemvWarps) {
    const int64_t n0 = rg * R;
    float acc[R][M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[r][m] = 0.0f;

    for (int i0 = 0; i0 < nsteps; i0 += U) {
      uint4 hv[U][R], lv[U][R];
      float sc[U][R];
      // issue every load of the U steps first
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = (i0 + u) * 32 + lane;
        const bool cok = (i0 + u < nsteps) && (c < C);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool ok = cok && (n0 + r < N);
          const int64_t off = (n0 + r) * row_bytes + 16 * (int64_t)c;
          hv[u][r] = ok ? ldg_stream16(a.hi + off) : make_uint4(0, 0, 0, 0);
          if (MODE == 1) lv[u][r] = ok ? ldg_stream16(a.lo + off) : make_uint4(0, 0, 0, 0);
          sc[u][r] = (ok && !DEBUG) ? __half2float(__ushort_as_half(__ldg(a.scale + (n0 + r) * G + c / 4)))
                        : 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = (i0 + u) * 32 + lane;
        // lanes past the end compute zeros (every lane must reach the shuffles;
        // C is a multiple of 4, so the 4 lanes of a group agree on `cok`)
        const bool cok = (i0 + u < nsteps) && (c < C);
        const int cc = cok ? c : 0;
        const int g = cc >> 2;
        // activations of this chunk for every token (shared by the R rows)
        uint4 xa[M], xb[M];
        int corr[M];
        float xg[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          xa[m] = cok ? xs4[(m * 2 + 0) * C + cc] : make_uint4(0, 0, 0, 0);
          xb[m] = cok ? xs4[(m * 2 + 1) * C + cc] : make_uint4(0, 0, 0, 0);
          // offset correction of this lane's 32 columns
          corr[m] = cok ? OFF * rsum[m * C + cc] : 0;
          xg[m] = a.act_group ? __ldg(a.xscale + m * G + g) : 1.0f;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t h[4] = {hv[u][r].x, hv[u][r].y, hv[u][r].z, hv[u][r].w};
          uint32_t ev[4], od[4];  // operand bytes of even / odd columns
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            if (MODE == 0) {
              ev[w] = h[w] & 0x0F0F0F0Fu;
              od[w] = (h[w] >> 4) & 0x0F0F0F0Fu;
            } else {
              const uint32_t l[4] = {lv[u][r].x, lv[u][r].y, lv[u][r].z, lv[u][r].w};
              ev[w] = ((h[w] << 4) & 0xF0F0F0F0u) | (l[w] & 0x0F0F0F0Fu);
              od[w] = (h[w] & 0xF0F0F0F0u) | ((l[w] >> 4) & 0x0F0F0F0Fu);
            }
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            int p = -corr[m];
            p = dp4a_us(ev[0], xa[m].x, p);
            p = dp4a_us(od[0], xa[m].y, p);
            p = dp4a_us(ev[1], xa[m].z, p);
            p = dp4a_us(od[1], xa[m].w, p);
            p = dp4a_us(ev[2], xb[m].x, p);
            p = dp4a_us(od[2], xb[m].y, p);
            p = dp4a_us(ev[3], xb[m].z, p);
            p = dp4a_us(od[3], xb[m].w, p);
            if (DEBUG) {
              // exact group sum: the 4 lanes of a group are consecutive
              int s = p + __shfl_xor_sync(0xffffffffu, p, 1);
              s += __shfl_xor_sync(0xffffffffu, s, 2);
              if (cok && (cc & 3) == 0 && n0 + r < N) a.S[((int64_t)m * N + n0 + r) * G + g] = s;
            } else {
              const float f = (float)p;  // |p| < 2^24: exact
              acc[r][m] = a.act_group ? fmaf(f, sc[u][r] * xg[m], acc[r][m])
                                      : fmaf(f, sc[u][r], acc[r][m]);
            }
          }
        }
      }
    }
    if (!DEBUG) {
      // ---- epilogue: reduce over the warp, apply token scale (and 1/16)
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < M; ++m) acc[r][m] = warp_sum(acc[r][m]);
      if (lane < R * M) {
        const int r = lane / M, m = lane % M;
        float v = 0.0f;
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
#pragma unroll
          for (int mm = 0; mm < M; ++mm)
            if (rr == r && mm == m) v = acc[rr][mm];
        const int64_t n = n0 + r;
        if (n < N) {
          float out = a.act_group ? v : v * __ldg(a.xscale + m);
          if (MODE == 1) out *= 0.0625f;
          if (a.bias) out += __half2float(__ushort_as_half(__ldg(a.bias + n)));
          a.y[(int64_t)m * N + n] = out;
        }
      }
    }
  }
}

template <int MODE, int M, int R, int U, bool DEBUG>
static cudaError_t launch_gemv_t(const LinearArgs &a, cudaStream_t st) {
  auto kern = gemv_kernel<MODE, M, R, U, DEBUG>;
  const int64_t smem = gemv_smem_bytes(M, a.K);
  // per device: the shared-memory limit set so far and the occupancy at it
  static int set_smem[64] = {0};
  static int occ_smem[64] = {-1};
  static int occ[64] = {0};
  static int sms[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > 48 * 1024 && smem > set_smem[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    set_smem[dev] = (int)smem;
  }
  if (sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  if (occ_smem[dev] != (int)smem) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, (size_t)smem);
    if (e != cudaSuccess) return e;
    occ[dev] = per_sm < 1 ? 1 : per_sm;
    occ_smem[dev] = (int)smem;
  }
  const int64_t row_groups = (a.N + R - 1) / R;
  int64_t blocks = (row_groups + kGemvWarps - 1) / kGemvWarps;
  const int64_t cap = (int64_t)sms[dev] * occ[dev];
  if (blocks > cap) blocks = cap;
  kern<<<(unsigned)blocks, kGemvThreads, (size_t)smem, st>>>(a);
  return cudaGetLastError();
}

// Rows per warp: enough row groups to give every SM several warps.
template <int MODE, int M, bool DEBUG>
static cudaError_t dispatch_rows(const LinearArgs &a, cudaStream_t st) {
  if (DEBUG) return launch_gemv_t<MODE, M, 1, 4, true>(a, st);
  if (a.N >= 8192) return launch_gemv_t<MODE, M, 2, 4, false>(a, st);
  return launch_gemv_t<MODE, M, 1, 4, false>(a, st);
}

template <int MODE, bool DEBUG>
static cudaError_t dispatch_m(const LinearArgs &a, cudaStream_t st) {
  switch (a.M) {
    case 1: return dispatch_rows<MODE, 1, DEBUG>(a, st);
    case 2: return dispatch_rows<MODE, 2, DEBUG>(a, st);
    case 3: return dispatch_rows<MODE, 3, DEBUG>(a, st);
    case 4: return dispatch_rows<MODE, 4, DEBUG>(a, st);
    case 5: return dispatch_rows<MODE, 5, DEBUG>(a, st);
    case 6: return dispatch_rows<MODE, 6, DEBUG>(a, st);
    case 7: return dispatch_rows<MODE, 7, DEBUG>(a, st);
    case 8: return dispatch_rows<MODE, 8, DEBUG>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(const LinearArgs &a, cudaStream_t st) {
  const bool debug = a.S != nullptr;
  if (a.mode == 0) return debug ? dispatch_m<0, true>(a, st) : dispatch_m<0, false>(a, st);
  return debug ? dispatch_m<1, true>(a, st) : dispatch_m<1, false>(a, st);
}

}  // namespace bitnest
