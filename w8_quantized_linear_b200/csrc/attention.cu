// Decode attention over a nested KV cache (BitNest-Llama-3-8B model card,
// model table row "KV cache": nested at runtime, the draft reads KV4, the
// target KV8).  The cache uses the weights' nesting: every K (V) row of one
// token and one KV head (head_dim 128 = one group) is an 8-bit code split
// into a hi and a lo nibble plane with an fp16 scale (packed at runtime with
// bitnest_pack_weights); the draft dequantises (hi - 8) s and reads only the
// hi plane, the target (16 (hi - 8) + (lo - 8)) s / 16 from both.
//
// One new token: head h (of H) attends with KV head h / (H / Hkv) over the T
// cached tokens, softmax(q K^T / sqrt(D)) V.
//
// The cache is a pure HBM stream (130 or 260 bytes per token and KV head),
// so the tokens of a KV head are split over a cluster of up to 16 CTAs (two
// per SM: eight warps each, at most 128 registers a thread), every warp takes
// tiles of 16 tokens, and each CTA stores its partial softmax state into the
// shared memory of the cluster's first CTA (remote stores, no round trip),
// which merges them: one launch, no global scratch.
//
// Both products run on the tensor cores (mma.sync m16n8k16, fp16 inputs,
// fp32 accumulation), on the integer codes themselves, exact in fp16; the
// scales are applied in fp32:
//   scores:  S = Q K^T: A = the group's queries (rows = heads), B = codes of
//            16 tokens; the K (column) order is permuted so that a lane's
//            codes are one 16-byte piece of each plane row; score =
//            S * k_scale * 1/sqrt(D) in fp32;
//   output:  O^T = V^T P'^T with P' = p * v_scale * 2^-E split into two fp16
//            terms (hi + lo, 22 bits together); 2^E, per warp and tile, puts
//            the tile's largest v_scale in [1/2, 1), so P' stays clear of the
//            fp16 subnormals, and the running output is kept in units of the
//            last tile's 2^E (exact power-of-two rescales); A = codes of V
//            (rows = columns of V in a permuted order: a lane reads 8 bytes of
//            each plane row).
// The scores' accumulator layout is exactly the B operand the output product
// needs, so p never leaves the registers.  Online softmax per warp over its
// tiles; warps, then CTAs, merged with max-rescaling.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace bitnest {

namespace attn {

constexpr int kD = 128;       // head dimension (one scale group)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSplit = 16;
constexpr int kTile = 16;     // tokens per warp step

// D = A (16x16 f16, row) * B (16x8 f16, col) + C, fp32
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte codes u of 8 columns from one 32-bit word of each plane: even columns
// (the low nibbles) in `ev`, odd columns in `od`, byte b for plane byte b.
// Draft: u = hi nibble; target: u = (hi << 4) | lo.
template <int MODE>
__device__ __forceinline__ void codes(uint32_t hw, uint32_t lw, uint32_t &ev, uint32_t &od) {
  if (MODE == 0) {
    ev = hw & 0x0F0F0F0Fu;
    od = (hw >> 4) & 0x0F0F0F0Fu;
  } else {
    ev = ((hw << 4) & 0xF0F0F0F0u) | (lw & 0x0F0F0F0Fu);
    od = (hw & 0xF0F0F0F0u) | ((lw >> 4) & 0x0F0F0F0Fu);
  }
}

// fp16 pair (byte b of x, byte b of y) as codes u - offset: 0x6400 | u is the
// half 1024 + u, and 1024 + u - (1024 + offset) is exact.
template <int MODE>
__device__ __forceinline__ uint32_t pair(uint32_t x, uint32_t y, int b) {
  const uint32_t sel = (uint32_t)b | ((uint32_t)(b + 4) << 8);
  const uint32_t t = (prmt(x, y, sel) & 0x00FF00FFu) | 0x64006400u;
  // -(1024 + offset) in both halves: -1032 (draft) = 0xE408, -1160 (target) = 0xE488
  constexpr uint32_t kOff = MODE ? 0xE488E488u : 0xE408E408u;
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(kOff));
  return r;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float half_bits(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Cluster helpers (distributed shared memory).
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// distributed shared memory is used only once every CTA of the cluster has
// started: each thread arrives at entry and waits before its first access
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// Store v at the same shared-memory offset as `p` in CTA `rank` of the cluster.
__device__ __forceinline__ void st_cluster(float *p, uint32_t rank, float v) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// Shared memory (dynamic): the warps' states, then the cluster's CTAs'
// merged states (filled in the first CTA only).
template <int GQ>
struct Smem {
  float m[kWarps][GQ], l[kWarps][GQ];
  float o[kWarps][GQ][kD];
  float pm[kMaxSplit][GQ], pl[kMaxSplit][GQ];
  float po[kMaxSplit][GQ][kD];
};

// One tile's loads for one lane (gid = lane / 4, tig = lane % 4): K rows of
// tokens gid and 8 + gid (16 bytes of each plane at byte 16 tig), V rows of
// tokens 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 (8 bytes at byte 8 gid), and
// the K / V scales of those four tokens.  Tokens at or past t_end read zeros.
struct TileRegs {
  uint4 kh[2], kl[2];
  uint2 vh[4], vl[4];
  uint16_t ks[4], vs[4];
};

template <int MODE>
__device__ __forceinline__ void load_tile(TileRegs &r, int t0, int t_end, int64_t Hkv, int j,
                                          int gid, int tig, const uint8_t *__restrict__ k_hi,
                                          const uint8_t *__restrict__ k_lo,
                                          const uint16_t *__restrict__ k_scale,
                                          const uint8_t *__restrict__ v_hi,
                                          const uint8_t *__restrict__ v_lo,
                                          const uint16_t *__restrict__ v_scale) {
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int t = t0 + 8 * n + gid;
    r.kh[n] = r.kl[n] = make_uint4(0, 0, 0, 0);
    if (t < t_end) {
      const int64_t off = ((int64_t)t * Hkv + j) * (kD / 2) + 16 * tig;
      r.kh[n] = __ldg(reinterpret_cast<const uint4 *>(k_hi + off));
      if (MODE) r.kl[n] = __ldg(reinterpret_cast<const uint4 *>(k_lo + off));
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + 2 * tig + (i & 1) + 8 * (i >> 1);
    r.vh[i] = r.vl[i] = make_uint2(0, 0);
    r.ks[i] = r.vs[i] = 0;
    if (t < t_end) {
      const int64_t row = (int64_t)t * Hkv + j;
      const int64_t off = row * (kD / 2) + 8 * gid;
      r.vh[i] = __ldg(reinterpret_cast<const uint2 *>(v_hi + off));
      if (MODE) r.vl[i] = __ldg(reinterpret_cast<const uint2 *>(v_lo + off));
      r.ks[i] = __ldg(k_scale + row);
      r.vs[i] = __ldg(v_scale + row);
    }
  }
}

template <int MODE, int GQ>
__global__ void __launch_bounds__(kThreads, 2) nested_attention_kernel(
    const uint16_t *__restrict__ q, int Hkv, int T, int per_cta,
    const uint8_t *__restrict__ k_hi, const uint8_t *__restrict__ k_lo,
    const uint16_t *__restrict__ k_scale, const uint8_t *__restrict__ v_hi,
    const uint8_t *__restrict__ v_lo, const uint16_t *__restrict__ v_scale,
    float *__restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem<GQ> &sh = *reinterpret_cast<Smem<GQ> *>(smem_raw);
  const int j = blockIdx.y;         // KV head
  const int split = blockIdx.x;     // this CTA's token range (its rank in the cluster)
  const int nsplit = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int c_begin = split * per_cta;
  const int c_end = min(T, c_begin + per_cta);
  cluster_arrive();
  griddep_wait();  // q (and the cache) may come from the preceding kernel
  griddep_launch_dependents();

  // queries of head gid of the group as the scores' A operand: k-step ks,
  // K slots 2 tig, 2 tig + 1 <- columns 32 tig + 4 ks + {0, 1}, slots 2 tig + 8,
  // 2 tig + 9 <- columns 32 tig + 4 ks + {2, 3}; rows 8..15 (a1, a3) are zero
  uint32_t qa[8][2];
  {
    uint4 qv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    if (gid < GQ) {
      const uint4 *qr = reinterpret_cast<const uint4 *>(q + (int64_t)(j * GQ + gid) * kD + 32 * tig);
      qv[0] = __ldg(qr);
      qv[1] = __ldg(qr + 1);
      uint4 q2 = __ldg(qr + 2), q3 = __ldg(qr + 3);
      const uint32_t w[16] = {qv[0].x, qv[0].y, qv[0].z, qv[0].w, qv[1].x, qv[1].y, qv[1].z,
                              qv[1].w, q2.x,    q2.y,    q2.z,    q2.w,    q3.x,    q3.y,
                              q3.z,    q3.w};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {  // columns 4 ks .. 4 ks + 3 = halves 2 ks, 2 ks + 1
        qa[ks][0] = w[2 * ks];
        qa[ks][1] = w[2 * ks + 1];
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) qa[ks][0] = qa[ks][1] = 0u;
    }
  }
  const float rsd = 0.088388347648318440550f;  // 1 / sqrt(128)

  float m_run = -INFINITY, l_run = 0.0f;  // head gid (lanes gid < GQ)
  int e_run = 0;                          // o holds the output in units of 2^e_run
  float o[8][4];                          // O^T fragments: m-tile mt, heads 2 tig, 2 tig + 1
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[mt][i] = 0.0f;

  const int ntiles = (c_end - c_begin + kTile - 1) / kTile;  // <= 0 for an empty range
  for (int ti = warp; ti < ntiles; ti += kWarps) {
    const int t0 = c_begin + ti * kTile;
    TileRegs cur;
    load_tile<MODE>(cur, t0, c_end, Hkv, j, gid, tig, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale);

    // ------------------------------------------------ scores of 16 tokens
    float s[4];  // tokens 2 tig, 2 tig + 1, 8 + 2 tig, 9 + 2 tig of head gid
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const uint32_t hw[4] = {cur.kh[n].x, cur.kh[n].y, cur.kh[n].z, cur.kh[n].w};
      const uint32_t lw[4] = {cur.kl[n].x, cur.kl[n].y, cur.kl[n].z, cur.kl[n].w};
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int w = 0; w < 4; ++w) {  // plane word w: bytes 4 w .. 4 w + 3 = k-steps 2 w, 2 w + 1
        uint32_t ev, od;
        codes<MODE>(hw[w], lw[w], ev, od);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ks = 2 * w + h;
          mma_f16(d, qa[ks][0], 0u, qa[ks][1], 0u, pair<MODE>(ev, od, 2 * h),
                  pair<MODE>(ev, od, 2 * h + 1));
        }
      }
      s[2 * n] = d[0];
      s[2 * n + 1] = d[1];
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + 2 * tig + (i & 1) + 8 * (i >> 1);
      float f = half_bits(cur.ks[i]);
      if (MODE) f *= 0.0625f;
      s[i] = (t < c_end && gid < GQ) ? s[i] * f * rsd : -INFINITY;
      tmax = fmaxf(tmax, s[i]);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    // online softmax of head gid (a head with no token yet keeps corr = 1)
    const float m_new = fmaxf(m_run, tmax);
    const bool live = m_new != -INFINITY;
    const float corr = live ? __expf(m_run - m_new) : 1.0f;
    float p[4], psum = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p[i] = live ? __expf(s[i] - m_new) : 0.0f;
      psum += p[i];
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l_run = l_run * corr + psum;
    m_run = m_new;
    // p' = p * v_scale (/ 16) * 2^-e as hi + lo fp16 terms: the B operand of
    // the output product (k = token, n = head gid); 2^e from the tile's
    // largest v_scale (the same in every lane), 0 when they are all zero
    float vf[4], vmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      vf[i] = half_bits(cur.vs[i]);
      if (MODE) vf[i] *= 0.0625f;
      vmax = fmaxf(vmax, vf[i]);
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o2));
    // vmax = f 2^(b - 127), f in [1, 2): e = b - 126 puts vmax 2^-e in [1/2, 1)
    const int e_tile = vmax > 0.0f ? (int)((__float_as_uint(vmax) >> 23) & 0xFFu) - 126 : e_run;
    const float down = __uint_as_float((uint32_t)(127 - e_tile) << 23);  // 2^-e_tile
    float pv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pv[i] = p[i] * vf[i] * down;
    const uint32_t bh0 = pack_half2(pv[0], pv[1]), bh1 = pack_half2(pv[2], pv[3]);
    const float2 r0 = __half22float2(*reinterpret_cast<const __half2 *>(&bh0));
    const float2 r1 = __half22float2(*reinterpret_cast<const __half2 *>(&bh1));
    const uint32_t bl0 = pack_half2(pv[0] - r0.x, pv[1] - r0.y);
    const uint32_t bl1 = pack_half2(pv[2] - r1.x, pv[3] - r1.y);
    // rescale the output of heads 2 tig, 2 tig + 1 (their corr is held by
    // lanes 8 tig, 8 tig + 4) and from units 2^e_run to 2^e_tile
    const float unit = __uint_as_float((uint32_t)(127 + e_run - e_tile) << 23);
    const float c0 = __shfl_sync(0xffffffffu, corr, 8 * tig) * unit;
    const float c1 = __shfl_sync(0xffffffffu, corr, 8 * tig + 4) * unit;
    e_run = e_tile;
    // the running maxima and the unit settle after a few tiles: then the
    // output needs no rescaling
    const bool rescale = __any_sync(0xffffffffu, c0 != 1.0f || c1 != 1.0f);
    // ------------------------------------------------ O^T += V^T P'^T
    uint32_t ev[4][2], od[4][2];  // tokens 2 tig, 2 tig + 1, 8 + 2 tig, 9 + 2 tig; bytes 0..7
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      codes<MODE>(cur.vh[i].x, cur.vl[i].x, ev[i][0], od[i][0]);
      codes<MODE>(cur.vh[i].y, cur.vl[i].y, ev[i][1], od[i][1]);
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {  // plane byte 8 gid + mt: columns 16 gid + 2 mt, + 1
      const int w = mt >> 2, b = mt & 3;
      const uint32_t a0 = pair<MODE>(ev[0][w], ev[1][w], b);  // even column, tokens 2 tig, + 1
      const uint32_t a1 = pair<MODE>(od[0][w], od[1][w], b);  // odd column
      const uint32_t a2 = pair<MODE>(ev[2][w], ev[3][w], b);  // tokens 8 + 2 tig, 9 + 2 tig
      const uint32_t a3 = pair<MODE>(od[2][w], od[3][w], b);
      if (rescale) {
        o[mt][0] *= c0;
        o[mt][1] *= c1;
        o[mt][2] *= c0;
        o[mt][3] *= c1;
      }
      mma_f16(o[mt], a0, a1, a2, a3, bh0, bh1);
      mma_f16(o[mt], a0, a1, a2, a3, bl0, bl1);
    }
  }

  // ------------------------------------------------ merge the warps
  {  // the output back from units of 2^e_run
    const float up = __uint_as_float((uint32_t)(127 + e_run) << 23);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[mt][i] *= up;
  }
  if (gid < GQ && tig == 0) {
    sh.m[warp][gid] = m_run;
    sh.l[warp][gid] = l_run;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int col = 16 * gid + 2 * mt;
    if (2 * tig < GQ) {
      sh.o[warp][2 * tig][col] = o[mt][0];
      sh.o[warp][2 * tig][col + 1] = o[mt][2];
    }
    if (2 * tig + 1 < GQ) {
      sh.o[warp][2 * tig + 1][col] = o[mt][1];
      sh.o[warp][2 * tig + 1][col + 1] = o[mt][3];
    }
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster has started
  // this CTA's state, merged over its warps, into slot `split` of the first
  // CTA of the cluster
  const uint32_t rank = cluster_rank();
  for (int e = threadIdx.x; e < GQ * kD; e += kThreads) {
    const int g = e / kD, c = e - g * kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh.m[w][g]);
    float num = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (sh.m[w][g] == -INFINITY) continue;  // a warp that saw no token
        const float f = __expf(sh.m[w][g] - M);
        num += f * sh.o[w][g][c];
        den += f * sh.l[w][g];
      }
    }
    st_cluster(&sh.po[rank][g][c], 0u, num);
    if (c == 0) {
      st_cluster(&sh.pm[rank][g], 0u, M);
      st_cluster(&sh.pl[rank][g], 0u, den);
    }
  }
  cluster_sync();  // every CTA's state is in the first CTA
  if (rank == 0) {
    for (int e = threadIdx.x; e < GQ * kD; e += kThreads) {
      const int g = e / kD, c = e - g * kD;
      float M = -INFINITY;
      for (int r = 0; r < nsplit; ++r) M = fmaxf(M, sh.pm[r][g]);
      float num = 0.0f, den = 0.0f;
      for (int r = 0; r < nsplit; ++r) {
        const float mr = sh.pm[r][g];
        if (mr == -INFINITY) continue;  // a CTA that saw no token
        const float f = __expf(mr - M);
        num += f * sh.po[r][g][c];
        den += f * sh.pl[r][g];
      }
      out[(int64_t)(j * GQ + g) * kD + c] = num / den;
    }
  }
}

// Tokens per CTA: a cluster of up to 16 CTAs per KV head, each at least 64
// tokens (a multiple of 16).
inline int split_count(int64_t T, int max_split) {
  int s = (int)((T + 63) / 64);
  return s < 1 ? 1 : (s > max_split ? max_split : s);
}

template <int MODE, int GQ>
cudaError_t launch_g(const uint16_t *q, int64_t Hkv, int64_t T, const uint8_t *k_hi,
                     const uint8_t *k_lo, const uint16_t *k_scale, const uint8_t *v_hi,
                     const uint8_t *v_lo, const uint16_t *v_scale, float *out, cudaStream_t st) {
  auto kern = nested_attention_kernel<MODE, GQ>;
  // 16-CTA clusters are past the portable size: ask for them, and fall back
  // to 8 where the device will not place them
  for (int max_split = kMaxSplit; max_split >= 8; max_split /= 2) {
    const int S = split_count(T, max_split);
    const int per = (int)(((T + S - 1) / S + kTile - 1) / kTile * kTile);
    if (S > 8) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) {
        (void)cudaGetLastError();
        continue;
      }
    }
    constexpr int smem = (int)sizeof(Smem<GQ>);
    cudaError_t e0 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e0 != cudaSuccess) return e0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)Hkv);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    if (S > 8) {
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        continue;
      }
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, q, (int)Hkv, (int)T, per, k_hi, k_lo, k_scale,
                                       v_hi, v_lo, v_scale, out);
    if (e == cudaSuccess) return cudaSuccess;
    if (S <= 8) return e;
    (void)cudaGetLastError();
  }
  return cudaErrorLaunchFailure;
}

template <int MODE>
cudaError_t launch_mode(const uint16_t *q, int64_t H, int64_t Hkv, int64_t T, const uint8_t *k_hi,
                        const uint8_t *k_lo, const uint16_t *k_scale, const uint8_t *v_hi,
                        const uint8_t *v_lo, const uint16_t *v_scale, float *out,
                        cudaStream_t st) {
  switch (H / Hkv) {
    case 1: return launch_g<MODE, 1>(q, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale, out, st);
    case 2: return launch_g<MODE, 2>(q, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale, out, st);
    case 4: return launch_g<MODE, 4>(q, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale, out, st);
    case 8: return launch_g<MODE, 8>(q, Hkv, T, k_hi, k_lo, k_scale, v_hi, v_lo, v_scale, out, st);
    default: return cudaErrorInvalidValue;
  }
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
