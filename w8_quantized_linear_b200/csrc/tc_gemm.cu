// tcgen05 tensor-core path of the bit-nested linear layer (any M).
//
// BitNest-Llama-3-8B model card, section "Files": the draft weight code is
// hi - 8 and the target code 16 (hi - 8) + (lo - 8) = ((hi << 4) | lo) - 136.
// Both are formed here as ONE unsigned byte per weight (hi, or (hi<<4)|lo)
// so a single kind::i8 MMA (u8 weights x s8 activations -> s32) per 32
// columns does the work; the constant offset (8 or 136) times the
// activation group sum is folded into the epilogue.
//
// Tile: 128 weight rows (the MMA's M, TMEM lanes) x BT tokens (the MMA's N),
// one 128-column group per pipeline stage.  The group scales differ per
// (row, group), so the int32 accumulator of every group is drained from TMEM
// and scaled in fp32; two TMEM accumulators let the drain of group g overlap
// the MMA of group g + 1.
//
// Warp roles (15 warps):
//   0      TMA producer: activation tile (128-byte swizzle) and the hi / lo
//          plane tiles of the group, one mbarrier per stage (no multicast)
//   1      TMEM owner and MMA issuer (one thread)
//   2      per-group column constants: magic - offset * activation group sum
//          (and the per-group activation scale for o_proj-style inputs)
//   3..6   plane -> byte transform into the swizzled K-major MMA operand
//   7..14  epilogue: TMEM -> registers, exact int -> fp32, scale, accumulate
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace bitnest {

namespace tc {

constexpr int BW = 128;  // weight rows per tile
constexpr int kMaxStages = 4;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpPrep = 2;
constexpr int kWarpXf0 = 3, kNumXf = 4;
constexpr int kWarpEpi0 = 7, kNumEpi = 8;
constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;
// 1.5 * 2^23: adding an integer |s| < 2^22 to this bit pattern gives the
// float 1.5 * 2^23 + s exactly, so int -> float is one integer add.
constexpr int kMagicI = 0x4B400000;
constexpr float kMagicF = 12582912.0f;

struct Params {
  const uint16_t *scale;   // fp16 [N, G]
  const float *xscale;     // [M] or [M, G]
  const int32_t *xsum;     // [M, G]
  const uint16_t *bias;    // [N] or null
  float *y;                // [M, N]
  int32_t *S;              // debug sums [M, N, G]
  int M, N, G;
  int act_group;
  int stages;
  int sc_pitch;            // halves per row of the staged scale block (odd word count)
};

__host__ __device__ constexpr int tmem_cols(int bt) {
  return 2 * bt < 32 ? 32 : 2 * bt;  // 2 * bt is a power of two for bt in {16,32,64,128}
}

struct Layout {
  int a, b, h, l, sc, cv, xv, bars, total;
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout smem_layout(int mode, int bt, int stages, int G, int pitch) {
  Layout L;
  int o = 0;
  L.a = o;
  o += stages * BW * 128;
  L.b = o;
  o += stages * bt * 128;
  L.h = o;
  o += stages * BW * 64;
  L.l = o;
  o += mode ? stages * BW * 64 : 0;
  L.sc = o;
  o += align_up(BW * pitch * 2, 16);
  L.cv = o;
  o += stages * bt * 4;
  L.xv = o;
  o += stages * bt * 4;
  o = align_up(o, 8);
  L.bars = o;
  o += (5 * kMaxStages + 4) * 8 + 16;
  L.total = o + 1024;  // slack to align the base to 1024 bytes
  return L;
}

template <int MODE, int BT, bool DEBUG>
__global__ void __launch_bounds__(kThreads, 1)
    tc_linear_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, const Params p) {
  constexpr int OFF = CodeOffset<MODE>::value;
  constexpr int COLS = BT / 2;            // columns per epilogue warp
  constexpr int CH = COLS < 32 ? COLS : 32;  // columns per TMEM load
  constexpr uint32_t IDESC = umma_idesc_u8s8(BW, BT);
  constexpr int TCOLS = tmem_cols(BT);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int S = p.stages, G = p.G;
  const Layout L = smem_layout(MODE, BT, S, G, p.sc_pitch);
  uint8_t *sA = smem + L.a;
  uint8_t *sB = smem + L.b;
  uint8_t *sH = smem + L.h;
  uint8_t *sL = smem + L.l;
  __half *sSc = reinterpret_cast<__half *>(smem + L.sc);
  int32_t *sCv = reinterpret_cast<int32_t *>(smem + L.cv);
  float *sXv = reinterpret_cast<float *>(smem + L.xv);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *fullIn = bars;                    // TMA landed (q, hi, lo)
  uint64_t *emptyIn = bars + kMaxStages;      // MMA done with the stage
  uint64_t *fullA = bars + 2 * kMaxStages;    // transformed operand written
  uint64_t *fullC = bars + 3 * kMaxStages;    // column constants written
  uint64_t *emptyC = bars + 4 * kMaxStages;   // epilogue done with the constants
  uint64_t *accFull = bars + 5 * kMaxStages;  // [2] accumulator ready
  uint64_t *accEmpty = accFull + 2;           // [2] accumulator drained
  uint32_t *tslot = reinterpret_cast<uint32_t *>(accEmpty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BW, m0 = blockIdx.y * BT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullIn[s], 1);
      mbar_init(&emptyIn[s], 1);
      mbar_init(&fullA[s], kNumXf);
      mbar_init(&fullC[s], 1);
      mbar_init(&emptyC[s], kNumEpi);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accFull[b], 1);
      mbar_init(&accEmpty[b], kNumEpi);
    }
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tslot, TCOLS);
    tmem_relinquish();
  }
  if (warp >= kWarpEpi0 && !DEBUG) {
    // stage this tile's group scales, [row][pitch] fp16 (odd word pitch: the
    // per-group column reads of 32 rows hit 32 different banks)
    const int t = threadIdx.x - kWarpEpi0 * 32;
    for (int i = t; i < BW * G; i += kNumEpi * 32) {
      const int r = i / G, g = i - r * G;
      const int n = n0 + r;
      const uint16_t v = n < p.N ? __ldg(p.scale + (int64_t)n * G + g) : (uint16_t)0;
      sSc[r * p.sc_pitch + g] = __ushort_as_half(v);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == kWarpTma) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_hi);
      if (MODE) prefetch_tmap(&tm_lo);
      const uint32_t bytes = BT * 128 + BW * 64 * (MODE ? 2 : 1);
      int issued = 0;
      for (int g = 0; g < G; ++g) {
        const int s = g % S;
        if (!mbar_wait(&emptyIn[s], ((g / S) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&fullIn[s], bytes);
        tma_load_2d(sB + s * BT * 128, &tm_q, &fullIn[s], g * 128, m0);
        tma_load_2d(sH + s * BW * 64, &tm_hi, &fullIn[s], g * 64, n0);
        if (MODE) tma_load_2d(sL + s * BW * 64, &tm_lo, &fullIn[s], g * 64, n0);
        ++issued;
      }
      if (issued < G) {  // gave up: let the copies already issued land
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(&fullIn[i % S], (i / S) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int g = 0; g < G && ok; ++g) {
        const int s = g % S, b = g & 1;
        ok = mbar_wait(&fullA[s], (g / S) & 1) && mbar_wait(&accEmpty[b], ((g >> 1) & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad = umma_desc_sw128(sA + s * BW * 128);
        const uint64_t bd = umma_desc_sw128(sB + s * BT * 128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 4 x K=32 bytes inside the 128-byte row
          umma_i8(tmem + b * BT, ad + 2 * kk, bd + 2 * kk, IDESC, kk > 0 ? 1u : 0u);
        umma_commit(&emptyIn[s]);
        umma_commit(&accFull[b]);
      }
      // the last accumulator must be complete before TMEM is released
      if (ok && G > 0) mbar_wait(&accFull[(G - 1) & 1], ((G - 1) >> 1) & 1);
    }
  } else if (warp == kWarpPrep) {
    // ------------------------------------- per-group column constants
    for (int g = 0; g < G; ++g) {
      const int s = g % S;
      if (!mbar_wait_warp(&emptyC[s], ((g / S) & 1) ^ 1)) break;
      for (int j = lane; j < BT; j += 32) {
        const int m = m0 + j;
        const int r = m < p.M ? __ldg(p.xsum + (int64_t)m * G + g) : 0;
        sCv[s * BT + j] = kMagicI - OFF * r;
        if (p.act_group) sXv[s * BT + j] = m < p.M ? __ldg(p.xscale + (int64_t)m * G + g) : 0.0f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&fullC[s]);
    }
  } else if (warp < kWarpEpi0) {
    // ------------------------------------------ plane -> operand bytes
    const int t = threadIdx.x - kWarpXf0 * 32;  // 0..127
    const int qd = t & 3;                         // 32-column quarter of the group
    for (int g = 0; g < G; ++g) {
      const int s = g % S;
      if (!mbar_wait_warp(&fullIn[s], (g / S) & 1)) break;
      const uint8_t *hs = sH + s * BW * 64;
      const uint8_t *ls = sL + s * BW * 64;
      uint8_t *as = sA + s * BW * 128;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int r = pass * 32 + (t >> 2);
        const uint4 h = *reinterpret_cast<const uint4 *>(hs + r * 64 + qd * 16);
        uint4 l = make_uint4(0, 0, 0, 0);
        if (MODE) l = *reinterpret_cast<const uint4 *>(ls + r * 64 + qd * 16);
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
        const uint32_t lw[4] = {l.x, l.y, l.z, l.w};
        uint32_t out[8];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t ev, od;  // bytes of columns 8w + {0,2,4,6} and 8w + {1,3,5,7}
          if (MODE == 0) {
            ev = hw[w] & 0x0F0F0F0Fu;
            od = (hw[w] >> 4) & 0x0F0F0F0Fu;
          } else {
            ev = ((hw[w] << 4) & 0xF0F0F0F0u) | (lw[w] & 0x0F0F0F0Fu);
            od = (hw[w] & 0xF0F0F0F0u) | ((lw[w] >> 4) & 0x0F0F0F0Fu);
          }
          out[2 * w] = prmt(ev, od, 0x5140);      // columns 8w + 0..3
          out[2 * w + 1] = prmt(ev, od, 0x7362);  // columns 8w + 4..7
        }
        // 16-byte chunks 2qd and 2qd+1 of the 128-byte row, 128-byte swizzle
        const int c0 = 2 * qd, c1 = 2 * qd + 1;
        *reinterpret_cast<uint4 *>(as + r * 128 + ((c0 ^ (r & 7)) << 4)) =
            make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4 *>(as + r * 128 + ((c1 ^ (r & 7)) << 4)) =
            make_uint4(out[4], out[5], out[6], out[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&fullA[s]);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int e = warp - kWarpEpi0;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = e >> 2;
    const int row = quarter * 32 + lane;
    const int n = n0 + row;
    const int col0 = half * COLS;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    float acc[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) acc[j] = 0.0f;
    for (int g = 0; g < G; ++g) {
      const int s = g % S, b = g & 1;
      if (!mbar_wait_warp(&fullC[s], (g / S) & 1)) break;
      if (!mbar_wait_warp(&accFull[b], (g >> 1) & 1)) break;
      tc_fence_after();
      const float sg = DEBUG ? 0.0f : __half2float(sSc[row * p.sc_pitch + g]);
      const int32_t *cv = sCv + s * BT + col0;
      const float *xv = sXv + s * BT + col0;
#pragma unroll
      for (int c = 0; c < COLS; c += CH) {
        uint32_t d[CH];
        tmem_ld<CH>(tmem + lane_addr + b * BT + col0 + c, d);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const int bits = (int)d[j] + cv[c + j];  // 1.5 * 2^23 + exact group sum
          if (DEBUG) {
            const int m = m0 + col0 + c + j;
            if (m < p.M && n < p.N) p.S[((int64_t)m * p.N + n) * G + g] = bits - kMagicI;
          } else {
            const float f = __int_as_float(bits) - kMagicF;
            acc[c + j] = p.act_group ? fmaf(f, sg * xv[c + j], acc[c + j])
                                     : fmaf(f, sg, acc[c + j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accEmpty[b]);
        mbar_arrive(&emptyC[s]);
      }
    }
    if (!DEBUG && n < p.N) {
      const float bias = p.bias ? __half2float(__ushort_as_half(__ldg(p.bias + n))) : 0.0f;
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        const int m = m0 + col0 + j;
        if (m < p.M) {
          float out = p.act_group ? acc[j] : acc[j] * __ldg(p.xscale + m);
          if (MODE) out *= 0.0625f;
          p.y[(int64_t)m * p.N + n] = out + bias;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

// ----------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2D uint8 tensor map: rows x cols (cols contiguous), box box_rows x box_cols.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int pick_bt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

int sc_pitch(int G) {
  int words = (G + 1) / 2;
  words |= 1;  // odd number of 32-bit words per row
  return 2 * words;
}

int pick_stages(int mode, int bt, int G, int max_smem) {
  for (int s = kMaxStages; s >= 2; --s)
    if (smem_layout(mode, bt, s, G, sc_pitch(G)).total <= max_smem) return s;
  return 0;
}

constexpr int kMaxSmem = 227 * 1024;

template <int MODE, int BT, bool DEBUG>
cudaError_t launch_t(const LinearArgs &a, cudaStream_t st) {
  const int G = (int)(a.K / kGroup);
  const int stages = pick_stages(MODE, BT, G, kMaxSmem);
  if (stages == 0) return cudaErrorInvalidValue;
  const int pitch = sc_pitch(G);
  const Layout L = smem_layout(MODE, BT, stages, G, pitch);
  CUtensorMap mq, mh, ml;
  if (!make_map(&mq, a.xq, (uint64_t)a.M, (uint64_t)a.K, BT, 128,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mh, a.hi, (uint64_t)a.N, (uint64_t)(a.K / 2), BW, 64,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (MODE) {
    if (!make_map(&ml, a.lo, (uint64_t)a.N, (uint64_t)(a.K / 2), BW, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    ml = mh;
  }
  Params p;
  p.scale = a.scale;
  p.xscale = a.xscale;
  p.xsum = a.xsum;
  p.bias = a.bias;
  p.y = a.y;
  p.S = a.S;
  p.M = (int)a.M;
  p.N = (int)a.N;
  p.G = G;
  p.act_group = a.act_group;
  p.stages = stages;
  p.sc_pitch = pitch;
  auto kern = tc_linear_kernel<MODE, BT, DEBUG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.N + BW - 1) / BW), (unsigned)((a.M + BT - 1) / BT));
  kern<<<grid, kThreads, L.total, st>>>(mq, mh, ml, p);
  return cudaGetLastError();
}

template <int MODE, bool DEBUG>
cudaError_t launch_mode(const LinearArgs &a, cudaStream_t st) {
  switch (pick_bt(a.M)) {
    case 16: return launch_t<MODE, 16, DEBUG>(a, st);
    case 32: return launch_t<MODE, 32, DEBUG>(a, st);
    case 64: return launch_t<MODE, 64, DEBUG>(a, st);
    default: return launch_t<MODE, 128, DEBUG>(a, st);
  }
}

}  // namespace tc

cudaError_t read_wait_timeout(int *flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_wait_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_wait_timeout, &zero, sizeof(int));
}

bool tc_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || M > (int64_t)1 << 30 || N > (int64_t)1 << 30) return false;
  const int G = (int)(K / kGroup);
  return tc::pick_stages(1, tc::pick_bt(M), G, tc::kMaxSmem) >= 2;
}

cudaError_t launch_tc(const LinearArgs &a, cudaStream_t st) {
  const bool debug = a.S != nullptr;
  if (a.mode == 0)
    return debug ? tc::launch_mode<0, true>(a, st) : tc::launch_mode<0, false>(a, st);
  return debug ? tc::launch_mode<1, true>(a, st) : tc::launch_mode<1, false>(a, st);
}

}  // namespace bitnest
