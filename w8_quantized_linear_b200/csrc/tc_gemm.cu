// tcgen05 tensor-core path of the bit-nested linear layer (any M; the
// prefill-sized GEMM and the middle of the batch sweep).
//
// BitNest-Llama-3-8B model card, section "Files": the draft weight code is
// hi - 8 and the target code 16 (hi - 8) + (lo - 8) = ((hi << 4) | lo) - 136.
// Both are formed here as ONE unsigned byte per weight (hi, or (hi<<4)|lo)
// so a single kind::i8 MMA (u8 weights x s8 activations -> s32) per 32
// columns does the work; the constant offset (8 or 136) times the
// activation group sum is removed in the drain.
//
// Tile: 128 weight rows (the MMA's M, TMEM lanes) x BT tokens (the MMA's N,
// up to 128), one 128-column group per pipeline stage.  The group scales
// differ per (row, group), so the int32 accumulator of every group is
// drained from TMEM and scaled in fp32 (the model card's per-group scale);
// three TMEM accumulators let the drain of a group run while the MMAs of the
// next two proceed.
//
// The weight operand never touches shared memory: each thread of the
// transform warps owns one weight row, reads its plane bytes of the group
// from a 64-byte-swizzled TMA tile (conflict-free, one row per lane) and
// writes the 128 operand bytes into a TMEM slot of the stage, from which the
// MMA reads A.  Shared memory then carries only the activation tile (the
// MMA's B), the plane tiles and the per-group constants: the operand's store
// and the MMA's reads of it were the bulk of the shared-memory traffic that
// bounded this kernel.
//
// The drain turns each int32 group sum into fp32 exactly with one integer
// add: the bit pattern of 1.5 * 2^23 minus offset * sum(q) (one constant per
// token and group) plus the raw sum is the float 1.5 * 2^23 + exact group
// sum (|sum| < 2^22); one packed subtract and one packed fma per two
// elements finish it.  The drain reads a whole group out of TMEM, hands the
// accumulator back to the MMA and only then does the arithmetic.
//
// The drain reads each accumulator in 32-column chunks, the load of the next
// chunk in flight while the current one is turned into fp32 sums.
// Persistent: one CTA per SM walks the tiles (token tiles fastest, so the
// CTAs of a wave share weight rows in L2) and every role runs ahead into the
// next tile while the epilogue finishes the current one.
//
// Warp roles (16 warps, four warpgroups):
//   0..3   plane -> byte operand (shared-memory planes -> TMEM, one row per
//          thread); without caller group sums also the tokens' sums of the
//          group (from the landed activation tile)
//   4      TMA producer: activation tile (128-byte swizzle) and the hi / lo
//          plane tiles of the group, one mbarrier per stage (this CTA only)
//   5, 6   MMA issuers (one thread each), even and odd groups; warp 5 owns
//          the tensor memory
//   7      per-group constants: row scales, per-token constants c (and the
//          per-group activation scales for o_proj)
//   8..15  epilogue: TMEM -> registers -> fp32 running sums (two warps per
//          TMEM lane quarter, half of the tokens each)
// The other warpgroups hand registers to the epilogue (setmaxnreg), which
// holds a tile row's running sums and a whole group of the accumulator.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace bitnest {

namespace tc {

constexpr int BW = 128;  // weight rows per tile
constexpr int kMaxStages = 8;
constexpr int kWarpXf0 = 0, kNumXf = 4;  // one warpgroup
constexpr int kXfThreads = 32 * kNumXf;
// two MMA issuers on alternate groups: one thread issues an MMA only every
// ~50 cycles, about as long as the tensor core takes to run one of 128 x 128
// x 32, so a single issuer with its waits between groups cannot keep it busy
constexpr int kWarpTma = kNumXf, kWarpMma0 = kNumXf + 1, kNumMma = 2;
constexpr int kWarpPrep = kNumXf + 3;
// groups' MMA completion: one barrier per group in a ring whose length is a
// multiple of the stage count (2, 3 or 4) and of the accumulator count (3)
constexpr int kDone = 12;
constexpr int kWarpEpi0 = kNumXf + 4, kNumEpi = 8;  // two epilogue warps per TMEM lane quarter
constexpr int kWarps = kWarpEpi0 + kNumEpi;
constexpr int kThreads = kWarps * 32;
// registers per thread at launch: 65536 / threads, rounded down to the
// allocation unit of 8
constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
// 1.5 * 2^23: its bit pattern plus an integer |s| < 2^22 is the float
// 1.5 * 2^23 + s exactly
constexpr uint32_t kMagicI = 0x4B400000u;
constexpr float kMagicF = 12582912.0f;
// registers per thread of each warpgroup; together within the launch
// allocation
constexpr int kRegXf = 56, kRegMisc = 96, kRegEpi = 176;
static_assert(32 * kNumXf * kRegXf + 128 * kRegMisc + 32 * kNumEpi * kRegEpi <=
                  kThreads * kLaunchRegs,
              "register pool");

template <int BT>
struct Cfg {
  static constexpr int NACC = 3;                      // TMEM accumulators
  static constexpr int CSLOTS = 16;                   // per-group constant slots
  static constexpr int CBATCH = 4;                    // groups of constants per round trip
  static constexpr int COLS = BT / 2;                 // tokens per epilogue warp
  static constexpr int CH = COLS < 32 ? COLS : 32;    // columns per TMEM load
};

struct Params {
  const uint16_t *scale;   // fp16 [N, G]
  const float *xscale;     // [M] or [M, G]
  const int32_t *xsum;     // [M, G] (unused when the kernel forms the sums)
  const uint16_t *bias;    // [N] or null
  float *y;                // [M, N]
  int32_t *S;              // debug sums [M, N, G]
  // split K: each (row tile, token tile) is cut into `splits` ranges of `gps`
  // groups; a range's partial sums go to ws, and the last of the splits to
  // finish a warp's sub-block adds them (in split order) and writes y
  float *ws;               // [row tiles x token tiles][splits][BW][BT] (splits > 1)
  int *cnt;                // [row tiles x token tiles][kNumEpi] arrival counters, zero
                           // (at the start of the scratch, ws after them)
  int M, N, K, G;
  int mt;                  // token tiles
  int splits, gps;         // K ranges per tile and groups per range
  int tiles;               // row tiles x token tiles x splits
  int stages;
};

// Work item `tile`: its (row tile, token tile) index, K range and groups.
struct TileCoord {
  int tmn, split, n0, m0, g0, g1;
};
template <int BT, bool SPLIT>
__device__ __forceinline__ TileCoord tile_coord(const Params &p, int tile) {
  TileCoord c;
  c.split = SPLIT ? tile % p.splits : 0;
  c.tmn = SPLIT ? tile / p.splits : tile;
  c.n0 = (c.tmn / p.mt) * BW;
  c.m0 = (c.tmn % p.mt) * BT;
  c.g0 = SPLIT ? c.split * p.gps : 0;
  c.g1 = SPLIT ? min(p.G, c.g0 + p.gps) : p.G;
  return c;
}

// Tensor memory: three accumulators of bt columns, then one 32-column slot
// of the weight operand per pipeline stage (128 bytes of K per lane).
constexpr int kStagesMax = 4;
__host__ __device__ constexpr int tmem_abase(int bt) { return (3 * bt + 31) / 32 * 32; }
__host__ __device__ constexpr int tmem_cols(int bt) {
  // rounded up to a power of two >= 32
  return tmem_abase(bt) + 32 * kStagesMax <= 256 ? 256 : 512;
}

__host__ __device__ constexpr int stage_bytes(int mode, int bt) {
  // operand B (bt x 128 B, 128-byte swizzle), hi (and lo) plane tiles
  // (128 x 64 B each, 64-byte swizzle); stages start on 1024-byte boundaries
  return (bt * 128 + (mode ? 2 : 1) * BW * 64 + 1023) / 1024 * 1024;
}

// one constant slot: row scales (128 fp32), per-token constants c (int32)
// and activation scales (bt x 4 B each)
__host__ __device__ constexpr int cslot_bytes(int bt) { return BW * 4 + 2 * bt * 4; }

__host__ __device__ constexpr int cslots(int) { return 16; }

// mbarriers: fullB, fullA [kMaxStages each], done [kDone], fullC, emptyC
// [16 each], accEmpty [4]
constexpr int kBarriers = 2 * kMaxStages + kDone + 2 * 16 + 4;

__host__ __device__ constexpr int smem_total(int mode, int bt, int stages) {
  return 1024 + stages * stage_bytes(mode, bt) + cslots(bt) * cslot_bytes(bt) + kBarriers * 8 +
         16;
}

// Float pairs in 64-bit registers and the packed f32x2 operations on them.
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t pack_i2(int lo, int hi) {  // the bit patterns
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}


// XS: the kernel forms the tokens' group sums itself (no caller xsum).
template <int MODE, int BT, bool ACTG, bool DEBUG, bool SPLIT, bool XS>
__global__ void __launch_bounds__(kThreads, 1)
    tc_linear_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, const Params p) {
  using C = Cfg<BT>;
  constexpr int OFF = CodeOffset<MODE>::value;
  constexpr int NACC = C::NACC, CS = C::CSLOTS, COLS = C::COLS, CH = C::CH;
  constexpr uint32_t IDESC = umma_idesc_u8s8(BW, BT);
  constexpr int TCOLS = tmem_cols(BT);
  constexpr int STAGE = stage_bytes(MODE, BT);
  constexpr int CSLOT = cslot_bytes(BT);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int S = p.stages;
  // stage s: [B bt x 128][hi 8 KB][lo 8 KB]; its weight operand is in tensor
  // memory (slot s)
  auto sB = [&](int s) { return smem + s * STAGE; };
  auto sH = [&](int s) { return smem + s * STAGE + BT * 128; };
  auto sL = [&](int s) { return smem + s * STAGE + BT * 128 + BW * 64; };
  // constant slot c: [row scales][per-token constants][act. scales]
  uint8_t *cbase = smem + S * STAGE;
  auto sSg = [&](int c) { return reinterpret_cast<float *>(cbase + c * CSLOT); };
  auto sCv = [&](int c) { return reinterpret_cast<int32_t *>(sSg(c) + BW); };
  auto sXv = [&](int c) { return reinterpret_cast<float *>(sCv(c) + BT); };
  uint64_t *bars = reinterpret_cast<uint64_t *>(cbase + CS * CSLOT);
  uint64_t *fullB = bars;                      // activation and plane tiles landed
  uint64_t *fullA = bars + kMaxStages;         // byte operand written (the tiles landed)
  uint64_t *done = bars + 2 * kMaxStages;      // [kDone] the group's MMAs complete:
                                               // stage and accumulator readable / free
  uint64_t *fullC = done + kDone;              // [CS] per-group constants written
  uint64_t *emptyC = fullC + CS;               // [CS] epilogue done with them
  uint64_t *accEmpty = emptyC + CS;            // [NACC] accumulator read out
  uint32_t *tslot = reinterpret_cast<uint32_t *>(accEmpty + NACC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&fullA[s], kNumXf);
    }
    for (int c = 0; c < CS; ++c) {
      mbar_init(&fullC[c], XS ? 1 + kNumXf : 1);  // one prep warp per slot
      mbar_init(&emptyC[c], kNumEpi);
    }
    for (int d = 0; d < kDone; ++d) mbar_init(&done[d], 1);
    for (int b = 0; b < NACC; ++b) mbar_init(&accEmpty[b], kNumEpi);
    fence_barrier_init();
  }
  if (warp == kWarpMma0) {
    tmem_alloc(tslot, TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // the next kernel may start its prologue; the activations, their sums and
  // scales come from the preceding one (waited for below, before each read)
  griddep_launch_dependents();

  // Each warpgroup's branch starts with its register count (the epilogue
  // holds the fp32 running sums), so the compiler allocates every role
  // within what it has.
  if (warp < kWarpXf0 + kNumXf) {
    setmaxnreg_dec<kRegXf>();
    // ---------------------------------------------- plane -> operand bytes
    // thread t: weight row t of the tile (TMEM lane t, in this warp's lane
    // quarter): its 64 hi (and lo) plane bytes of the group -> 128 operand
    // bytes, written to the stage's TMEM slot as 32 columns
    const int t = threadIdx.x - kWarpXf0 * 32;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int sw = (t >> 1) & 3;  // the plane tiles' 64-byte swizzle: chunk c sits at c ^ sw
    int s = 0, it = 0;
    uint32_t ph = 0;  // stage slot and the parity of its current fill
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
      const TileCoord tc = tile_coord<BT, SPLIT>(p, tile);
      for (int g = tc.g0; g < tc.g1; ++g, ++it) {
        ok = mbar_wait_warp(&fullB[s], ph);
        if (!ok) break;
        const uint8_t *hs = sH(s) + t * 64;
        const uint8_t *ls = sL(s) + t * 64;
        const uint32_t at = tmem + lane_base + (uint32_t)(tmem_abase(BT) + 32 * s);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // columns 64 half .. 64 half + 63
          uint32_t out[16];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {  // plane chunk c = 2 half + cc: 32 columns
            const int c = 2 * half + cc;
            const uint4 h = *reinterpret_cast<const uint4 *>(hs + ((c ^ sw) << 4));
            uint4 l = make_uint4(0, 0, 0, 0);
            if (MODE) l = *reinterpret_cast<const uint4 *>(ls + ((c ^ sw) << 4));
            const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
            const uint32_t lw[4] = {l.x, l.y, l.z, l.w};
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
              out[8 * cc + 2 * w] = prmt(ev, od, 0x5140);      // columns 8w + 0..3
              out[8 * cc + 2 * w + 1] = prmt(ev, od, 0x7362);  // columns 8w + 4..7
            }
          }
          tmem_st16(at + 16 * half, out);
        }
        tmem_st_wait();
        tc_fence_before();
        int cs = 0;
        if constexpr (XS) {
          // the tokens' sums of this group from the landed activation tile
          // (rows of 128 bytes in the 128-byte swizzle): eight threads per
          // row, one 16-byte chunk each; c = bits(1.5 * 2^23) - offset * sum
          cs = it % CS;
          ok = mbar_wait_warp(&emptyC[cs], ((it / CS) & 1) ^ 1);
          if (!ok) break;
          int32_t *cv = sCv(cs);
          const uint8_t *bs = sB(s);
          const int q = t & 7;
#pragma unroll 4
          for (int r0 = 0; r0 < BT; r0 += kXfThreads / 8) {
            const int r = r0 + (t >> 3);
            uint4 w = make_uint4(0, 0, 0, 0);
            if (r < BT) w = *reinterpret_cast<const uint4 *>(bs + r * 128 + ((q ^ (r & 7)) << 4));
            int sum = __dp4a((int)w.x, 0x01010101, 0);
            sum = __dp4a((int)w.y, 0x01010101, sum);
            sum = __dp4a((int)w.z, 0x01010101, sum);
            sum = __dp4a((int)w.w, 0x01010101, sum);
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            if (q == 0 && r < BT) cv[r] = (int)kMagicI - OFF * sum;
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&fullA[s]);
          if (XS) mbar_arrive(&fullC[cs]);
        }
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp < kWarpEpi0) {
    setmaxnreg_dec<kRegMisc>();
    if (warp == kWarpTma) {
    // --------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_hi);
      if (MODE) prefetch_tmap(&tm_lo);
      griddep_wait();
      int it = 0, s = 0, fd = 0;  // fd: done slot of group it - S
      uint32_t fdph = 0;
      bool ok = true;
      constexpr uint32_t bytes = BT * 128 + BW * 64 * (MODE ? 2 : 1);
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord<BT, SPLIT>(p, tile);
        const int n0 = tc.n0, m0 = tc.m0;
        for (int g = tc.g0; g < tc.g1; ++g, ++it) {
          if (it >= S) {  // the stage's previous group: its MMAs are complete
            if (!mbar_wait(&done[fd], fdph)) {
              ok = false;
              break;
            }
            if (++fd == kDone) {
              fd = 0;
              fdph ^= 1u;
            }
          }
          mbar_arrive_expect_tx(&fullB[s], bytes);
          tma_load_2d(sB(s), &tm_q, &fullB[s], g * 128, m0);
          tma_load_2d(sH(s), &tm_hi, &fullB[s], g * 64, n0);
          if (MODE) tma_load_2d(sL(s), &tm_lo, &fullB[s], g * 64, n0);
          if (++s == S) s = 0;
        }
      }
      if (!ok)  // gave up: let the copies already issued land
        for (int i = (it > S ? it - S : 0); i < it; ++i)
          mbar_wait_final(&fullB[i % S], (i / S) & 1);
    }
    } else if (warp < kWarpMma0 + kNumMma) {
    // ----------------------------------------------------------- MMA issuers
    // issuer i takes the groups it = i, i + 2, ...: it waits for the group's
    // operand (written after the tiles landed, so it implies them) and its
    // accumulator, issues the four MMAs and one commit that tells the TMA
    // producer (stage free) and the epilogue (accumulator full).  Counts,
    // slots and phases are kept incrementally for every group.
    if (lane == 0) {
      const int mine = warp - kWarpMma0;
      int it = 0, s = 0, b = 0, d = 0, ld = 0;
      uint32_t ph = 0, bph = 0, dph = 0, ldph = 0;
      bool issued = false;
      const uint64_t bd0 = umma_desc_sw128(sB(0));
      const uint32_t at0 = tmem + (uint32_t)tmem_abase(BT);  // the weight operand slots
      constexpr uint64_t kStageDesc = STAGE >> 4;  // descriptor address unit: 16 bytes
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord<BT, SPLIT>(p, tile);
        for (int g = tc.g0; g < tc.g1; ++g, ++it) {
          if ((it & 1) == mine) {
            ok = mbar_wait(&fullA[s], ph) && mbar_wait(&accEmpty[b], bph ^ 1u);
            if (!ok) break;
            tc_fence_after();
            const uint64_t bd = bd0 + (uint64_t)s * kStageDesc;
            const uint32_t at = at0 + (uint32_t)(32 * s);
            const uint32_t dt = tmem + (uint32_t)(b * BT);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // 4 x K=32: 8 TMEM columns of A, 32 bytes of B
              umma_i8_ta(dt, at + 8 * kk, bd + 2 * kk, IDESC, kk > 0 ? 1u : 0u);
            umma_commit(&done[d]);
            issued = true;
            ld = d;
            ldph = dph;
          }
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
          if (++b == NACC) {
            b = 0;
            bph ^= 1u;
          }
          if (++d == kDone) {
            d = 0;
            dph ^= 1u;
          }
        }
      }
      // every MMA this thread issued must be complete before TMEM is released
      // (also after a wait gave up): its commits complete in order
      if (issued) mbar_wait_final(&done[ld], ldph);
    }
    } else if (warp == kWarpPrep) {
    // ----------------------------------------------- per-group constants
    // CBATCH groups per round trip: lane i holds rows i + 32 r (r < 4) and
    // tokens i + 32 u (u < BT / 32, at least one), all loads of a batch
    // issued before the first use.
    constexpr int TU = BT < 32 ? 1 : BT / 32;
    constexpr int CB = C::CBATCH;
    griddep_wait();
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
      const TileCoord tc = tile_coord<BT, SPLIT>(p, tile);
      const int n0 = tc.n0, m0 = tc.m0, G1 = tc.g1, G = p.G;
      for (int gb = tc.g0; gb < G1 && ok; gb += CB) {
        uint16_t sv[4][CB];
        int rv[TU][CB];
        float xv[TU][CB];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int n = n0 + lane + 32 * r;
#pragma unroll
          for (int k = 0; k < CB; ++k)
            sv[r][k] = (!DEBUG && n < p.N && gb + k < G1) ? __ldg(p.scale + (int64_t)n * G + gb + k)
                                                           : (uint16_t)0;
        }
#pragma unroll
        for (int u = 0; u < TU; ++u) {
          const int j = lane + 32 * u, m = m0 + j;
          const bool in = j < BT && m < p.M;
#pragma unroll
          for (int k = 0; k < CB; ++k) {
            rv[u][k] = (!XS && in && gb + k < G1) ? __ldg(p.xsum + (int64_t)m * G + gb + k) : 0;
            xv[u][k] = (ACTG && in && gb + k < G1) ? __ldg(p.xscale + (int64_t)m * G + gb + k)
                                                   : 0.0f;
          }
        }
#pragma unroll
        for (int k = 0; k < CB; ++k) {
          if (gb + k >= G1) break;
          const int c = it % CS;
          ok = mbar_wait_warp(&emptyC[c], ((it / CS) & 1) ^ 1);
          if (!ok) break;
          float *sg = sSg(c);
          int32_t *cv = sCv(c);
          float *xs = sXv(c);
#pragma unroll
          for (int r = 0; r < 4; ++r) sg[lane + 32 * r] = __half2float(__ushort_as_half(sv[r][k]));
#pragma unroll
          for (int u = 0; u < TU; ++u) {
            const int j = lane + 32 * u;
            if (j < BT) {
              if (!XS) cv[j] = (int)kMagicI - OFF * rv[u][k];
              if (ACTG) xs[j] = xv[u][k];
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&fullC[c]);
          ++it;
        }
      }
    }
    }
  } else {
    setmaxnreg_inc<kRegEpi>();
    // -------------------------------------------------------------- epilogue
    const int e = warp - kWarpEpi0;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = e >> 2;
    const int row = quarter * 32 + lane;
    const int col0 = half * COLS;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    griddep_wait();  // y may still be read by the preceding kernel
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord<BT, SPLIT>(p, tile);
      const int n = tc.n0 + row, m0 = tc.m0;
      // running sums of the tile row, as float pairs in 64-bit registers (the
      // packed fma's operands, so no pair is assembled per instruction)
      uint64_t acc2[COLS / 2];
#pragma unroll
      for (int j = 0; j < COLS / 2; ++j) acc2[j] = 0ull;
      for (int g = tc.g0; g < tc.g1; ++g, ++it) {
        if (!ok) continue;  // after a give-up: no more waits, but every tile still arrives below
        const int cs = it % CS, b = it % NACC;
        ok = mbar_wait_warp(&fullC[cs], (it / CS) & 1) &&
             mbar_wait_warp(&done[it % kDone], (it / kDone) & 1);
        if (!ok) continue;
        tc_fence_after();
        const float sg = sSg(cs)[row];
        const int32_t *cv = sCv(cs) + col0;
        const float *xv = sXv(cs) + col0;
        // the whole group is read out and the accumulator handed back to the
        // MMA before the arithmetic
        const uint32_t ta0 = tmem + lane_addr + b * BT + col0;
        uint32_t dd[COLS];
#pragma unroll
        for (int c = 0; c < COLS; c += CH)
          tmem_ld<CH>(ta0 + c, *reinterpret_cast<uint32_t(*)[CH]>(dd + c));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accEmpty[b]);
#pragma unroll
        for (int c = 0; c < COLS; c += CH) {
          const uint32_t *d = dd + c;
          if (DEBUG) {
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              const int m = m0 + col0 + c + j;
              if (m < p.M && n < p.N)
                p.S[((int64_t)m * p.N + n) * p.G + g] = (int)d[j] + cv[c + j] - (int)kMagicI;
            }
          } else {
            const uint64_t nm = pack_f2(-kMagicF, -kMagicF);
            const uint64_t sg2 = pack_f2(sg, sg);
#pragma unroll
            for (int j = 0; j < CH; j += 4) {
              const int4 c4 = *reinterpret_cast<const int4 *>(cv + c + j);
              // 1.5 * 2^23 + exact group sum, as a float, minus the magic
              uint64_t f01 = pack_i2((int)d[j] + c4.x, (int)d[j + 1] + c4.y);
              uint64_t f23 = pack_i2((int)d[j + 2] + c4.z, (int)d[j + 3] + c4.w);
              f01 = add_f2(f01, nm);
              f23 = add_f2(f23, nm);
              uint64_t s01 = sg2, s23 = sg2;
              if (ACTG) {
                const float4 x4 = *reinterpret_cast<const float4 *>(xv + c + j);
                s01 = pack_f2(sg * x4.x, sg * x4.y);
                s23 = pack_f2(sg * x4.z, sg * x4.w);
              }
              acc2[(c + j) / 2] = fma_f2(f01, s01, acc2[(c + j) / 2]);
              acc2[(c + j) / 2 + 1] = fma_f2(f23, s23, acc2[(c + j) / 2 + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyC[cs]);
      }
      float acc[COLS];
#pragma unroll
      for (int j = 0; j < COLS / 2; ++j) unpack_f2(acc2[j], acc[2 * j], acc[2 * j + 1]);
      if constexpr (SPLIT && !DEBUG) {
        // this range's partial sums of the warp's sub-block (rows of its lane
        // quarter, its columns), then one arrival per warp; the last of the
        // splits to arrive adds them all in split order.  A warp whose wait
        // gave up still arrives (its partials are invalid, and so is y: the
        // flag says so), so every counter returns to zero.
        float *part = p.ws + ((int64_t)tc.tmn * p.splits) * (BW * BT) + row * BT + col0;
        if (ok) {
#pragma unroll
          for (int j = 0; j < COLS; j += 4)
            *reinterpret_cast<float4 *>(part + (int64_t)tc.split * (BW * BT) + j) =
                make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(&p.cnt[tc.tmn * kNumEpi + e], 1) == p.splits - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        if (lane == 0) p.cnt[tc.tmn * kNumEpi + e] = 0;  // ready for the next call
        if (!ok) continue;
#pragma unroll
        for (int j = 0; j < COLS; ++j) acc[j] = 0.0f;
        for (int sp = 0; sp < p.splits; ++sp) {
#pragma unroll
          for (int j = 0; j < COLS; j += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(part + (int64_t)sp * (BW * BT) + j));
            acc[j] += v.x;
            acc[j + 1] += v.y;
            acc[j + 2] += v.z;
            acc[j + 3] += v.w;
          }
        }
      }
      if (!DEBUG && ok && n < p.N) {
        const float bias = p.bias ? __half2float(__ushort_as_half(__ldg(p.bias + n))) : 0.0f;
#pragma unroll
        for (int j = 0; j < COLS; ++j) {
          const int m = m0 + col0 + j;
          if (m < p.M) {
            float out = ACTG ? acc[j] : acc[j] * __ldg(p.xscale + m);
            if (MODE) out *= 0.0625f;
            p.y[(int64_t)m * p.N + n] = out + bias;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma0) {
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

// Token tile: the smallest of 16 .. 128 that holds M (128 from there on).
int pick_bt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

int pick_stages(int mode, int bt, int max_smem) {
  for (int s = kStagesMax; s >= 2; --s)
    if (smem_total(mode, bt, s) <= max_smem) return s;
  return 0;
}

constexpr int kMaxSmem = 227 * 1024;

int num_sms() {
  static int sms[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  return sms[dev] > 0 ? sms[dev] : 148;
}

// Split-K plan of a shape: a (row tile, token tile) grid that fills fewer
// than half of the SMs is cut along K into ranges of at least four groups,
// about one work item per SM in all.  Scratch: the arrival counters (one
// per epilogue warp and tile) at a fixed place, the start, so that calls of
// any shapes can share one scratch (each leaves its counters zero, and no
// shape's partial tiles reach another's counters); then the partial tiles.
constexpr int kMaxCntTiles = 256;
constexpr int64_t kCntBytes = int64_t(kMaxCntTiles) * kNumEpi * 4;  // 8 KB
struct SplitPlan {
  int splits, gps;
  int64_t tmn, bytes;
};
SplitPlan split_plan(int64_t M, int64_t N, int64_t K, int bt) {
  SplitPlan sp;
  const int G = (int)(K / kGroup);
  sp.tmn = ((N + BW - 1) / BW) * ((M + bt - 1) / bt);
  const int sms = num_sms();
  int s = 1;
  if (sp.tmn * 2 <= sms && sp.tmn <= kMaxCntTiles) {
    s = (int)(sms / sp.tmn);
    if (s > G / 4) s = G / 4;
    if (s < 1) s = 1;
  }
  sp.gps = (G + s - 1) / s;
  sp.splits = (G + sp.gps - 1) / sp.gps;  // no empty range
  sp.bytes = sp.splits == 1 ? 0 : kCntBytes + sp.tmn * sp.splits * BW * bt * 4;
  return sp;
}

// The register split hands out the launch allocation of kLaunchRegs
// registers per thread; a kernel built with fewer would make the increase
// wait for registers that do not exist, so it is not launched.
template <typename Kern>
cudaError_t check_register_pool(Kern kern) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  return fa.numRegs == kLaunchRegs ? cudaSuccess : cudaErrorInvalidConfiguration;
}

template <int MODE, int BT, bool ACTG, bool DEBUG, bool XS>
cudaError_t launch_t(const LinearArgs &a, cudaStream_t st) {
  // split K only where the plan asks for it: the unsplit kernel carries none
  // of the partial-tile code
  const int G = (int)(a.K / kGroup);
  const int stages = pick_stages(MODE, BT, kMaxSmem);
  if (stages == 0) return cudaErrorInvalidValue;
  CUtensorMap mq, mh, ml;
  if (!make_map(&mq, a.xq, (uint64_t)a.M, (uint64_t)a.K, BT, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mh, a.hi, (uint64_t)a.N, (uint64_t)(a.K / 2), BW, 64, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  if (MODE) {
    if (!make_map(&ml, a.lo, (uint64_t)a.N, (uint64_t)(a.K / 2), BW, 64,
                  CU_TENSOR_MAP_SWIZZLE_64B))
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
  p.K = (int)a.K;
  p.G = G;
  p.mt = (int)((a.M + BT - 1) / BT);
  p.splits = 1;
  p.gps = G;
  p.ws = nullptr;
  p.cnt = nullptr;
  if (a.ws && !DEBUG) {
    const SplitPlan sp = split_plan(a.M, a.N, a.K, BT);
    if (sp.splits > 1) {
      if (a.ws_bytes < sp.bytes) return cudaErrorInvalidValue;
      p.splits = sp.splits;
      p.gps = sp.gps;
      p.cnt = static_cast<int *>(a.ws);
      p.ws = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + kCntBytes);
    }
  }
  const int64_t tiles = ((a.N + BW - 1) / BW) * (int64_t)p.mt * p.splits;
  if (tiles > (1 << 30)) return cudaErrorInvalidValue;
  p.tiles = (int)tiles;
  p.stages = stages;
  const int grid = p.tiles < num_sms() ? p.tiles : num_sms();
  const int smem = smem_total(MODE, BT, stages);
  constexpr bool kCanSplit = !DEBUG;
  auto kern = (kCanSplit && p.splits > 1) ? tc_linear_kernel<MODE, BT, ACTG, DEBUG, kCanSplit, XS>
                                          : tc_linear_kernel<MODE, BT, ACTG, DEBUG, false, XS>;
  cudaError_t e = check_register_pool(kern);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, st, a.overlap, mq, mh,
                 ml, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int MODE, int BT, bool DEBUG>
cudaError_t launch_g(const LinearArgs &a, cudaStream_t st) {
  const bool xs = a.xsum == nullptr;  // no caller sums: the kernel forms them
  // the debug sums take no activation scale: no per-group scale variant
  if constexpr (!DEBUG) {
    if (a.act_group != 0)
      return xs ? launch_t<MODE, BT, true, false, true>(a, st)
                : launch_t<MODE, BT, true, false, false>(a, st);
  }
  return xs ? launch_t<MODE, BT, false, DEBUG, true>(a, st)
            : launch_t<MODE, BT, false, DEBUG, false>(a, st);
}

template <int MODE, bool DEBUG>
cudaError_t launch_mode(const LinearArgs &a, cudaStream_t st) {
  switch (pick_bt(a.M)) {
    case 16: return launch_g<MODE, 16, DEBUG>(a, st);
    case 32: return launch_g<MODE, 32, DEBUG>(a, st);
    case 64: return launch_g<MODE, 64, DEBUG>(a, st);
    default: return launch_g<MODE, 128, DEBUG>(a, st);
  }
}

}  // namespace tc

// Test hook: one warp waits, with the kernels' own bounded wait (cut to
// 200 us of device time), on an mbarrier that nothing ever arrives at.  The
// wait gives up and sets this translation unit's g_wait_timeout, which
// read_wait_timeout reports; nothing faults or hangs.
__global__ void wait_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  (void)mbar_wait(&bar, 0, 200000ull);  // phase 0 never completes
}

cudaError_t launch_wait_probe(cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

cudaError_t read_wait_timeout(int *flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_wait_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_wait_timeout, &zero, sizeof(int));
}

bool tc_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || M > (int64_t)1 << 30 || N > (int64_t)1 << 30) return false;
  if (K < kGroup || K % kGroup != 0 || K > ((int64_t)1 << 30)) return false;
  return tc::pick_stages(1, tc::pick_bt(M), tc::kMaxSmem) >= 2;
}

// Library-owned split-K scratch for bitnest_linear_static_ws: zero at module
// load (so its arrival counters start at zero) and left zero by every call.
// The largest split plan is one 128 x 128 fp32 partial tile per SM plus the
// counters: under 10 MB on 148 SMs.
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

// Its device address, looked up once per device (the first caller on a
// device does the lookup; the others wait for it).
cudaError_t tc_static_ws(void **ws) {
  static std::once_flag once[64];
  static void *addr[64] = {nullptr};
  static cudaError_t err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev] {
    void *p = nullptr;
    err[dev] = cudaGetSymbolAddress(&p, g_static_ws);
    if (err[dev] == cudaSuccess && !p) err[dev] = cudaErrorInvalidSymbol;
    addr[dev] = p;
  });
  if (err[dev] != cudaSuccess) return err[dev];
  *ws = addr[dev];
  return cudaSuccess;
}

// After a bounded wait gave up inside a split call, the counters of the
// static scratch may hold arrivals of that call: clear them (no allocation).
cudaError_t tc_static_ws_clear_counters(cudaStream_t st) {
  void *ws = nullptr;
  cudaError_t e = tc_static_ws(&ws);
  if (e != cudaSuccess) return e;
  return cudaMemsetAsync(ws, 0, (size_t)tc::kCntBytes, st);
}

int64_t tc_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (!tc_supported(M, N, K)) return 0;
  return tc::split_plan(M, N, K, tc::pick_bt(M)).bytes;
}

cudaError_t launch_tc(const LinearArgs &a, cudaStream_t st) {
  const bool debug = a.S != nullptr;
  if (a.mode == 0)
    return debug ? tc::launch_mode<0, true>(a, st) : tc::launch_mode<0, false>(a, st);
  return debug ? tc::launch_mode<1, true>(a, st) : tc::launch_mode<1, false>(a, st);
}

}  // namespace bitnest
