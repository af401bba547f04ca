// Decode GEMV of the bit-nested linear layer with a TMA shared-memory ring.
//
// BitNest-Llama-3-8B model card, section "Files": the draft reads the hi plane
// only (W4 = (hi - 8) * scale); the target reads both planes
// (W8 = (16 (hi - 8) + (lo - 8)) * scale / 16 = (((hi << 4) | lo) - 136) * scale / 16).
//
// The decode layer is a pure HBM stream: every weight byte is read once.  One
// persistent CTA per SM.  A producer warp streams the CTA's 16-row blocks with
// one TMA box per plane per stage (16 rows x 4096 columns = 32 KB, landed with
// the 128-byte swizzle) into a ring of shared-memory stages.  On this part the
// TMA streaming rate of an SM is set by a per-stage cost far more than by the
// bytes, so stages are large and carry nothing else: the 16-bit group scales
// are read by the consumers with 8-byte loads issued a stage ahead.
//
// Eight consumer warps each own four 128-column groups of a stage.  The
// per-group integer sums go through the integer tensor-core MMA
// (mma.sync m16n8k32, u8 weight bytes x s8 activations -> s32, 16 rows x 8
// token slots x 32 columns): the weight byte is the nibble (draft) or
// (hi << 4) | lo (target), unpacked in registers; the accumulator starts at
// -offset * sum(q) of the group, so the MMA result is the exact group sum.
// A dp4a inner loop needs about twice the issue slots of this and could not
// keep up with HBM at 2 warps per scheduler.  The K-permutation that lets a
// plane word's low / high nibbles feed the fragments without byte shuffles is
// applied to the staged activations instead (even / odd columns).  Each warp
// accumulates its groups' scaled sums in fp32 and hands the partial sums of a
// 16-row block to a reducer warp, which adds them in a fixed warp order and
// writes y while the consumers go on with the next block.
//
// With programmatic dependent launch the weight stream starts while the
// preceding kernel (the activation quantiser) still runs; the consumers wait
// for it (griddepcontrol.wait) before they read the activations.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace bitnest {
namespace gv {

constexpr int kConsumerWarps = 8;                      // four 128-column groups each per stage
constexpr int kGroupsPerWarp = 4;
constexpr int kProducerWarp = kConsumerWarps;          // TMA producer
constexpr int kReducerWarp = kConsumerWarps + 1;       // adds the warps' partial sums, writes y
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kRows = 16;                              // weight rows per stage (the MMA's M)
constexpr int kStepCols = 4096;                        // columns per stage = 32 groups
constexpr int kSegs = kStepCols / 256;                 // 128-byte plane segments per row
constexpr int kPlaneBytes = kRows * kStepCols / 2;     // 32 KB: one TMA box per plane
constexpr int kMaxStages = 8;
constexpr int kRedSlots = 4;  // row blocks whose partial sums can be in flight (2 for 16 slots)
// Weight bytes the producer issues (per CTA) before the activations are
// loaded: the stream starts while the preceding kernel runs, yet the memory
// queues are short again when the consumers' activation loads go out (two
// draft stages, one target stage).
constexpr int kPreBytes = 64 * 1024;
constexpr int kScaleSmemMax = 32 * 1024;  // the CTA's group scales are staged once
constexpr int kSmemBudget = 227 * 1024;

struct Params {
  const uint16_t *scale;
  const int8_t *xq;
  const float *xscale;
  const uint16_t *bias;
  float *y;
  int32_t *S;
  int M, N, K, G, Cp, Gp, nks, NB, stages;
};

__host__ __device__ constexpr int stage_bytes(int mode) { return (mode ? 2 : 1) * kPlaneBytes; }

// row pitch (halves) of the staged group scales: an odd number of 16-byte
// units, so rows are copied in 16-byte pieces and the 8 rows a warp reads
// with one 8-byte load each fall in different banks (row r starts at bank
// 4 (odd r mod 8))
__host__ __device__ inline int scale_pitch(int G) { return 8 * (((G + 7) / 8) | 1); }

// staged activations [M][2][Cp] x 16 B, group sums [Gp][8], group act. scales
// [Gp][8], the CTA's group scales [nb * 16][pitch] fp16, partial-sum slots
// [kRedSlots][warps][128] and their counters
// token slots of the MMA's N side: one 8-column block up to 8 tokens, two
// up to 16 (then two partial-sum slots instead of four: the staged codes
// take the shared memory)
__host__ __device__ constexpr int token_slots(int M) { return M > 8 ? 16 : 8; }
__host__ __device__ constexpr int red_slots(int M) { return M > 8 ? 2 : kRedSlots; }

__host__ __device__ inline int fixed_bytes(int M, int K, bool actg, int nb) {
  const int nks = (K + kStepCols - 1) / kStepCols;
  const int Cp = nks * (kStepCols / 32), Gp = nks * (kStepCols / kGroup);
  const int G = K / kGroup, TS = token_slots(M);
  int o = M * Cp * 32 + Gp * TS * 4 + (actg ? Gp * TS * 4 : 0) +
          (nb * kRows * scale_pitch(G) * 2 + 15) / 16 * 16 + red_slots(M) * kConsumerWarps * 16 * TS * 4;
  return (o + 1023) / 1024 * 1024;
}

__host__ inline int smem_total(int mode, int M, bool actg, int K, int nb, int stages) {
  return 1024 + fixed_bytes(M, K, actg, nb) + stages * stage_bytes(mode) +
         (2 * kMaxStages + 2 * kRedSlots + 1) * 8;
}

// D = A (16x32 u8) * B (32x8 s8) + C, int32.  Not volatile: a pure function
// of its operands, so the compiler may interleave independent MMA chains.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1, const int (&c)[4]) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]),
        "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, uint64_t *bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// MMA row g (0..7) reads stage row perm(g) (and perm(g) + 8): rows whose
// swizzle phases differ by 4 share a shared-memory wavefront, so the 16-byte
// loads of a warp hit 32 different banks.
__device__ __forceinline__ int perm_row(int g) { return (g >> 1) + ((g & 1) << 2); }

// Asynchronous 16-byte copy global -> shared (L2 only).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint32_t w, int hi) {
  return __half2float(__ushort_as_half((uint16_t)(hi ? (w >> 16) : (w & 0xFFFFu))));
}


template <int MODE, int M, bool ACTG, bool DEBUG>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap tm_hi,
                    const __grid_constant__ CUtensorMap tm_lo, const Params p) {
  constexpr int OFF = CodeOffset<MODE>::value;
  constexpr int STAGE = stage_bytes(MODE);
  constexpr int GS = kStepCols / kGroup;  // groups per stage (32)
  constexpr int TS = token_slots(M);      // token slots: 8 or 16
  constexpr int NTB = TS / 8;             // 8-token column blocks of the MMA
  constexpr int RED = 16 * TS;            // partial sums of a row block per warp
  constexpr int RS = red_slots(M);        // partial-sum slots in flight

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int Cp = p.Cp, Gp = p.Gp, G = p.G, S = p.stages;
  uint4 *xs4 = reinterpret_cast<uint4 *>(smem);                    // [M][2][Cp]
  int32_t *sr = reinterpret_cast<int32_t *>(smem + M * Cp * 32);   // [Gp][TS] group sums
  float *sxg = reinterpret_cast<float *>(sr + Gp * TS);            // [Gp][TS] group act. scales
  const int nb = (p.NB - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int sp = scale_pitch(G);
  __half *ssc = reinterpret_cast<__half *>(sxg + (ACTG ? Gp * TS : 0));  // [nb * 16][sp]
  float *red = reinterpret_cast<float *>(
      reinterpret_cast<uint8_t *>(ssc) + (nb * kRows * sp * 2 + 15) / 16 * 16);  // [slots][warps][RED]
  uint8_t *ring = smem + fixed_bytes(M, p.K, ACTG, nb);            // 1024-aligned stages
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + S * STAGE);
  uint64_t *empty = full + kMaxStages;
  uint64_t *part_full = empty + kMaxStages;       // [kRedSlots]: all warps' partials written
  uint64_t *slot_free = part_full + kRedSlots;    // [kRedSlots]: partials read out
  uint64_t *act_issued = slot_free + kRedSlots;   // every consumer warp issued its activation loads

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int i = 0; i < kRedSlots; ++i) {
      mbar_init(&part_full[i], kConsumerWarps);
      mbar_init(&slot_free[i], 1);
    }
    mbar_init(act_issued, kConsumerWarps);
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();

  if (warp == kReducerWarp) {
    // ------------------------------------------------------------- reducer
    // every consumer warp holds a K-slice of the same 16 x 8 outputs of a
    // row block; add the eight in a fixed warp order and write y
    if (DEBUG) return;
    griddep_wait();  // the token scales come from the preceding kernel
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = perm_row(gid), r1 = r0 + 8;
    const int t0 = 2 * tig;
    float xt[NTB][2];  // token scales of tokens t0, t0 + 1 of each column block
#pragma unroll
    for (int b = 0; b < NTB; ++b)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tk = 8 * b + t0 + e;
        xt[b][e] = (!ACTG && tk < M) ? __ldg(p.xscale + tk) : 0.0f;
      }
    for (int k = 0; k < nb; ++k) {
      const int slot = k % RS;
      if (!mbar_wait_warp(&part_full[slot], (k / RS) & 1)) return;
      const float *rb = red + slot * (kConsumerWarps * RED);
      const int row0 = ((int)blockIdx.x + k * (int)gridDim.x) * kRows;
#pragma unroll
      for (int b = 0; b < NTB; ++b) {
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float4 pv = *reinterpret_cast<const float4 *>(rb + w * RED + b * 128 + lane * 4);
          v[0] += pv.x;
          v[1] += pv.y;
          v[2] += pv.z;
          v[3] += pv.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = 8 * b + t0 + (i & 1);
          const int n = row0 + ((i >> 1) ? r1 : r0);
          if (tk < M && n < p.N) {
            float out = v[i];
            if (!ACTG) out *= xt[b][i & 1];
            if (MODE) out *= 0.0625f;
            if (p.bias) out += __half2float(__ushort_as_half(__ldg(p.bias + n)));
            p.y[(int64_t)tk * p.N + n] = out;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_free[slot]);
    }
    return;
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_hi);
      if (MODE) prefetch_tmap(&tm_lo);
      int it = 0;
      bool ok = true;
      for (int k = 0; k < nb && ok; ++k) {
        const int row0 = ((int)blockIdx.x + k * (int)gridDim.x) * kRows;
        for (int ks = 0; ks < p.nks; ++ks, ++it) {
          const int s = it % S;
          // the rest of the stream queues behind the activation loads
          if (it == kPreBytes / STAGE && !mbar_wait(act_issued, 0)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], STAGE);
          uint8_t *st = ring + s * STAGE;
          tma_load_3d(st, &tm_hi, &full[s], 0, row0, ks * kSegs);
          if (MODE) tma_load_3d(st + kPlaneBytes, &tm_lo, &full[s], 0, row0, ks * kSegs);
        }
      }
      if (!ok)  // gave up: let the copies already issued land before leaving
        for (int i = (it > S ? it - S : 0); i < it; ++i) mbar_wait(&full[i % S], (i / S) & 1);
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  constexpr int NT = kConsumerWarps * 32;
  // The group scales of every row this CTA owns (16-byte pieces: G is a
  // multiple of 8), copied asynchronously: all of them are in flight at
  // once.  Like the planes they do not come from the preceding kernel, so
  // this starts before the wait.
  if (!DEBUG) {
    const int cpr = G / 8;
    for (int i = threadIdx.x; i < nb * kRows * cpr; i += NT) {
      const int rl = i / cpr, c = i - rl * cpr;
      const int n = ((int)blockIdx.x + (rl / kRows) * (int)gridDim.x) * kRows + rl % kRows;
      uint4 *dst = reinterpret_cast<uint4 *>(ssc + rl * sp) + c;
      if (n < p.N)
        cp_async16(dst, reinterpret_cast<const uint4 *>(p.scale + (int64_t)n * G) + c);
      else
        *dst = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  griddep_wait();  // the activations are written by the preceding kernel
  const int C = p.K / 32;
  // token slots M..7 of the group sums (the MMA's unused columns) are zero
  if constexpr (M < TS)
    for (int i = threadIdx.x; i < Gp * (TS - M); i += NT)
      sr[(i / (TS - M)) * TS + M + i % (TS - M)] = 0;
  // activations (and per-group activation scales): every load of this
  // thread first (one round trip), then the permuted stores and the group
  // sums, formed here from the codes themselves
  constexpr int XB = 8;  // activation items per batch
  constexpr int RB = 4;  // activation-scale items per batch
  for (int bx = 0, br = 0; bx < M * Cp || (ACTG && br < Gp * TS); bx += XB * NT, br += RB * NT) {
    uint4 va[XB], vb[XB];
    float xv[RB];
#pragma unroll
    for (int u = 0; u < XB; ++u) {
      const int item = bx + threadIdx.x + u * NT;
      va[u] = make_uint4(0, 0, 0, 0);
      vb[u] = make_uint4(0, 0, 0, 0);
      if (item < M * Cp) {
        const int m = item / Cp, c = item - m * Cp;
        if (c < C) {  // zero padding past K
          const uint4 *src = reinterpret_cast<const uint4 *>(p.xq + (int64_t)m * p.K + 32 * c);
          va[u] = __ldg(src);
          vb[u] = __ldg(src + 1);
        }
      }
    }
    if (ACTG) {
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int i = br + threadIdx.x + u * NT;
        const int g = i / TS, m = i % TS;
        const bool in = i < Gp * TS && m < M && g < G;
        xv[u] = in ? __ldg(p.xscale + m * G + g) : 0.0f;
      }
    }
    if (bx == 0) {  // loads of the first batch issued: the weight stream may go on
      __syncwarp();
      if (lane == 0) mbar_arrive(act_issued);
    }
#pragma unroll
    for (int u = 0; u < XB; ++u) {
      // items bx + threadIdx.x + u NT: the four 32-column chunks of a group
      // are four consecutive lanes (Cp and NT are multiples of 4), so every
      // lane takes part in the shuffles below
      const int item = bx + threadIdx.x + u * NT;
      const uint32_t w[8] = {va[u].x, va[u].y, va[u].z, va[u].w,
                             vb[u].x, vb[u].y, vb[u].z, vb[u].w};
      int r = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) r = __dp4a((int)w[i], 0x01010101, r);
      r += __shfl_xor_sync(0xffffffffu, r, 1);
      r += __shfl_xor_sync(0xffffffffu, r, 2);
      if (item < M * Cp) {
        const int m = item / Cp, c = item - m * Cp;
        uint32_t e[4], o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          e[i] = prmt(w[2 * i], w[2 * i + 1], 0x6420);  // columns 8i + 0,2,4,6
          o[i] = prmt(w[2 * i], w[2 * i + 1], 0x7531);  // columns 8i + 1,3,5,7
        }
        xs4[(m * 2 + 0) * Cp + c] = make_uint4(e[0], o[0], e[1], o[1]);
        xs4[(m * 2 + 1) * Cp + c] = make_uint4(e[2], o[2], e[3], o[3]);
        if ((c & 3) == 0) sr[(c >> 2) * TS + m] = r;  // group c / 4 of token m (0 past K)
      }
    }
    if (ACTG) {
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int i = br + threadIdx.x + u * NT;
        if (i < Gp * TS) sxg[i] = xv[u];
      }
    }
  }
  cp_async_wait_all();
  asm volatile("bar.sync 1, %0;" ::"r"(NT) : "memory");

  const int gid = lane >> 2, tig = lane & 3;  // MMA fragment coordinates
  const int r0 = perm_row(gid), r1 = r0 + 8;  // stage rows of this thread's A rows
  const int tok0 = 2 * tig, tok1 = 2 * tig + 1;
  // byte offset of this thread's 16-byte chunk of group jl (0..31), row r
  auto chunk_off = [&](int jl, int r) {
    const int seg = jl >> 1, c = ((jl & 1) << 2) + tig;
    return seg * (kRows * 128) + r * 128 + ((c ^ (r & 7)) << 4);
  };

  // after a wait gives up, no more waits are attempted; the warp runs out its
  // loops without work (there is no CTA barrier it could be left at)
  bool ok = true;
  int it = 0;
  for (int k = 0; k < nb; ++k) {
    const int row0 = ((int)blockIdx.x + k * (int)gridDim.x) * kRows;
    float acc[NTB][4];
#pragma unroll
    for (int b = 0; b < NTB; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = 0.0f;
    for (int ks = 0; ks < p.nks && ok; ++ks, ++it) {
      uint2 sc_cur0 = make_uint2(0, 0), sc_cur1 = make_uint2(0, 0);
      if (!DEBUG) {  // this warp's four group scales of rows r0, r1
        const int gq = ks * GS + warp * kGroupsPerWarp;
        if (gq < G) {
          sc_cur0 = *reinterpret_cast<const uint2 *>(ssc + (k * kRows + r0) * sp + gq);
          sc_cur1 = *reinterpret_cast<const uint2 *>(ssc + (k * kRows + r1) * sp + gq);
        }
      }
      const int s = it % S;
      ok = mbar_wait_warp(&full[s], (it / S) & 1);
      if (!ok) break;
      const uint8_t *st = ring + s * STAGE;
#pragma unroll
      for (int q = 0; q < kGroupsPerWarp; ++q) {
        const int jl = warp * kGroupsPerWarp + q;  // group within the stage
        const int g = ks * GS + jl;                 // global group index
        const int off0 = chunk_off(jl, r0), off1 = chunk_off(jl, r1);
        const uint4 h0 = *reinterpret_cast<const uint4 *>(st + off0);
        const uint4 h1 = *reinterpret_cast<const uint4 *>(st + off1);
        uint4 l0 = make_uint4(0, 0, 0, 0), l1 = make_uint4(0, 0, 0, 0);
        if (MODE) {
          l0 = *reinterpret_cast<const uint4 *>(st + kPlaneBytes + off0);
          l1 = *reinterpret_cast<const uint4 *>(st + kPlaneBytes + off1);
        }
        // activations of tokens gid (and gid + 8), 32-column chunk 4g + tig,
        // permuted even/odd: the MMA's B operand of each 8-token column block
        uint32_t xe[NTB][4], xo[NTB][4];
        // the accumulator starts at -offset * sum(q) of the group: the MMA
        // result is the exact group sum of q * weight code
        int d[NTB][4];
#pragma unroll
        for (int b = 0; b < NTB; ++b) {
          uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
          const int tk = 8 * b + gid;
          if (tk < M) {
            const int c = g * 4 + tig;
            xa = xs4[(tk * 2 + 0) * Cp + c];
            xb = xs4[(tk * 2 + 1) * Cp + c];
          }
          xe[b][0] = xa.x; xe[b][1] = xa.z; xe[b][2] = xb.x; xe[b][3] = xb.z;
          xo[b][0] = xa.y; xo[b][1] = xa.w; xo[b][2] = xb.y; xo[b][3] = xb.w;
          const int2 rr = *reinterpret_cast<const int2 *>(sr + g * TS + 8 * b + tok0);
          d[b][0] = -OFF * rr.x;
          d[b][1] = -OFF * rr.y;
          d[b][2] = -OFF * rr.x;
          d[b][3] = -OFF * rr.y;
        }
        const uint32_t hw0[4] = {h0.x, h0.y, h0.z, h0.w}, hw1[4] = {h1.x, h1.y, h1.z, h1.w};
        const uint32_t lw0[4] = {l0.x, l0.y, l0.z, l0.w}, lw1[4] = {l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {  // 4 x K=32 columns of the group
          uint32_t a[4];
          if (MODE == 0) {
            a[0] = hw0[jj] & 0x0F0F0F0Fu;
            a[1] = hw1[jj] & 0x0F0F0F0Fu;
            a[2] = (hw0[jj] >> 4) & 0x0F0F0F0Fu;
            a[3] = (hw1[jj] >> 4) & 0x0F0F0F0Fu;
          } else {
            a[0] = ((hw0[jj] << 4) & 0xF0F0F0F0u) | (lw0[jj] & 0x0F0F0F0Fu);
            a[1] = ((hw1[jj] << 4) & 0xF0F0F0F0u) | (lw1[jj] & 0x0F0F0F0Fu);
            a[2] = (hw0[jj] & 0xF0F0F0F0u) | ((lw0[jj] >> 4) & 0x0F0F0F0Fu);
            a[3] = (hw1[jj] & 0xF0F0F0F0u) | ((lw1[jj] >> 4) & 0x0F0F0F0Fu);
          }
#pragma unroll
          for (int b = 0; b < NTB; ++b) mma_u8s8(d[b], a, xe[b][jj], xo[b][jj], d[b]);
        }
        if (DEBUG) {
          const int n0 = row0 + r0, n1 = row0 + r1;
          if (g < G) {
#pragma unroll
            for (int b = 0; b < NTB; ++b) {
              const int t0 = 8 * b + tok0, t1 = 8 * b + tok1;
              if (t0 < M && n0 < p.N) p.S[((int64_t)t0 * p.N + n0) * G + g] = d[b][0];
              if (t1 < M && n0 < p.N) p.S[((int64_t)t1 * p.N + n0) * G + g] = d[b][1];
              if (t0 < M && n1 < p.N) p.S[((int64_t)t0 * p.N + n1) * G + g] = d[b][2];
              if (t1 < M && n1 < p.N) p.S[((int64_t)t1 * p.N + n1) * G + g] = d[b][3];
            }
          }
        } else {
          const float s0 = half_bits_to_float(q < 2 ? sc_cur0.x : sc_cur0.y, q & 1);
          const float s1 = half_bits_to_float(q < 2 ? sc_cur1.x : sc_cur1.y, q & 1);
#pragma unroll
          for (int b = 0; b < NTB; ++b) {
            float x0 = 1.0f, x1 = 1.0f;
            if (ACTG) {
              const float2 xg = *reinterpret_cast<const float2 *>(sxg + g * TS + 8 * b + tok0);
              x0 = xg.x;
              x1 = xg.y;
            }
            // |d| < 2^24: the conversions are exact
            acc[b][0] = fmaf((float)d[b][0], ACTG ? s0 * x0 : s0, acc[b][0]);
            acc[b][1] = fmaf((float)d[b][1], ACTG ? s0 * x1 : s0, acc[b][1]);
            acc[b][2] = fmaf((float)d[b][2], ACTG ? s1 * x0 : s1, acc[b][2]);
            acc[b][3] = fmaf((float)d[b][3], ACTG ? s1 * x1 : s1, acc[b][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!DEBUG && ok) {
      // deposit this warp's partial sums of the row block for the reducer
      const int slot = k % RS;
      if (k >= RS) ok = mbar_wait_warp(&slot_free[slot], ((k / RS) - 1) & 1);
      if (ok) {
        float *rb = red + slot * (kConsumerWarps * RED);
#pragma unroll
        for (int b = 0; b < NTB; ++b)
          *reinterpret_cast<float4 *>(rb + warp * RED + b * 128 + lane * 4) =
              make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&part_full[slot]);
      }
    }
  }
}

// ---------------------------------------------------------------- host side
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

bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, uint64_t rows,
              uint64_t cols, uint32_t box_rows, uint32_t box_cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int sms[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  return sms[dev] > 0 ? sms[dev] : 148;
}

// The plane as [segments of 128 bytes][rows][128 bytes]: a box of 16 rows x
// 8 segments lands in shared memory as [segment][row][128 B] with the 128-byte
// swizzle, the layout the MMA fragment loads read without bank conflicts.
bool make_plane_map(CUtensorMap *m, const void *base, uint64_t N, uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, N, K / 256};
  cuuint64_t strides[2] = {K / 2, 128};
  cuuint32_t box[3] = {128, (cuuint32_t)kRows, (cuuint32_t)kSegs};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int M, bool ACTG, bool DEBUG>
cudaError_t launch_t(const LinearArgs &a, cudaStream_t st) {
  Params p;
  p.scale = a.scale;
  p.xq = a.xq;
  p.xscale = a.xscale;
  p.bias = a.bias;
  p.y = a.y;
  p.S = a.S;
  p.M = (int)a.M;
  p.N = (int)a.N;
  p.K = (int)a.K;
  p.G = (int)(a.K / kGroup);
  p.nks = (int)((a.K + kStepCols - 1) / kStepCols);
  p.Cp = p.nks * (kStepCols / 32);
  p.Gp = p.nks * (kStepCols / kGroup);
  p.NB = (int)((a.N + kRows - 1) / kRows);
  // balanced grid: every CTA gets ceil(NB / grid) or one fewer 16-row blocks
  const int sms = num_sms();
  const int per = (p.NB + sms - 1) / sms;
  const int grid = (p.NB + per - 1) / per;
  const int fixed = smem_total(MODE, M, ACTG, p.K, per, 0);
  int stages = (kSmemBudget - fixed) / stage_bytes(MODE);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  p.stages = stages;
  const int smem = smem_total(MODE, M, ACTG, p.K, per, stages);

  CUtensorMap mh, ml;
  if (!make_plane_map(&mh, a.hi, (uint64_t)a.N, (uint64_t)a.K)) return cudaErrorInvalidValue;
  ml = mh;
  if (MODE && !make_plane_map(&ml, a.lo, (uint64_t)a.N, (uint64_t)a.K)) return cudaErrorInvalidValue;

  auto kern = gemv_tma_kernel<MODE, M, ACTG, DEBUG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, st, a.overlap, mh, ml,
                 p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int MODE, bool DEBUG>
cudaError_t dispatch_m(const LinearArgs &a, cudaStream_t st) {
  const bool g = a.act_group != 0 && !DEBUG;
#define BITNEST_GV_CASE(MM) \
  case MM: return g ? launch_t<MODE, MM, true, DEBUG>(a, st) : launch_t<MODE, MM, false, DEBUG>(a, st);
  switch (a.M) {
    BITNEST_GV_CASE(1)
    BITNEST_GV_CASE(2)
    BITNEST_GV_CASE(3)
    BITNEST_GV_CASE(4)
    BITNEST_GV_CASE(5)
    BITNEST_GV_CASE(6)
    BITNEST_GV_CASE(7)
    BITNEST_GV_CASE(8)
    BITNEST_GV_CASE(9)
    BITNEST_GV_CASE(10)
    BITNEST_GV_CASE(11)
    BITNEST_GV_CASE(12)
    BITNEST_GV_CASE(13)
    BITNEST_GV_CASE(14)
    BITNEST_GV_CASE(15)
    BITNEST_GV_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef BITNEST_GV_CASE
}

}  // namespace gv

bool gemv_tma_supported(int64_t M, int64_t N, int64_t K) {
  // the scale rows are read as 32-bit words and G is a multiple of 8
  if (M < 1 || M > 16 || N < 1 || K % 1024 != 0 || K > (1 << 20)) return false;
  const int64_t NB = (N + gv::kRows - 1) / gv::kRows;
  const int sms = gv::num_sms();
  const int64_t per = (NB + sms - 1) / sms;
  const int G = (int)(K / kGroup);
  if (per * gv::kRows * gv::scale_pitch(G) * 2 > gv::kScaleSmemMax) return false;
  return gv::smem_total(1, (int)M, true, (int)K, (int)per, 2) <= gv::kSmemBudget;
}

cudaError_t launch_gemv_tma(const LinearArgs &a, cudaStream_t st) {
  const bool debug = a.S != nullptr;
  if (a.mode == 0) return debug ? gv::dispatch_m<0, true>(a, st) : gv::dispatch_m<0, false>(a, st);
  return debug ? gv::dispatch_m<1, true>(a, st) : gv::dispatch_m<1, false>(a, st);
}

cudaError_t read_wait_timeout_gemv(int *flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_wait_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_wait_timeout, &zero, sizeof(int));
}

}  // namespace bitnest
