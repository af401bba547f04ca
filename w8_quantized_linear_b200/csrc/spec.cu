// Speculative decoding rounds with the nested weights, on the device.
//
// BitNest-Llama-3-8B model card, opening paragraph: the W4A8 draft (hi plane)
// proposes tokens and the W8A8 target (hi and lo planes) verifies all of them
// in one pass, so the output equals the target's greedy output; model table
// row "Default draft length": gamma = 3.  The model is a small synthetic one
// built from the nested linear layer (the pages give none):
//   input at position p : x0 = fp16(E[t_p] + 0.5 E[t_{p-1}])   (t_{-1} := t_0)
//   layer l             : x_{l+1} = fp16(tanh(W_l x_l)),  W_l nested [d, d]
//   head                : logits = W_head x_L,             W_head nested [V, d]
//   next token          : argmax, the lowest index among equal maxima.
// A round: gamma draft steps at M = 1, one target pass over the gamma + 1
// positions at M = gamma + 1, then the accept step appends the agreed prefix
// of the draft tokens and the target's token after it.  The sequence, its
// length and the round statistics live in device memory, so no round reads
// anything back to the host and a round can be captured in a CUDA graph.
#include <cstring>

#include "bitnest.h"
#include "common.cuh"
#include "launch.h"

namespace bitnest {
namespace spec {

constexpr int kThreads = 256;

// token i of the sequence followed by the draft tokens (clamped into the vocabulary)
__device__ __forceinline__ int token_at(const int32_t *seq, int L, const int32_t *draft, int i,
                                        int vocab) {
  const int t = i < L ? seq[i] : draft[i - L];
  return min(max(t, 0), vocab - 1);
}

// Block m: the input of position q = len - 1 + q0 + m of (sequence ++ draft):
// fp16(E[t_q] + 0.5 E[t_{q-1}]); the sum of two fp16 values (one halved) is
// exact in fp32, so the result is the correctly rounded sum.
__global__ void __launch_bounds__(kThreads) embed_kernel(const uint16_t *__restrict__ E, int vocab,
                                                         int dim, const int32_t *seq,
                                                         const int32_t *len, const int32_t *draft,
                                                         int q0, uint16_t *__restrict__ x) {
  const int L = *len;
  const int q = L - 1 + q0 + (int)blockIdx.x;
  const int cur = token_at(seq, L, draft, q, vocab);
  const int prev = token_at(seq, L, draft, q > 0 ? q - 1 : 0, vocab);
  const uint4 *ec = reinterpret_cast<const uint4 *>(E + (int64_t)cur * dim);
  const uint4 *ep = reinterpret_cast<const uint4 *>(E + (int64_t)prev * dim);
  uint4 *out = reinterpret_cast<uint4 *>(x + (int64_t)blockIdx.x * dim);
  for (int v = threadIdx.x; v < dim / 8; v += kThreads) {
    const uint4 a = __ldg(ec + v), b = __ldg(ep + v);
    const __half2 *ha = reinterpret_cast<const __half2 *>(&a);
    const __half2 *hb = reinterpret_cast<const __half2 *>(&b);
    uint4 r;
    __half2 *hr = reinterpret_cast<__half2 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __half22float2(ha[i]), fb = __half22float2(hb[i]);
      hr[i] = __floats2half2_rn(fa.x + 0.5f * fb.x, fa.y + 0.5f * fb.y);
    }
    out[v] = r;
  }
}

// x = fp16(tanh(y)), elementwise
__global__ void __launch_bounds__(kThreads) act_kernel(const float *__restrict__ y, int64_t n,
                                                       uint16_t *__restrict__ x) {
  for (int64_t i = blockIdx.x * (int64_t)kThreads + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * kThreads)
    x[i] = __half_as_ushort(__float2half_rn(tanhf(y[i])));
}

// Block m: out[m] = argmax of row m of logits [M, vocab] (lowest index among
// equal maxima).
__global__ void __launch_bounds__(kThreads) argmax_kernel(const float *__restrict__ logits,
                                                          int vocab, int32_t *out) {
  const float *row = logits + (int64_t)blockIdx.x * vocab;
  float best = -INFINITY;
  int idx = 0x7fffffff;
  for (int i = threadIdx.x; i < vocab; i += kThreads) {
    const float v = row[i];
    if (v > best) {  // indices rise along the thread's walk: first maximum kept
      best = v;
      idx = i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (ob > best || (ob == best && oi < idx)) {
      best = ob;
      idx = oi;
    }
  }
  __shared__ float sb[kThreads / 32];
  __shared__ int si[kThreads / 32];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sb[warp] = best;
    si[warp] = idx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kThreads / 32; ++w)
      if (sb[w] > best || (sb[w] == best && si[w] < idx)) {
        best = sb[w];
        idx = si[w];
      }
    out[blockIdx.x] = idx == 0x7fffffff ? 0 : idx;
  }
}

// stats: [0] rounds, [1] tokens appended, [2] draft tokens accepted,
// [3] set when a write would pass the sequence's capacity (nothing written)
__global__ void accept_kernel(int gamma, const int32_t *draft, const int32_t *verify, int32_t *seq,
                              int64_t cap, int32_t *len, int32_t *stats) {
  if (threadIdx.x != 0) return;
  int k = 0;
  while (k < gamma && draft[k] == verify[k]) ++k;
  const int L = *len;
  if ((int64_t)L + k + 1 > cap) {
    stats[3] = 1;
    return;
  }
  for (int i = 0; i < k; ++i) seq[L + i] = draft[i];
  seq[L + k] = verify[k];
  *len = L + k + 1;
  stats[0] += 1;
  stats[1] += k + 1;
  stats[2] += k;
}

__global__ void append_kernel(const int32_t *tok, int32_t *seq, int64_t cap, int32_t *len,
                              int32_t *stats) {
  if (threadIdx.x != 0) return;
  const int L = *len;
  if ((int64_t)L + 1 > cap) {
    stats[3] = 1;
    return;
  }
  seq[L] = *tok;
  *len = L + 1;
  stats[1] += 1;
}

// Scratch of a round: activations, codes, scales, layer outputs, draft and
// verify tokens, each on a 256-byte boundary.
struct Work {
  uint16_t *x;
  int8_t *xq;
  float *xs;
  float *y;
  int32_t *draft, *verify;
  int64_t bytes;
};

inline int64_t up256(int64_t b) { return (b + 255) / 256 * 256; }

Work layout(void *base, int64_t vocab, int64_t dim, int gamma) {
  const int64_t M = gamma + 1;
  const int64_t wide = vocab > dim ? vocab : dim;
  Work w;
  int64_t o = 0;
  auto take = [&](int64_t b) {
    const int64_t at = o;
    o += up256(b);
    return static_cast<uint8_t *>(base) + at;
  };
  w.x = reinterpret_cast<uint16_t *>(take(M * dim * 2));
  w.xq = reinterpret_cast<int8_t *>(take(M * dim));
  w.xs = reinterpret_cast<float *>(take(M * 4));
  w.y = reinterpret_cast<float *>(take(M * wide * 4));
  w.draft = reinterpret_cast<int32_t *>(take(gamma > 0 ? gamma * 4 : 4));
  w.verify = reinterpret_cast<int32_t *>(take(M * 4));
  w.bytes = o;
  return w;
}

// One pass of the model over M positions starting at q0 of (sequence ++
// draft): tokens of `out` (M of them) from the argmax of the logits.
int forward(const bitnest_spec_model *m, int mode, int M, int q0, const int32_t *seq,
            const int32_t *len, const int32_t *draft, const Work &w, int32_t *out,
            cudaStream_t st) {
  const int V = (int)m->vocab, d = (int)m->dim;
  embed_kernel<<<M, kThreads, 0, st>>>(m->embed, V, d, seq, len, draft, q0, w.x);
  if (cudaGetLastError() != cudaSuccess) return BITNEST_ERR_CUDA;
  const int path = BITNEST_PATH_AUTO | BITNEST_PATH_OVERLAP;
  for (int64_t l = 0; l < m->layers; ++l) {
    int s = bitnest_quantize_linear(mode, m->hi[l], mode ? m->lo[l] : nullptr, m->scale[l], w.x, M,
                                    d, d, w.y, 0, nullptr, w.xq, w.xs, nullptr, path, st);
    if (s != BITNEST_OK) return s;
    const int64_t n = (int64_t)M * d;
    const int blocks = (int)((n + kThreads - 1) / kThreads);
    act_kernel<<<blocks, kThreads, 0, st>>>(w.y, n, w.x);
    if (cudaGetLastError() != cudaSuccess) return BITNEST_ERR_CUDA;
  }
  int s = bitnest_quantize_linear(mode, m->head_hi, mode ? m->head_lo : nullptr, m->head_scale,
                                  w.x, M, V, d, w.y, 0, nullptr, w.xq, w.xs, nullptr, path, st);
  if (s != BITNEST_OK) return s;
  argmax_kernel<<<M, kThreads, 0, st>>>(w.y, V, out);
  return cudaGetLastError() == cudaSuccess ? BITNEST_OK : BITNEST_ERR_CUDA;
}

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

int check_model(const bitnest_spec_model *m) {
  if (!m || !m->embed || !m->head_hi || !m->head_lo || !m->head_scale) return BITNEST_ERR_INVALID_ARG;
  if (m->vocab < 1 || m->vocab > (1 << 30) || m->dim < 128 || m->dim % 128 != 0 ||
      m->dim > (1 << 20) || m->layers < 0 || m->layers > 4096)
    return BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (m->layers > 0 && (!m->hi || !m->lo || !m->scale)) return BITNEST_ERR_INVALID_ARG;
  for (int64_t l = 0; l < m->layers; ++l) {
    if (!m->hi[l] || !m->lo[l] || !m->scale[l]) return BITNEST_ERR_INVALID_ARG;
    if (misaligned(m->hi[l]) || misaligned(m->lo[l]) || misaligned(m->scale[l]))
      return BITNEST_ERR_MISALIGNED;
  }
  if (misaligned(m->embed) || misaligned(m->head_hi) || misaligned(m->head_lo) ||
      misaligned(m->head_scale))
    return BITNEST_ERR_MISALIGNED;
  return BITNEST_OK;
}

int check_run(const bitnest_spec_model *m, int gamma, int32_t *seq, int64_t cap, int32_t *len,
              int32_t *stats, void *work, int64_t work_bytes) {
  int s = check_model(m);
  if (s != BITNEST_OK) return s;
  if (gamma < 0 || gamma + 1 > BITNEST_GEMV_MAX_M) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (!seq || !len || !stats || !work || cap < 1) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(work) || misaligned(seq) || misaligned(len) || misaligned(stats))
    return BITNEST_ERR_MISALIGNED;
  if (work_bytes < layout(nullptr, m->vocab, m->dim, gamma).bytes) return BITNEST_ERR_INVALID_ARG;
  return BITNEST_OK;
}

}  // namespace spec
}  // namespace bitnest

using namespace bitnest;

extern "C" {

int64_t bitnest_spec_work_bytes(int64_t vocab, int64_t dim, int gamma) {
  if (vocab < 1 || dim < 128 || dim % 128 != 0 || gamma < 0 || gamma + 1 > BITNEST_GEMV_MAX_M)
    return -BITNEST_ERR_UNSUPPORTED_SHAPE;
  return spec::layout(nullptr, vocab, dim, gamma).bytes;
}

int bitnest_spec_rounds(const bitnest_spec_model *m, int gamma, int rounds, int32_t *seq,
                        int64_t cap, int32_t *len, int32_t *stats, void *work, int64_t work_bytes,
                        void *stream) {
  if (rounds < 0) return BITNEST_ERR_INVALID_ARG;
  int s = spec::check_run(m, gamma, seq, cap, len, stats, work, work_bytes);
  if (s != BITNEST_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const spec::Work w = spec::layout(work, m->vocab, m->dim, gamma);
  for (int r = 0; r < rounds; ++r) {
    for (int j = 0; j < gamma; ++j) {  // draft: position len - 1 + j, one token each
      s = spec::forward(m, BITNEST_DRAFT, 1, j, seq, len, w.draft, w, w.draft + j, st);
      if (s != BITNEST_OK) return s;
    }
    // verify: the target on positions len - 1 .. len - 1 + gamma at once
    s = spec::forward(m, BITNEST_TARGET, gamma + 1, 0, seq, len, w.draft, w, w.verify, st);
    if (s != BITNEST_OK) return s;
    spec::accept_kernel<<<1, 32, 0, st>>>(gamma, w.draft, w.verify, seq, cap, len, stats);
    if (cudaGetLastError() != cudaSuccess) return BITNEST_ERR_CUDA;
  }
  return BITNEST_OK;
}

int bitnest_spec_greedy(const bitnest_spec_model *m, int steps, int32_t *seq, int64_t cap,
                        int32_t *len, int32_t *stats, void *work, int64_t work_bytes,
                        void *stream) {
  if (steps < 0) return BITNEST_ERR_INVALID_ARG;
  int s = spec::check_run(m, 0, seq, cap, len, stats, work, work_bytes);
  if (s != BITNEST_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const spec::Work w = spec::layout(work, m->vocab, m->dim, 0);
  for (int i = 0; i < steps; ++i) {
    s = spec::forward(m, BITNEST_TARGET, 1, 0, seq, len, w.draft, w, w.verify, st);
    if (s != BITNEST_OK) return s;
    spec::append_kernel<<<1, 32, 0, st>>>(w.verify, seq, cap, len, stats);
    if (cudaGetLastError() != cudaSuccess) return BITNEST_ERR_CUDA;
  }
  return BITNEST_OK;
}

}  // extern "C"
