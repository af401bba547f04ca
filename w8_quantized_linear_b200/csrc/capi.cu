// C ABI of the BitNest nested W4/W8 linear layer: host-side argument checks
// and dispatch to the sm_100a kernels.  Declarations and the contract of each
// entry point are in include/bitnest.h.
#include <stdint.h>

#include "bitnest.h"
#include "common.cuh"
#include "launch.h"

using namespace bitnest;

namespace {

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? BITNEST_OK : BITNEST_ERR_CUDA; }

// K must be a positive multiple of the group size; M, N non-negative.
int check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K <= 0 || K % kGroup != 0) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  // 32-bit grid / index limits of the kernels
  if (K > (int64_t)1 << 24 || N > (int64_t)1 << 31 || M > (int64_t)1 << 31)
    return BITNEST_ERR_UNSUPPORTED_SHAPE;
  return BITNEST_OK;
}

int check_linear(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                 const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                 int64_t N, int64_t K, const float *y, int act_group, const uint16_t *bias) {
  if (mode != BITNEST_DRAFT && mode != BITNEST_TARGET) return BITNEST_ERR_INVALID_ARG;
  if (act_group != 0 && act_group != kGroup) return BITNEST_ERR_INVALID_ARG;
  int s = check_shape(M, N, K);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;  // empty problem: pointers are not inspected
  if (!hi || !scale || !xq || !xscale || !y) return BITNEST_ERR_INVALID_ARG;
  if (mode == BITNEST_TARGET && !lo) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(hi) || misaligned(scale) || misaligned(xq) || misaligned(xscale) ||
      (xsum && misaligned(xsum)) || misaligned(y) || (bias && misaligned(bias)) ||
      (mode == BITNEST_TARGET && misaligned(lo)))
    return BITNEST_ERR_MISALIGNED;
  return BITNEST_OK;
}

// The TMA-ring GEMV where it applies; with split-K scratch available, the
// tensor-core path before the plain-load GEMV (whose single pass over a long
// K with up to 8 tokens is slower than K split across the GPU).
int pick_path(int mode, int64_t M, int64_t N, int64_t K, bool ws = false) {
  (void)mode;
  if (gemv_tma_supported(M, N, K)) return BITNEST_PATH_GEMV;
  if (ws && tc_ws_bytes(M, N, K) > 0) return BITNEST_PATH_TC;
  if (gemv_fits(M, K)) return BITNEST_PATH_GEMV;
  return BITNEST_PATH_TC;
}

int run_linear(const LinearArgs &a, int path, cudaStream_t st) {
  if (path == BITNEST_PATH_AUTO) path = pick_path(a.mode, a.M, a.N, a.K);
  if (path == BITNEST_PATH_GEMV) {
    if (gemv_tma_supported(a.M, a.N, a.K)) return cuda_status(launch_gemv_tma(a, st));
    if (!gemv_fits(a.M, a.K)) return BITNEST_ERR_UNSUPPORTED_SHAPE;
    return cuda_status(launch_gemv(a, st));
  }
  if (path == BITNEST_PATH_TC) {
    if (!tc_supported(a.M, a.N, a.K)) return BITNEST_ERR_UNSUPPORTED_SHAPE;
    return cuda_status(launch_tc(a, st));
  }
  return BITNEST_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

const char *bitnest_status_string(int status) {
  switch (status) {
    case BITNEST_OK: return "ok";
    case BITNEST_ERR_INVALID_ARG: return "invalid argument";
    case BITNEST_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BITNEST_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case BITNEST_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int bitnest_version(void) { return 100; }

int bitnest_device_wait_timeout(int reset) {
  int f1 = 0, f2 = 0;
  if (read_wait_timeout(&f1, reset != 0) != cudaSuccess) return -BITNEST_ERR_CUDA;
  if (read_wait_timeout_gemv(&f2, reset != 0) != cudaSuccess) return -BITNEST_ERR_CUDA;
  // a split call that gave up may have left arrivals in the counters of the
  // library's static scratch: the reset clears them as well
  if (reset && f1) {
    if (tc_static_ws_clear_counters(nullptr) != cudaSuccess) return -BITNEST_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return -BITNEST_ERR_CUDA;
  }
  return (f1 | f2) ? 1 : 0;
}

int bitnest_debug_wait_probe(void *stream) {
  return cuda_status(launch_wait_probe((cudaStream_t)stream));
}

int bitnest_pack_planes(const uint8_t *uh, const uint8_t *ul, int64_t N, int64_t K,
                        uint8_t *hi, uint8_t *lo, void *stream) {
  int s = check_shape(0, N, K);
  if (s != BITNEST_OK) return s;
  if (N == 0) return BITNEST_OK;
  if (!uh || !hi || (ul && !lo)) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(uh) || misaligned(hi) || (ul && (misaligned(ul) || misaligned(lo))))
    return BITNEST_ERR_MISALIGNED;
  if (N == 0) return BITNEST_OK;
  return cuda_status(launch_pack(uh, ul, N, K, hi, lo, (cudaStream_t)stream));
}

int bitnest_pack_weights(const uint16_t *w, int64_t N, int64_t K, uint8_t *hi, uint8_t *lo,
                         uint16_t *scale, void *stream) {
  int s = check_shape(0, N, K);
  if (s != BITNEST_OK) return s;
  if (N == 0) return BITNEST_OK;
  if (!w || !hi || !lo || !scale) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(w) || misaligned(hi) || misaligned(lo) || misaligned(scale))
    return BITNEST_ERR_MISALIGNED;
  return cuda_status(launch_pack_weights(w, N, K, hi, lo, scale, (cudaStream_t)stream));
}

int bitnest_quantize_act(const uint16_t *x, int64_t M, int64_t K, int act_group, int8_t *xq,
                         float *xscale, int32_t *xsum, void *stream) {
  if (act_group != 0 && act_group != kGroup) return BITNEST_ERR_INVALID_ARG;
  int s = check_shape(M, 0, K);
  if (s != BITNEST_OK) return s;
  if (M == 0) return BITNEST_OK;
  if (!x || !xq || !xscale) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(x) || misaligned(xq) || misaligned(xscale) || (xsum && misaligned(xsum)))
    return BITNEST_ERR_MISALIGNED;
  if (M == 0) return BITNEST_OK;
  return cuda_status(launch_quantize(x, M, K, act_group, xq, xscale, xsum, (cudaStream_t)stream));
}

int bitnest_hadamard_quantize_act(const uint16_t *x, int64_t M, int64_t K, int8_t *xq,
                                  float *xscale, int32_t *xsum, void *stream) {
  int s = check_shape(M, 0, K);
  if (s != BITNEST_OK) return s;
  if (!hadamard_supported(K)) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BITNEST_OK;
  if (!x || !xq || !xscale) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(x) || misaligned(xq) || misaligned(xscale) || (xsum && misaligned(xsum)))
    return BITNEST_ERR_MISALIGNED;
  return cuda_status(launch_hadamard_quantize(x, M, K, xq, xscale, xsum, (cudaStream_t)stream));
}

int bitnest_nested_attention(int mode, const uint16_t *q, int64_t H, int64_t Hkv, int64_t D,
                             int64_t T, const uint8_t *k_hi, const uint8_t *k_lo,
                             const uint16_t *k_scale, const uint8_t *v_hi, const uint8_t *v_lo,
                             const uint16_t *v_scale, float *out, void *stream) {
  if (mode != BITNEST_DRAFT && mode != BITNEST_TARGET) return BITNEST_ERR_INVALID_ARG;
  if (!nested_attention_supported(H, Hkv, D, T)) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (!q || !k_hi || !k_scale || !v_hi || !v_scale || !out) return BITNEST_ERR_INVALID_ARG;
  if (mode == BITNEST_TARGET && (!k_lo || !v_lo)) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(q) || misaligned(k_hi) || misaligned(k_scale) || misaligned(v_hi) ||
      misaligned(v_scale) || misaligned(out) ||
      (mode == BITNEST_TARGET && (misaligned(k_lo) || misaligned(v_lo))))
    return BITNEST_ERR_MISALIGNED;
  return cuda_status(launch_nested_attention(mode, q, H, Hkv, T, k_hi,
                                             mode == BITNEST_TARGET ? k_lo : nullptr, k_scale,
                                             v_hi, mode == BITNEST_TARGET ? v_lo : nullptr,
                                             v_scale, out, (cudaStream_t)stream));
}

int bitnest_act_group_sums(const int8_t *xq, int64_t M, int64_t K, int32_t *xsum,
                           void *stream) {
  int s = check_shape(M, 0, K);
  if (s != BITNEST_OK) return s;
  if (M == 0) return BITNEST_OK;
  if (!xq || !xsum) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(xq) || misaligned(xsum)) return BITNEST_ERR_MISALIGNED;
  if (M == 0) return BITNEST_OK;
  return cuda_status(launch_act_group_sums(xq, M, K, xsum, (cudaStream_t)stream));
}

int bitnest_select_path(int mode, int64_t M, int64_t N, int64_t K) {
  return pick_path(mode, M, N, K);
}

int bitnest_linear_path(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                        const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                        int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                        int path, void *stream) {
  const bool overlap = (path & BITNEST_PATH_OVERLAP) != 0;
  path &= ~BITNEST_PATH_OVERLAP;
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return BITNEST_ERR_INVALID_ARG;
  int s = check_linear(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y, act_group, bias);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;
  LinearArgs a{mode, hi, mode == BITNEST_TARGET ? lo : nullptr, scale, xq, xscale, xsum,
               bias, y, nullptr, M, N, K, act_group, overlap};
  return run_linear(a, path, (cudaStream_t)stream);
}

int64_t bitnest_linear_ws_bytes(int mode, int64_t M, int64_t N, int64_t K, int path) {
  path &= ~BITNEST_PATH_OVERLAP;
  if (mode != BITNEST_DRAFT && mode != BITNEST_TARGET) return -BITNEST_ERR_INVALID_ARG;
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return -BITNEST_ERR_INVALID_ARG;
  if (check_shape(M, N, K) != BITNEST_OK) return -BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return 0;
  if (path == BITNEST_PATH_AUTO) path = pick_path(mode, M, N, K, true);
  return path == BITNEST_PATH_TC ? tc_ws_bytes(M, N, K) : 0;
}

int bitnest_linear_ws(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                      const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                      int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                      int path, void *ws, int64_t ws_bytes, void *stream) {
  const bool overlap = (path & BITNEST_PATH_OVERLAP) != 0;
  path &= ~BITNEST_PATH_OVERLAP;
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return BITNEST_ERR_INVALID_ARG;
  int s = check_linear(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y, act_group, bias);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;
  if (path == BITNEST_PATH_AUTO) path = pick_path(mode, M, N, K, true);
  const int64_t need = path == BITNEST_PATH_TC ? tc_ws_bytes(M, N, K) : 0;
  if (need > 0) {
    if (!ws || ws_bytes < need) return BITNEST_ERR_INVALID_ARG;
    if (misaligned(ws)) return BITNEST_ERR_MISALIGNED;
  }
  LinearArgs a{mode, hi, mode == BITNEST_TARGET ? lo : nullptr, scale, xq, xscale, xsum,
               bias, y, nullptr, M, N, K, act_group, overlap};
  if (need > 0) {
    a.ws = ws;
    a.ws_bytes = ws_bytes;
  }
  return run_linear(a, path, (cudaStream_t)stream);
}

int bitnest_linear_static_ws(int mode, const uint8_t *hi, const uint8_t *lo,
                             const uint16_t *scale, const int8_t *xq, const float *xscale,
                             const int32_t *xsum, int64_t M, int64_t N, int64_t K, float *y,
                             int act_group, const uint16_t *bias, int path, void *stream) {
  static_assert(kStaticWsBytes == BITNEST_STATIC_WS_BYTES, "scratch size");
  const bool overlap = (path & BITNEST_PATH_OVERLAP) != 0;
  path &= ~BITNEST_PATH_OVERLAP;
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return BITNEST_ERR_INVALID_ARG;
  int s = check_linear(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y, act_group, bias);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;
  if (path == BITNEST_PATH_AUTO) path = pick_path(mode, M, N, K, true);
  const int64_t need = path == BITNEST_PATH_TC ? tc_ws_bytes(M, N, K) : 0;
  if (need > kStaticWsBytes) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  LinearArgs a{mode, hi, mode == BITNEST_TARGET ? lo : nullptr, scale, xq, xscale, xsum,
               bias, y, nullptr, M, N, K, act_group, overlap};
  if (need > 0) {
    void *ws = nullptr;
    if (tc_static_ws(&ws) != cudaSuccess) return BITNEST_ERR_CUDA;
    a.ws = ws;
    a.ws_bytes = kStaticWsBytes;
  }
  return run_linear(a, path, (cudaStream_t)stream);
}

int bitnest_linear(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                   const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                   int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                   void *stream) {
  return bitnest_linear_path(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y, act_group,
                             bias, BITNEST_PATH_AUTO, stream);
}

int bitnest_quantize_linear(int mode, const uint8_t *hi, const uint8_t *lo,
                            const uint16_t *scale, const uint16_t *x, int64_t M, int64_t N,
                            int64_t K, float *y, int act_group, const uint16_t *bias,
                            int8_t *xq, float *xscale, int32_t *xsum, int path, void *stream) {
  const bool overlap = (path & BITNEST_PATH_OVERLAP) != 0;
  path &= ~BITNEST_PATH_OVERLAP;
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return BITNEST_ERR_INVALID_ARG;
  int s = check_linear(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y, act_group, bias);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;
  if (!x) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(x)) return BITNEST_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;
  LinearArgs a{mode, hi, mode == BITNEST_TARGET ? lo : nullptr, scale, xq, xscale, xsum,
               bias, y, nullptr, M, N, K, act_group, overlap};
  if (path == BITNEST_PATH_AUTO) path = pick_path(mode, M, N, K);
  // the layer's shape is checked before anything is launched
  if (path == BITNEST_PATH_GEMV && !gemv_tma_supported(M, N, K) && !gemv_fits(M, K))
    return BITNEST_ERR_UNSUPPORTED_SHAPE;
  if (path == BITNEST_PATH_TC && !tc_supported(M, N, K)) return BITNEST_ERR_UNSUPPORTED_SHAPE;
  s = cuda_status(launch_quantize(x, M, K, act_group, xq, xscale, xsum, st));
  if (s != BITNEST_OK) return s;
  return run_linear(a, path, st);
}

int bitnest_debug_group_sums(int mode, const uint8_t *hi, const uint8_t *lo,
                             const int8_t *xq, const int32_t *xsum, int64_t M, int64_t N,
                             int64_t K, int32_t *S, int path, void *stream) {
  if (path < BITNEST_PATH_AUTO || path > BITNEST_PATH_TC) return BITNEST_ERR_INVALID_ARG;
  if (mode != BITNEST_DRAFT && mode != BITNEST_TARGET) return BITNEST_ERR_INVALID_ARG;
  int s = check_shape(M, N, K);
  if (s != BITNEST_OK) return s;
  if (M == 0 || N == 0) return BITNEST_OK;
  if (!hi || !xq || !S || (mode == BITNEST_TARGET && !lo)) return BITNEST_ERR_INVALID_ARG;
  if (misaligned(hi) || misaligned(xq) || (xsum && misaligned(xsum)) || misaligned(S) ||
      (mode == BITNEST_TARGET && misaligned(lo)))
    return BITNEST_ERR_MISALIGNED;
  if (M == 0 || N == 0) return BITNEST_OK;
  LinearArgs a{mode, hi, mode == BITNEST_TARGET ? lo : nullptr, nullptr, xq, nullptr, xsum,
               nullptr, nullptr, S, M, N, K, 0, false};
  return run_linear(a, path, (cudaStream_t)stream);
}

}  // extern "C"
