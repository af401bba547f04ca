// Internal launchers (C++), called only by the C ABI in capi.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnest {

struct LinearArgs {
  int mode;               // 0 draft, 1 target
  const uint8_t *hi;      // [N, K/2]
  const uint8_t *lo;      // [N, K/2] (target)
  const uint16_t *scale;  // fp16 [N, K/128]
  const int8_t *xq;       // [M, K]
  const float *xscale;    // [M] or [M, K/128]
  const int32_t *xsum;    // [M, K/128] or null (the kernels form the sums)
  const uint16_t *bias;   // fp16 [N] or null
  float *y;               // [M, N]
  int32_t *S;             // debug group sums [M, N, K/128] (null unless debug)
  int64_t M, N, K;
  int act_group;          // 0 or 128
  bool overlap;           // launch with programmatic dependent launch
  // scratch of the tensor-core path's split K (null: no split), its bytes;
  // its counter area is zero before the call and zero again after it
  void *ws = nullptr;
  int64_t ws_bytes = 0;
};

cudaError_t launch_pack(const uint8_t *uh, const uint8_t *ul, int64_t N, int64_t K, uint8_t *hi,
                        uint8_t *lo, cudaStream_t st);
cudaError_t launch_pack_weights(const uint16_t *w, int64_t N, int64_t K, uint8_t *hi,
                                uint8_t *lo, uint16_t *scale, cudaStream_t st);
cudaError_t launch_quantize(const uint16_t *x, int64_t M, int64_t K, int act_group, int8_t *xq,
                            float *xs, int32_t *xsum, cudaStream_t st);
cudaError_t launch_act_group_sums(const int8_t *xq, int64_t M, int64_t K, int32_t *xsum,
                                  cudaStream_t st);
// Decode attention over a nested KV cache (D = 128, H / Hkv in {1,2,4,8}).
bool nested_attention_supported(int64_t H, int64_t Hkv, int64_t D, int64_t T);
cudaError_t launch_nested_attention(int mode, const uint16_t *q, int64_t H, int64_t Hkv,
                                    int64_t T, const uint8_t *k_hi, const uint8_t *k_lo,
                                    const uint16_t *k_scale, const uint8_t *v_hi,
                                    const uint8_t *v_lo, const uint16_t *v_scale, float *out,
                                    cudaStream_t st);
// Hadamard rotation x H / sqrt(K) + per-token quantisation (K = p or 28 p,
// p a power of two, K <= 32768).
bool hadamard_supported(int64_t K);
cudaError_t launch_hadamard_quantize(const uint16_t *x, int64_t M, int64_t K, int8_t *xq,
                                     float *xs, int32_t *xsum, cudaStream_t st);

// Largest M * K the GEMV kernels can stage in shared memory.
bool gemv_fits(int64_t M, int64_t K);
cudaError_t launch_gemv(const LinearArgs &a, cudaStream_t st);

// TMA-ring decode GEMV (K a multiple of 1024).
bool gemv_tma_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_tma(const LinearArgs &a, cudaStream_t st);
cudaError_t read_wait_timeout_gemv(int *flag, bool reset);

// tcgen05 tensor-core GEMM (any M).
bool tc_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_tc(const LinearArgs &a, cudaStream_t st);
// Scratch bytes the tensor-core path splits K with for this shape (0: none).
int64_t tc_ws_bytes(int64_t M, int64_t N, int64_t K);
// Size and device address (looked up once per device) of the library's own
// static split-K scratch.
constexpr int64_t kStaticWsBytes = int64_t(12) << 20;
cudaError_t tc_static_ws(void **ws);
// Zero the arrival counters of that scratch (after a bounded wait gave up).
cudaError_t tc_static_ws_clear_counters(cudaStream_t st);

// The flag a bounded wait sets when it gives up (synchronous read).
cudaError_t read_wait_timeout(int *flag, bool reset);
// Test hook: a wait that gives up (sets the flag above).
cudaError_t launch_wait_probe(cudaStream_t st);

}  // namespace bitnest
