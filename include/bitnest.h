/*
 * bitnest.h -- C ABI of the BitNest bit-nested W4/W8 quantised linear layer
 * on NVIDIA B200 (sm_100a).
 *
 * What the layer computes (BitNest-Llama-3-8B model card, section "Files",
 * planes.safetensors entry, and the model table rows "Weights" and
 * "Activations"): one stored 8-bit weight code serves two precisions.
 *   hi, lo : uint8 [N, K/2] planes of unsigned nibbles u = q + 8; byte j of a
 *            row holds column 2j in its low nibble and column 2j+1 in its high
 *            nibble.
 *   scale  : fp16 [N, K/128], one scale per 128-column group.
 *   draft  (W4A8) reads hi only:   W4[n,k] = (hi - 8) * scale
 *   target (W8A8) reads hi and lo: W8[n,k] = (16*(hi - 8) + (lo - 8)) * scale / 16
 *   activations are symmetric int8, one scale per token (per 128-column
 *   group for o_proj): x[m,k] ~= xq[m,k] * xscale.
 *   y[m,n] = sum_k (xq[m,k] * xscale) * W[n,k] (+ bias[n]).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers to row-major, contiguous
 *     arrays; the caller allocates, owns and frees them.  The library
 *     allocates no memory and keeps no state beyond cached device
 *     attributes and driver entry points.
 *   - fp16 arrays are passed as their IEEE binary16 bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously on it; the entry points are re-entrant.
 *   - Every argument check runs on the host, before anything is launched.  A
 *     failed check returns a non-zero BITNEST_ERR_* status and launches
 *     nothing.  A launch failure returns BITNEST_ERR_CUDA.  Faults during
 *     execution surface at the caller's next synchronisation.
 *   - M == 0 or N == 0 is an empty problem: BITNEST_OK, nothing launched, and
 *     the pointers are not inspected (after mode / group / K are checked).
 *   - K must be a positive multiple of 128 (the group size).
 *   - Base pointers must be 16-byte aligned (BITNEST_ERR_MISALIGNED).
 */
#ifndef BITNEST_H_
#define BITNEST_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Which model reads the planes. */
#define BITNEST_DRAFT 0  /* W4A8: hi plane only        */
#define BITNEST_TARGET 1 /* W8A8: hi and lo planes    */

/* Kernel family for bitnest_linear_path. */
#define BITNEST_PATH_AUTO 0 /* the library picks (see bitnest_select_path)          */
#define BITNEST_PATH_GEMV 1 /* decode GEMV (planes streamed by TMA, integer
                               mma.sync group sums), M <= BITNEST_GEMV_MAX_M
                               (<= 8 where K is not a multiple of 1024) */
#define BITNEST_PATH_TC 2   /* tcgen05 kind::i8 tensor-core GEMM, any M              */

#define BITNEST_GEMV_MAX_M 16 /* largest M the GEMV kernels are built for */

/* May be OR-ed into the `path` of bitnest_linear_path: the layer kernel is
 * launched with programmatic dependent launch and starts streaming hi, lo and
 * scale before the preceding kernel on the stream has finished; it waits for
 * that kernel only before it reads xq / xscale / xsum.  Safe when no kernel
 * still running on the stream writes the planes or the scales (a
 * bitnest_quantize_act call right before is always safe: it waits for its own
 * predecessor before it lets the next kernel start).  Setting the environment
 * variable BITNEST_PDL=0 before the first call turns programmatic dependent
 * launch off for every kernel of the library (profilers that replay captured
 * graphs cannot replay such launches). */
#define BITNEST_PATH_OVERLAP 0x100

/* Status codes. */
#define BITNEST_OK 0
#define BITNEST_ERR_INVALID_ARG 1       /* null pointer, bad mode / group / path        */
#define BITNEST_ERR_UNSUPPORTED_SHAPE 2 /* K not a positive multiple of 128, sizes < 0 */
#define BITNEST_ERR_MISALIGNED 3        /* a base pointer is not 16-byte aligned       */
#define BITNEST_ERR_CUDA 4              /* a CUDA launch or driver call failed         */

/* Human-readable name of a status code (static storage, never NULL). */
const char *bitnest_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int bitnest_version(void);

/* Every wait of the layer kernels on another warp or on a copy is bounded
 * (a few seconds of device time); a wait that gives up sets a device flag and
 * the kernel winds down without finishing its output.  Returns that flag for
 * the current device (1: some launch since the last reset gave up, its
 * outputs are invalid; 0: none), or -BITNEST_ERR_CUDA.  Synchronous: reads
 * device memory.  reset != 0 clears the flag after reading it and, when it
 * was set, also zeroes the arrival counters of the static split-K scratch
 * (see bitnest_linear_static_ws).  A split-K call that gave up leaves the
 * counters of caller scratch at zero as well: its warps still arrive. */
int bitnest_device_wait_timeout(int reset);

/* Test hook for the flag above: launches one warp that waits, with the
 * kernels' bounded wait (cut to 200 us of device time), on an mbarrier that
 * nothing arrives at.  The wait gives up, sets the flag and the kernel
 * returns; nothing faults or hangs.  Asynchronous on `stream`; clear the flag with
 * bitnest_device_wait_timeout(1) afterwards, or later bounded waits give up
 * at once. */
int bitnest_debug_wait_probe(void *stream);

/*
 * Build the planes and scales of one layer from its fp16 weights
 * (BitNest-Llama-3-8B model card, opening paragraph: the high nibble is a
 * 4-bit model fitted first, the low nibble the closed-form residual back to
 * 8 bits; section "Files": u = q + 8, one fp16 scale per 128 columns).  The
 * card fits the high nibble with GPTQ, which needs calibration data; this
 * packer rounds it to nearest instead:
 *   s  = fp16(max|W| / 7) per row and 128-column group (0 for an all-zero
 *        group, whose nibbles are then 8),
 *   t  = W / s (fp32, correctly rounded),
 *   hi = rne(t) + 8,  lo = clamp(rne(16 (t - (hi - 8))), -8, 7) + 8.
 * The draft W4 = (hi - 8) s is then within s/2 of W and the target W8 within
 * s/16 (s/32 where lo is not clamped).
 *   w      : fp16 [N, K] weights (finite).
 *   hi, lo : uint8 [N, K/2] planes (outputs, the card's byte layout).
 *   scale  : fp16 [N, K/128] (output).
 * K must be a positive multiple of 128; checks and errors as the other
 * entry points.
 */
int bitnest_pack_weights(const uint16_t *w, int64_t N, int64_t K, uint8_t *hi, uint8_t *lo,
                         uint16_t *scale, void *stream);

/*
 * The down_proj input path: online Hadamard rotation (model card, model
 * table row "Rotation": R4 online Hadamard on down_proj inputs) fused with
 * the per-token quantiser.  The card ships its R4 matrices, not their
 * construction; this library's reading:
 *   x_rot = x H / sqrt(K), H of order K:
 *     K = p (a power of two)      : Sylvester's matrix (-1)^popcount(i & j);
 *     K = 28 p (p a power of two) : H = H28 (x) H_p (Kronecker product, the
 *        order-28 factor outer), H28 = I + S from Paley's construction I
 *        over GF(27) = GF(3)[x] / (x^3 - x - 1).
 *   Then, per token, as bitnest_quantize_act with act_group 0 on the fp32
 *   rotated values: xscale = max|x_rot| / 127, xq = rne(x_rot / xscale),
 *   xsum = per-128-group sums of xq.
 * The rotation runs in fp32 (a Walsh-Hadamard transform per length-p block,
 * then the order-28 mix), so x_rot carries fp32 rounding: a code may differ
 * by one from that of the exact rotation where x_rot / xscale is within
 * rounding of a half-integer.
 *   x : fp16 [M, K];  xq : int8 [M, K];  xscale : fp32 [M];
 *   xsum : int32 [M, K/128] or NULL.
 * K must be p or 28 p as above, a multiple of 128 and at most 32768
 * (else BITNEST_ERR_UNSUPPORTED_SHAPE); e.g. down_proj's K = 14336 = 28 x 512.
 */
int bitnest_hadamard_quantize_act(const uint16_t *x, int64_t M, int64_t K, int8_t *xq,
                                  float *xscale, int32_t *xsum, void *stream);

/*
 * Decode attention of one new token over a nested KV cache (model card,
 * model table row "KV cache": nested at runtime, the draft reads KV4, the
 * target KV8).  The card does not give the cache layout; this library's
 * reading is the weights' nesting: each K (V) row of one token and one KV
 * head, D = 128 values, is packed by bitnest_pack_weights (planes and one
 * fp16 scale per row); the draft dequantises (hi - 8) s and reads only the
 * hi planes, the target (16 (hi - 8) + (lo - 8)) s / 16.
 *   q                   : fp16 [H, D], the new token's query heads.
 *   k_hi, k_lo, v_hi, v_lo : uint8 [T * Hkv, D/2] planes, row t * Hkv + j
 *                         = token t, KV head j (lo planes only for TARGET).
 *   k_scale, v_scale    : fp16 [T * Hkv, D/128] = [T * Hkv, 1].
 *   out                 : fp32 [H, D];  head h attends with KV head
 *                         h / (H / Hkv):  softmax(q K^T / sqrt(D)) V.
 * D must be 128, H / Hkv one of 1, 2, 4, 8, T >= 1 (else
 * BITNEST_ERR_UNSUPPORTED_SHAPE).  Both products run on the tensor cores with
 * fp16 operands that are exact (the queries as given, the integer codes) and
 * fp32 accumulation; the scales and the softmax are fp32, and p * v_scale
 * enters as two fp16 terms (22 bits): within 1e-3 of an exact evaluation in
 * the normalised error max |out - ref| / (|ref| + 1e-3 rms(ref)).  One launch:
 * the tokens of each KV head are split over a thread-block cluster of up to
 * 16 CTAs (8 where the device cannot place 16), merged in the cluster's
 * shared memory; nothing is allocated, no scratch is needed.
 */
int bitnest_nested_attention(int mode, const uint16_t *q, int64_t H, int64_t Hkv, int64_t D,
                             int64_t T, const uint8_t *k_hi, const uint8_t *k_lo,
                             const uint16_t *k_scale, const uint8_t *v_hi, const uint8_t *v_lo,
                             const uint16_t *v_scale, float *out, void *stream);

/*
 * Pack unpacked nibbles into the planes of the model card's layout
 * ("Files": byte j holds column 2j in its low nibble, 2j+1 in its high).
 *   uh, ul : uint8 [N, K] nibble values; only the low 4 bits are used.
 *            ul may be NULL (then lo is not written; lo may be NULL too).
 *   hi, lo : uint8 [N, K/2] outputs.
 * K must be a positive multiple of 128.
 */
int bitnest_pack_planes(const uint8_t *uh, const uint8_t *ul, int64_t N, int64_t K,
                        uint8_t *hi, uint8_t *lo, void *stream);

/*
 * Symmetric int8 activation quantiser (model table row "Activations").
 *   x         : fp16 [M, K] activations (finite values).
 *   act_group : 0   -> one scale per token;   xscale is fp32 [M]
 *               128 -> one scale per (token, 128-column group) (o_proj);
 *                      xscale is fp32 [M, K/128].
 *   xq        : int8 [M, K] output, q = clamp(rne(x / s), -127, 127) with
 *               s = max|x| / 127 computed in fp32 (correctly rounded
 *               division, round-half-even); an all-zero span gives s = 0, q = 0.
 *   xsum      : int32 [M, K/128] output, xsum[m,g] = sum of xq[m,k] over the
 *               128 columns of group g; may be NULL (not written).
 *               bitnest_linear needs it (see there).
 */
int bitnest_quantize_act(const uint16_t *x, int64_t M, int64_t K, int act_group, int8_t *xq,
                         float *xscale, int32_t *xsum, void *stream);

/*
 * Per-128-group sums of already quantised activations:
 *   xsum[m, g] = sum_{k in group g} xq[m, k]   (int32 [M, K/128]).
 * An optional input of the layer entry points (they form the sums
 * themselves when given none).
 */
int bitnest_act_group_sums(const int8_t *xq, int64_t M, int64_t K, int32_t *xsum,
                           void *stream);

/*
 * The nested linear layer, y = dequant(xq, xscale) * W^T (+ bias), with W the
 * draft (mode = BITNEST_DRAFT, W4A8) or target (BITNEST_TARGET, W8A8) weight.
 *   hi, lo    : uint8 [N, K/2] planes; lo is ignored (may be NULL) for DRAFT
 *               and required for TARGET.
 *   scale     : fp16 [N, K/128] group scales.
 *   xq        : int8 [M, K] quantised activations.
 *   xscale    : fp32 [M] (act_group 0) or [M, K/128] (act_group 128).
 *   xsum      : int32 [M, K/128] group sums of xq, or NULL.  The kernels fold
 *               the planes' unsigned-nibble offset (8 for hi, 136 for the
 *               combined byte) into one correction per (token, group), which
 *               needs these sums: the decode GEMV always forms them from the
 *               codes it stages; the tensor-core path takes them from here
 *               when given (they must match xq, as bitnest_quantize_act's
 *               do) and otherwise forms them from the activation tiles it
 *               loads.  The result is the same either way.
 *   y         : fp32 [M, N] output.
 *   bias      : fp16 [N] or NULL.
 * Integer group sums are exact (int32); the epilogue is fp32, so y agrees
 * with an exact evaluation to within fp32 summation rounding.
 */
int bitnest_linear(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                   const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                   int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                   void *stream);

/* bitnest_linear with an explicit kernel family (BITNEST_PATH_*, optionally
 * OR-ed with BITNEST_PATH_OVERLAP).  PATH_GEMV requires M <= BITNEST_GEMV_MAX_M,
 * and M <= 8 where K is not a multiple of 1024, and the tokens' codes must fit
 * the kernel's shared memory (else BITNEST_ERR_UNSUPPORTED_SHAPE). */
int bitnest_linear_path(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                        const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                        int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                        int path, void *stream);

/*
 * bitnest_linear_path with caller-provided scratch `ws` (device memory,
 * 16-byte aligned, ws_bytes long) that the tensor-core path uses to split K
 * when the layer has too few (row tile, token tile) pairs to fill the GPU
 * (few output rows and tokens, long K: e.g. down_proj, N = 4096, K = 14336,
 * at M <= 128).  The split ranges' fp32 partial sums go to ws; the last range
 * to finish each sub-block adds them in a fixed order, so results do not
 * depend on timing.  They agree with bitnest_linear_path's to within fp32
 * summation rounding (the group sums themselves are the same exact int32).
 *   ws, ws_bytes : at least bitnest_linear_ws_bytes(mode, M, N, K, path)
 *                  bytes (BITNEST_ERR_INVALID_ARG if fewer).  When that is 0
 *                  ws may be NULL and the call is bitnest_linear_path.
 * The first 8 KB of ws hold arrival counters that must be zero before the
 * first call (cudaMemset once); every call leaves them zero, also one whose
 * bounded wait gave up, so one ws can serve calls of any shapes.  Calls sharing one ws must not run at the same
 * time (calls in order on one stream are fine).
 * With BITNEST_PATH_AUTO the choice may differ from bitnest_select_path's:
 * where the TMA-ring GEMV does not apply and K would be split, the
 * tensor-core path is taken (e.g. 5..8 tokens with K = 14336).
 * Other arguments, checks and errors: as bitnest_linear_path.
 */
int bitnest_linear_ws(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                      const int8_t *xq, const float *xscale, const int32_t *xsum, int64_t M,
                      int64_t N, int64_t K, float *y, int act_group, const uint16_t *bias,
                      int path, void *ws, int64_t ws_bytes, void *stream);

/*
 * bitnest_linear_ws without caller scratch and without any allocation: the
 * split-K partial sums and counters live in one file-scope static device
 * array of the library, BITNEST_STATIC_WS_BYTES (12 MiB) per device, zero
 * from module load and left zero by every call (a call whose bounded wait
 * gave up also leaves them zero; clearing the timeout flag zeroes them once
 * more).  (The BitNest pages have no counterpart to this entry point: it is a
 * deployment convenience of this library.)  The library calls no cudaMalloc /
 * cudaFree here; the first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, once per device, thread-safe) and caches it.
 * cudaDeviceReset unloads the module: the cached address is stale after it.
 *   - A problem whose split needs more than BITNEST_STATIC_WS_BYTES returns
 *     BITNEST_ERR_UNSUPPORTED_SHAPE, launching nothing.
 *   - Every call on a device shares the one array: calls that overlap in
 *     time (on different streams or threads) race and give wrong results.
 *     Calls in order on one stream are safe, BITNEST_PATH_OVERLAP included.
 *   - Make the first call on each device outside CUDA stream capture (the
 *     address lookup is not a capturable operation); later calls may be
 *     captured.
 * Results are bit-identical to bitnest_linear_ws's for the same arguments.
 * Other arguments, checks and errors: as bitnest_linear_ws.
 */
#define BITNEST_STATIC_WS_BYTES (12LL << 20)
int bitnest_linear_static_ws(int mode, const uint8_t *hi, const uint8_t *lo,
                             const uint16_t *scale, const int8_t *xq, const float *xscale,
                             const int32_t *xsum, int64_t M, int64_t N, int64_t K, float *y,
                             int act_group, const uint16_t *bias, int path, void *stream);

/* Scratch bytes bitnest_linear_ws uses for this problem and path (0 when the
 * path does not split K).  Host only; -BITNEST_ERR_INVALID_ARG for a bad
 * mode or path, -BITNEST_ERR_UNSUPPORTED_SHAPE for a bad shape. */
int64_t bitnest_linear_ws_bytes(int mode, int64_t M, int64_t N, int64_t K, int path);

/*
 * Activation quantiser and nested linear layer in one call: the same results
 * as bitnest_quantize_act(x, M, K, act_group, xq, xscale, xsum) followed by
 * bitnest_linear_path(mode, hi, lo, scale, xq, xscale, xsum, M, N, K, y,
 * act_group, bias, path), bit for bit in xq / xscale / xsum and y.
 *   x                 : fp16 [M, K] activations (finite values).
 *   xq, xscale        : outputs as in bitnest_quantize_act (required).
 *   xsum              : output as in bitnest_quantize_act, or NULL (then not
 *                       written, and the layer forms the sums itself).
 * The quantiser and the layer kernel run back to back on `stream`; with
 * BITNEST_PATH_OVERLAP the layer kernel streams its weights while the
 * quantiser runs.  Argument checks and
 * error behaviour are those of bitnest_linear_path plus: x non-NULL and
 * 16-byte aligned.
 */
int bitnest_quantize_linear(int mode, const uint8_t *hi, const uint8_t *lo,
                            const uint16_t *scale, const uint16_t *x, int64_t M, int64_t N,
                            int64_t K, float *y, int act_group, const uint16_t *bias,
                            int8_t *xq, float *xscale, int32_t *xsum, int path, void *stream);

/*
 * Speculative decoding with the nested weights (BitNest-Llama-3-8B model
 * card, opening paragraph: the W4A8 draft proposes tokens and the W8A8
 * target verifies every one of them, so the output is exactly the target's
 * greedy output; model table row "Default draft length": gamma = 3).  The
 * pages give no model; these entry points run a small synthetic one built
 * from the nested linear layer (bitnest_quantize_linear per layer):
 *   input at position p : x0 = fp16(E[t_p] + 0.5 E[t_{p-1}])   (t_{-1} := t_0)
 *   layer l             : x_{l+1} = fp16(tanh(W_l x_l)),  W_l nested [dim, dim]
 *   head                : logits = W_head x_L,             W_head nested [vocab, dim]
 *   next token          : argmax of the logits, lowest index among equal maxima
 * A round: gamma draft steps (draft weights, one token each), one target pass
 * over the gamma + 1 positions together, then the accept step appends the
 * leading draft tokens the target agrees with and the target's own token
 * after them (1 .. gamma + 1 tokens).  The sequence, its length and the
 * statistics live in device memory: nothing is read back to the host, and
 * the rounds can be captured in a CUDA graph.
 *   model  : host struct; embed fp16 [vocab, dim]; hi / lo / scale are HOST
 *            arrays of `layers` DEVICE pointers (planes uint8 [dim, dim/2],
 *            scales fp16 [dim, dim/128]); head planes [vocab, dim/2], scales
 *            [vocab, dim/128].  dim a positive multiple of 128.
 *   seq    : int32 [cap] device, tokens 0 .. *len - 1 on entry (*len >= 1);
 *            tokens are appended.  The caller keeps cap >= *len + rounds *
 *            (gamma + 1) (greedy: + steps); a write that would pass cap is
 *            not made and sets stats[3].
 *   len    : int32 device scalar, updated in place.
 *   stats  : int32 [4] device, accumulated: rounds, tokens appended, draft
 *            tokens accepted, capacity overflow flag.
 *   work   : device scratch of bitnest_spec_work_bytes(vocab, dim, gamma)
 *            bytes (16-byte aligned), owned by the caller.
 * gamma in 0 .. BITNEST_GEMV_MAX_M - 1.  Checks and errors as the other
 * entry points; everything is asynchronous on `stream`.
 */
typedef struct bitnest_spec_model {
  int64_t vocab, dim, layers;
  const uint16_t *embed;
  const uint8_t *const *hi;
  const uint8_t *const *lo;
  const uint16_t *const *scale;
  const uint8_t *head_hi;
  const uint8_t *head_lo;
  const uint16_t *head_scale;
} bitnest_spec_model;

/* Scratch bytes of a round (or of greedy decoding with gamma = 0);
 * -BITNEST_ERR_UNSUPPORTED_SHAPE for a bad shape.  Host only. */
int64_t bitnest_spec_work_bytes(int64_t vocab, int64_t dim, int gamma);

/* `rounds` speculative rounds with draft length `gamma`. */
int bitnest_spec_rounds(const bitnest_spec_model *model, int gamma, int rounds, int32_t *seq,
                        int64_t cap, int32_t *len, int32_t *stats, void *work,
                        int64_t work_bytes, void *stream);

/* `steps` tokens of the target's own greedy decoding (one position per step):
 * the sequence speculative rounds must reproduce. */
int bitnest_spec_greedy(const bitnest_spec_model *model, int steps, int32_t *seq, int64_t cap,
                        int32_t *len, int32_t *stats, void *work, int64_t work_bytes,
                        void *stream);

/* The kernel family BITNEST_PATH_AUTO picks for this problem (host only,
 * launches nothing).  Returns BITNEST_PATH_GEMV or BITNEST_PATH_TC. */
int bitnest_select_path(int mode, int64_t M, int64_t N, int64_t K);

/*
 * Test hook: the exact int32 group sums the kernels of `path` form,
 *   S[m, n, g] = sum_{k in g} xq[m,k] * code[n,k],
 * code = hi - 8 (DRAFT) or 16*(hi - 8) + (lo - 8) (TARGET), written to
 * S int32 [M, N, K/128].  Same inner loops as bitnest_linear_path; xsum as
 * there (may be NULL).
 */
int bitnest_debug_group_sums(int mode, const uint8_t *hi, const uint8_t *lo,
                             const int8_t *xq, const int32_t *xsum, int64_t M, int64_t N,
                             int64_t K, int32_t *S, int path, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BITNEST_H_ */
