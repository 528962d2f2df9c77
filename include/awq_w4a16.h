/*
 * awq_w4a16.h — C ABI of the AWQ W4A16 g128 library for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are web pages, cited by title and section):
 *
 *   "AWQ: Activation-aware Weight Quantization for LLM Compression and
 *   Acceleration" (llm-awq README mirror), "Usage" steps 1-3 and
 *   "Installation" step 3: 4-bit weights quantized in groups of 128 along the
 *   input dimension, 16-bit activations, CUDA kernels for the context (GEMM)
 *   and decode (GEMV) stages.
 *   "transformers - AWQ" (HF guide translation), section 2: the
 *   quantization_config {quant_method: awq, zero_point: true, group_size: 128,
 *   bits: 4, version: gemm}.
 *   CSDN VPTQ blog, section "02.02 AWQ": salient input channels are found
 *   from activation statistics and protected by scaling them up through an
 *   equivalent transform (weights times s, activations divided by s).
 *
 * Steps of the path and their entry points:
 *   a1  awq_activation_scale  s_k = max(mean_m |x_mk|, 1e-8)^alpha;  x'_mk = fp16(x_mk / s_k)
 *       awq_scale_activations x'_mk = fp16(x_mk / s_k) with a stored s
 *   a2  awq_quantize_g128     w'_nk = fp16(W_nk * s_k); per group of 128 k:
 *                             S = fp16(max(hi-lo, 1e-5)/15), z = clamp(rint(-lo/S), 0, 15),
 *                             q = clamp(rint(w'/S) + z, 0, 15)      (fp32, round half to even)
 *   a3  awq_w4a16_gemv        y[M,N] = x'[M,K] . ((q - z) * S)^T, M <= 32  (fp32 accumulate, fp16 out)
 *   a4  awq_w4a16_gemm        the same for any M (tensor-core prefill kernel);
 *       awq_gemm_plan         its launch plan for a shape (token tile, K split)
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller. The library
 *     allocates no memory and never synchronizes, except awq_poll_device_status
 *     and the test hooks awq_debug_set_wait_budget_ns and
 *     awq_debug_drop_first_copy, which say so.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and runs asynchronously; outputs are valid once the stream reaches
 *     that point.
 *   - Arguments are checked on the host before anything is launched. A bad
 *     argument returns an error code and launches nothing. No call aborts the
 *     process or throws.
 *   - fp16 buffers hold IEEE binary16 bit patterns (uint16_t here).
 *   - Outputs must not alias inputs.
 *   - Only device ordinals with compute capability 10.0 are supported
 *     (AWQ_ERR_UNSUPPORTED otherwise).
 *
 * Packed layout, version 2 (awq_layout_version() == 2): "tile-major".
 *   Rows are grouped in 16-row tiles, Ntiles = ceil(N/16). Along K the
 *   groups are padded to an even count: G = K/128, G2 = ceil(G/2) group
 *   pairs, KTp = 4*G2 64-k tiles per tile. Padding rows and padding groups
 *   hold code 0, scale 0, zero 0. With
 *     n = 16*T + 8*h + r                  (T tile, h half, r row)
 *     k = 64*kt + 16*t + 4*s + 2*e1 + e0  (kt 64-k tile, t column block, s step, e slot)
 *     g = k / 128
 *   qweight: uint32[Ntiles*KTp*128];  code q[n][k] sits in word
 *            (T*KTp + kt)*128 + (4*r + t)*4 + s,  nibble h + 2*e1 + 4*e0
 *            (bits 4*nibble .. 4*nibble+3).  The 16 bytes of words
 *            (.., 4r+t, 0..3) are exactly the m16n8k16 A-fragments of one lane
 *            (rows r, r+8; k in [16t, 16t+16) of a 64-k tile).
 *   scales:  fp16[Ntiles*2*G2*16]; S[n][g] at (T*2*G2 + g)*16 + 2*r + h
 *   zeros:   uint8[Ntiles*2*G2*8]; z[n][g] in byte (T*2*G2 + g)*8 + r,
 *            low nibble for h = 0, high nibble for h = 1.
 *   So one tile and group pair is 2048 bytes of codes, 64 of scales and 16
 *   of zeros, and each tile's codes, scales and zeros run contiguously along
 *   K: a range of (tile, group pair) items is one contiguous byte range of
 *   each array.
 *   Base pointers of qweight, scales, zeros, x, x' and y must be 16-byte aligned.
 */
#ifndef AWQ_W4A16_H_
#define AWQ_W4A16_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* the same type cudaStream_t points to */
typedef struct CUstream_st* awq_stream_t;

typedef enum {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, size out of range */
  AWQ_ERR_UNSUPPORTED = 2,   /* configuration or device not built (bits != 4, group != 128, ...) */
  AWQ_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
  AWQ_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  AWQ_ERR_TIMEOUT = 5,       /* a kernel gave up a bounded wait (reported by awq_poll_device_status) */
  AWQ_ERR_BOUNDS = 6         /* debug builds (-DAWQ_DEBUG_BOUNDS) only: a kernel's index check failed and
                                the access was skipped (reported by awq_poll_device_status) */
} awq_status_t;

/* Packed-layout version; bumps whenever the layout above changes. */
AWQ_API int awq_layout_version(void);

/* Static, human-readable name of a status code. Never NULL. */
AWQ_API const char* awq_status_string(int status);

/* AWQ_OK iff (bits, group_size, zero_point) is a built configuration: bits 4
 * or 3, group size 128, zero point 1 or 0 — (4, 128, 1) is the
 * quantization_config of "transformers - AWQ" section 2 and the quant_config
 * of the AutoAWQ section of the llmstudio.ru page; INT3-g128 is in the model
 * zoo of the llm-awq README. AWQ_ERR_UNSUPPORTED otherwise (group size 64
 * included). Pure host function. */
AWQ_API awq_status_t awq_check_config(int bits, int group_size, int zero_point);

/* Sizes in bytes of the packed arrays for an N x K layer: Ntiles*G2 times
 * 2048 (qweight), 64 (scales) and 16 (zeros). 0 if N < 1, N > 2^31 - 128,
 * K < 128, K % 128 != 0 or 16*Ntiles*K > 2^34. Pure host functions. */
AWQ_API size_t awq_qweight_bytes(int N, int K);
AWQ_API size_t awq_scales_bytes(int N, int K);
AWQ_API size_t awq_zeros_bytes(int N, int K);

/* a1. Activation statistic and activation scaling (CSDN blog "02.02 AWQ":
 * scales from activation statistics; equivalent transform).
 *   x        fp16 [M, K] row-major (device).
 *   s_out    fp32 [K] (device): s_k = max(mean_m |x_mk|, 1e-8)^alpha, computed in
 *            float64 (the column sum is exact: integers in units of 2^-24) and
 *            rounded to fp32; alpha = 0.5 uses the correctly rounded square root.
 *   x_scaled fp16 [M, K] (device) or NULL: x'_mk = fp16_rn(fp32(x_mk) / s_k)
 *            (IEEE fp32 division).
 * Requires 1 <= M, 1 <= K, K % 8 == 0. alpha must be finite. */
AWQ_API awq_status_t awq_activation_scale(const uint16_t* x, int M, int K, float alpha,
                                  float* s_out, uint16_t* x_scaled, awq_stream_t stream);

/* a1 (inference form). x'_mk = fp16_rn(fp32(x_mk) / s_k) with a stored s
 * (calibrated once by awq_activation_scale); the activation half of the
 * equivalent transform of CSDN "02.02 AWQ".
 *   x        fp16 [M, K] row-major (device);  s  fp32 [K] (device, 16-byte aligned)
 *   x_scaled fp16 [M, K] (device).
 * Bit-identical to the x_scaled output of awq_activation_scale for the same s.
 * Requires 1 <= M, 1 <= K, K % 8 == 0. */
AWQ_API awq_status_t awq_scale_activations(const uint16_t* x, const float* s, int M, int K, uint16_t* x_scaled,
                                   awq_stream_t stream);

/* a2. Fold + asymmetric 4-bit group quantizer, group size 128 along K
 * ("Usage" steps 1-3 of the llm-awq README: --w_bit 4 --q_group_size 128,
 * --q_backend real; HF config zero_point true).
 *   W          fp16 [N, K] row-major (device).
 *   fold_scale fp32 [K] (device) or NULL (= all ones, no fold).
 *   qweight, scales, zeros: outputs in packed layout v2, sizes from awq_*_bytes.
 * Codes, scales and zeros are bit-identical to the rules in the file header
 * (every step IEEE fp32, round to nearest even). Requires N >= 1, K >= 128,
 * K % 128 == 0. Values with |W*s| >= 65520 overflow fp16 to inf; the result is
 * then defined by the same IEEE rules but is not a useful quantization. */
AWQ_API awq_status_t awq_quantize_g128(const uint16_t* W, const float* fold_scale, int N, int K,
                               uint32_t* qweight, uint16_t* scales, uint8_t* zeros,
                               awq_stream_t stream);

/* a2 variants: the same fold and group quantizer for the other configurations
 * the pages name — INT3-g128 (model-zoo table of the llm-awq README) and the
 * symmetric form (zero_point false; AutoAWQ section of the llmstudio.ru page:
 * zero_point selects asymmetric quantization).
 *   bits       4 or 3; 3-bit codes (0..7) occupy the same 4-bit slots of packed
 *              layout v2 (same sizes, same linear kernels).
 *   group_size 128 (64 returns AWQ_ERR_UNSUPPORTED: every kernel here works on
 *              128-k groups; the oracle defines g64 for a future layout).
 *   zero_point 1: asymmetric, S = fp16(max(hi - lo, 1e-5) / (2^bits - 1)),
 *              z = clamp(rint(-lo / S), 0, 2^bits - 1);
 *              0: symmetric, S = fp16(max(max|w'|, 1e-5) / (2^(bits-1) - 1)),
 *              z = 2^(bits-1) (stored in `zeros` like any zero point);
 *              q = clamp(rint(w' / S) + z, 0, 2^bits - 1) in both cases.
 * Other arguments, layout, errors and the no-early-start rule as for
 * awq_quantize_g128, which is awq_quantize(..., 4, 128, 1, ...). The linear
 * entry points dequantize every variant as (q - z) * S unchanged. */
AWQ_API awq_status_t awq_quantize(const uint16_t* W, const float* fold_scale, int N, int K, int bits,
                                  int group_size, int zero_point, uint32_t* qweight, uint16_t* scales,
                                  uint8_t* zeros, awq_stream_t stream);

/* a3. Decode W4A16 linear layer (context: "Installation" step 3 of the llm-awq
 * README, W4A16 decode kernels).
 *   x  fp16 [M, K] row-major (the scaled activations x'), 1 <= M <= 32.
 *   y  fp16 [M, N] row-major.
 * y = x . dequant^T with fp32 accumulation; dequant(q) = (q - z) * S.
 * Bitwise reproducible from call to call. Requires N >= 1, K >= 128,
 * K % 128 == 0.
 * Weight prefetch and overlap: the kernel starts reading qweight, scales and
 * zeros as soon as it is resident, and lets the next kernel of `stream` launch
 * at once (programmatic dependent launch); x and y are touched only after the
 * preceding kernel of `stream` has completed and its writes are visible. So a
 * run of consecutive decode calls on one stream overlaps: each may start
 * reading its weights while the earlier ones still run, back to the most
 * recent stream operation that is not a decode call. The packed weights must
 * be complete before that operation lets later work start: true for weights
 * written by any earlier kernel or copy (ordinary kernels and copies let later
 * work start only when they complete), and for awq_quantize_g128, which lets
 * no later kernel start before its writes are visible. A kernel that writes
 * packed weights must not trigger programmatic dependent launch before those
 * writes. */
AWQ_API awq_status_t awq_w4a16_gemv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                            const uint8_t* zeros, uint16_t* y, int M, int N, int K,
                            awq_stream_t stream);

/* a4. Prefill W4A16 linear layer (tcgen05 tensor cores, TMEM accumulators,
 * TMA-fed pipeline). Same arguments and result as awq_w4a16_gemv, any M >= 1
 * (M <= 2^31-1 / K). Weights are dequantized to fp16 ((q - z) * S rounded
 * once) before the fp16 x fp16 -> fp32 tensor-core products. */
AWQ_API awq_status_t awq_w4a16_gemm(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                            const uint8_t* zeros, uint16_t* y, int M, int N, int K,
                            awq_stream_t stream);

/* Convenience dispatch: the decode kernel of awq_w4a16_gemv for M <= 32 (same
 * weight-prefetch rule), awq_w4a16_gemm otherwise, and also for M <= 32 when
 * the decode kernel's full-size configuration does not fit in shared memory
 * (very wide layers at M > 8; on B200 the prefill kernel is the faster one
 * there). Measured on B200 at M = 2..32 over the Llama-2 7B and 70B layer
 * shapes, the decode kernel is 1.1x to 8x faster everywhere else. */
AWQ_API awq_status_t awq_w4a16_linear(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                              const uint8_t* zeros, uint16_t* y, int M, int N, int K,
                              awq_stream_t stream);

/* Fused-module epilogues ("transformers - AWQ" section 3: the attention
 * projections fused in the order query, key, value, with num_key_value_heads
 * below num_attention_heads giving narrower keys and values; the MLP layers
 * fused in the order gate, up, down). Same arguments, layout and weight
 * prefetch rule as awq_w4a16_linear (the decode kernel for M <= 32, the
 * prefill kernel above), with the output written differently:
 *
 * awq_w4a16_linear_qkv: the weight holds N = Nq + 2*Nkv rows (Nq query rows,
 *   then Nkv key rows, then Nkv value rows); the output goes to
 *   yq [M, Nq], yk [M, Nkv], yv [M, Nkv] (fp16, row-major, 16-byte aligned).
 *   Requires Nq >= 1, Nkv >= 1.
 *
 * awq_w4a16_linear_silu_mul: the weight holds N = 2*I rows (I gate rows,
 *   then I up rows), I a multiple of 16; the output is
 *   h [M, I] = SiLU(x . Wgate^T) * (x . Wup^T), SiLU(v) = v / (1 + e^-v),
 *   evaluated in fp32 on the fp32 sums (the pages name the fused MLP of Llama
 *   and Mistral, whose gate activation is SiLU), fp16 output. */
AWQ_API awq_status_t awq_w4a16_linear_qkv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                          const uint8_t* zeros, uint16_t* yq, uint16_t* yk, uint16_t* yv,
                                          int M, int Nq, int Nkv, int K, awq_stream_t stream);
AWQ_API awq_status_t awq_w4a16_linear_silu_mul(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                               const uint8_t* zeros, uint16_t* h, int M, int I, int K,
                                               awq_stream_t stream);

/* AWQ scale search (llm-awq README "Usage" step 1: the AWQ search picks the
 * scales on calibration data; CSDN VPTQ blog "02.02 AWQ": scales from offline
 * activation statistics, no backpropagation). For each candidate exponent
 * alpha_i the whole path runs on the calibration rows:
 *   s = max(mean_m |x_mk|, 1e-8)^alpha_i, x' = fp16(x / s), codes of fold(W, s),
 *   y_i = x' . dequant^T (fp16, the decode or prefill kernel by M),
 *   err[i] = sum_{m,n} (y_ref[m,n] - y_i[m,n])^2 in float64,
 * with y_ref = x . W^T (fp16 inputs, fp32 accumulation) computed once.
 *   x       fp16 [M, K] calibration rows (device);  W fp16 [N, K] (device)
 *   alphas  float [n_alpha] HOST array of candidates (finite), 1 <= n_alpha <= 4096
 *   err     double [n_alpha] (device, 8-byte aligned): the squared errors
 *   best    int [1] (device): index of the first smallest err
 *   workspace (device, 16-byte aligned) of at least
 *           awq_search_workspace_bytes(M, N, K) bytes; the library allocates nothing.
 * The workspace holds y_ref, y_i, s, x', the packed weights of the candidate
 * being scored and the error reduction's partial sums; its contents after the
 * call are those of the last candidate. Errors are reproducible from call to
 * call (fixed reduction order). Requires 1 <= M <= 1048560, K >= 128,
 * K % 128 == 0, M*N and M*K < 2^31. */
AWQ_API size_t awq_search_workspace_bytes(int M, int N, int K);
AWQ_API awq_status_t awq_search_alpha(const uint16_t* x, const uint16_t* W, int M, int N, int K,
                                      const float* alphas, int n_alpha, double* err, int* best,
                                      void* workspace, size_t workspace_bytes, awq_stream_t stream);

/* The scale search above for callers that cannot allocate device memory: code
 * that runs inside a host program which owns all of the GPU's memory (a serving
 * engine with a preallocated pool, a plugin that is handed no allocator), and
 * code that must not call cudaMalloc/cudaFree because they synchronize the
 * device and stall the other streams' work. The paper has no counterpart; this
 * is a library convenience. Arguments, results and status codes are those of
 * awq_search_alpha, and so are the errors, bit for bit; the workspace is
 * instead a fixed array of AWQ_SEARCH_NOALLOC_SCRATCH_BYTES (64 MiB) in the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits. Nothing here calls cudaMalloc, cudaFree or any
 * allocating library routine.
 *   Limit: awq_search_workspace_bytes(M, N, K) <= AWQ_SEARCH_NOALLOC_SCRATCH_BYTES
 *   (e.g. a 4096 x 4096 layer with up to 1781 calibration rows, 8192 x 8192 with
 *   up to 491); larger shapes return AWQ_ERR_INVALID_ARG and launch nothing.
 *   Set-up: the first call on a device, with that device current, looks up the
 *   array's device address; make that first call before any stream capture.
 *   Sharing: all calls on a device use the same array, which keeps the last
 *   call's contents (no byte of it needs to start at zero: each call writes
 *   everything it reads). Calls whose work can overlap on the GPU (streams not
 *   ordered with each other) race on the array and give undefined errors:
 *   order them on one stream or with events. */
#define AWQ_SEARCH_NOALLOC_SCRATCH_BYTES (64u << 20)
AWQ_API awq_status_t awq_search_alpha_noalloc(const uint16_t* x, const uint16_t* W, int M, int N, int K,
                                              const float* alphas, int n_alpha, double* err, int* best,
                                              awq_stream_t stream);

/* Synchronizes `stream`, then reads and clears the device status word of the
 * current device. Returns AWQ_ERR_TIMEOUT if a kernel since the last poll gave
 * up a bounded wait (its outputs are then undefined), AWQ_ERR_CUDA if the
 * stream reports an error, AWQ_ERR_BOUNDS (debug builds only) if a kernel's
 * index check failed, AWQ_OK otherwise.
 * The status word is one per device, shared by every stream and launch of this
 * library on it: a timeout raised by a kernel of another stream since the last
 * poll is reported (and cleared) here too. With several streams, synchronize
 * all of them before polling to attribute a timeout to the work just done. */
AWQ_API awq_status_t awq_poll_device_status(awq_stream_t stream);

/* Test hook: sets the time (ns) after which a bounded wait inside a kernel
 * gives up on the current device (0 restores the default of 2 s). Synchronous.
 * A kernel that gives up sets the status read by awq_poll_device_status,
 * drains its own copies and tensor-core work in flight, frees its tensor
 * memory and returns. */
AWQ_API awq_status_t awq_debug_set_wait_budget_ns(unsigned long long ns);

/* Test hook: nonzero makes the producer of the quantizer and of the decode
 * kernel skip the copies of its first pipeline stage, so the consumers' wait
 * on that stage can only end by running out its budget (shorten it with
 * awq_debug_set_wait_budget_ns). The kernel then behaves as described there.
 * 0 restores normal operation. Synchronous; current device. */
AWQ_API awq_status_t awq_debug_drop_first_copy(int enable);

/* The launch plan awq_w4a16_gemm (and the fused prefill entry points)
 * would take for an M x K by K x N layer on a GPU with num_sms SMs: the
 * token tile (*token_tile: 32, 64, 128 or 256 tokens per tile), the K
 * split (*k_split: 1, or 2 when the two CTAs of a thread-block cluster
 * share tiles, each over half of K) and *split_tiles, how many of the
 * layer's tiles are shared that way (all of them, or only those left
 * for the last round after whole rounds of one tile per SM). epilogue:
 * 0 plain, 1 q/k/v split, 2 gate/up SiLU·up (N = 2 I, I a multiple of
 * 16). Host-only; honours awq_debug_set_gemm_split. AWQ_ERR_INVALID_ARG
 * for null outputs or the shapes the linear entry points reject. */
AWQ_API awq_status_t awq_gemm_plan(int M, int N, int K, int epilogue, int num_sms, int* token_tile, int* k_split,
                                   long long* split_tiles);

/* Test hook: the prefill kernel's K split. 0 (the default) lets the
 * library's round model choose, per launch, whether the two CTAs of a
 * thread-block cluster share output tiles (each over half of K, their
 * fp32 partial sums added in a fixed order); 1 never splits, 2 splits
 * every tile, 3 takes the mixed form (whole rounds of one tile per CTA,
 * then the remaining tiles split) on a grid of 3 CTA pairs, so that small
 * layers run both kinds of work item. Results agree within fp32 rounding
 * of the split sum. Host-side setting for all devices, read at each
 * launch; AWQ_ERR_INVALID_ARG for other values. */
AWQ_API awq_status_t awq_debug_set_gemm_split(int ks);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* AWQ_W4A16_H_ */
