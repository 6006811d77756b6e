/*
 * zq.h -- C ABI of libzq, the B200 (sm_100a) fused quantized linear layer of
 * ZeroQuant ("ZeroQuant: Efficient and Affordable Post-Training Quantization
 * for Large-Scale Transformers", arXiv 2206.01861).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - All tensor pointers are DEVICE pointers into memory the caller owns and
 *    keeps alive until the work queued on `stream` has finished.  fp16 tensors
 *    are passed as `void*` holding IEEE binary16 values.
 *  - Matrices are row-major and dense: X[T][K] (tokens x hidden),
 *    W[N][K] (output features x hidden; the paper's W in R^{n x m} with one
 *    row per output), Y[T][N].
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and on the device that is current for the calling thread.
 *  - Argument errors are reported synchronously (ZQ_ERR_NULL / _SHAPE /
 *    _ALIGN / _UNSUPPORTED) and nothing is launched.  Launch failures return
 *    ZQ_ERR_CUDA.  A kernel that gives up a bounded device-side wait records
 *    the fact in a per-device status word that zq_device_status() reports.
 *  - Group of output row o when N rows are split into g contiguous groups:
 *    group(o) = floor(o*g/N).
 *  - Rounding: round half to even everywhere.  Every floating-point step is
 *    one IEEE round-to-nearest operation in a stated order: a single add,
 *    multiply, divide or square root, except in the LayerNorm variance, whose
 *    squared deviations are accumulated with fused multiply-adds (one
 *    rounding each).  Results are therefore bit-for-bit reproducible and do
 *    not depend on the launch configuration.
 */
#ifndef ZQ_H_
#define ZQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t */
typedef struct CUstream_st* zq_stream_t;

typedef enum {
  ZQ_OK = 0,
  ZQ_ERR_NULL = 1,        /* a required pointer is NULL */
  ZQ_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  ZQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  ZQ_ERR_UNSUPPORTED = 4, /* valid request this build does not handle (e.g. bits) */
  ZQ_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed */
  ZQ_ERR_TIMEOUT = 6      /* a kernel gave up a bounded wait (zq_device_status) */
} zq_status;

/* Human-readable name of a status code (static storage). */
const char* zq_status_str(int status);

/* ABI version of this header (major*100 + minor). */
int zq_abi_version(void);

/*
 * zq_quantize_weights_groupwise -- offline group-wise symmetric weight
 * quantization (Sec. 3.4 "Group-wise Weight Quantization", Eq. 2).
 *   W      fp16 [N][K]; N rows split into g contiguous groups.
 *   bits   8: Wq is int8 [N][K].  4: Wq is uint8 [N][K/2], two signed
 *          two's-complement nibbles per byte: of each eight consecutive k
 *          (k = 8m..8m+7), byte 4m+i of the row holds k = 8m+i in its low
 *          nibble and k = 8m+4+i in its high nibble.
 *   s_grp  fp32 [g]: S_i = amax_i / qmax with amax_i = max |W| over group i,
 *          qmax = 127 (bits 8) or 7 (bits 4).  q = clamp(rne(w * (qmax/amax_i)),
 *          -qmax, qmax); a group that is all zero gets S_i = 0 and q = 0.
 * Requirements: 1 <= g <= N, K >= 1, K % 16 == 0 (K % 32 == 0 for bits 4),
 * pointers 16-byte aligned.
 */
zq_status zq_quantize_weights_groupwise(const void* W, int N, int K, int g, int bits, void* Wq,
                                        float* s_grp, zq_stream_t stream);

/*
 * zq_ln_quant -- fused LayerNorm + token-wise dynamic INT8 quantization
 * (Sec. 3.4 "Token-wise Activation Quantization" and "Kernel fusion for
 * token-wise activation quantization"; Fig. 2 right, first box).
 *   X      fp16 [T][K] input rows (tokens).
 *   gamma  fp16 [K] or NULL.  NULL selects quant-only mode: y = x.
 *   beta   fp16 [K] or NULL (= 0).  Ignored when gamma is NULL.
 *   eps    LayerNorm epsilon (added to the biased variance).
 *   Xq     int8 [T][K] output, s_tok fp32 [T] output:
 *          y = fp16(((x - mean) * rstd) * gamma + beta) in fp32, with
 *          mean = S/K and biased var = Q/K, where S sums x and Q sums
 *          (x - mean)^2 in a fixed order: chunks of 8 consecutive values in
 *          index order, chunk sums combined by a zero-padded pairwise tree;
 *          rstd = 1/sqrt(var + eps);
 *          s_tok[t] = amax_t/127 with amax_t = max_k |y|,
 *          Xq = clamp(rne(y * (127/amax_t)), -127, 127); zero rows give 0.
 *   Y_ln   fp16 [T][K] or NULL: also store y (unfused form, for checking).
 * Requirements: T >= 0 (T == 0 is a no-op), 16 <= K <= 32768, K % 16 == 0,
 * pointers 16-byte aligned.
 */
zq_status zq_ln_quant(const void* X, const void* gamma, const void* beta, int T, int K, float eps,
                      int8_t* Xq, float* s_tok, void* Y_ln, zq_stream_t stream);

/*
 * zq_bias_act_quant -- token-wise dynamic INT8 quantization fused into a
 * bias-add or a GeLU (Sec. 3.4 "Kernel fusion for token-wise activation
 * quantization": the quantization is fused with the preceding LayerNorm,
 * GeLU or bias-add, so the fp16 activation never makes a DRAM round trip).
 *   X      fp16 [T][K] input rows (tokens), e.g. a GEMM's fp16 output.
 *   bias   fp16 [K] or NULL (no add).
 *   act    ZQ_ACT_NONE: v = f32(x) + f32(bias) (one fp32 add), y = fp16(v);
 *          ZQ_ACT_GELU: y = fp16(gelu(v)), GeLU in its exact form
 *          gelu(v) = 0.5 v (1 + erf(v / sqrt 2)) = v * 0.5 erfc(-v / sqrt 2),
 *          evaluated in fp32 with a Chebyshev approximation of erfc
 *          (fractional error below 1.2e-7; y may differ from a correctly
 *          rounded GeLU by one fp16 ulp).
 *   Xq, s_tok  the token quantization of y, as in zq_ln_quant:
 *          s_tok[t] = amax_t/127 with amax_t = max_k |y|,
 *          Xq = clamp(rne(y * (127/amax_t)), -127, 127); zero rows give 0.
 *   Y_act  fp16 [T][K] or NULL: also store y.
 * Requirements: as zq_ln_quant; act is ZQ_ACT_NONE or ZQ_ACT_GELU
 * (else ZQ_ERR_UNSUPPORTED).
 */
typedef enum { ZQ_ACT_NONE = 0, ZQ_ACT_GELU = 1 } zq_act;
zq_status zq_bias_act_quant(const void* X, const void* bias, int T, int K, int act, int8_t* Xq,
                            float* s_tok, void* Y_act, zq_stream_t stream);

/*
 * zq_static_quant -- static (per-tensor) INT8 activation quantization, the
 * prior post-training scheme the pages contrast with token-wise quantization
 * (Sec. 3.4 "Token-wise Activation Quantization": a scale calibrated offline
 * and frozen).  For comparison with zq_ln_quant's quant-only mode.
 *   X      fp16 [T][K].
 *   amax   the calibrated range A (0 <= A <= 65504), e.g. moving averages of
 *          calibration batches' max and min, A = max(|x_max|, |x_min|).
 *   Xq     int8 [T][K]: clamp(rne(x * (127/A)), -127, 127) (0 when A = 0).
 *   s_tok  fp32 [T]: A/127 for every token, so the GEMMs consume it unchanged.
 * Requirements: as zq_ln_quant (pointers X and Xq 16-byte aligned).
 */
zq_status zq_static_quant(const void* X, int T, int K, float amax, int8_t* Xq, float* s_tok,
                          zq_stream_t stream);

/*
 * zq_gemm_w8a8 -- INT8 x INT8 GEMM with the dequantization fused into the
 * epilogue (Sec. 3.4 "CUTLASS INT8 GEMM" and "Dequantization fused into the
 * GEMM epilogue"; Fig. 2 right, second box).
 *   Xq, s_tok   int8 [T][K] and fp32 [T] from zq_ln_quant.
 *   Wq, s_grp   int8 [N][K] and fp32 [g] from zq_quantize_weights_groupwise.
 *   bias        fp16 [N] or NULL (= 0).
 *   Y           fp16 [T][N]:
 *               acc[t][o] = sum_k Xq[t][k]*Wq[o][k]   (exact, int32)
 *               Y[t][o] = fp16(((f32(acc)*s_tok[t]) * s_grp[group(o)]) + f32(bias[o]))
 *   acc_dbg     int32 [T][N] or NULL: also store acc (for checking).
 * Runs on tcgen05 tensor cores, except for T <= 2 (INT8) or T <= 4 (INT4
 * weights), a memory-bound matrix-vector product that runs on CUDA cores
 * (dp4a, exact int32).  Small T (weight-streaming) tensor-core shapes split
 * K across SMs: the exact int32 partial sums go to the library workspace
 * and a second kernel on the same stream adds them and dequantizes.
 * The library workspace is one device buffer per device, grown with
 * cudaMalloc the first time a call needs more than it holds (see
 * zq_workspace_reserve to size it up front); calls that use it on
 * different streams must not overlap.  Growing it never frees the old
 * buffer (it stays allocated until the process exits), so a CUDA graph
 * captured before a growth stays valid.  A call that would grow it while
 * `stream` is being captured returns ZQ_ERR_UNSUPPORTED and launches
 * nothing: size the workspace before the capture (an eager call of the
 * same shape, or zq_workspace_reserve).
 * Requirements: T >= 0 (T == 0 is a no-op), N >= 8, N % 8 == 0,
 * 16 <= K <= 133136, K % 16 == 0 (so that 127*127*K < 2^31), 1 <= g <= N,
 * pointers 16-byte aligned.
 */
zq_status zq_gemm_w8a8(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                       const float* s_grp, int g, const void* bias, int T, int N, int K, void* Y,
                       int32_t* acc_dbg, zq_stream_t stream);

/*
 * zq_gemm_w4a8 -- as zq_gemm_w8a8 with INT4 weights (Sec. 3.4 "Which weights
 * get INT4": FFN weights in INT4).  Wq4 is uint8 [N][K/2] in the layout of
 * zq_quantize_weights_groupwise(bits=4).  The nibbles are widened to int8
 * codes before the tensor-core MMAs read them:
 *   - T >= 512 (prefill): once per call, by an HBM-bound pass into the
 *     library workspace (N*K bytes), which the INT8 GEMM then reads;
 *   - 128 < T < 512: in shared memory, inside each token-row tile;
 *   - 4 < T <= 128: in tensor memory (the MMA's A operand), inside each
 *     weight-row tile;
 *   - T <= 4: in registers, on the CUDA-core matrix-vector path.
 * Requirements as zq_gemm_w8a8, plus K % 32 == 0 and K <= 132096.
 */
zq_status zq_gemm_w4a8(const int8_t* Xq, const float* s_tok, const uint8_t* Wq4,
                       const float* s_grp, int g, const void* bias, int T, int N, int K, void* Y,
                       int32_t* acc_dbg, zq_stream_t stream);

/*
 * zq_widen_int4_weights -- the INT4 unpack step on its own (Sec. 3.4 "Which
 * weights get INT4": INT4 weights are converted to INT8 before the INT8
 * GEMM): packed codes to int8 codes, an HBM-bound pass.  zq_gemm_w4a8 runs
 * it itself at prefill token counts; calling it separately lets a caller
 * widen a layer's INT4 weights ahead of time, for example on a second
 * stream while other GEMMs run, and then call zq_gemm_w8a8 on the result
 * (which gives the same outputs as zq_gemm_w4a8).
 *   Wq4    uint8 [N][K/2] in the layout of zq_quantize_weights_groupwise(bits=4).
 *   Wq8    int8 [N][K] output, caller-owned: Wq8[o][k] = the signed code of
 *          weight (o, k), in -8..7 (-8 never occurs in quantized weights).
 * Requirements: N >= 1, K >= 32, K % 32 == 0, pointers 16-byte aligned.
 * Asynchronous on `stream`; argument errors return before any launch.
 */
zq_status zq_widen_int4_weights(const uint8_t* Wq4, int N, int K, int8_t* Wq8, zq_stream_t stream);

/*
 * zq_gemm_w8a16 -- the quantized linear layer with FP16 activations and
 * group-wise INT8 weights (W8A16: the summary page's "Main Quantitative
 * Results", Table 4; also the GPT-NeoX self-attention input that stays in
 * FP16 while its weights are INT8, "INT4/INT8 Mixed-Precision Quantization").
 *   X           fp16 [T][K], row-major (no activation quantization).
 *   Wq, s_grp   int8 [N][K] and fp32 [g] from zq_quantize_weights_groupwise.
 *   bias        fp16 [N] or NULL (= 0).
 *   Y           fp16 [T][N]:
 *               acc[t][o] = sum_k x[t][k] * Wq[o][k]   (fp32 accumulation on
 *                           tcgen05 tensor cores, codes exact in fp16; the
 *                           summation order is the hardware's)
 *               Y[t][o] = fp16(f32(acc * s_grp[group(o)]) + f32(bias[o]))
 *               i.e. X * (Wq * S)^T + bias with each row's group scale
 *               applied after the K sum, where it factors out exactly.
 *   acc_dbg     fp32 [T][N] or NULL: also store acc (for checking).
 * Runs on tcgen05 tensor cores (kind::f16), except for T <= 4: a
 * memory-bound matrix-vector product on CUDA cores (exact products, fp32
 * fma sums).  From T = 1024 the codes are first widened to fp16 integers in
 * the library workspace (2*N*K bytes, an HBM-bound pass) and the GEMM reads
 * them by TMA, on single CTAs or CTA pairs; below that each tile widens its
 * codes in shared memory.  ZQ_OPT_GEMM_PATH = 3 forces the matrix-vector
 * path (T <= 4), 4 the widening pass, 1 or 2 the in-tile widening;
 * ZQ_OPT_CTA_PAIR = 2 forces 256-row units shared by a CTA pair (with the
 * in-tile widening they measured slower and are never chosen automatically).
 * Requirements: T >= 0 (T == 0 is a no-op), N >= 8, N % 8 == 0,
 * 16 <= K <= 2^20, K % 16 == 0, 1 <= g <= N, pointers 16-byte aligned.
 * Errors: as zq_gemm_w8a8 (argument errors before any launch).
 */
zq_status zq_gemm_w8a16(const void* X, const int8_t* Wq, const float* s_grp, int g,
                        const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                        zq_stream_t stream);

/*
 * zq_gemm_w4a16 -- as zq_gemm_w8a16 with INT4 weights (the W4/8A16
 * configurations of "INT4/INT8 Mixed-Precision Quantization": INT4 FFN
 * weights with FP16 activations).  Wq4 is uint8 [N][K/2] in the layout of
 * zq_quantize_weights_groupwise(bits=4); the kernel widens the nibbles to
 * fp16 in shared memory.  Requirements as zq_gemm_w8a16, plus K % 32 == 0.
 */
zq_status zq_gemm_w4a16(const void* X, const uint8_t* Wq4, const float* s_grp, int g,
                        const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                        zq_stream_t stream);

/*
 * zq_gemm_w8a8_noalloc -- zq_gemm_w8a8 for callers that must not let a
 * library allocate device memory: a serving runtime that owns the whole
 * device memory pool, a process whose memory budget is fixed up front, or
 * code that cannot afford the device-wide synchronisation that cudaMalloc /
 * cudaFree may cause.  It has no counterpart in the paper; it exists only
 * for such callers.
 *   Same arguments, results and requirements as zq_gemm_w8a8.  The caller
 *   still owns and passes every input and output.  The scratch memory of the
 *   split-K reduction (small token counts) comes from a fixed array of
 *   8 MiB in device memory that the library declares statically; every GPU
 *   that loads the library holds it until the process exits, and no call of
 *   this function allocates or frees anything.
 *   It chooses the same kernel and tiling as zq_gemm_w8a8.
 *   Limit: when that plan's split-K reduction would need more than the
 *   array holds (splits * T * N int32 partial sums above 8 MiB), the call
 *   plans again with as many K splits as fit (one split needs no scratch).
 *   Only a split count forced through ZQ_OPT_SPLIT_K that does not fit is
 *   refused: ZQ_ERR_SHAPE, without launching.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   All calls on a device share the one array: calls whose work may overlap
 *   on the GPU (for example on different streams) race on it and give wrong
 *   results.
 */
zq_status zq_gemm_w8a8_noalloc(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                               const float* s_grp, int g, const void* bias, int T, int N, int K,
                               void* Y, int32_t* acc_dbg, zq_stream_t stream);

/*
 * zq_device_status -- synchronize `stream`, then read and clear the status
 * word of the current device.  Returns ZQ_OK, ZQ_ERR_TIMEOUT when a kernel
 * gave up a bounded wait since the last call (*detail receives the kernel's
 * wait-site code, may be NULL), or ZQ_ERR_CUDA when synchronization failed.
 */
zq_status zq_device_status(zq_stream_t stream, int* detail);

/*
 * zq_set_option / zq_get_option -- process-wide tuning switches used by
 * tests and benchmarks to force one kernel variant.  0 always means
 * "automatic".  Unknown keys return ZQ_ERR_UNSUPPORTED.
 *   ZQ_OPT_GEMM_PATH   1 = token rows on the MMA M side (prefill tiling),
 *                      2 = weight rows on the MMA M side (weight streaming),
 *                      3 = CUDA-core matrix-vector product (T <= 4, else
 *                          ZQ_ERR_UNSUPPORTED); automatic at T <= 4 with
 *                          INT4 weights and at T <= 2 with INT8 ones;
 *                      4 = the codes widened into the workspace first:
 *                          zq_gemm_w4a8 then runs the INT8 GEMM (automatic
 *                          at T >= 512), the FP16-activation GEMMs the fp16
 *                          GEMM (automatic at T >= 1024); zq_gemm_w8a8
 *                          returns ZQ_ERR_UNSUPPORTED.
 *   ZQ_OPT_GEMM_BN     MMA N tile width for path 1 (a multiple of 16, 16..256);
 *                      the FP16-activation GEMMs accept 128 or 256 (other
 *                      values: ZQ_ERR_UNSUPPORTED) and ignore the path.
 *   ZQ_OPT_SPLIT_K     number of K splits for path 2 (1 = none); for path 1,
 *                      the number of K parts of each tile of a partial last
 *                      wave (automatic: for rows of K >= 12288 when that
 *                      wave is less than half full).
 *   ZQ_OPT_MAX_CTAS    cap on the number of CTAs of the GEMM (persistent grid).
 *   ZQ_OPT_CTA_PAIR    path 1: 1 = one CTA per 128 x BN
 *                      tile, 2 = CTA pairs sharing 256 x BN tiles (tcgen05
 *                      cta_group::2); automatic picks pairs for large K.
 */
typedef enum {
  ZQ_OPT_GEMM_PATH = 1,
  ZQ_OPT_GEMM_BN = 2,
  ZQ_OPT_SPLIT_K = 3,
  ZQ_OPT_MAX_CTAS = 4,
  ZQ_OPT_CTA_PAIR = 5
} zq_option;
zq_status zq_set_option(int key, int value);
int zq_get_option(int key);

/*
 * zq_workspace_reserve -- grow the library workspace of the current device
 * to at least `bytes` now (cudaMalloc; nothing happens if it is that large
 * already), so that later GEMM calls of up to that need allocate nothing.
 * The need of a call: 4 * splits * T * N bytes for a split-K weight-streaming
 * plan, plus N * K bytes (rounded up to 256) when zq_gemm_w4a8 widens its
 * codes (T >= 512, or ZQ_OPT_GEMM_PATH = 4); 2 * N * K bytes when an
 * FP16-activation GEMM widens its codes (T >= 1024, or path 4).  Synchronous; call it
 * outside stream capture.  A growth keeps the previous buffer allocated (for
 * graphs captured with it) and takes at least a quarter more than the
 * previous size, rounded up to 2 MiB.  Returns ZQ_ERR_CUDA if the
 * allocation fails.
 */
zq_status zq_workspace_reserve(unsigned long long bytes);

/*
 * zq_launch_count -- number of kernel launches this library has issued in
 * this process, on every device and stream (a launch recorded into a CUDA
 * graph counts once, when it is recorded; its replays do not go through the
 * library).  Benchmarks use the difference over one recorded step.
 */
unsigned long long zq_launch_count(void);

/*
 * zq_debug_wait_timeout -- launches one CTA that waits on a shared-memory
 * barrier nothing ever arrives at.  The wait is bounded: after about a
 * second it records ZQ_ERR_TIMEOUT in the status word and the kernel
 * returns.  Exists to test the bounded-wait path without a real fault.
 */
zq_status zq_debug_wait_timeout(zq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ZQ_H_ */
