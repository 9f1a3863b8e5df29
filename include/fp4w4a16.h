/*
 * fp4w4a16.h -- C interface of the B200 (sm_100a) FP4 weight-quantization
 * and W4A16 GEMM library (libfp4w4a16.so).
 *
 * Method: 4-bit floating-point (ExMy) post-training quantization of linear
 * layer weights and the matrix multiply that consumes them, as described on
 * the LLM-FP4 summary page "首个支持4-bit浮点量化的LLM来了" (sections on the
 * floating-point number formula, scale-and-clip, compare-and-quantize, the
 * efficient matrix multiplication, the format/range search, and the
 * pre-shifted exponent bias) with two codes packed per byte as in the
 * "为什么我们需要4-bit浮点量化" tutorial, section 2.2.
 *
 * Conventions for every entry point:
 *  - Tensor arguments are DEVICE pointers allocated and owned by the caller.
 *    The library never allocates or frees device memory; scratch space is
 *    passed in as `workspace`.
 *  - Layouts are row-major and contiguous.  bf16 and fp16 tensors are passed
 *    as uint16_t bit patterns.  Tensor base pointers must be 16-byte
 *    aligned (FP4_ERR_MISALIGNED otherwise); scale arrays 4-byte aligned.
 *  - Argument errors are detected on the host before anything is launched
 *    and returned synchronously; nothing is written in that case.
 *  - Work is enqueued on `stream` and is asynchronous; a launch failure
 *    returns FP4_ERR_CUDA.  Problems only the GPU can see (a non-finite
 *    input, an fp16 scale overflow, a pipeline wait that timed out) set bits
 *    of a per-device status word read by fp4_get_device_status().
 *  - Empty problems (a zero dimension) succeed without launching, except
 *    that fp4_gemm with K == 0 writes zeros to Y.
 *  - The library keeps per-device state that it sets up on first use (the
 *    status word's address, kernel attributes, the address of the built-in
 *    calibration buffer).  It belongs to the context that was current then:
 *    after cudaDeviceReset the library must not be called on that device
 *    again in the same process.
 *  - Weight layouts produced by fp4_quantize and read by fp4_gemm:
 *      packed [N][K/2] uint8: element k of row n is nibble (k & 1) of byte
 *                             k/2, low nibble first (even k in bits 0..3);
 *      scales [N][K/group]    fp32 or fp16, one per (row, group of `group`
 *                             consecutive k).
 *    Code = sign<<3 | exponent<<m | mantissa; magnitude index = code & 7.
 */
#ifndef FP4W4A16_H
#define FP4W4A16_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FP4_API __attribute__((visibility("default")))
#else
#define FP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp4_status {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum  */
    FP4_ERR_UNSUPPORTED_SHAPE = 2, /* K % group, K % 32, group not 32/64/128 */
    FP4_ERR_MISALIGNED = 3,        /* a tensor pointer is not 16-byte aligned */
    FP4_ERR_WORKSPACE = 4,         /* workspace missing or too small          */
    FP4_ERR_CUDA = 5,              /* a CUDA call or launch failed            */
    FP4_ERR_DEVICE_STATUS = 6      /* fp4_get_device_status found a flag set  */
} fp4_status;

/* 4-bit formats (exponent bits / mantissa bits, bias 2^(e-1)-1):
 *   E1M2 {0,.5,1,1.5,2,2.5,3,3.5}   E2M1 {0,.5,1,1.5,2,3,4,6}
 *   E3M0 {0,.25,.5,1,2,4,8,16}  (magnitudes of codes 0..7; codes 8..15 are
 *   the negatives).  FP4_FMT_AUTO asks fp4_quantize to search the format. */
typedef enum fp4_format { FP4_E1M2 = 0, FP4_E2M1 = 1, FP4_E3M0 = 2, FP4_FMT_AUTO = -1 } fp4_format;

typedef enum fp4_scale_dtype { FP4_SCALE_F32 = 0, FP4_SCALE_F16 = 1 } fp4_scale_dtype;

/* GEMM engine selection for fp4_gemm_ex (fp4_gemm always uses AUTO). */
typedef enum fp4_engine { FP4_ENGINE_AUTO = 0, FP4_ENGINE_DECODE = 1, FP4_ENGINE_TENSOR = 2 } fp4_engine;
/* Extent of the absmax behind one weight scale (fp4_quantize_blocks). */
typedef enum fp4_granularity { FP4_GRAN_GROUP = 0, FP4_GRAN_CHANNEL = 1, FP4_GRAN_HEAD = 2 } fp4_granularity;
/* Output activation fused into the GEMM epilogue (fp4_gemm_act). */
typedef enum fp4_act { FP4_ACT_NONE = 0, FP4_ACT_SILU = 1, FP4_ACT_GELU = 2, FP4_ACT_SILU_GATE = 3 } fp4_act;

/* Bits of the device status word. */
#define FP4_DEV_NONFINITE_INPUT 0x1 /* NaN/Inf met in W or X                   */
#define FP4_DEV_SCALE_OVERFLOW 0x2  /* a group scale does not fit in fp16       */
#define FP4_DEV_WAIT_TIMEOUT 0x4    /* a pipeline wait gave up; output invalid  */
#define FP4_DEV_LAYOUT 0x8          /* a kernel's shared-memory base lacked the alignment its layout needs; nothing written */

/* Version of this interface (major * 100 + minor). */
FP4_API int fp4_abi_version(void);

/* Human-readable name of a status code (static string). */
FP4_API const char *fp4_status_string(fp4_status s);

/* ------------------------------------------------------------------------
 * fp4_quantize -- scale-and-clip, optional format / range search,
 * compare-and-quantize, pack.  (LLM-FP4 summary page: scale-and-clip,
 * eq. (2)-(4); compare-and-quantize, eq. (5); format and range search;
 * pre-shifted exponent bias folded into the weights.)
 *
 * For every row n and group gi of `group` consecutive k:
 *   W'[n,k] = W[n,k] * 2^chan_shift[k]            (chan_shift NULL: W' = W)
 *   A       = max |W'| over the group              (fp32)
 *   s       = R(fl32(fl32(A * c_j) / Qmax_f))      R = identity (fp32 scales)
 *                                                  or fp16 round-to-nearest-even
 *   c_j     = fl32(2^(-j/8)), j = 0..7: a real-valued exponent bias acting as
 *             a scale (j = 0 is plain absmax scaling)
 *   code    = signbit(W') << 3 | nearest magnitude index of fl32(|W'| / s),
 *             ties to the even index, saturating at index 7; s == 0 gives
 *             index 0.
 * Search: the candidates are formats {fmt} (or all three if fmt ==
 * FP4_FMT_AUTO) times j in {0} (or 0..7 if bias_search != 0).  The chosen
 * candidate minimises SSE = sum (W' - v*s)^2 over the whole tensor (fp64);
 * the first strict minimum in (format, j) order wins.
 *
 *   W          [N][K] fp32, device.
 *   group      32, 64 or 128; K % group == 0 and K % 32 == 0.
 *   chan_shift [K] int8 device (values in [-126, 0]) or NULL.
 *   sdt        scale storage type.
 *   packed     [N][K/2] uint8 out.   scales [N][K/group] fp32/fp16 out.
 *   choice     device int32[2] out: {format, j}.  Required.
 *   sse        device double[24] out or NULL: SSE of candidate f*8+j for the
 *              candidates evaluated; NaN for the others.
 *   workspace  device scratch of fp4_quantize_workspace_size(...) bytes
 *              (may be NULL when that size is 0).  Its contents need no
 *              initialisation and are undefined afterwards.
 * Device status: FP4_DEV_NONFINITE_INPUT, FP4_DEV_SCALE_OVERFLOW.
 * ---------------------------------------------------------------------- */
FP4_API size_t fp4_quantize_workspace_size(int N, int K, int group, fp4_format fmt, int bias_search);
FP4_API fp4_status fp4_quantize(const float *W, int N, int K, int group, fp4_format fmt, int bias_search,
                        const int8_t *chan_shift, fp4_scale_dtype sdt, uint8_t *packed, void *scales,
                        int32_t *choice, double *sse, void *workspace, size_t ws_bytes,
                        cudaStream_t stream);

/* ------------------------------------------------------------------------
 * fp4_quantize_blocks -- fp4_quantize with the scale's absmax taken over a
 * coarser block, and the bias index chosen per block.  (Granularities of
 * the HiFloat4 page, section 3.1 "权重量化策略": scales grouped per
 * attention head; of the "量化技术详解" page, section "量化分类" by
 * granularity, and the per_channel option of the 4-bit float tutorial,
 * section 4.2: one scale per output channel; the search of the LLM-FP4
 * summary page applied to each block instead of the whole tensor.)
 *
 *   gran FP4_GRAN_GROUP    block = `group` consecutive k of a row (as
 *                          fp4_quantize);
 *        FP4_GRAN_CHANNEL  block = a whole row (one output channel);
 *        FP4_GRAN_HEAD     block = N/heads consecutive rows (an attention
 *                          head of a q/k/v projection); N % heads == 0.
 *   Channel and head blocks need K % 128 == 0.
 *   A    = max |W'| over the block; s = R(fl32(fl32(A * c_j) / Qmax_f)) as
 *          in fp4_quantize, written to every [n][k/group] slot the block
 *          covers, so fp4_gemm reads the result with the same `group`.
 *   bias_index 0..7: that c_j for every block; -1: each block takes the j
 *          with the smallest SSE over its own elements (fp64; first strict
 *          minimum in j order; the SSE is summed in a fixed order, so the
 *          choice does not depend on timing).  fmt is fixed (not AUTO): the
 *          GEMM decodes one format per tensor.
 *   jmap       device int8 [blocks] out or NULL: the bias index of each
 *              block (blocks: N*K/group, N or heads, in row order).
 *   workspace  fp4_quantize_blocks_workspace_size(...) bytes (NULL when
 *              0), no initialisation; channel/head searches keep 64 bytes
 *              per 128 weights there.
 * Device status: FP4_DEV_NONFINITE_INPUT, FP4_DEV_SCALE_OVERFLOW.
 * ---------------------------------------------------------------------- */
FP4_API size_t fp4_quantize_blocks_workspace_size(int N, int K, int group, fp4_granularity gran, int heads,
                                                  int bias_index);
FP4_API fp4_status fp4_quantize_blocks(const float *W, int N, int K, int group, fp4_granularity gran, int heads,
                                       fp4_format fmt, int bias_index, const int8_t *chan_shift,
                                       fp4_scale_dtype sdt, uint8_t *packed, void *scales, int8_t *jmap,
                                       void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * fp4_dequantize -- W_hat[n,k] = fl32(v(code[n,k]) * s[n, k/group]), the
 * weights the GEMM multiplies by (test aid).  W_hat [N][K] fp32 out.
 * ---------------------------------------------------------------------- */
FP4_API fp4_status fp4_dequantize(const uint8_t *packed, const void *scales, fp4_scale_dtype sdt,
                          fp4_format fmt, int N, int K, int group, float *W_hat, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Pre-shifted exponent bias (LLM-FP4 summary page, section on the
 * pre-shifted exponent bias): a per-channel activation maximum from
 * calibration data is split into one per-tensor real factor rho times a
 * per-channel power of two 2^e_k; 2^e_k is folded into the weights
 * (pass it as chan_shift to fp4_quantize), rho stays with the activations.
 *
 * fp4_preshift_calibrate:
 *   c_k = max_m |X[m,k]|, rho = max_k c_k (1 if X is all zero),
 *   e_k = ceil(log2(c_k / rho)) clamped to [-126, 0], 0 when c_k == 0.
 *   X [M][K] bf16; shift [K] int8 out; rho device float out.
 *   workspace: fp4_preshift_workspace_size(M, K) bytes, no initialisation.
 *   Device status: FP4_DEV_NONFINITE_INPUT.
 * fp4_preshift_apply:
 *   Xt[m,k] = bf16_rne(fl32(fl32(X[m,k] * 2^-e_k) / rho)), |Xt| <= 1.
 *   Xt may not alias X.  The GEMM then takes x_scale = rho.
 * ---------------------------------------------------------------------- */
FP4_API size_t fp4_preshift_workspace_size(int M, int K);
FP4_API fp4_status fp4_preshift_calibrate(const uint16_t *X, int M, int K, int8_t *shift, float *rho,
                                  void *workspace, size_t ws_bytes, cudaStream_t stream);
FP4_API fp4_status fp4_preshift_apply(const uint16_t *X, int M, int K, const int8_t *shift, const float *rho,
                              uint16_t *Xt, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * fp4_preshift_calibrate_noalloc -- the method has no counterpart for this
 * call: it is fp4_preshift_calibrate for callers that cannot obtain device
 * memory when they calibrate (for instance a runtime that fixes its whole
 * device-memory plan at start-up and forbids allocation afterwards, or a
 * plug-in that receives tensors but no allocator).  It takes no workspace
 * and allocates nothing; its scratch is a 256 KB buffer inside the library
 * that every GPU loading the library keeps until the process exits.
 *   Same arguments and results as fp4_preshift_calibrate (bit-identical
 *   shift and rho).  K must be <= 65536: larger K returns FP4_ERR_WORKSPACE.
 *   The first call on a device looks up the buffer's device address (with
 *   that device current); make that first call before any stream capture.
 *   All calls share the buffer: calls whose work overlaps on a GPU race and
 *   must be ordered by the caller.  No part of it needs initialising.
 * ---------------------------------------------------------------------- */
FP4_API fp4_status fp4_preshift_calibrate_noalloc(const uint16_t *X, int M, int K, int8_t *shift, float *rho,
                                                  cudaStream_t stream);

/* ------------------------------------------------------------------------
 * 4-bit activations with the pre-shifted exponent bias (LLM-FP4 summary
 * page, section on the pre-shifted exponent bias: activations are quantized
 * with one per-tensor real factor, the per-channel powers of two having
 * moved into the weights; efficient matrix multiplication: both scale
 * factors are taken out of the low-bit product).
 *
 * fp4_act_quantize:
 *   s_a  = fl32(fl32(rho * c_j) / Qmax_f)                    (fp32)
 *   X'   = fl32(X[m,k] * 2^-shift[k])                        (shift NULL: X)
 *   code = signbit(X') << 3 | nearest magnitude index of fl32(|X'| / s_a),
 *          ties to the even index, saturating at index 7 (values beyond
 *          the calibrated range clip to +-Qmax * s_a).
 *   X [M][K] bf16 device, K % 8 == 0; shift [K] int8 (values in [-126, 0],
 *   from fp4_preshift_calibrate) or NULL; rho device float (positive,
 *   finite: else FP4_DEV_NONFINITE_INPUT and a_scale = NaN); fmt
 *   E1M2/E2M1/E3M0; j 0..7.  packed [M][K/2] uint8 out (low nibble
 *   first); a_scale device float out (s_a, written even when M == 0).
 * Device status: FP4_DEV_NONFINITE_INPUT.
 *
 * fp4_gemm_w4a4:
 *   Y[m,n] = bf16( act( s_a * sum_k v_a(a[m,k]) * v(w[n,k]) * s[n,k/group] ) )
 *   apacked [M][K/2] from fp4_act_quantize in format afmt, a_scale its s_a;
 *   the weights, act and Y as for fp4_gemm_act.  E2M1 activations with
 *   E2M1 weights at group 128, M > 64, with apacked and packed 32-byte
 *   aligned, multiply as 4-bit codes on tcgen05.mma kind::f8f6f4 (no
 *   dequantization; each group's code-product sum is exact in fp32, then
 *   scaled by s[n,g] in fp32).  Every other case expands the activation
 *   values (exact in bf16) into the workspace and runs fp4_gemm_act's
 *   engines on them.
 *   workspace  fp4_gemm_w4a4_workspace_size(M, N, K) bytes, zero-filled
 *              once before first use (its first part is the GEMM
 *              workspace, with the same rules).
 * ---------------------------------------------------------------------- */
FP4_API fp4_status fp4_act_quantize(const uint16_t *X, int M, int K, const int8_t *shift, const float *rho,
                                    fp4_format fmt, int j, uint8_t *packed, float *a_scale, cudaStream_t stream);
FP4_API size_t fp4_gemm_w4a4_workspace_size(int M, int N, int K);
FP4_API fp4_status fp4_gemm_w4a4(const uint8_t *apacked, fp4_format afmt, const float *a_scale,
                                 const uint8_t *packed, const void *scales, fp4_scale_dtype sdt, fp4_format fmt,
                                 int M, int N, int K, int group, fp4_act act, uint16_t *Y, void *workspace,
                                 size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * fp4_gemm -- Y = bf16( x_scale * X . dequant(W)^T ), fp32 accumulation.
 * (LLM-FP4 summary page, efficient matrix multiplication: the per-group
 * scales are applied outside the 4-bit products.)
 *
 *   Y[m,n] = bf16_rne( rho * sum_k X[m,k] * v(code[n,k]) * s[n, k/group] )
 *
 *   X        [M][K] bf16 device.   packed/scales as written by fp4_quantize.
 *   fmt      the format the weights were quantized in (not AUTO).
 *   x_scale  device float (rho from fp4_preshift_calibrate) or NULL for 1.
 *   Y        [M][N] bf16 out; must not alias the inputs.
 *   workspace 16-byte aligned, not overlapping the other buffers, of
 *            fp4_gemm_workspace_size() bytes, ZERO-FILLED ONCE before its
 *            first use (e.g. cudaMemsetAsync).  Its first 64 KB hold the
 *            decode engine's per-tile counters, which every call leaves at
 *            zero again (a call that set FP4_DEV_WAIT_TIMEOUT may not: zero
 *            the workspace again after that error); the rest holds, per
 *            engine, partial tiles of split tiles and activations prepared
 *            once per call.  The tensor engine's E2M1 path stores the
 *            activations there in f16, each row scaled by a power of two
 *            that brings its largest magnitude into [2^14, 2^15) (exact;
 *            elements more than 2^31 below the row maximum round to the f16
 *            subnormal grid), the factor undone in fp32 in the epilogue;
 *            the decode engine does the same per 128- or 256-element slice
 *            in shared memory.  Every bf16 activation is accepted.  With the
 *            automatic engine a workspace that is too small (or NULL) falls
 *            back to the tensor engine's bf16 path.
 * Engines (fp4_gemm_engine_for reports the choice).  Group 128: the decode
 * engine for M <= 8, and for 9 <= M <= 16 where the row-block kernel keeps
 * two block buffers (shared-memory fit of the staged activations); the
 * tensor engine otherwise.  Groups 32/64: the decode engine for M <= 8.
 * The group-128 decode engine has three kernels:
 *   - row-block (M <= 16, the activations [M][K] staged once per CTA in
 *     shared memory): each CTA takes whole 16-row blocks over all of K,
 *     bulk-copied; codes convert in registers (hardware e2m1 -> f16 for
 *     E2M1, exact bf16 bit placement otherwise) into warp-level MMAs.  No
 *     workspace.  Used when splits == 0 and the activations fit;
 *   - streaming (M <= 16): one persistent CTA per SM over an even split of
 *     all (row tile, 16 KB code chunk) units, streamed by TMA; a tile split
 *     between CTAs is summed by the CTA that completes it, in CTA order, so
 *     the result does not depend on timing.  Needs the workspace;
 *   - tensor-memory (17 <= M <= 64, on request only): dequantize warps
 *     write the codes to tensor memory as the A operand of tcgen05 MMAs.
 * The tensor engine stages TMA tiles, dequantizes them in shared memory and
 * runs tcgen05 MMAs into tensor memory, one group per pipeline stage.  Each
 * group scale is applied in fp32.  Groups 32/64 decode through a lookup
 * table into warp-level MMAs (no workspace).
 * Stream order: the GEMM kernels are launched as programmatic dependents
 * and start copying `packed` and `scales` before the kernel ahead of them
 * in the stream has finished; X, x_scale and Y are touched only after it
 * has.  Codes and scales written by the kernel directly ahead of a GEMM
 * call must therefore be separated from it by another stream operation
 * (any other kernel, copy or memset); fp4_quantize ends with such a launch.
 * Device status: FP4_DEV_WAIT_TIMEOUT, FP4_DEV_LAYOUT.
 * ---------------------------------------------------------------------- */
FP4_API size_t fp4_gemm_workspace_size(int M, int N, int K);
FP4_API fp4_status fp4_gemm(const uint16_t *X, const uint8_t *packed, const void *scales,
                    fp4_scale_dtype sdt, fp4_format fmt, int M, int N, int K, int group,
                    const float *x_scale, uint16_t *Y, void *workspace, size_t ws_bytes,
                    cudaStream_t stream);

/* fp4_gemm with an explicit engine and split count (0 = automatic); meant
 * for tests and tuning.  For the tensor engine `splits` is the split-K
 * count (at most 8); for the group-128 decode engine it is the number of
 * CTAs.  The decode engine accepts M <= 64 at group 128 (and needs the
 * workspace: FP4_ERR_WORKSPACE otherwise) and M <= 8 at groups 32/64;
 * larger M returns FP4_ERR_UNSUPPORTED_SHAPE. */
FP4_API fp4_status fp4_gemm_ex(const uint16_t *X, const uint8_t *packed, const void *scales,
                       fp4_scale_dtype sdt, fp4_format fmt, int M, int N, int K, int group,
                       const float *x_scale, uint16_t *Y, void *workspace, size_t ws_bytes,
                       fp4_engine engine, int splits, cudaStream_t stream);

/* fp4_gemm_ex with an output activation applied in the epilogue, in fp32,
 * to the finished value before the bf16 rounding (HiFloat4 page, section 5
 * "性能优化实战案例", optimisation measures: the fused Quant-GeLU-Dequant
 * operator; here the activations stay 16-bit, so the fusion is the
 * activation of the layer output inside the GEMM):
 *
 *   Y[m,n] = bf16_rne( act( rho * sum_k X[m,k] * v(code[n,k]) * s[n,k/group] ) )
 *
 *   act  FP4_ACT_NONE: identity; FP4_ACT_SILU: y / (1 + exp(-y));
 *        FP4_ACT_GELU: y * (1 + erf(y / sqrt 2)) / 2;
 *        FP4_ACT_SILU_GATE: gate and up projections fused in one call (the
 *        MLP of the LLaMA-shaped workloads): the weight rows are
 *        interleaved, row 2i the gate row and row 2i+1 the up row of output
 *        column i (quantize [W_gate; W_up] with its rows interleaved that
 *        way), N is even, and Y is [M][N/2] with
 *          Y[m,i] = bf16_rne( silu(y[m,2i]) * y[m,2i+1] ),
 *        y the product above; group 128 only (FP4_ERR_UNSUPPORTED_SHAPE
 *        otherwise).  Anything else returns FP4_ERR_INVALID_ARG.
 * Every engine and kernel supports NONE, SILU and GELU, with the other
 * arguments as for fp4_gemm_ex; the group-128 kernels also SILU_GATE.  The
 * activation is computed once per output after any split-K sum. */
FP4_API fp4_status fp4_gemm_act(const uint16_t *X, const uint8_t *packed, const void *scales,
                        fp4_scale_dtype sdt, fp4_format fmt, int M, int N, int K, int group,
                        const float *x_scale, fp4_act act, uint16_t *Y, void *workspace, size_t ws_bytes,
                        fp4_engine engine, int splits, cudaStream_t stream);

/* Engine fp4_gemm runs for this shape (FP4_ENGINE_DECODE or
 * FP4_ENGINE_TENSOR); host-only, no device call.  Non-positive sizes or an
 * unsupported group return FP4_ENGINE_AUTO. */
FP4_API fp4_engine fp4_gemm_engine_for(int M, int N, int K, int group);

/* ------------------------------------------------------------------------
 * fp4_get_device_status -- synchronises `stream`, copies the current
 * device's status word (FP4_DEV_* bits) to *host_code and, when `clear` is
 * non-zero, resets it.  Returns FP4_ERR_DEVICE_STATUS when a bit is set.
 * ---------------------------------------------------------------------- */
FP4_API fp4_status fp4_get_device_status(int32_t *host_code, int clear, cudaStream_t stream);

/* Test knob: bound, in microseconds, of every pipeline wait in the tensor
 * engine (default 2,000,000).  Values < 1 restore the default.  A test sets
 * it small to check that a wait which cannot complete reports
 * FP4_DEV_WAIT_TIMEOUT instead of hanging. */
FP4_API void fp4_set_wait_timeout_us(long long us);

/* Failure-detection check: launches one CTA that waits, with the bound
 * timeout_us (1 .. 10,000,000), on a barrier nothing arrives on.  The wait
 * must give up and set FP4_DEV_WAIT_TIMEOUT; no fault, trap or hang.  The
 * page has no counterpart: this only tests the library's bounded waits. */
FP4_API fp4_status fp4_selftest_bounded_wait(long long timeout_us, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4W4A16_H */
