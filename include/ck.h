/*
 * ck.h — C ABI of the B200 (sm_100a) ConvRot256 INT8 linear library (libck.so).
 *
 * The method (sources are web pages, cited by title and section):
 *  - comfy-kitchen 0.2.40 (PyPI page), "Huawei Ascend backend" and "HIP backend":
 *    quantize_int8_rowwise, quantize_and_rotate_rowwise (a ConvRot rotation
 *    fused with the dynamic per-row INT8 quantiser) and int8_linear (that
 *    quantiser on the activation, then an INT8 matmul).
 *  - sglang PR "Tune Kitchen INT8 row splitting for SM120", "Accuracy Test":
 *    BF16 activations and bias, INT8 weights, FP32 row scales, ConvRot256;
 *    outputs do not depend on how the M rows are split across calls.
 *  - ComfyUI-AppleSilicon-FP8 README, "What it fixes" row 17: rotate the
 *    activation online, quantise it per row, INT8 x INT8 -> INT32, with the
 *    per-row rescale and the bias fused into the store epilogue; row 12: the
 *    INT32 sums stay inside the int32 range.
 *
 * Definitions this library implements (the pages name the steps but print no
 * formulas; these are the readings taken):
 *  - ConvRot256: along K, every block of 256 consecutive values is replaced by
 *    its normalised Walsh-Hadamard transform, computed in fp32 as 8 butterfly
 *    stages h = 1, 2, 4, ..., 128 ((a, c) -> (a + c, a - c) on indices i and
 *    i + h with bit h of i clear), then multiplied by 1/16.
 *  - Per-row quantisation of a rotated row y[0..K): s = absmax(y) / 127
 *    (one IEEE fp32 division), q[k] = round-half-even(y[k] / s) clamped to
 *    [-127, 127] (-128 is never produced). A row of zeros gets s = 0, q = 0.
 *  - Linear: acc[m][n] = sum_k Qx[m][k] * Qw[n][k] in int32 (exact for
 *    K <= 132864), then Y[m][n] = bf16_rne(((float(acc) * s_x[m]) * s_w[n])
 *    + float(bias[n])), every step an fp32 operation rounded to nearest even;
 *    a NULL bias adds +0.0f.
 *
 * Conventions for every entry point:
 *  - Every pointer argument is DEVICE memory (cudaMalloc, a PyTorch CUDA
 *    tensor, ...) on the current device, owned by the caller. The library
 *    allocates nothing, keeps no pointer after returning, and never
 *    synchronises the stream or the device (except ck_get_device_error,
 *    ck_clear_device_error and ck_checked_violations).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and runs asynchronously: on CK_OK the results are valid once the
 *    stream reaches that point.
 *  - All matrices are row-major. BF16 values are passed as their 16-bit
 *    patterns (ck_bf16 is binary-compatible with __nv_bfloat16).
 *  - Arguments are validated on the host before anything is launched; a
 *    non-CK_OK status means nothing was enqueued. Checks, in order:
 *    CK_ERR_INVALID_VALUE (NULL pointer where one is required, negative size,
 *    K <= 0, ldx < K), CK_ERR_UNSUPPORTED_SHAPE (K % 256 != 0, K > 132864,
 *    N % 8 != 0, M or N >= 2^31), CK_ERR_MISALIGNED (an address or row stride
 *    not 16-byte aligned where stated), CK_ERR_WORKSPACE, then
 *    CK_ERR_ARCH (current device is not compute capability 10.0) and
 *    CK_ERR_CUDA (a CUDA runtime call or launch failed).
 *  - M == 0 (and N == 0 for the linear) is valid and enqueues nothing.
 *  - The functions are thread-safe and may be called concurrently on
 *    different streams; calls that write the same buffers must be ordered
 *    by the caller.
 *  - Device-side waits inside the kernels are bounded (about 4 s). If one
 *    runs out the kernel records CK_ERR_DEVICE_TIMEOUT in a per-device error
 *    word, stops its work and returns; outputs of that call are then
 *    undefined. ck_get_device_error() reports it.
 */
#ifndef CK_H_
#define CK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t. */
typedef struct CUstream_st *ck_stream_t;

/* A bfloat16 value as its bit pattern. */
typedef uint16_t ck_bf16;

typedef enum ck_status {
    CK_OK = 0,
    CK_ERR_INVALID_VALUE = 1,
    CK_ERR_UNSUPPORTED_SHAPE = 2,
    CK_ERR_MISALIGNED = 3,
    CK_ERR_WORKSPACE = 4,
    CK_ERR_ARCH = 5,
    CK_ERR_CUDA = 6,
    CK_ERR_DEVICE_TIMEOUT = 7
} ck_status;

/* Largest K for which |acc| <= K * 127^2 stays below 2^31, rounded down to a
 * multiple of 256. */
#define CK_MAX_K 132864

/*
 * Offline weight preparation (ComfyUI-AppleSilicon-FP8 README, row 17: the
 * weights of a ConvRot checkpoint are stored rotated; sglang PR, Accuracy
 * Test: INT8 weights with FP32 row scales).
 *   W   [N, K] fp32, row stride K, 16-byte aligned.  (input)
 *   Qw  [N, K] int8, row stride K, 16-byte aligned.  (output) ConvRot256 of
 *       each row of W, quantised per row.
 *   s_w [N] fp32, 16-byte aligned.                   (output) row scales.
 * Requires K % 256 == 0 and K <= CK_MAX_K; N >= 0.
 */
ck_status ck_rotate_quant_weight(const float *W, int64_t N, int64_t K, int8_t *Qw, float *s_w,
                                 ck_stream_t stream);

/*
 * quantize_and_rotate_rowwise (comfy-kitchen, "Huawei Ascend backend" and
 * "HIP backend": the fused ConvRot quantiser): ConvRot256 of every row of X,
 * then dynamic per-row INT8 quantisation, in one pass over X.
 *   X   [M, K] bf16 with row stride ldx elements (ldx >= K, ldx % 8 == 0),
 *       16-byte aligned.                                      (input)
 *   Qx  [M, K] int8, row stride K, 16-byte aligned.            (output)
 *   s_x [M] fp32, 4-byte aligned.                              (output)
 * Requires K % 256 == 0 and K <= CK_MAX_K.
 */
ck_status ck_quantize_rotate_rowwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                     int8_t *Qx, float *s_x, ck_stream_t stream);

/*
 * quantize_int8_rowwise (comfy-kitchen, "Huawei Ascend backend"): the same
 * per-row quantiser without the rotation. Same arguments and rules as
 * ck_quantize_rotate_rowwise.
 */
ck_status ck_quantize_int8_rowwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                   int8_t *Qx, float *s_x, ck_stream_t stream);

/* Input activations for the *_act entry points (each bf16 input becomes the
 * bf16 value nearest to the exact act(x), then is rotated and quantised). */
typedef enum ck_act {
    CK_ACT_NONE = 0,
    CK_ACT_RELU = 1,      /* max(x, 0) */
    CK_ACT_SILU = 2,      /* x / (1 + e^-x) */
    CK_ACT_GELU_TANH = 3  /* 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) */
} ck_act;

/*
 * quantize_and_rotate_rowwise with an input activation (comfy-kitchen 0.2.40,
 * "HIP backend": int8_linear(input_act=...) folds the activation into the
 * fused ConvRot quantiser's load, so act(x) is never written to memory).
 * Each element x becomes the bf16 value nearest to the exact act(x) (ties to
 * even; no bf16 input's exact act(x) lies on or near a midpoint, except
 * |x| < 2^-120, where act(x) is just above x/2 and x/2 rounds with ties
 * going up) before ConvRot256; act is a ck_act value (CK_ERR_INVALID_VALUE
 * otherwise). The list of activations and their formulas are a reading: the
 * page names the argument only. The kernel evaluates act in fp32 (its own
 * e^x: Cody-Waite reduction and a degree-7 Taylor polynomial) and redoes in
 * double precision every value whose fp32 result lies near a bf16 rounding
 * midpoint, so the stored bf16 values are those of the definition; for silu
 * and gelu_tanh each CTA evaluates that once per bf16 input with |x| in
 * [2^-9, 2^7) into a table, and the other inputs have closed forms (x, -0
 * or x/2) or take the double path. Other arguments as for
 * ck_quantize_rotate_rowwise.
 */
ck_status ck_quantize_rotate_rowwise_act(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                         int act, int8_t *Qx, float *s_x, ck_stream_t stream);

/*
 * dequantize_int8_simple / dequantize_int8_simple_dtype (comfy-kitchen 0.2.40,
 * "Huawei Ascend backend"): Y[m][k] = float(Q[m][k]) * s, one fp32 rounding,
 * with s = s[0] for the whole tensor (per_row == 0) or s[m] per row
 * (per_row != 0). out_bf16 == 0 stores fp32 Y [rows, K]; otherwise the
 * product is rounded to bf16 (the _dtype form). Q 16-B aligned, K % 16 == 0,
 * s 4-B aligned, Y 16-B aligned.
 */
ck_status ck_dequantize_int8(const int8_t *Q, const float *s, int64_t rows, int64_t K,
                             int per_row, int out_bf16, void *Y, ck_stream_t stream);

/*
 * quantize_int8_tensorwise (same page): one scale for the whole tensor,
 * s = absmax(X) / 127, Q = round-half-even(X / s) clamped to [-127, 127]; a
 * zero tensor gives s = 0 and zero codes. No rotation (quantising this way
 * before ConvRot is the ~16% error negative control of the
 * ComfyUI-AppleSilicon-FP8 README, row 17). X [M, K] bf16 with row stride ldx
 * (16-B aligned rows, K % 8 == 0), Q [M, K] int8, s one fp32 (its memory is
 * also used for the absmax while the three kernels run).
 */
ck_status ck_quantize_int8_tensorwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                      int8_t *Q, float *s, ck_stream_t stream);

/*
 * Bytes of device workspace ck_int8_linear needs for M rows of K features:
 * the INT8 codes (M*K bytes) and the row scales (4*M bytes), each part
 * rounded up to 256 bytes. Returns 0 for M <= 0 or K <= 0.
 */
size_t ck_int8_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * int8_linear (comfy-kitchen, "Huawei Ascend backend"; ComfyUI-AppleSilicon-FP8
 * README, row 17): Y = bf16(((INT32 GEMM of the rotated, per-row quantised X
 * with Qw) * s_x) * s_w + bias). Two kernels on `stream`: the fused
 * rotate+quantise pass writes the codes and row scales into `workspace`, then
 * the tcgen05 INT8 GEMM applies the epilogue as it stores Y. M may be any
 * size (no row splitting): the ragged last tile is handled in the same launch.
 *   X         [M, K] bf16, row stride ldx (ldx >= K, ldx % 8 == 0), 16-B aligned.
 *   Qw        [N, K] int8 (already rotated, from ck_rotate_quant_weight),
 *             row stride K, 16-B aligned.
 *   s_w       [N] fp32, 16-B aligned.
 *   bias      [N] bf16, 16-B aligned, or NULL (adds +0.0f).
 *   Y         [M, N] bf16, row stride N, 16-B aligned.   (output)
 *   workspace >= ck_int8_linear_workspace_bytes(M, K) bytes, 256-B aligned;
 *             its contents on return are the codes (first M*K bytes) and the
 *             row scales (at offset round_up(M*K, 256)).
 * Requires K % 256 == 0, K <= CK_MAX_K, N % 8 == 0.
 */
ck_status ck_int8_linear(const ck_bf16 *X, int64_t ldx, const int8_t *Qw, const float *s_w,
                         const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                         void *workspace, size_t workspace_bytes, ck_stream_t stream);

/*
 * ck_int8_linear with an input activation: Y = linear(act(X)) with act
 * applied inside the quantiser's load (see ck_quantize_rotate_rowwise_act).
 * CK_ACT_NONE gives exactly ck_int8_linear.
 */
ck_status ck_int8_linear_act(const ck_bf16 *X, int64_t ldx, int act, const int8_t *Qw,
                             const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                             int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                             ck_stream_t stream);

/*
 * Input RMSNorm with a residual (comfy-kitchen 0.2.40, "Huawei Ascend backend":
 * int8_linear accepts the input RMSNorm and residual arguments and applies
 * them with shared helpers apart from its GEMM; the page prints no formula).
 * Reading:
 *   h   = bf16_rne(fl32(x + r)) (a bf16 tensor addition), or h = x when
 *         residual is NULL;
 *   residual_out = h (when residual_out is not NULL);
 *   Y_k = the bf16 value nearest to h_k g_k / sqrt(mean_k(h_k^2) + eps) (the
 *         exact real value; g_k = 1 when g is NULL), ties to even.
 * The kernel sums the squares and forms Y in double precision (each h^2 and
 * h g exact), so Y is that rounding except where the exact value lies within
 * about 2^-36 (relative) of a bf16 rounding midpoint, where the summation
 * order can decide the neighbour.
 *   X            [M, K] bf16, row stride ldx (>= K, % 8 == 0), 16-B aligned.
 *   residual     [M, K] bf16, row stride ldr, or NULL.
 *   residual_out [M, K] bf16, row stride ldo, or NULL (output); it may alias
 *                X or residual (in-place update of the residual stream).
 *   g            [K] bf16 weight, or NULL.
 *   eps          > 0 and finite.
 *   Y            [M, K] bf16, row stride K (output; must not overlap the inputs).
 * All pointers 16-B aligned, strides multiples of 8; K % 256 == 0,
 * K <= CK_MAX_K. One kernel on `stream`, one warp per row.
 */
ck_status ck_rmsnorm_residual(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual, int64_t ldr,
                              ck_bf16 *residual_out, int64_t ldo, const ck_bf16 *g, float eps,
                              int64_t M, int64_t K, ck_bf16 *Y, ck_stream_t stream);

/* Largest K for which ck_int8_linear_norm normalises inside the quantiser. */
#define CK_NORM_FUSED_MAX_K 14336

/*
 * quantize_and_rotate_rowwise on the input RMSNorm of X (comfy-kitchen
 * 0.2.40, "Huawei Ascend backend": int8_linear's input RMSNorm and residual
 * arguments), in one kernel: the normalised values (defined as in
 * ck_rmsnorm_residual) are formed in the quantiser's staged load, rotated and
 * quantised; only residual_out (when given), Qx and s_x are written.
 * Arguments as in ck_rmsnorm_residual for X, residual, residual_out, g, eps,
 * and as in ck_quantize_rotate_rowwise for Qx [M, K] and s_x [M].
 * K <= CK_NORM_FUSED_MAX_K (CK_ERR_UNSUPPORTED_SHAPE otherwise).
 */
ck_status ck_quantize_rotate_rowwise_norm(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual,
                                          int64_t ldr, ck_bf16 *residual_out, int64_t ldo,
                                          const ck_bf16 *g, float eps, int64_t M, int64_t K,
                                          int8_t *Qx, float *s_x, ck_stream_t stream);

/*
 * ck_int8_linear on the input RMSNorm of X (with an optional residual), as
 * the page's int8_linear takes them. For K <= CK_NORM_FUSED_MAX_K the
 * normalisation runs inside the ConvRot quantiser's staged load (x and the
 * residual staged together, the residual output written from there, the sum
 * of squares in double, each normalised value rounded to bf16 as
 * ck_rmsnorm_residual defines it and then rotated and quantised), so the
 * normalised rows never reach memory; larger K runs ck_rmsnorm_residual into
 * the workspace first. Then the INT8 GEMM. Arguments as in
 * ck_rmsnorm_residual and ck_int8_linear. Workspace:
 * ck_int8_linear_norm_workspace_bytes(M, K) bytes, 256-B aligned (the codes
 * and row scales, as ck_int8_linear's; for K > CK_NORM_FUSED_MAX_K the
 * normalised rows come first).
 */
size_t ck_int8_linear_norm_workspace_bytes(int64_t M, int64_t K);
ck_status ck_int8_linear_norm(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual,
                              int64_t ldr, ck_bf16 *residual_out, int64_t ldo, const ck_bf16 *g,
                              float eps, const int8_t *Qw, const float *s_w, const ck_bf16 *bias,
                              ck_bf16 *Y, int64_t M, int64_t N, int64_t K, void *workspace,
                              size_t workspace_bytes, ck_stream_t stream);

/*
 * ck_int8_linear_act for activations and outputs in HOST memory, with the
 * PCIe copies overlapped with the kernels. The rows are processed in chunks of
 * chunk_rows (the last one ragged): chunk c is copied to the device while
 * chunk c-1 is quantised and multiplied and chunk c-2 is copied back, so the
 * call takes about as long as the larger of its two transfers. The results
 * are those of ck_int8_linear_act row for row (rows are independent:
 * sglang PR "Tune Kitchen INT8 row splitting for SM120", Accuracy Test).
 *
 *   X_host  [M, K] bf16, row stride ldx (ldx >= K) elements, host memory.
 *           (input; page-locked memory - cudaHostAlloc, cudaHostRegister,
 *           torch pin_memory - lets the copies run asynchronously; pageable
 *           memory gives the same results without the overlap)
 *   Qw, s_w, bias: device memory, as for ck_int8_linear.
 *   Y_host  [M, N] bf16, row stride N, host memory.   (output)
 *   chunk_rows  rows per chunk (> 0). 2048 keeps a chunk's GEMM a few waves
 *           long on a B200 for the N of the pages' workloads while the
 *           first copy in and the last copy out, which nothing overlaps,
 *           stay short.
 *   workspace   >= ck_int8_linear_host_workspace_bytes(chunk_rows, N, K)
 *           bytes of device memory, 256-B aligned (two input and two output
 *           chunk buffers, the chunk's codes and row scales).
 *
 * Ordering: the copies and kernels run on three streams the library creates
 * once per device (together with the events that link them); they start
 * after the work already queued on `stream`, and `stream` waits for the last
 * copy back, so work queued on `stream` afterwards - or a synchronize of it -
 * sees Y_host complete. Calls on one device are queued on the same internal
 * streams in the order they are made. Nothing here blocks the host (apart
 * from what the driver does for pageable memory). Validation failures
 * enqueue nothing; a CUDA error returned while chunks are being enqueued
 * (CK_ERR_CUDA) can leave earlier chunks queued, and Y_host is then
 * undefined.
 */
size_t ck_int8_linear_host_workspace_bytes(int64_t chunk_rows, int64_t N, int64_t K);
ck_status ck_int8_linear_host(const ck_bf16 *X_host, int64_t ldx, int act, const int8_t *Qw,
                              const float *s_w, const ck_bf16 *bias, ck_bf16 *Y_host, int64_t M,
                              int64_t N, int64_t K, int64_t chunk_rows, void *workspace,
                              size_t workspace_bytes, ck_stream_t stream);

/*
 * convrot_w4a4_linear (comfy-kitchen 0.2.40, "Huawei Ascend backend": ConvRot
 * then signed INT4 quantisation of both operands; activation codes stay in
 * INT8 storage; packed weights are unpacked to INT8 for INT32 accumulation;
 * the result is scaled like int8_linear's). Readings: s = absmax / 7, codes
 * round-half-even(y / s) clamped to [-7, 7]; two weight codes per byte,
 * element 2j in the low nibble of byte j, each nibble 4-bit two's complement.
 */

/* Offline: ConvRot256 + per-row signed INT4 of fp32 W [N, K] (16-B aligned).
 * Qw4 [N, K/2] bytes (16-B aligned), s_w [N] fp32 (16-B aligned). */
ck_status ck_rotate_quant_weight_int4(const float *W, int64_t N, int64_t K, uint8_t *Qw4,
                                      float *s_w, ck_stream_t stream);

/* Packed INT4 [N, K/2] -> int8 codes [N, K] (both 16-B aligned). */
ck_status ck_unpack_int4(const uint8_t *Qw4, int64_t N, int64_t K, int8_t *Qw, ck_stream_t stream);

/* ConvRot256 + per-row signed INT4 codes (in int8 storage, [-7, 7]) of bf16
 * X; arguments as for ck_quantize_rotate_rowwise. */
ck_status ck_quantize_rotate_rowwise_int4(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                          int8_t *Qx, float *s_x, ck_stream_t stream);

/* Workspace of ck_convrot_w4a4_linear: activation codes (M*K), row scales
 * (4*M) and the unpacked weights (N*K), each part rounded up to 256 bytes. */
size_t ck_convrot_w4a4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Y = bf16(((INT32 GEMM of the INT4 codes of rotated X with the unpacked
 * weights) * s_x) * s_w + bias): the INT4 quantiser, the unpack kernel and
 * the INT8 tcgen05 GEMM on `stream`. Arguments as for ck_int8_linear, with
 * Qw4 [N, K/2] packed codes (16-B aligned) and the workspace sized by
 * ck_convrot_w4a4_linear_workspace_bytes (256-B aligned). */
ck_status ck_convrot_w4a4_linear(const ck_bf16 *X, int64_t ldx, const uint8_t *Qw4,
                                 const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                                 int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                                 ck_stream_t stream);

/* convrot_w4a4_linear on weights unpacked once, offline (ck_unpack_int4 of
 * the packed codes: Qw [N, K] int8 in [-7, 7], 16-B aligned): the INT4
 * quantiser into the workspace (ck_int8_linear_workspace_bytes(M, K) bytes,
 * 256-B aligned: codes, then row scales) and the INT8 GEMM, with no unpack
 * per call; results equal ck_convrot_w4a4_linear's. Static weights trade
 * N * K / 2 more bytes of weight memory for the per-call unpack (1.5 N K
 * bytes of traffic and a kernel). Other arguments as for ck_int8_linear. */
ck_status ck_convrot_w4a4_linear_unpacked(const ck_bf16 *X, int64_t ldx, const int8_t *Qw,
                                          const float *s_w, const ck_bf16 *bias, ck_bf16 *Y,
                                          int64_t M, int64_t N, int64_t K, void *workspace,
                                          size_t workspace_bytes, ck_stream_t stream);

/*
 * The GEMM and fused epilogue alone, on activations already quantised (by
 * ck_quantize_rotate_rowwise):
 *   Qx [M, K] int8 (16-B aligned), s_x [M] fp32 (4-B aligned), Qw/s_w/bias/Y as
 *   for ck_int8_linear. Requires K % 256 == 0, K <= CK_MAX_K, N % 8 == 0.
 */
ck_status ck_int8_gemm_rowscale(const int8_t *Qx, const float *s_x, const int8_t *Qw,
                                const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                                int64_t N, int64_t K, ck_stream_t stream);

/*
 * ConvRot NVFP4 (ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix",
 * section 5-1, nvfp4_gemm.py: FP4 E2M1 codes, one scale per 16 values along
 * K in the cuBLAS 128 x 4 blocked layout, a per-tensor scale, dequantisation
 * as value x (per-tensor scale x block scale), a_dq @ w_dq.T + bias).
 * Readings (the pages print no quantiser), on ConvRot256-rotated rows y:
 *   s_t = amax(tensor) / 2688                       (fp32 division; 6 x 448)
 *   b   = E4M3 of (amax(block of 16) / 6) / s_t, round to nearest even,
 *         saturating at 448 (0 when s_t == 0)
 *   q   = E2M1 of y / (float(b) * s_t), round to nearest even, saturating at
 *         6, sign kept (+0 when the divisor is 0)
 * Codes: [rows, K/2] bytes, element 2j in the low nibble of byte j (the
 * tensor cores' order). Scales: ck_nvfp4_scale_bytes(rows, K) bytes, E4M3,
 * blocked: the scale of row r, column c = k/16 sits at
 *   ((r/128) * (K/64) + c/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4 + c%4,
 * rows padded to a multiple of 128 with zero bytes. s_t: one fp32 in device
 * memory. Requires K % 256 == 0 and K <= 32768; pointers 16-B aligned (s_t
 * 4-B). Codes and scales are bit-exact against the CPU oracle.
 */
size_t ck_nvfp4_scale_bytes(int64_t rows, int64_t K);

/* bf16 X [M, K] (row stride ldx) -> Q [M, K/2], S, *s_t (all device). Two
 * passes over X: the rotated tensor's absmax, then the codes. */
ck_status ck_quantize_rotate_nvfp4(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                   uint8_t *Q, uint8_t *S, float *s_t, ck_stream_t stream);

/* Offline: fp32 W [N, K] (row stride K) -> Qw [N, K/2], Sw, *s_tw. */
ck_status ck_rotate_quant_weight_nvfp4(const float *W, int64_t N, int64_t K, uint8_t *Qw,
                                       uint8_t *Sw, float *s_tw, ck_stream_t stream);

/* Decoding as the page's dequantiser, in fp32: out[r][k] =
 * e2m1(code) * (s_t * e4m3(scale)); hi_first != 0 reads the high nibble of
 * each byte as the first of its two elements (the page's default order). */
ck_status ck_dequantize_nvfp4(const uint8_t *Q, const uint8_t *S, const float *s_t, int64_t rows,
                              int64_t K, int hi_first, float *out, ck_stream_t stream);

/* Block-scaled FP4 GEMM (tcgen05 kind::mxf4nvf4) with the epilogue
 * Y = bf16_rne(fl(acc * fl(s_ta * s_tw)) + float(bias)); acc is the tensor
 * cores' fp32 sum of the exact products (summation order theirs), so Y
 * matches the oracle within the float accumulation bound, not bit for bit.
 * Requires N % 8 == 0 (plus the constraints above). */
ck_status ck_nvfp4_gemm(const uint8_t *Qa, const uint8_t *Sa, const float *s_ta,
                        const uint8_t *Qw, const uint8_t *Sw, const float *s_tw,
                        const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                        ck_stream_t stream);

/* ConvRot NVFP4 linear: quantise X (ck_quantize_rotate_nvfp4) into the
 * workspace, then ck_nvfp4_gemm. Workspace: codes, scales and s_t of X, each
 * part rounded up to 256 bytes, 256-B aligned. */
size_t ck_convrot_nvfp4_linear_workspace_bytes(int64_t M, int64_t K);
ck_status ck_convrot_nvfp4_linear(const ck_bf16 *X, int64_t ldx, const uint8_t *Qw,
                                  const uint8_t *Sw, const float *s_tw, const ck_bf16 *bias,
                                  ck_bf16 *Y, int64_t M, int64_t N, int64_t K, void *workspace,
                                  size_t workspace_bytes, ck_stream_t stream);

/* Size of the device array that ck_int8_linear_noalloc uses as its
 * workspace: 32 MiB, enough for ck_int8_linear_workspace_bytes(M, K) of e.g.
 * M = 4096, K = 7936 or M = 1024, K = 32512. */
#define CK_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * ck_int8_linear without a caller workspace, for callers that cannot allocate
 * device memory (a plugin inside an engine that owns all device memory and
 * gives it no workspace, code with a memory budget fixed at start-up, code
 * that must not risk the device-wide synchronisation cudaFree can cause).
 * The pages have no counterpart to this entry point; it exists for such
 * callers only. Arguments and results are those of ck_int8_linear minus the
 * workspace: the activation codes and row scales go to one file-scope device
 * array of CK_NOALLOC_SCRATCH_BYTES instead, which every GPU that loads this
 * part of the library holds until the process exits. Calls need
 * ck_int8_linear_workspace_bytes(M, K) <= CK_NOALLOC_SCRATCH_BYTES, else
 * CK_ERR_WORKSPACE is returned and nothing is launched. All calls on a device
 * share the array (it keeps the last call's contents; each call rewrites all
 * it reads, so nothing needs clearing), so calls whose work overlaps on the
 * GPU race and give wrong results: order them. The first call on a device
 * looks up the array's device address with that device current; make that
 * first call before any stream capture (the lookup is repeated after the
 * device's context changes, e.g. after cudaDeviceReset). Argument checks and
 * their order are ck_int8_linear's (CK_ERR_INVALID_VALUE, then
 * CK_ERR_UNSUPPORTED_SHAPE, then CK_ERR_MISALIGNED), then the size check,
 * then CK_ERR_ARCH. Allocates nothing.
 */
ck_status ck_int8_linear_noalloc(const ck_bf16 *X, int64_t ldx, const int8_t *Qw, const float *s_w,
                                 const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                                 ck_stream_t stream);

/* A static, human-readable name for a status code. */
const char *ck_status_string(ck_status status);

/*
 * Synchronises the current device, then returns CK_ERR_DEVICE_TIMEOUT if any
 * kernel of this library on it gave up on a bounded wait since the last
 * ck_clear_device_error(), CK_ERR_CUDA if the synchronisation itself failed,
 * else CK_OK.
 */
ck_status ck_get_device_error(void);

/* Resets the current device's error word (synchronous with the device). */
ck_status ck_clear_device_error(void);

/*
 * The checked build. libck_checked.so is this library compiled with
 * CK_CHECKED: its kernels test index invariants at their memory accesses
 * (global stores and loads inside their tensor's rows and columns,
 * shared-memory accesses and bulk copies inside the CTA's allocation, TMEM
 * columns inside the allocation). A failed check skips the access and sets
 * its class bit (1 global store, 2 global load, 4 shared memory, 8 bulk copy,
 * 16 TMEM) in a device word; nothing traps. A bulk copy that was skipped
 * leaves its stage's wait to run out, which ck_get_device_error() then
 * reports as CK_ERR_DEVICE_TIMEOUT. ck_is_checked_build() returns 1 in that
 * build and 0 in libck.so. ck_checked_violations() synchronises the current
 * device, returns the class bits set since its last call on that device and
 * clears them (0 in libck.so; bit 31 if the words could not be read).
 */
int ck_is_checked_build(void);
unsigned ck_checked_violations(void);

/* ---- test hooks (used by the test suite; stable, but not part of the method) ---- */

/*
 * The INT32 accumulators of the GEMM, without the epilogue:
 *   acc [M, N] int32, row stride N, 16-B aligned.  (output)
 * Same kernel and tiling as ck_int8_gemm_rowscale.
 */
ck_status ck_test_int8_gemm_i32(const int8_t *Qx, const int8_t *Qw, int32_t *acc, int64_t M,
                                int64_t N, int64_t K, ck_stream_t stream);

/* Same as ck_quantize_int8_rowwise (the quantiser without the rotation). */
ck_status ck_test_quantize_rowwise_norotate(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                            int8_t *Qx, float *s_x, ck_stream_t stream);

/*
 * The input activation alone, exactly as the quantiser applies it before the
 * rotation (same device code), on n bf16 values:
 *   X [n] bf16 (input), Y [n] bf16 (output), both 16-B aligned; n % 256 == 0;
 *   act a ck_act value.
 * Lets the tests compare every possible bf16 input with the definition.
 */
ck_status ck_test_input_act(const ck_bf16 *X, int64_t n, int act, ck_bf16 *Y, ck_stream_t stream);

/*
 * The per-row divisor and reciprocal of the rotated quantiser, for n row
 * absmax values (all device memory, fp32, n elements each):
 *   amax [n] (input), div [n], rc [n] (outputs); q = 127 (INT8) or 7 (INT4).
 * For amax >= 2^-103 (finite) div is the IEEE quotient fl(amax / q), which
 * the row scale is derived from, and rc the reciprocal of div that the fast
 * rounding path multiplies by (within 2^-24 + 2^-43 of 1 / div relative);
 * smaller absmax values take the quantiser's exact path (div = the row
 * scale, rc = 0). CK_ERR_INVALID_VALUE for n < 0, another q, or a null
 * pointer with n > 0. Lets the tests compare the division with the IEEE
 * quotient for every fp32 significand.
 */
ck_status ck_test_row_quant_params(const float *amax, int64_t n, int q, float *div, float *rc,
                                   ck_stream_t stream);

/*
 * The INT8 tensor-core ceiling, measured: on every pair of SMs the GEMM uses
 * (*pairs receives their number), mmas_per_pair back-to-back
 * tcgen05.mma.cta_group::2.kind::i8 of the GEMM's shape (M 256, N 256, K 32:
 * 2 * 256 * 256 * 32 operations each) on shared-memory operands, with no
 * global-memory traffic. Time it with events on `stream`; the operation count
 * is 4194304 * mmas_per_pair * *pairs. No counterpart in the pages: it gives
 * the INT8 GEMM's roofline a measured denominator.
 */
ck_status ck_test_i8_mma_peak(int64_t mmas_per_pair, int *pairs, ck_stream_t stream);

/*
 * One thread whose index check fails on purpose (class bit 4, shared memory)
 * with no memory access behind it: in libck_checked.so the next
 * ck_checked_violations() then returns 4; in libck.so nothing happens. It
 * shows that the checked build's words are set, read and cleared.
 */
ck_status ck_test_checked_fire(ck_stream_t stream);

/*
 * Fault injection for the bounded waits, host side only: with mode 1 the next
 * GEMM launch (INT8 or NVFP4) on this thread's current device runs with its TMA producer
 * issuing nothing, so the MMA warp's wait for the first stage can never be
 * satisfied; the kernel must then record CK_ERR_DEVICE_TIMEOUT and return
 * instead of hanging. The flag is consumed by that launch. mode 0 clears it.
 * wait_limit_ns (> 0) replaces the default bound (about 4 s) for that launch.
 */
ck_status ck_test_inject_producer_stall(int mode, int64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* CK_H_ */
