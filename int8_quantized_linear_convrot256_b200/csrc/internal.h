// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "ck.h"

namespace ck {

// ---- host-side checks shared by the entry points (api.cu)

// ck_int8_linear's argument checks before its workspace size check, in its
// order (CK_ERR_INVALID_VALUE, CK_ERR_UNSUPPORTED_SHAPE, CK_ERR_MISALIGNED);
// with_workspace = false leaves the workspace pointer out.
ck_status check_linear_args(const void *X, int64_t ldx, const void *Qw, const void *s_w,
                            const void *bias, const void *Y, int64_t M, int64_t N, int64_t K,
                            const void *workspace, bool with_workspace);
// CK_OK on a B200 (compute capability 10.0) current device, else CK_ERR_ARCH or
// CK_ERR_CUDA; *generation changes whenever the device's context changed
// (e.g. after cudaDeviceReset), so per-context caches know to refresh.
ck_status check_current_device(unsigned *generation);

// ---- fused ConvRot256 + per-row INT8 quantiser (quant_rotate.cu)

// Rows of bf16 (bit patterns) with row stride ldx; rotate=false skips ConvRot.
// err is the device error word (bounded waits of the staged variant).
// act: input activation applied before the rotation (0 none, 1 relu, 2 silu,
// 3 tanh-form gelu); only with rotate. qmax: 127 (INT8 codes) or 7 (signed
// INT4 codes in int8 storage, rotate only, no act).
cudaError_t launch_quant_rows_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   bool rotate, int act, int qmax, int8_t *Q, float *S,
                                   unsigned *err, int num_sms, cudaStream_t stream);

// The input RMSNorm (h = bf16(x + r) written to Rout when given, y = the
// bf16 rounding of h g / sqrt(mean(h^2) + eps)) fused into the ConvRot256
// INT8 quantiser's staged load: codes Q [M, K] and row scales S of y, which
// never reaches memory. *launched is false when the rows do not fit the
// staging buffers (then nothing ran); Rout may alias X or R.
cudaError_t launch_quant_norm_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   const uint16_t *R, int64_t ldr, uint16_t *Rout, int64_t ldo,
                                   const uint16_t *g, float eps, int8_t *Q, float *S,
                                   unsigned *err, int num_sms, cudaStream_t stream,
                                   bool *launched);

// Test hook: the input activation of n bf16 values (n % 256 == 0) as the
// staged quantiser applies it (0 none, 1 relu, 2 silu, 3 tanh-form gelu).
cudaError_t launch_test_row_quant_params(const float *amax, int64_t n, int q, float *div,
                                         float *rc, cudaStream_t stream);
cudaError_t launch_test_input_act(const uint16_t *X, int64_t n, int act, uint16_t *Y,
                                  cudaStream_t stream);

// Rows of fp32 with row stride K (offline weight preparation), always rotated;
// int4_packed: signed INT4 codes packed two per byte into Q [N, K/2].
cudaError_t launch_quant_rows_f32(const float *W, int64_t N, int64_t K, bool int4_packed,
                                  int8_t *Q, float *S, cudaStream_t stream);

// ConvRot NVFP4 quantisation (codes [rows, K/2], blocked scales of s_bytes
// bytes, per-tensor scale in *s_t) and decoding to fp32.
cudaError_t launch_quant_nvfp4_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                    uint8_t *Q, uint8_t *S, size_t s_bytes, float *s_t,
                                    unsigned *err, int num_sms, cudaStream_t stream);
cudaError_t launch_quant_nvfp4_f32(const float *W, int64_t N, int64_t K, uint8_t *Q, uint8_t *S,
                                   size_t s_bytes, float *s_t, cudaStream_t stream);
cudaError_t launch_dequant_nvfp4(const uint8_t *Q, const uint8_t *S, const float *s_t,
                                 int64_t rows, int64_t K, bool hi_first, float *out, int num_sms,
                                 cudaStream_t stream);
// Packed signed INT4 [rows, K/2] -> int8 [rows, K].
cudaError_t launch_unpack_int4(const uint8_t *Q4, int64_t rows, int64_t K, int8_t *Q8,
                               int num_sms, cudaStream_t stream);

// ---- input RMSNorm with a residual (rmsnorm.cu): Y [M, K] (row stride K) =
// bf16((h * inv) * g), h = bf16(x + r) (x without R) also written to Rout
// when given (row stride ldo; it may alias X or R).
cudaError_t launch_rmsnorm_rows(const uint16_t *X, int64_t ldx, const uint16_t *R, int64_t ldr,
                                uint16_t *Rout, int64_t ldo, const uint16_t *g, float eps,
                                int64_t M, int64_t K, uint16_t *Y, cudaStream_t stream);

// ---- dequantize_int8_simple(_dtype), quantize_int8_tensorwise (dequant.cu)

cudaError_t launch_dequantize_int8(const int8_t *Q, const float *S, int64_t rows, int64_t K,
                                   bool per_row, bool out_bf16, void *Y, int num_sms,
                                   cudaStream_t stream);

// s receives the tensor's scale (used as scratch for the absmax first).
cudaError_t launch_quantize_int8_tensorwise(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                            int8_t *Q, float *s, int num_sms, cudaStream_t stream);

// ---- tcgen05 INT8 GEMM with fused epilogue (gemm_i8_tcgen05.cu)

struct GemmParams {
    const float *s_x;       // [M]
    const float *s_w;       // [N]
    const uint16_t *bias;   // [N] bf16 bits or nullptr
    uint16_t *Y;            // [M, N] bf16 bits (epilogue mode)
    int32_t *acc;           // [M, N] int32 (raw accumulator mode)
    int M, N, K;
    unsigned *err;          // device error word
    uint64_t wait_limit_ns; // bound on every device-side wait
    int stall_producer;     // test hook: TMA producer issues nothing
};

// Tile sizes of the GEMM (also used by the host to build the TMA boxes).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;

// Which GEMM variant runs for an M x N output, and its grid: the 2-SM
// (cta_group::2, 256 x 256 tiles per CTA pair) kernel when M > 128 and pairs
// fit on the device, else the 1-SM 128 x 256 kernel. A's TMA box is always
// kGemmBM rows; B's box is b_box_rows rows.
struct GemmPlan {
    bool pair;
    int b_box_rows;
    int grid;
};

cudaError_t plan_gemm(int M, int N, int num_sms, GemmPlan *plan);

// tmY: bf16 [M, N] output, box {kGemmYBoxCols, kGemmYBoxRows}, 64-byte
// swizzle (used by the 2-SM kernel's epilogue; ignored in raw mode).
constexpr int kGemmYBoxCols = 32;
constexpr int kGemmYBoxRows = 32;

cudaError_t launch_gemm_i8(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmY,
                           const GemmParams &p, bool raw_i32, const GemmPlan &plan,
                           cudaStream_t stream);

// INT8 tensor-core peak probe: `mmas` back-to-back pair MMAs of the GEMM's
// shape (2 * 256 * 256 * 32 ops each) per CTA pair, on every pair of SMs the
// GEMM would use; *pairs_out receives the number of pairs launched.
cudaError_t launch_i8_mma_peak(int64_t mmas, unsigned *err, uint64_t limit_ns, int *pairs_out,
                               cudaStream_t stream);

// ---- block-scaled NVFP4 GEMM with fused epilogue (gemm_nvfp4_tcgen05.cu)

struct Nvfp4GemmParams {
    const uint8_t *sfa;     // blocked E4M3 scales of A (rows padded to 128)
    const uint8_t *sfb;     // blocked E4M3 scales of B
    const float *s_ta;      // per-tensor scales (device scalars)
    const float *s_tb;
    const uint16_t *bias;   // [N] bf16 bits or nullptr
    uint16_t *Y;            // [M, N] bf16 bits
    int M, N, K;
    unsigned *err;
    uint64_t wait_limit_ns;
    int stall_producer;     // test hook: the loads are never issued
};

constexpr int kNvfp4BM = 128;      // rows of A per tile (TMA box rows)
constexpr int kNvfp4BN = 128;      // rows of B per tile
constexpr int kNvfp4BKBytes = 128; // packed bytes of K per stage (256 values)

// The 2-SM kernel (256 x 256 tiles per CTA pair) runs when M > 128 and
// allow_pair, else the 1-SM 128 x 128 kernel. tmA / tmB: the packed codes
// (boxes of 128 bytes x 128 rows, 128-byte swizzle); tmSFA / tmSFB: the
// blocked scales as rows of 256 bytes (boxes of 256 bytes x 8 rows).
cudaError_t launch_gemm_nvfp4(const CUtensorMap &tmA, const CUtensorMap &tmB,
                              const CUtensorMap &tmSFA, const CUtensorMap &tmSFB,
                              const Nvfp4GemmParams &p, int num_sms, bool allow_pair,
                              cudaStream_t stream);

// Test hook: one thread failing an index check (class bit kChkShared), no access.
cudaError_t launch_test_checked_fire(cudaStream_t stream);

// The CK_CHECKED build's per-file check words (class bits of failed checks),
// read and cleared; always 0 in the normal build.
unsigned check_word_quant();
unsigned check_word_gemm_i8();
unsigned check_word_gemm_nvfp4();
unsigned check_word_dequant();
unsigned check_word_rmsnorm();

}  // namespace ck
