// C ABI of libck.so: host-side validation, per-device state, TMA tensor maps
// and the launches. Declarations and the contract of every entry point are in
// include/ck.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "ck.h"
#include "ck_device.cuh"
#include "internal.h"

namespace {

// Per-device error word for bounded waits that ran out (CK_ERR_DEVICE_TIMEOUT).
__device__ unsigned g_device_error;

constexpr int kMaxDevices = 64;
constexpr int64_t kBlock = 256;

struct DeviceState {
    bool ready = false;
    bool arch_ok = false;
    int num_sms = 0;
    unsigned *err = nullptr;
    CUcontext ctx = nullptr;  // the context the cached addresses belong to
    unsigned generation = 0;  // bumped whenever the state is rebuilt
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_get = nullptr;

thread_local int t_stall_next = 0;
thread_local int64_t t_stall_limit_ns = 0;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

ck_status check_k(int64_t K) {
    if (K <= 0) return CK_ERR_INVALID_VALUE;
    if (K % kBlock != 0 || K > CK_MAX_K) return CK_ERR_UNSUPPORTED_SHAPE;
    return CK_OK;
}

// The context current on this thread, created by the runtime if there is
// none yet (cudaSetDevice initialises the device's primary context).
ck_status current_context(int dev, CUcontext *ctx) {
    if (!g_ctx_get) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return CK_ERR_CUDA;
        g_ctx_get = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    }
    *ctx = nullptr;
    if (g_ctx_get(ctx) != CUDA_SUCCESS) return CK_ERR_CUDA;
    if (*ctx == nullptr) {
        if (cudaSetDevice(dev) != cudaSuccess || g_ctx_get(ctx) != CUDA_SUCCESS || !*ctx)
            return CK_ERR_CUDA;
    }
    return CK_OK;
}

// Returns the state of the current device, initialising it once per context
// (arch check, SM count, address of the error word, tensor-map encoder). A
// new context on the device (after cudaDeviceReset, or a different context
// made current) rebuilds it: the cached addresses belonged to the old one.
ck_status device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CK_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return CK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    CUcontext ctx = nullptr;
    if (current_context(dev, &ctx) != CK_OK) return CK_ERR_CUDA;
    DeviceState &st = g_dev[dev];
    if (st.ready && st.ctx != ctx) {
        st.ready = false;
        st.err = nullptr;
    }
    if (!st.ready) {
        st.ctx = ctx;
        ++st.generation;
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return CK_ERR_CUDA;
        st.arch_ok = (major == 10 && minor == 0);
        st.num_sms = sms;
        if (st.arch_ok) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return CK_ERR_CUDA;
            st.err = static_cast<unsigned *>(p);
            if (!g_encode) {
                void *fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                        cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || fn == nullptr)
                    return CK_ERR_CUDA;
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
        }
        st.ready = true;
    }
    if (!st.arch_ok) return CK_ERR_ARCH;
    *out = &st;
    return CK_OK;
}

// Row-major [rows, K] int8 matrix, box = box_rows x 128 bytes, 128-byte swizzle,
// out-of-range elements read as zero.
ck_status make_tmap_i8(CUtensorMap *tm, const void *base, int64_t rows, int64_t K, int box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(ck::kGemmBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CK_OK : CK_ERR_CUDA;
}

// Row-major [M, N] bf16 output, box = 32 columns x 32 rows, 64-byte swizzle.
ck_status make_tmap_y(CUtensorMap *tm, const void *base, int64_t M, int64_t N) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(ck::kGemmYBoxCols),
                         static_cast<cuuint32_t>(ck::kGemmYBoxRows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CK_OK : CK_ERR_CUDA;
}

// Blocked NVFP4 scales viewed as rows of 256 bytes; box = 8 rows (2 KB, four
// 512-byte scale tiles), no swizzle.
ck_status make_tmap_sf(CUtensorMap *tm, const void *base, size_t bytes) {
    cuuint64_t dims[2] = {256, static_cast<cuuint64_t>(bytes / 256)};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, 8};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CK_OK : CK_ERR_CUDA;
}

ck_status run_gemm(const int8_t *Qx, const float *s_x, const int8_t *Qw, const float *s_w,
                   const ck_bf16 *bias, ck_bf16 *Y, int32_t *acc, int64_t M, int64_t N, int64_t K,
                   DeviceState *st, cudaStream_t stream) {
    ck::GemmPlan plan{};
    if (ck::plan_gemm(static_cast<int>(M), static_cast<int>(N), st->num_sms, &plan) != cudaSuccess)
        return CK_ERR_CUDA;
    CUtensorMap tmA, tmB;
    std::memset(&tmA, 0, sizeof tmA);
    std::memset(&tmB, 0, sizeof tmB);
    ck_status s = make_tmap_i8(&tmA, Qx, M, K, ck::kGemmBM);
    if (s != CK_OK) return s;
    s = make_tmap_i8(&tmB, Qw, N, K, plan.b_box_rows);
    if (s != CK_OK) return s;
    CUtensorMap tmY;
    std::memset(&tmY, 0, sizeof tmY);
    if (Y != nullptr) {
        s = make_tmap_y(&tmY, Y, M, N);
        if (s != CK_OK) return s;
    }
    ck::GemmParams p{};
    p.s_x = s_x;
    p.s_w = s_w;
    p.bias = bias;
    p.Y = Y;
    p.acc = acc;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.err = st->err;
    p.wait_limit_ns = ck::kDefaultWaitLimitNs;
    p.stall_producer = 0;
    if (t_stall_next) {
        p.stall_producer = 1;
        if (t_stall_limit_ns > 0) p.wait_limit_ns = static_cast<uint64_t>(t_stall_limit_ns);
        t_stall_next = 0;
        t_stall_limit_ns = 0;
    }
    cudaError_t e = ck::launch_gemm_i8(tmA, tmB, tmY, p, acc != nullptr, plan, stream);
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status quant_common(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx, int8_t *Qx,
                       float *s_x, bool rotate, int act, ck_stream_t stream, int qmax = 127) {
    if (M < 0 || act < CK_ACT_NONE || act > CK_ACT_GELU_TANH) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (ldx < K && K > 0) return CK_ERR_INVALID_VALUE;
    if (M > 0 && (!X || !Qx || !s_x)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (M >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return CK_OK;
    if (!aligned16(X) || !aligned16(Qx) || !aligned4(s_x) || ldx % 8 != 0) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_quant_rows_bf16(X, M, K, ldx, rotate, act, qmax, Qx, s_x, st->err,
                                               st->num_sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status gemm_args(const int8_t *Qx, const int8_t *Qw, const void *Y, int64_t M, int64_t N,
                    int64_t K) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (M > 0 && N > 0 && (!Qx || !Qw || !Y)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    return CK_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

ck_status weight_common(const float *W, int64_t N, int64_t K, void *Qw, float *s_w, bool int4,
                        ck_stream_t stream) {
    if (N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (N > 0 && (!W || !Qw || !s_w)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return CK_OK;
    if (!aligned16(W) || !aligned16(Qw) || !aligned16(s_w)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_quant_rows_f32(W, N, K, int4, static_cast<int8_t *>(Qw), s_w,
                                              reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

// Streams and events of ck_int8_linear_host, created once per device
// context (a new context, e.g. after cudaDeviceReset, gets new ones; the old
// handles died with their context).
struct HostPipe {
    bool ready = false;
    unsigned generation = 0;
    cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
    cudaEvent_t entry = nullptr, done = nullptr;
    cudaEvent_t in_done[2] = {}, x_free[2] = {}, y_ready[2] = {}, y_free[2] = {};
    std::mutex m;
};
HostPipe g_pipe[kMaxDevices];

ck_status host_pipe(const DeviceState *st, HostPipe **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    HostPipe &hp = g_pipe[dev];
    if (hp.ready && hp.generation != st->generation) hp.ready = false;
    if (!hp.ready) {
        hp.generation = st->generation;
        const unsigned ef = cudaEventDisableTiming;
        bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&hp.entry, ef) == cudaSuccess &&
                  cudaEventCreateWithFlags(&hp.done, ef) == cudaSuccess;
        for (int i = 0; ok && i < 2; ++i)
            ok = cudaEventCreateWithFlags(&hp.in_done[i], ef) == cudaSuccess &&
                 cudaEventCreateWithFlags(&hp.x_free[i], ef) == cudaSuccess &&
                 cudaEventCreateWithFlags(&hp.y_ready[i], ef) == cudaSuccess &&
                 cudaEventCreateWithFlags(&hp.y_free[i], ef) == cudaSuccess;
        if (!ok) return CK_ERR_CUDA;
        hp.ready = true;
    }
    *out = &hp;
    return CK_OK;
}

}  // namespace

namespace ck {

ck_status check_linear_args(const void *X, int64_t ldx, const void *Qw, const void *s_w,
                            const void *bias, const void *Y, int64_t M, int64_t N, int64_t K,
                            const void *workspace, bool with_workspace) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && N > 0 && (!X || !Qw || !s_w || !Y || (with_workspace && !workspace)))
        return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(Qw) || !aligned16(s_w) || !aligned16(Y) ||
        (bias && !aligned16(bias)) ||
        (with_workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return CK_ERR_MISALIGNED;
    return CK_OK;
}

ck_status check_current_device(unsigned *generation) {
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    *generation = st->generation;
    return CK_OK;
}

}  // namespace ck

extern "C" {

ck_status ck_rotate_quant_weight(const float *W, int64_t N, int64_t K, int8_t *Qw, float *s_w,
                                 ck_stream_t stream) {
    return weight_common(W, N, K, Qw, s_w, false, stream);
}

ck_status ck_rotate_quant_weight_int4(const float *W, int64_t N, int64_t K, uint8_t *Qw4,
                                      float *s_w, ck_stream_t stream) {
    return weight_common(W, N, K, Qw4, s_w, true, stream);
}

ck_status ck_unpack_int4(const uint8_t *Qw4, int64_t N, int64_t K, int8_t *Qw, ck_stream_t stream) {
    if (N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (N > 0 && (!Qw4 || !Qw)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return CK_OK;
    if (!aligned16(Qw4) || !aligned16(Qw)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_unpack_int4(Qw4, N, K, Qw, st->num_sms,
                                           reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_quantize_rotate_rowwise_int4(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                          int8_t *Qx, float *s_x, ck_stream_t stream) {
    return quant_common(X, M, K, ldx, Qx, s_x, true, CK_ACT_NONE, stream, 7);
}

ck_status ck_dequantize_int8(const int8_t *Q, const float *s, int64_t rows, int64_t K,
                             int per_row, int out_bf16, void *Y, ck_stream_t stream) {
    if (rows < 0 || K <= 0) return CK_ERR_INVALID_VALUE;
    if (rows > 0 && (!Q || !s || !Y)) return CK_ERR_INVALID_VALUE;
    if (K % 16 != 0) return CK_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0) return CK_OK;
    if (!aligned16(Q) || !aligned4(s) || !aligned16(Y)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    ck_status st_ = device_state(&st);
    if (st_ != CK_OK) return st_;
    cudaError_t e = ck::launch_dequantize_int8(Q, s, rows, K, per_row != 0, out_bf16 != 0, Y,
                                               st->num_sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_quantize_int8_tensorwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                      int8_t *Q, float *s, ck_stream_t stream) {
    if (M < 0 || K <= 0 || ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && (!X || !Q || !s)) return CK_ERR_INVALID_VALUE;
    if (K % 8 != 0) return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return CK_OK;
    if (!aligned16(X) || !aligned16(Q) || !aligned4(s) || ldx % 8 != 0) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    ck_status st_ = device_state(&st);
    if (st_ != CK_OK) return st_;
    cudaError_t e = ck::launch_quantize_int8_tensorwise(X, M, K, ldx, Q, s, st->num_sms,
                                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

size_t ck_convrot_w4a4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return round256(size_t(M) * size_t(K)) + round256(size_t(M) * 4) +
           round256(size_t(N) * size_t(K));
}

ck_status ck_quantize_rotate_rowwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                     int8_t *Qx, float *s_x, ck_stream_t stream) {
    return quant_common(X, M, K, ldx, Qx, s_x, true, CK_ACT_NONE, stream);
}

ck_status ck_quantize_rotate_rowwise_act(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                         int act, int8_t *Qx, float *s_x, ck_stream_t stream) {
    return quant_common(X, M, K, ldx, Qx, s_x, true, act, stream);
}

ck_status ck_quantize_int8_rowwise(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                   int8_t *Qx, float *s_x, ck_stream_t stream) {
    return quant_common(X, M, K, ldx, Qx, s_x, false, CK_ACT_NONE, stream);
}

ck_status ck_test_quantize_rowwise_norotate(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                            int8_t *Qx, float *s_x, ck_stream_t stream) {
    return quant_common(X, M, K, ldx, Qx, s_x, false, CK_ACT_NONE, stream);
}

size_t ck_int8_linear_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return round256(size_t(M) * size_t(K)) + round256(size_t(M) * 4);
}

ck_status ck_int8_linear_act(const ck_bf16 *X, int64_t ldx, int act, const int8_t *Qw,
                             const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                             int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                             ck_stream_t stream) {
    if (act < CK_ACT_NONE || act > CK_ACT_GELU_TANH) return CK_ERR_INVALID_VALUE;
    ck_status s = ck::check_linear_args(X, ldx, Qw, s_w, bias, Y, M, N, K, workspace, true);
    if (s != CK_OK || M == 0 || N == 0) return s;
    if (workspace_bytes < ck_int8_linear_workspace_bytes(M, K)) return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    int8_t *Qx = static_cast<int8_t *>(workspace);
    float *s_x = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                           round256(size_t(M) * size_t(K)));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e =
        ck::launch_quant_rows_bf16(X, M, K, ldx, true, act, 127, Qx, s_x, st->err, st->num_sms, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st, cs);
}

ck_status ck_int8_linear(const ck_bf16 *X, int64_t ldx, const int8_t *Qw, const float *s_w,
                         const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                         void *workspace, size_t workspace_bytes, ck_stream_t stream) {
    return ck_int8_linear_act(X, ldx, CK_ACT_NONE, Qw, s_w, bias, Y, M, N, K, workspace,
                              workspace_bytes, stream);
}

// Arguments of the input RMSNorm (ck_rmsnorm_residual's rules), M > 0.
static ck_status check_norm(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual, int64_t ldr,
                            const ck_bf16 *residual_out, int64_t ldo, const ck_bf16 *g, float eps,
                            int64_t K) {
    if (!X || ldx < K || (residual && ldr < K) || (residual_out && ldo < K) ||
        !(eps > 0.0f) || !(eps <= 3.4e38f))
        return CK_ERR_INVALID_VALUE;
    if (!aligned16(X) || ldx % 8 != 0 || (residual && (!aligned16(residual) || ldr % 8 != 0)) ||
        (residual_out && (!aligned16(residual_out) || ldo % 8 != 0)) || (g && !aligned16(g)))
        return CK_ERR_MISALIGNED;
    return CK_OK;
}

ck_status ck_rmsnorm_residual(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual, int64_t ldr,
                              ck_bf16 *residual_out, int64_t ldo, const ck_bf16 *g, float eps,
                              int64_t M, int64_t K, ck_bf16 *Y, ck_stream_t stream) {
    if (M < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s != CK_OK) return s;
    if (M == 0) return CK_OK;
    if (!Y) return CK_ERR_INVALID_VALUE;
    s = check_norm(X, ldx, residual, ldr, residual_out, ldo, g, eps, K);
    if (s != CK_OK) return s;
    if (!aligned16(Y)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_rmsnorm_rows(X, ldx, residual, ldr, residual_out, ldo, g, eps, M, K,
                                            Y, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_quantize_rotate_rowwise_norm(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual,
                                          int64_t ldr, ck_bf16 *residual_out, int64_t ldo,
                                          const ck_bf16 *g, float eps, int64_t M, int64_t K,
                                          int8_t *Qx, float *s_x, ck_stream_t stream) {
    if (M < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (M > 0 && (!X || !Qx || !s_x)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (K > CK_NORM_FUSED_MAX_K || M >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return CK_OK;
    s = check_norm(X, ldx, residual, ldr, residual_out, ldo, g, eps, K);
    if (s != CK_OK) return s;
    if (!aligned16(Qx) || !aligned4(s_x)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    bool launched = false;
    cudaError_t e = ck::launch_quant_norm_bf16(X, M, K, ldx, residual, ldr, residual_out, ldo, g,
                                               eps, Qx, s_x, st->err, st->num_sms,
                                               reinterpret_cast<cudaStream_t>(stream), &launched);
    return (e == cudaSuccess && launched) ? CK_OK : CK_ERR_CUDA;
}

size_t ck_int8_linear_norm_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    if (K <= CK_NORM_FUSED_MAX_K) return ck_int8_linear_workspace_bytes(M, K);
    return round256(size_t(M) * size_t(K) * 2) + ck_int8_linear_workspace_bytes(M, K);
}

ck_status ck_int8_linear_norm(const ck_bf16 *X, int64_t ldx, const ck_bf16 *residual,
                              int64_t ldr, ck_bf16 *residual_out, int64_t ldo, const ck_bf16 *g,
                              float eps, const int8_t *Qw, const float *s_w, const ck_bf16 *bias,
                              ck_bf16 *Y, int64_t M, int64_t N, int64_t K, void *workspace,
                              size_t workspace_bytes, ck_stream_t stream) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (M > 0 && N > 0 && (!X || !Qw || !s_w || !Y || !workspace)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    s = check_norm(X, ldx, residual, ldr, residual_out, ldo, g, eps, K);
    if (s != CK_OK) return s;
    if (!aligned16(Qw) || !aligned16(s_w) || !aligned16(Y) || (bias && !aligned16(bias)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CK_ERR_MISALIGNED;
    if (workspace_bytes < ck_int8_linear_norm_workspace_bytes(M, K)) return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (K <= CK_NORM_FUSED_MAX_K) {
        // the normalisation inside the quantiser's staged load
        int8_t *Qx = reinterpret_cast<int8_t *>(base);
        float *s_x = reinterpret_cast<float *>(base + round256(size_t(M) * size_t(K)));
        bool launched = false;
        cudaError_t e = ck::launch_quant_norm_bf16(X, M, K, ldx, residual, ldr, residual_out, ldo,
                                                   g, eps, Qx, s_x, st->err, st->num_sms, cs,
                                                   &launched);
        if (e != cudaSuccess || !launched) return CK_ERR_CUDA;
        return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st, cs);
    }
    ck_bf16 *Xn = reinterpret_cast<ck_bf16 *>(base);
    int8_t *Qx = reinterpret_cast<int8_t *>(base + round256(size_t(M) * size_t(K) * 2));
    float *s_x = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(Qx) +
                                           round256(size_t(M) * size_t(K)));
    cudaError_t e = ck::launch_rmsnorm_rows(X, ldx, residual, ldr, residual_out, ldo, g, eps, M, K,
                                            Xn, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    e = ck::launch_quant_rows_bf16(Xn, M, K, K, true, CK_ACT_NONE, 127, Qx, s_x, st->err,
                                   st->num_sms, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st, cs);
}

size_t ck_int8_linear_host_workspace_bytes(int64_t chunk_rows, int64_t N, int64_t K) {
    if (chunk_rows <= 0 || N <= 0 || K <= 0) return 0;
    const size_t r = size_t(chunk_rows);
    return 2 * round256(r * size_t(K) * 2) + 2 * round256(r * size_t(N) * 2) +
           ck_int8_linear_workspace_bytes(chunk_rows, K);
}

ck_status ck_int8_linear_host(const ck_bf16 *X_host, int64_t ldx, int act, const int8_t *Qw,
                              const float *s_w, const ck_bf16 *bias, ck_bf16 *Y_host, int64_t M,
                              int64_t N, int64_t K, int64_t chunk_rows, void *workspace,
                              size_t workspace_bytes, ck_stream_t stream) {
    if (M < 0 || N < 0 || chunk_rows <= 0 || act < CK_ACT_NONE || act > CK_ACT_GELU_TANH)
        return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && N > 0 && (!X_host || !Qw || !s_w || !Y_host || !workspace))
        return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) ||
        chunk_rows >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(Qw) || !aligned16(s_w) || (bias && !aligned16(bias)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CK_ERR_MISALIGNED;
    if (workspace_bytes < ck_int8_linear_host_workspace_bytes(chunk_rows, N, K))
        return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    HostPipe *hp = nullptr;
    s = host_pipe(st, &hp);
    if (s != CK_OK) return s;
    std::lock_guard<std::mutex> lock(hp->m);

    const size_t r = size_t(chunk_rows);
    uint8_t *base = static_cast<uint8_t *>(workspace);
    const size_t xb_bytes = round256(r * size_t(K) * 2), yb_bytes = round256(r * size_t(N) * 2);
    ck_bf16 *xb[2] = {reinterpret_cast<ck_bf16 *>(base),
                      reinterpret_cast<ck_bf16 *>(base + xb_bytes)};
    ck_bf16 *yb[2] = {reinterpret_cast<ck_bf16 *>(base + 2 * xb_bytes),
                      reinterpret_cast<ck_bf16 *>(base + 2 * xb_bytes + yb_bytes)};
    int8_t *Qx = reinterpret_cast<int8_t *>(base + 2 * xb_bytes + 2 * yb_bytes);
    float *s_x = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(Qx) +
                                           round256(r * size_t(K)));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    // start after the caller's queued work and after the previous call
    if (cudaEventRecord(hp->entry, cs) != cudaSuccess) return CK_ERR_CUDA;
    for (cudaStream_t q : {hp->in, hp->comp, hp->out})
        if (cudaStreamWaitEvent(q, hp->entry, 0) != cudaSuccess ||
            cudaStreamWaitEvent(q, hp->done, 0) != cudaSuccess)
            return CK_ERR_CUDA;
    const int64_t nchunks = (M + chunk_rows - 1) / chunk_rows;
    for (int64_t c = 0; c < nchunks; ++c) {
        const int b = int(c & 1);
        const int64_t r0 = c * chunk_rows;
        const int64_t rows = M - r0 < chunk_rows ? M - r0 : chunk_rows;
        // copy in (buffer b was last read by the quantiser of chunk c - 2)
        if (c >= 2 && cudaStreamWaitEvent(hp->in, hp->x_free[b], 0) != cudaSuccess)
            return CK_ERR_CUDA;
        if (cudaMemcpy2DAsync(xb[b], size_t(K) * 2, X_host + r0 * ldx, size_t(ldx) * 2,
                              size_t(K) * 2, size_t(rows), cudaMemcpyHostToDevice,
                              hp->in) != cudaSuccess ||
            cudaEventRecord(hp->in_done[b], hp->in) != cudaSuccess)
            return CK_ERR_CUDA;
        // quantise + GEMM (output buffer b was last read by the copy out of chunk c - 2)
        if (cudaStreamWaitEvent(hp->comp, hp->in_done[b], 0) != cudaSuccess ||
            (c >= 2 && cudaStreamWaitEvent(hp->comp, hp->y_free[b], 0) != cudaSuccess))
            return CK_ERR_CUDA;
        if (ck::launch_quant_rows_bf16(xb[b], rows, K, K, true, act, 127, Qx, s_x, st->err,
                                       st->num_sms, hp->comp) != cudaSuccess ||
            cudaEventRecord(hp->x_free[b], hp->comp) != cudaSuccess)
            return CK_ERR_CUDA;
        s = run_gemm(Qx, s_x, Qw, s_w, bias, yb[b], nullptr, rows, N, K, st, hp->comp);
        if (s != CK_OK) return s;
        if (cudaEventRecord(hp->y_ready[b], hp->comp) != cudaSuccess) return CK_ERR_CUDA;
        // copy out
        if (cudaStreamWaitEvent(hp->out, hp->y_ready[b], 0) != cudaSuccess ||
            cudaMemcpyAsync(Y_host + r0 * N, yb[b], size_t(rows) * size_t(N) * 2,
                            cudaMemcpyDeviceToHost, hp->out) != cudaSuccess ||
            cudaEventRecord(hp->y_free[b], hp->out) != cudaSuccess)
            return CK_ERR_CUDA;
    }
    // the copy-out stream's last work follows every kernel and copy above
    if (cudaStreamWaitEvent(hp->out, hp->x_free[(nchunks - 1) & 1], 0) != cudaSuccess ||
        cudaEventRecord(hp->done, hp->out) != cudaSuccess ||
        cudaStreamWaitEvent(cs, hp->done, 0) != cudaSuccess)
        return CK_ERR_CUDA;
    return CK_OK;
}

// ---------------------------------------------------------------- NVFP4

size_t ck_nvfp4_scale_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return size_t((rows + 127) / 128) * 128 * size_t(K / 16);
}

namespace {
constexpr int64_t kNvfp4MaxK = 32768;

ck_status nvfp4_check_k(int64_t K) {
    if (K <= 0) return CK_ERR_INVALID_VALUE;
    if (K % kBlock != 0 || K > kNvfp4MaxK) return CK_ERR_UNSUPPORTED_SHAPE;
    return CK_OK;
}
}  // namespace

ck_status ck_quantize_rotate_nvfp4(const ck_bf16 *X, int64_t M, int64_t K, int64_t ldx,
                                   uint8_t *Q, uint8_t *S, float *s_t, ck_stream_t stream) {
    if (M < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = nvfp4_check_k(K);
    if (s == CK_ERR_INVALID_VALUE || ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && (!X || !Q || !S || !s_t)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (M >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return CK_OK;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(Q) || !aligned16(S) || !aligned4(s_t))
        return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return ck::launch_quant_nvfp4_bf16(X, M, K, ldx, Q, S, ck_nvfp4_scale_bytes(M, K), s_t,
                                       st->err, st->num_sms,
                                       reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CK_OK
               : CK_ERR_CUDA;
}

ck_status ck_rotate_quant_weight_nvfp4(const float *W, int64_t N, int64_t K, uint8_t *Qw,
                                       uint8_t *Sw, float *s_tw, ck_stream_t stream) {
    if (N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = nvfp4_check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (N > 0 && (!W || !Qw || !Sw || !s_tw)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N >= (int64_t(1) << 31)) return CK_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return CK_OK;
    if (!aligned16(W) || !aligned16(Qw) || !aligned16(Sw) || !aligned4(s_tw))
        return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return ck::launch_quant_nvfp4_f32(W, N, K, Qw, Sw, ck_nvfp4_scale_bytes(N, K), s_tw,
                                      reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CK_OK
               : CK_ERR_CUDA;
}

ck_status ck_dequantize_nvfp4(const uint8_t *Q, const uint8_t *S, const float *s_t, int64_t rows,
                              int64_t K, int hi_first, float *out, ck_stream_t stream) {
    if (rows < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = nvfp4_check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (rows > 0 && (!Q || !S || !s_t || !out)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (rows == 0) return CK_OK;
    if (!aligned16(Q) || !aligned16(out) || !aligned4(s_t)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return ck::launch_dequant_nvfp4(Q, S, s_t, rows, K, hi_first != 0, out, st->num_sms,
                                    reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CK_OK
               : CK_ERR_CUDA;
}

namespace {
ck_status nvfp4_gemm_checked(const uint8_t *Qa, const uint8_t *Sa, const float *s_ta,
                             const uint8_t *Qw, const uint8_t *Sw, const float *s_tw,
                             const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                             DeviceState *st, cudaStream_t stream) {
    CUtensorMap tmA, tmB, tmSFA, tmSFB;
    std::memset(&tmA, 0, sizeof tmA);
    std::memset(&tmB, 0, sizeof tmB);
    std::memset(&tmSFA, 0, sizeof tmSFA);
    std::memset(&tmSFB, 0, sizeof tmSFB);
    ck_status s = make_tmap_i8(&tmA, Qa, M, K / 2, ck::kNvfp4BM);
    if (s != CK_OK) return s;
    s = make_tmap_i8(&tmB, Qw, N, K / 2, ck::kNvfp4BN);
    if (s != CK_OK) return s;
    s = make_tmap_sf(&tmSFA, Sa, ck_nvfp4_scale_bytes(M, K));
    if (s != CK_OK) return s;
    s = make_tmap_sf(&tmSFB, Sw, ck_nvfp4_scale_bytes(N, K));
    if (s != CK_OK) return s;
    ck::Nvfp4GemmParams p{};
    p.sfa = Sa;
    p.sfb = Sw;
    p.s_ta = s_ta;
    p.s_tb = s_tw;
    p.bias = bias;
    p.Y = Y;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.err = st->err;
    p.wait_limit_ns = ck::kDefaultWaitLimitNs;
    p.stall_producer = 0;
    if (t_stall_next) {
        p.stall_producer = 1;
        if (t_stall_limit_ns > 0) p.wait_limit_ns = static_cast<uint64_t>(t_stall_limit_ns);
        t_stall_next = 0;
        t_stall_limit_ns = 0;
    }
    return ck::launch_gemm_nvfp4(tmA, tmB, tmSFA, tmSFB, p, st->num_sms, true, stream) ==
                   cudaSuccess
               ? CK_OK
               : CK_ERR_CUDA;
}
}  // namespace

ck_status ck_nvfp4_gemm(const uint8_t *Qa, const uint8_t *Sa, const float *s_ta,
                        const uint8_t *Qw, const uint8_t *Sw, const float *s_tw,
                        const ck_bf16 *bias, ck_bf16 *Y, int64_t M, int64_t N, int64_t K,
                        ck_stream_t stream) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = nvfp4_check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (M > 0 && N > 0 && (!Qa || !Sa || !s_ta || !Qw || !Sw || !s_tw || !Y))
        return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(Qa) || !aligned16(Sa) || !aligned16(Qw) || !aligned16(Sw) || !aligned4(s_ta) ||
        !aligned4(s_tw) || !aligned16(Y) || (bias && !aligned16(bias)))
        return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return nvfp4_gemm_checked(Qa, Sa, s_ta, Qw, Sw, s_tw, bias, Y, M, N, K, st,
                              reinterpret_cast<cudaStream_t>(stream));
}

size_t ck_convrot_nvfp4_linear_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return round256(size_t(M) * size_t(K / 2)) + round256(ck_nvfp4_scale_bytes(M, K)) + 256;
}

ck_status ck_convrot_nvfp4_linear(const ck_bf16 *X, int64_t ldx, const uint8_t *Qw,
                                  const uint8_t *Sw, const float *s_tw, const ck_bf16 *bias,
                                  ck_bf16 *Y, int64_t M, int64_t N, int64_t K, void *workspace,
                                  size_t workspace_bytes, ck_stream_t stream) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = nvfp4_check_k(K);
    if (s == CK_ERR_INVALID_VALUE || ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && N > 0 && (!X || !Qw || !Sw || !s_tw || !Y || !workspace))
        return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(Qw) || !aligned16(Sw) || !aligned4(s_tw) ||
        !aligned16(Y) || (bias && !aligned16(bias)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CK_ERR_MISALIGNED;
    if (workspace_bytes < ck_convrot_nvfp4_linear_workspace_bytes(M, K)) return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    uint8_t *Qa = base;
    uint8_t *Sa = base + round256(size_t(M) * size_t(K / 2));
    float *s_ta = reinterpret_cast<float *>(Sa + round256(ck_nvfp4_scale_bytes(M, K)));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (ck::launch_quant_nvfp4_bf16(X, M, K, ldx, Qa, Sa, ck_nvfp4_scale_bytes(M, K), s_ta,
                                    st->err, st->num_sms, cs) != cudaSuccess)
        return CK_ERR_CUDA;
    return nvfp4_gemm_checked(Qa, Sa, s_ta, Qw, Sw, s_tw, bias, Y, M, N, K, st, cs);
}

ck_status ck_convrot_w4a4_linear(const ck_bf16 *X, int64_t ldx, const uint8_t *Qw4,
                                 const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                                 int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                                 ck_stream_t stream) {
    if (M < 0 || N < 0) return CK_ERR_INVALID_VALUE;
    ck_status s = check_k(K);
    if (s == CK_ERR_INVALID_VALUE) return s;
    if (ldx < K) return CK_ERR_INVALID_VALUE;
    if (M > 0 && N > 0 && (!X || !Qw4 || !s_w || !Y || !workspace)) return CK_ERR_INVALID_VALUE;
    if (s != CK_OK) return s;
    if (N % 8 != 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return CK_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(Qw4) || !aligned16(s_w) || !aligned16(Y) ||
        (bias && !aligned16(bias)) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CK_ERR_MISALIGNED;
    if (workspace_bytes < ck_convrot_w4a4_linear_workspace_bytes(M, N, K)) return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    int8_t *Qx = reinterpret_cast<int8_t *>(base);
    float *s_x = reinterpret_cast<float *>(base + round256(size_t(M) * size_t(K)));
    int8_t *Qw = reinterpret_cast<int8_t *>(base + round256(size_t(M) * size_t(K)) +
                                            round256(size_t(M) * 4));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e =
        ck::launch_quant_rows_bf16(X, M, K, ldx, true, CK_ACT_NONE, 7, Qx, s_x, st->err, st->num_sms, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    e = ck::launch_unpack_int4(Qw4, N, K, Qw, st->num_sms, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st, cs);
}

ck_status ck_convrot_w4a4_linear_unpacked(const ck_bf16 *X, int64_t ldx, const int8_t *Qw,
                                          const float *s_w, const ck_bf16 *bias, ck_bf16 *Y,
                                          int64_t M, int64_t N, int64_t K, void *workspace,
                                          size_t workspace_bytes, ck_stream_t stream) {
    ck_status s = ck::check_linear_args(X, ldx, Qw, s_w, bias, Y, M, N, K, workspace, true);
    if (s != CK_OK || M == 0 || N == 0) return s;
    if (workspace_bytes < ck_int8_linear_workspace_bytes(M, K)) return CK_ERR_WORKSPACE;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    int8_t *Qx = reinterpret_cast<int8_t *>(base);
    float *s_x = reinterpret_cast<float *>(base + round256(size_t(M) * size_t(K)));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e =
        ck::launch_quant_rows_bf16(X, M, K, ldx, true, CK_ACT_NONE, 7, Qx, s_x, st->err, st->num_sms, cs);
    if (e != cudaSuccess) return CK_ERR_CUDA;
    return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st, cs);
}

ck_status ck_int8_gemm_rowscale(const int8_t *Qx, const float *s_x, const int8_t *Qw,
                                const float *s_w, const ck_bf16 *bias, ck_bf16 *Y, int64_t M,
                                int64_t N, int64_t K, ck_stream_t stream) {
    ck_status s = gemm_args(Qx, Qw, Y, M, N, K);
    if (s != CK_OK) return s;
    if (M > 0 && N > 0 && (!s_x || !s_w)) return CK_ERR_INVALID_VALUE;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(Qx) || !aligned4(s_x) || !aligned16(Qw) || !aligned16(s_w) || !aligned16(Y) ||
        (bias && !aligned16(bias)))
        return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return run_gemm(Qx, s_x, Qw, s_w, bias, Y, nullptr, M, N, K, st,
                    reinterpret_cast<cudaStream_t>(stream));
}

ck_status ck_test_int8_gemm_i32(const int8_t *Qx, const int8_t *Qw, int32_t *acc, int64_t M,
                                int64_t N, int64_t K, ck_stream_t stream) {
    ck_status s = gemm_args(Qx, Qw, acc, M, N, K);
    if (s != CK_OK) return s;
    if (M == 0 || N == 0) return CK_OK;
    if (!aligned16(Qx) || !aligned16(Qw) || !aligned16(acc)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    s = device_state(&st);
    if (s != CK_OK) return s;
    return run_gemm(Qx, nullptr, Qw, nullptr, nullptr, nullptr, acc, M, N, K, st,
                    reinterpret_cast<cudaStream_t>(stream));
}

ck_status ck_test_input_act(const ck_bf16 *X, int64_t n, int act, ck_bf16 *Y, ck_stream_t stream) {
    if (n < 0 || act < CK_ACT_NONE || act > CK_ACT_GELU_TANH) return CK_ERR_INVALID_VALUE;
    if (n > 0 && (!X || !Y)) return CK_ERR_INVALID_VALUE;
    if (n % 256 != 0) return CK_ERR_UNSUPPORTED_SHAPE;
    if (n == 0) return CK_OK;
    if (!aligned16(X) || !aligned16(Y)) return CK_ERR_MISALIGNED;
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_test_input_act(X, n, act, Y, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_test_row_quant_params(const float *amax, int64_t n, int q, float *div, float *rc,
                                   ck_stream_t stream) {
    if (n < 0 || (q != 127 && q != 7)) return CK_ERR_INVALID_VALUE;
    if (n > 0 && (!amax || !div || !rc)) return CK_ERR_INVALID_VALUE;
    if (n == 0) return CK_OK;
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_test_row_quant_params(amax, n, q, div, rc,
                                                     reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_test_i8_mma_peak(int64_t mmas_per_pair, int *pairs, ck_stream_t stream) {
    if (mmas_per_pair <= 0 || !pairs) return CK_ERR_INVALID_VALUE;
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    cudaError_t e = ck::launch_i8_mma_peak(mmas_per_pair, st->err, ck::kDefaultWaitLimitNs, pairs,
                                           reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status ck_test_checked_fire(ck_stream_t stream) {
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    return ck::launch_test_checked_fire(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CK_OK
               : CK_ERR_CUDA;
}

const char *ck_status_string(ck_status status) {
    switch (status) {
        case CK_OK: return "CK_OK";
        case CK_ERR_INVALID_VALUE: return "CK_ERR_INVALID_VALUE: null pointer, negative size, K <= 0 or ldx < K";
        case CK_ERR_UNSUPPORTED_SHAPE: return "CK_ERR_UNSUPPORTED_SHAPE: K % 256 != 0, K > 132864, N % 8 != 0 or M/N >= 2^31";
        case CK_ERR_MISALIGNED: return "CK_ERR_MISALIGNED: pointer or row stride not 16-byte aligned";
        case CK_ERR_WORKSPACE: return "CK_ERR_WORKSPACE: workspace smaller than ck_int8_linear_workspace_bytes";
        case CK_ERR_ARCH: return "CK_ERR_ARCH: current device is not compute capability 10.0 (B200)";
        case CK_ERR_CUDA: return "CK_ERR_CUDA: a CUDA runtime call or kernel launch failed";
        case CK_ERR_DEVICE_TIMEOUT: return "CK_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    }
    return "unknown ck_status";
}

ck_status ck_get_device_error(void) {
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    if (cudaDeviceSynchronize() != cudaSuccess) return CK_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, st->err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return CK_ERR_CUDA;
    return v ? static_cast<ck_status>(v) : CK_OK;
}

int ck_is_checked_build(void) {
#ifdef CK_CHECKED
    return 1;
#else
    return 0;
#endif
}

unsigned ck_checked_violations(void) {
#ifdef CK_CHECKED
    if (cudaDeviceSynchronize() != cudaSuccess) return 0x80000000u;
    return ck::check_word_quant() | ck::check_word_gemm_i8() | ck::check_word_gemm_nvfp4() |
           ck::check_word_dequant() | ck::check_word_rmsnorm();
#else
    return 0u;
#endif
}

ck_status ck_clear_device_error(void) {
    DeviceState *st = nullptr;
    ck_status s = device_state(&st);
    if (s != CK_OK) return s;
    if (cudaDeviceSynchronize() != cudaSuccess) return CK_ERR_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpy(st->err, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
        return CK_ERR_CUDA;
    return CK_OK;
}

ck_status ck_test_inject_producer_stall(int mode, int64_t wait_limit_ns) {
    if (mode != 0 && mode != 1) return CK_ERR_INVALID_VALUE;
    if (wait_limit_ns < 0) return CK_ERR_INVALID_VALUE;
    t_stall_next = mode;
    t_stall_limit_ns = mode ? wait_limit_ns : 0;
    return CK_OK;
}

}  // extern "C"
