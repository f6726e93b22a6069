// ck_int8_linear_noalloc: ck_int8_linear for callers that cannot allocate
// device memory.
//
// Some callers of this library are not allowed to call cudaMalloc: a plugin
// inside an inference engine that owns every byte of device memory and hands
// its plugins no workspace, code with a fixed memory budget planned at
// start-up, or code that must not risk the implicit device-wide
// synchronisation that cudaFree (and a growing allocator) can cause. For them
// the activation codes and row scales, which ck_int8_linear keeps in a
// caller-supplied workspace, live here in one file-scope device array of fixed
// size instead. The caller still passes X, the weights and Y.
//
// Costs and rules:
//  * Every GPU that loads this part of the library holds the array
//    (CK_NOALLOC_SCRATCH_BYTES) until the process exits.
//  * All calls on a device share the one array, and it keeps whatever the
//    last call left in it. Nothing in it has to start at zero: each call
//    rewrites every code and every row scale it later reads. Two calls whose
//    work overlaps on the GPU (different streams without ordering, or several
//    host threads) race on the array and corrupt each other's results; order
//    them, e.g. on one stream.
//  * The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current and caches it; make that
//    first call before any stream capture on the device. The lookup is done
//    again when the device's context changes (after cudaDeviceReset, or when
//    another context is made current), since the address belongs to a context.
//  * Problems whose codes and scales need more than the array holds
//    (ck_int8_linear_workspace_bytes(M, K) > CK_NOALLOC_SCRATCH_BYTES) are
//    rejected with CK_ERR_WORKSPACE before anything is launched.
//  * No cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ck.h"
#include "internal.h"

namespace {

// In host code this name is a host-side stand-in for the array, not its
// device address: never hand it to a kernel. Host code uses the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchAddr {
    void *ptr = nullptr;
    unsigned generation = 0;  // device-state generation the address was taken in
};
ScratchAddr g_scratch[kMaxDevices];

// Device address of the array on the current device (a B200: the caller has
// checked), looked up once per device context with that device current.
ck_status scratch_address(unsigned generation, void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchAddr &a = g_scratch[dev];
    if (a.ptr == nullptr || a.generation != generation) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();  // leave no sticky-looking error for the caller's next check
            return CK_ERR_CUDA;
        }
        a.ptr = p;
        a.generation = generation;
    }
    *out = a.ptr;
    return CK_OK;
}

}  // namespace

extern "C" ck_status ck_int8_linear_noalloc(const ck_bf16 *X, int64_t ldx, const int8_t *Qw,
                                            const float *s_w, const ck_bf16 *bias, ck_bf16 *Y,
                                            int64_t M, int64_t N, int64_t K, ck_stream_t stream) {
    // the checks of ck_int8_linear, in its order, then the array's size
    ck_status s = ck::check_linear_args(X, ldx, Qw, s_w, bias, Y, M, N, K, nullptr, false);
    if (s != CK_OK || M == 0 || N == 0) return s;
    if (ck_int8_linear_workspace_bytes(M, K) > CK_NOALLOC_SCRATCH_BYTES) return CK_ERR_WORKSPACE;
    unsigned generation = 0;
    s = ck::check_current_device(&generation);  // CK_ERR_ARCH before any symbol lookup
    if (s != CK_OK) return s;
    void *scratch = nullptr;
    s = scratch_address(generation, &scratch);
    if (s != CK_OK) return s;
    return ck_int8_linear(X, ldx, Qw, s_w, bias, Y, M, N, K, scratch, CK_NOALLOC_SCRATCH_BYTES,
                          stream);
}
