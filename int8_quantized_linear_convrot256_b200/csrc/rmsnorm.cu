// Input RMSNorm with a residual, before the ConvRot quantiser
// (comfy-kitchen 0.2.40, "Huawei Ascend backend": int8_linear accepts the input
// RMSNorm and residual arguments and applies them with shared helpers, apart
// from its GEMM; no formula is printed). Reading:
//   h   = bf16_rne(fl32(x + r))  (h = x without a residual); Rout = h
//   y_k = the bf16 value nearest to h_k g_k / sqrt(mean(h^2) + eps), the
//         exact real value (g_k = 1 without g)
// Evaluated in double precision: every h^2 and h g is exact in double; the
// sum of squares (each lane's share in index order, then a five-level xor
// butterfly), one division, one square root and one product per value carry
// a relative error below K 2^-53 + 2^-51, and cvt.rn.bf16.f64 rounds the
// double result once. So y is the exact value's rounding except within about
// 2^-36 (relative) of a bf16 rounding midpoint.
// Memory-bound: one warp per row, 16-byte loads and stores, two passes over
// the row (the second re-reads it from L2, or reads back Rout).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

constexpr int kNormRowsPerCta = 8;  // one warp per row

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Two doubles rounded once each to bf16 (cvt.rn.bf16.f64), packed low first.
__device__ __forceinline__ uint32_t pack_bf16x2_d(double lo, double hi) {
    const __nv_bfloat16 a = __double2bfloat16(lo), b = __double2bfloat16(hi);
    return uint32_t(*reinterpret_cast<const uint16_t *>(&a)) |
           (uint32_t(*reinterpret_cast<const uint16_t *>(&b)) << 16);
}

__device__ __forceinline__ uint4 ld16_nc(const uint16_t *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// A row's h in 16-byte pieces: from Rout when it was written, else
// recomputed. X, R and Rout go through coherent loads: Rout may alias X or R
// (each piece is read by the lane that then overwrites it).
__device__ __forceinline__ void load_h(const uint16_t *x, const uint16_t *r, const uint16_t *ro,
                                       int c, uint32_t (&h)[4]) {
    if (ro) {
        const uint4 v = *reinterpret_cast<const uint4 *>(ro + c);
        h[0] = v.x, h[1] = v.y, h[2] = v.z, h[3] = v.w;
        return;
    }
    const uint4 xv = *reinterpret_cast<const uint4 *>(x + c);
    h[0] = xv.x, h[1] = xv.y, h[2] = xv.z, h[3] = xv.w;
    if (r) {
        const uint4 rv = *reinterpret_cast<const uint4 *>(r + c);
        const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            h[q] = pack_bf16x2(__fadd_rn(bf16_lo(h[q]), bf16_lo(rw[q])),
                               __fadd_rn(bf16_hi(h[q]), bf16_hi(rw[q])));
    }
}

__global__ void __launch_bounds__(kNormRowsPerCta * 32)
rmsnorm_rows_kernel(const uint16_t *X, int64_t ldx, const uint16_t *R, int64_t ldr,
                    uint16_t *Rout, int64_t ldo, const uint16_t *__restrict__ g, float eps,
                    int64_t M, int K, uint16_t *__restrict__ Y) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = int64_t(blockIdx.x) * kNormRowsPerCta + warp;
    if (row >= M) return;  // whole warps leave together
    const int nb = K >> 8;
    const uint16_t *x = X + row * ldx;
    const uint16_t *r = R ? R + row * ldr : nullptr;
    uint16_t *ro = Rout ? Rout + row * ldo : nullptr;
    uint16_t *y = Y + row * int64_t(K);

    // pass 1: h (stored to Rout), the lane's partial sum of squares
    double p = 0.0;
    for (int i = 0; i < nb; ++i) {
        const int c = 256 * i + 8 * lane;
        uint32_t h[4];
        load_h(x, r, nullptr, c, h);
        if (ro) *reinterpret_cast<uint4 *>(ro + c) = make_uint4(h[0], h[1], h[2], h[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double lo = bf16_lo(h[q]), hi = bf16_hi(h[q]);
            p = __fma_rn(lo, lo, p);
            p = __fma_rn(hi, hi, p);
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) p = __dadd_rn(p, __shfl_xor_sync(0xFFFFFFFFu, p, m));
    const double inv = 1.0 / sqrt(p / double(K) + double(eps));

    // pass 2: y
    for (int i = 0; i < nb; ++i) {
        const int c = 256 * i + 8 * lane;
        uint32_t h[4];
        load_h(x, r, ro, c, h);
        uint32_t gw[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // bf16 1.0
        if (g) {
            const uint4 gv = ld16_nc(g + c);
            gw[0] = gv.x, gw[1] = gv.y, gw[2] = gv.z, gw[3] = gv.w;
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // h g is exact in double; one rounding for the product with inv
            const double lo = __dmul_rn(double(bf16_lo(h[q])) * double(bf16_lo(gw[q])), inv);
            const double hi = __dmul_rn(double(bf16_hi(h[q])) * double(bf16_hi(gw[q])), inv);
            o[q] = pack_bf16x2_d(lo, hi);
        }
        *reinterpret_cast<uint4 *>(y + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_rmsnorm_rows(const uint16_t *X, int64_t ldx, const uint16_t *R, int64_t ldr,
                                uint16_t *Rout, int64_t ldo, const uint16_t *g, float eps,
                                int64_t M, int64_t K, uint16_t *Y, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    const int64_t grid = (M + kNormRowsPerCta - 1) / kNormRowsPerCta;
    rmsnorm_rows_kernel<<<static_cast<unsigned>(grid), kNormRowsPerCta * 32, 0, stream>>>(
        X, ldx, R, ldr, Rout, ldo, g, eps, M, static_cast<int>(K), Y);
    return cudaGetLastError();
}

CK_DEFINE_CHECK_READER(check_word_rmsnorm)

}  // namespace ck
