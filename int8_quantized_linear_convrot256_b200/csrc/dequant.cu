// dequantize_int8_simple(_dtype) and quantize_int8_tensorwise (comfy-kitchen
// 0.2.40, "Huawei Ascend backend"). Memory-bound helpers around the linear:
//   dequantize: y = float(q) * s (one fp32 rounding; s per tensor or per
//               row), stored as fp32 or rounded to bf16;
//   tensorwise: s = absmax(X) / 127 over the whole tensor, then
//               q = round-half-even(x / s) clamped to [-127, 127].
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

// 16 codes per iteration: one 16-byte load, 64 (fp32) or 32 (bf16) bytes out.
template <bool kBF16>
__global__ void dequant_kernel(const int8_t *__restrict__ Q, const float *__restrict__ S,
                               int64_t K, bool per_row, void *__restrict__ Y, int64_t n16) {
    for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < n16;
         c += int64_t(gridDim.x) * blockDim.x) {
        const int64_t e0 = c * 16;
        const float sc = per_row ? S[e0 / K] : S[0];
        const uint4 raw = __ldcs(reinterpret_cast<const uint4 *>(Q) + c);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int q = int(int8_t((w[i >> 2] >> (8 * (i & 3))) & 0xFFu));
            f[i] = __fmul_rn(__int2float_rn(q), sc);
        }
        if (kBF16) {
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
                o[i] = *reinterpret_cast<const uint32_t *>(&h);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(Y) + 2 * c;
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
            float4 *dst = reinterpret_cast<float4 *>(Y) + 4 * c;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        }
    }
}

// Pass 1: absmax of the tensor into *amax_bits (zeroed by the host first);
// non-negative floats order like their bit patterns. 8 bf16 per thread step.
__global__ void absmax_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t K, int64_t ldx,
                              unsigned *amax_bits) {
    const int64_t per_row = K / 8;
    const int64_t n8 = M * per_row;
    float m = 0.0f;
    for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < n8;
         c += int64_t(gridDim.x) * blockDim.x) {
        const int64_t row = c / per_row, col = (c - row * per_row) * 8;
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(X + row * ldx + col));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)),
                               fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// Pass 2: codes with s = fl(amax / 127), the IEEE quotient rounded half-even.
__global__ void tensorwise_codes_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t K,
                                        int64_t ldx, const unsigned *amax_bits,
                                        int8_t *__restrict__ Q) {
    const float amax = __uint_as_float(*amax_bits);
    const float s = __fdiv_rn(amax, 127.0f);
    const int64_t per_row = K / 8;
    const int64_t n8 = M * per_row;
    for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < n8;
         c += int64_t(gridDim.x) * blockDim.x) {
        const int64_t row = c / per_row, col = (c - row * per_row) * 8;
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(X + row * ldx + col));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t b[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float x = __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
            int q = 0;
            if (amax != 0.0f) {
                float r = rintf(__fdiv_rn(x, s));
                r = fminf(fmaxf(r, -127.0f), 127.0f);
                q = int(r);
            }
            b[i >> 2] |= (uint32_t(q) & 0xFFu) << (8 * (i & 3));
        }
        *reinterpret_cast<uint2 *>(Q + row * K + col) = make_uint2(b[0], b[1]);
    }
}

// Pass 3: the scale itself, written over the absmax bits.
__global__ void tensorwise_scale_kernel(unsigned *amax_bits_then_scale) {
    const float amax = __uint_as_float(*amax_bits_then_scale);
    *reinterpret_cast<float *>(amax_bits_then_scale) = __fdiv_rn(amax, 127.0f);
}

unsigned grid_for(int64_t work, int num_sms) {
    const int64_t want = (work + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    return unsigned(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_dequantize_int8(const int8_t *Q, const float *S, int64_t rows, int64_t K,
                                   bool per_row, bool out_bf16, void *Y, int num_sms,
                                   cudaStream_t stream) {
    const int64_t n16 = rows * K / 16;
    if (n16 <= 0) return cudaSuccess;
    if (out_bf16)
        dequant_kernel<true><<<grid_for(n16, num_sms), 256, 0, stream>>>(Q, S, K, per_row, Y, n16);
    else
        dequant_kernel<false><<<grid_for(n16, num_sms), 256, 0, stream>>>(Q, S, K, per_row, Y, n16);
    return cudaGetLastError();
}

cudaError_t launch_quantize_int8_tensorwise(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                            int8_t *Q, float *s, int num_sms,
                                            cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(s, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    unsigned *bits = reinterpret_cast<unsigned *>(s);
    const unsigned g = grid_for(M * (K / 8), num_sms);
    absmax_kernel<<<g, 256, 0, stream>>>(X, M, K, ldx, bits);
    tensorwise_codes_kernel<<<g, 256, 0, stream>>>(X, M, K, ldx, bits, Q);
    tensorwise_scale_kernel<<<1, 1, 0, stream>>>(bits);
    return cudaGetLastError();
}

CK_DEFINE_CHECK_READER(check_word_dequant)

}  // namespace ck
