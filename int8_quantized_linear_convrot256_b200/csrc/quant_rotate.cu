// Fused ConvRot256 rotation + dynamic per-row INT8 quantisation for sm_100a.
//
// What is computed (comfy-kitchen 0.2.40, "Huawei Ascend backend" and "HIP
// backend": quantize_and_rotate_rowwise / quantize_int8_rowwise; sglang PR
// "Tune Kitchen INT8 row splitting for SM120", Accuracy Test: ConvRot256 and
// FP32 row scales; ComfyUI-AppleSilicon-FP8 README row 17: rotate online,
// then quantise per row):
//   every 256-block of a row -> 8 fp32 butterfly stages h = 1, 2, ..., 128,
//   then * 1/16; s = absmax(row) / 127; q = round-half-even(y / s) clamped to
//   [-127, 127]; a zero row gives s = 0 and q = 0.
//
// Design (HBM-bound: 2 B read + 1 B written per element, 4 B per row):
//  * One quad (4 consecutive lanes) owns one 256-block; each lane keeps 64
//    values in registers. Element e of the block sits in lane (e >> 3) & 3 of
//    the quad, register ((e >> 5) << 3) | (e & 7). Lane t therefore loads 8
//    contiguous values at e = 8t + 32j (j = 0..7): 16-byte loads, and each
//    quad reads 64 contiguous bytes per load instruction.
//  * Butterfly stages on element bits 0, 1, 2, 5, 6, 7 pair registers of the
//    same lane; stages on bits 3 and 4 (h = 8, 16) pair lanes t and t ^ 1,
//    t ^ 2 of the quad through one shuffle per value. Stages run in the order
//    h = 1, 2, 4, ..., 128 and each is one IEEE add or subtract per value,
//    so the result is bit-identical to the sequential definition.
//  * The whole row stays in registers of one CTA (rows_per_cta rows of
//    K/256 quads each); the row absmax is reduced through a shared-memory
//    atomicMax on the fp32 bit pattern (non-negative floats order like their
//    bits), so X is read from HBM exactly once. K > 32768 takes a two-pass
//    variant that re-reads the (L2-resident) row instead.
//  * Division: q needs round-half-even of the IEEE quotient fl(y / s). With
//    r = fl(1/s) and t = fl(y * r), |t - y/s| < 2^-16 and |fl(y/s) - y/s| <=
//    2^-17 when |y/s| < 128 (always: |y| <= absmax and s = fl(absmax/127)).
//    So if t is farther than 2^-14 from every half-integer, rint(t) equals
//    rint(fl(y / s)). Values closer than that (about 1 in 8000) and rows with
//    s < 2^-120 take the exact path rint(__fdiv_rn(y, s)). rint(t) itself uses
//    t + 1.5 * 2^23, whose low byte is then the two's-complement code; no
//    clamp is needed on the fast path because |y / s| <= 127 * (1 + 2^-23).
//  * No FMA contraction: every operation is an explicit _rn intrinsic.
#include <cuda_runtime.h>

#include <cstdint>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

constexpr int kBlock = 256;
constexpr int kVals = 64;  // values of a block held by one lane
constexpr int kMaxThreads = 512;
constexpr int kMaxRowsPerCta = kMaxThreads / 4;
constexpr int kTwoPassQuads = 128;  // quads per row in the two-pass variant
constexpr float kMagic = 12582912.0f;              // 1.5 * 2^23
constexpr float kNearHalf = 0.49993896484375f;     // 0.5 - 2^-14
constexpr float kMinFastScale = 7.52316384526264e-37f;  // 2^-120

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}

// Load lane t's 64 values of one block: base points at element 8t of the block.
__device__ __forceinline__ void load_block(const uint16_t *base, float (&v)[kVals]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 u = ld_stream_v4(base + 32 * j);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[8 * j + 2 * i] = __uint_as_float(w[i] << 16);
            v[8 * j + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

__device__ __forceinline__ void load_block(const float *base, float (&v)[kVals]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 a = __ldcs(reinterpret_cast<const float4 *>(base + 32 * j));
        const float4 b = __ldcs(reinterpret_cast<const float4 *>(base + 32 * j + 4));
        v[8 * j + 0] = a.x; v[8 * j + 1] = a.y; v[8 * j + 2] = a.z; v[8 * j + 3] = a.w;
        v[8 * j + 4] = b.x; v[8 * j + 5] = b.y; v[8 * j + 6] = b.z; v[8 * j + 7] = b.w;
    }
}

// Butterfly between registers r and r + R (R = 1, 2, 4, 8, 16, 32).
template <int R>
__device__ __forceinline__ void stage_regs(float (&v)[kVals]) {
#pragma unroll
    for (int r = 0; r < kVals; ++r) {
        if ((r & R) == 0) {
            const float a = v[r];
            const float c = v[r + R];
            v[r] = __fadd_rn(a, c);
            v[r + R] = __fsub_rn(a, c);
        }
    }
}

// Butterfly between lanes t and t ^ L of the quad (L = 1, 2). The lane with
// the bit clear holds a and computes a + c; the other holds c and computes
// a - c = fma(-1, c, a), a single rounding, the same value as the subtraction.
template <int L>
__device__ __forceinline__ void stage_lanes(float (&v)[kVals], int t) {
    const float sg = (t & L) ? -1.0f : 1.0f;
#pragma unroll
    for (int r = 0; r < kVals; ++r) {
        const float p = __shfl_xor_sync(0xFFFFFFFFu, v[r], L);
        v[r] = __fmaf_rn(sg, v[r], p);
    }
}

// ConvRot256 of the block spread over the quad: stages h = 1..128 in order.
__device__ __forceinline__ void rotate_block(float (&v)[kVals], int t) {
    stage_regs<1>(v);    // h = 1
    stage_regs<2>(v);    // h = 2
    stage_regs<4>(v);    // h = 4
    stage_lanes<1>(v, t);  // h = 8
    stage_lanes<2>(v, t);  // h = 16
    stage_regs<8>(v);    // h = 32
    stage_regs<16>(v);   // h = 64
    stage_regs<32>(v);   // h = 128
#pragma unroll
    for (int r = 0; r < kVals; ++r) v[r] = __fmul_rn(v[r], 0.0625f);
}

__device__ __forceinline__ float quad_absmax(const float (&v)[kVals]) {
    float m = 0.0f;
#pragma unroll
    for (int r = 0; r < kVals; ++r) m = fmaxf(m, fabsf(v[r]));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    return m;
}

// Exact path: the code as the definition states it, returned as the bit
// pattern of 1.5 * 2^23 + q (low byte = q in two's complement).
__device__ __forceinline__ uint32_t code_exact(float y, float s) {
    if (s == 0.0f) return __float_as_uint(kMagic);
    float q = rintf(__fdiv_rn(y, s));
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(q, kMagic));
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t ab = __byte_perm(a, b, 0x0040);
    const uint32_t cd = __byte_perm(c, d, 0x0040);
    return __byte_perm(ab, cd, 0x5410);
}

// Quantise lane t's 64 values with row scale s and store the codes: register
// group j holds elements 8t + 32j .. +7, stored as 8 contiguous bytes.
__device__ __forceinline__ void quantize_store(const float (&v)[kVals], float s, int8_t *qbase) {
    const bool fast = s >= kMinFastScale;
    const float rc = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t u[8];
        float dmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float t = __fmul_rn(v[8 * j + i], rc);
            const float m = __fadd_rn(t, kMagic);
            const float rt = __fsub_rn(m, kMagic);
            dmax = fmaxf(dmax, fabsf(__fsub_rn(t, rt)));
            u[i] = __float_as_uint(m);
        }
        if (!fast || dmax >= kNearHalf) {
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = code_exact(v[8 * j + i], s);
        }
        uint2 out;
        out.x = pack4(u[0], u[1], u[2], u[3]);
        out.y = pack4(u[4], u[5], u[6], u[7]);
        *reinterpret_cast<uint2 *>(qbase + 32 * j) = out;
    }
}

// Single pass: CTA = rows_per_cta rows x (K/256) quads, whole rows in registers.
template <bool kRotate, typename TIn>
__global__ void __launch_bounds__(kMaxThreads, 1)
quant_rows_kernel(const TIn *__restrict__ X, int64_t M, int K, int64_t ldx, int rows_per_cta,
                  int8_t *__restrict__ Q, float *__restrict__ S) {
    __shared__ unsigned s_amax[kMaxRowsPerCta];
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int row_local = quad / nb;
    const int blk = quad - row_local * nb;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + row_local;
    const bool active = row_local < rows_per_cta && row < M;
    const int col0 = blk * kBlock + 8 * t;

    if (tid < rows_per_cta) s_amax[tid] = 0u;

    float v[kVals];
    if (active) {
        load_block(X + row * ldx + col0, v);
    } else {
#pragma unroll
        for (int r = 0; r < kVals; ++r) v[r] = 0.0f;
    }
    if (kRotate) rotate_block(v, t);
    const float m = quad_absmax(v);
    __syncthreads();  // s_amax initialised
    if (active && t == 0) atomicMax(&s_amax[row_local], __float_as_uint(m));
    __syncthreads();
    if (!active) return;
    const float amax = __uint_as_float(s_amax[row_local]);
    const float s = __fdiv_rn(amax, 127.0f);
    if (blk == 0 && t == 0) S[row] = s;
    quantize_store(v, s, Q + row * static_cast<int64_t>(K) + col0);
}

// Two passes for long rows (K > 32768): one CTA per row, 128 quads; pass 1
// rotates every block and reduces the absmax, pass 2 reloads (from L2),
// rotates again and quantises.
template <bool kRotate, typename TIn>
__global__ void __launch_bounds__(kTwoPassQuads * 4, 1)
quant_rows_two_pass_kernel(const TIn *__restrict__ X, int64_t M, int K, int64_t ldx,
                           int8_t *__restrict__ Q, float *__restrict__ S) {
    __shared__ unsigned s_amax;
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int64_t row = blockIdx.x;
    if (tid == 0) s_amax = 0u;
    const TIn *xrow = X + row * ldx;
    float m = 0.0f;
    for (int b0 = 0; b0 < nb; b0 += kTwoPassQuads) {
        const int blk = b0 + quad;
        float v[kVals];
        if (blk < nb) {
            load_block(xrow + blk * kBlock + 8 * t, v);
        } else {
#pragma unroll
            for (int r = 0; r < kVals; ++r) v[r] = 0.0f;
        }
        if (kRotate) rotate_block(v, t);
        m = fmaxf(m, quad_absmax(v));
    }
    __syncthreads();
    if (t == 0) atomicMax(&s_amax, __float_as_uint(m));
    __syncthreads();
    const float amax = __uint_as_float(s_amax);
    const float s = __fdiv_rn(amax, 127.0f);
    if (tid == 0) S[row] = s;
    for (int b0 = 0; b0 < nb; b0 += kTwoPassQuads) {
        const int blk = b0 + quad;
        float v[kVals];
        if (blk < nb) {
            load_block(xrow + blk * kBlock + 8 * t, v);
        } else {
#pragma unroll
            for (int r = 0; r < kVals; ++r) v[r] = 0.0f;
        }
        if (kRotate) rotate_block(v, t);
        if (blk < nb) quantize_store(v, s, Q + row * static_cast<int64_t>(K) + blk * kBlock + 8 * t);
    }
}

// Rows per CTA for the single-pass kernel: the CTA has 4 * nb * R useful
// threads rounded up to whole warps; pick the R with the fewest idle lanes,
// then the CTA size closest to 256 threads.
int pick_rows_per_cta(int nb, int *threads_out) {
    int best_r = 1, best_t = ((4 * nb + 31) / 32) * 32;
    double best_waste = 2.0;
    int best_dist = 1 << 30;
    for (int r = 1; 4 * nb * r <= kMaxThreads; ++r) {
        const int used = 4 * nb * r;
        const int threads = ((used + 31) / 32) * 32;
        if (threads > kMaxThreads) break;
        const double waste = double(threads - used) / threads;
        const int dist = threads > 256 ? threads - 256 : 256 - threads;
        if (waste < best_waste - 1e-12 || (waste < best_waste + 1e-12 && dist < best_dist)) {
            best_waste = waste;
            best_dist = dist;
            best_r = r;
            best_t = threads;
        }
    }
    *threads_out = best_t;
    return best_r;
}

template <bool kRotate, typename TIn>
cudaError_t launch_rows(const TIn *X, int64_t M, int64_t K, int64_t ldx, int8_t *Q, float *S,
                        cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    const int nb = static_cast<int>(K / kBlock);
    if (4 * nb <= kMaxThreads) {
        int threads = 0;
        const int rows = pick_rows_per_cta(nb, &threads);
        const int64_t grid = (M + rows - 1) / rows;
        quant_rows_kernel<kRotate, TIn><<<static_cast<unsigned>(grid), threads, 0, stream>>>(
            X, M, static_cast<int>(K), ldx, rows, Q, S);
    } else {
        quant_rows_two_pass_kernel<kRotate, TIn>
            <<<static_cast<unsigned>(M), kTwoPassQuads * 4, 0, stream>>>(
                X, M, static_cast<int>(K), ldx, Q, S);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_rows_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   bool rotate, int8_t *Q, float *S, cudaStream_t stream) {
    return rotate ? launch_rows<true>(X, M, K, ldx, Q, S, stream)
                  : launch_rows<false>(X, M, K, ldx, Q, S, stream);
}

cudaError_t launch_quant_rows_f32(const float *W, int64_t N, int64_t K, int8_t *Q, float *S,
                                  cudaStream_t stream) {
    return launch_rows<true>(W, N, K, K, Q, S, stream);
}

}  // namespace ck
