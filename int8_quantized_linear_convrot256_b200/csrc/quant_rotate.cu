// Fused ConvRot256 rotation + dynamic per-row INT8 quantisation for sm_100a.
//
// What is computed (comfy-kitchen 0.2.40, "Huawei Ascend backend" and "HIP
// backend": quantize_and_rotate_rowwise / quantize_int8_rowwise; sglang PR
// "Tune Kitchen INT8 row splitting for SM120", Accuracy Test: ConvRot256 and
// FP32 row scales; ComfyUI-AppleSilicon-FP8 README row 17: rotate online,
// then quantise per row):
//   every 256-block of a row -> 8 fp32 butterfly stages h = 1, 2, ..., 128,
//   then * 1/16 (y); s = absmax(y) / 127; q = round-half-even(y / s) clamped
//   to [-127, 127]; a zero row gives s = 0 and q = 0.
//
// Design (HBM-bound: 2 B read + 1 B written per element, 4 B per row):
//  * One quad (4 consecutive lanes) owns one 256-block; each lane keeps 64
//    values in registers as 32 float2 pairs. Element e of the block sits in
//    lane (e >> 3) & 3 of the quad; within the lane, pair j holds elements
//    with e bit 0 = 0/1, j bit 0 = e bit 1, bit 1 = e bit 2, bits 2-4 = e
//    bits 5-7. Lane t therefore loads 8 contiguous values at e = 8t + 32i
//    (i = 0..7): 16-byte loads, each quad reading 64 contiguous bytes. In the
//    staged kernel odd quads read chunk i ^ 1 into register group i (so the
//    two quads of a quarter-warp use different shared-memory banks); the
//    h = 32 stage, which pairs groups i and i ^ 1, and the code stores
//    account for the swap.
//  * Butterfly stages h = 1, 2, ..., 128 run in that order; each is one IEEE
//    add or subtract per value (a - c as fma(c, -1, a): one rounding of the
//    exact difference). h = 1 pairs the two halves of a float2 (scalar ops;
//    in the staged kernel it is fused with the widening, add/sub.f32.bf16);
//    h = 2, 4, 32, 64, 128 pair whole float2s (packed add.f32x2 / fma.f32x2);
//    h = 8, 16 pair lanes t ^ 1, t ^ 2 of the quad through shuffles and one
//    packed fma(+-1, v, partner). Results are bit-identical to the
//    sequential definition.
//  * The exact * 1/16 is folded into the scale: with z = 16 y (the butterfly
//    output), amax_y = amax_z / 16 and s = fl(amax_z / 127) / 16 exactly, and
//    fl(y / s) = fl(z / fl(amax_z / 127)), as long as nothing is subnormal:
//    rows with amax_z >= 2^-103 take this path (values with |z| < 2^-122,
//    whose y would be subnormal, give code 0 either way: the divisor
//    fl(amax_z / 127) is at least 2^-110, so |z / divisor| < 2^-12).
//    Smaller rows follow the definition step by step (y = fl(z / 16), then the
//    exact division).
//  * Division: q needs round-half-even of the IEEE quotient fl(y / s). With
//    d the divisor (fl(amax_z / 127), one product and one fma, see
//    div_by_q) and r its reciprocal to within 2^-24 + 2^-43 (one Newton
//    step, see rcp_newton), the exact product z r is within
//    127.00001 (2^-24 + 2^-43) < 2^-17 of z/d, and |fl(z/d) - z/d| <= 2^-18
//    because |z/d| < 128; so if z r is farther than 2^-17 + 2^-18 from every
//    half-integer, rint(z r) = rint(fl(z/d)). One fma gives fl(z r + 1.5 * 2^23) =
//    1.5 * 2^23 + rint(z r), whose low byte is the two's-complement code (no
//    clamp is needed on that path); a second fma gives the distance of z r
//    to that integer. Groups that hold a value within 2^-16 of a
//    half-integer take rint(__fdiv_rn(z, d)) instead. The distance is
//    computed as fl(rint(z r) - z r) (error <= 2^-26), so a value that is
//    not redone lies more than 2^-16 - 2^-26 > 2^-17 + 2^-18 from every
//    half-integer; about 1 value in 30000 is redone.
//  * The whole row stays in registers of one CTA (rows_per_cta rows x K/256
//    quads); the row absmax is reduced through a shared-memory atomicMax on
//    the fp32 bit pattern, so X is read from HBM exactly once. BF16 rows are
//    staged into shared memory by 1-D bulk copies (cp.async.bulk) one row
//    group ahead of the compute, in a persistent grid, so HBM always has a
//    full row group per CTA in flight. K > 32768 takes a two-pass variant
//    (rows re-read from L2); fp32 weights (offline) take direct loads.
//  * No FMA contraction: every operation is an explicit _rn intrinsic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

constexpr int kBlock = 256;
constexpr int kPairs = 32;  // float2 pairs per lane per block (64 values)
constexpr int kMaxThreads = 512;
constexpr int kMaxRowsPerCta = kMaxThreads / 4;
constexpr int kTwoPassQuads = 128;                   // quads per row in the two-pass variant
constexpr float kMagic = 12582912.0f;                // 1.5 * 2^23
constexpr float kMagic4 = 3145728.0f;                // 1.5 * 2^21 (spacing 1/4 around it)
constexpr float kNearQuarter = 1.52587890625e-05f;   // 2^-16
constexpr float kNearHalf = 0.4999847412109375f;     // 0.5 - 2^-16
constexpr float kMinFastScale = 7.52316384526264e-37f;  // 2^-120
constexpr float kMinFoldAmax = 9.8607613152626476e-32f;  // 2^-103
constexpr size_t kBulkSmemBudget = 112 * 1024;       // per-CTA staging budget (all buffers)
constexpr int kBulkBufs = 2;                         // row groups staged per CTA of the INT8 quantiser (3 timed no faster)

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b with one rounding: b * (-1) is exact, then the sum is rounded once.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float2 widen_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ------------------------------------------------------------------ input_act
// int8_linear(input_act=...) (comfy-kitchen 0.2.40, "HIP backend"): each bf16
// input x becomes the bf16 value nearest to the exact act(x) (ties to even)
// before the rotation. relu; silu x / (1 + e^-x); gelu (tanh form)
// 0.5 x (1 + tanh(u)) = x / (1 + e^(-2u)), u = sqrt(2/pi) (x + 0.044715 x^3).
//
// Fast path, fp32: with v the exponent (-x, or -2u), e^v by Cody-Waite
// reduction v = n ln2 + r (ln2 = 16-bit head + tail) and a degree-7 Taylor
// polynomial of e^r (truncation below 2^-27), d = 1 + e, and the quotient
// x rcp.approx(d): within 4 fp32 ulps of the exact value for silu (whose v is
// exact) and within 4 + 3.5 |v| for gelu (the fp32 rounding of v, a few ulps,
// amplified by e^v when it is not negligible against 1). The bf16 rounding of
// the result is the exact value's unless it lies near a bf16 rounding
// midpoint: values within W = 8 (silu) or 8 + 4 |v| (gelu) fp32 ulps of one,
// and denominators above 1e36, are redone in double precision and rounded to
// bf16 from the double value directly. (The hardware's ex2.approx timed
// slower here: its error grows with |v|, and the wider windows it needs send
// more values to the double path.) The double
// result differs from the exact value by a few 2^-52 relative, far less than
// its distance from any midpoint for every bf16 input (the whole input set,
// 65,280 finite values, is checked against the CPU oracle).
// Where v > 182 the exact value's magnitude is below |x| e^-182 < 2^-134,
// half the smallest bf16 subnormal, for every bf16 x: the result is a zero
// with the sign of x, taken without a redo (gelu; for silu that needs
// x < -182, which goes to the double path).
// For |x| < 2^-120 the double evaluation gives x/2 exactly, which can sit on
// a midpoint between bf16 subnormals while the exact value lies just above
// x/2; there x/2 is rounded with ties going up.
constexpr int kActNone = 0;
constexpr int kActRelu = 1;
constexpr int kActSilu = 2;
constexpr int kActGeluTanh = 3;

// e^x of two values, branch-free: n = rint(x log2 e) by adding and removing
// 1.5 * 2^23 (round-to-nearest-even, |x log2 e| < 2^22 in range), k = n from
// the sum's bits; r = x - n ln2 (two fused steps, 16-bit head + tail);
// degree-7 Taylor polynomial of e^r by fused Horner steps (packed
// fma.f32x2); then p * 2^k as (p * 2^a) * 2^b with a = floor(k/2),
// b = ceil(k/2): p * 2^a is exact and normal (p >= 0.7, a >= -75). Outside
// [-104, 88.8] the limits 0 and +inf are selected.
__device__ __forceinline__ float2 act_exp2(float2 x) {
    const float kRound = 12582912.0f;  // 1.5 * 2^23
    const float2 m = __fadd2_rn(__fmul2_rn(x, make_float2(1.442695f, 1.442695f)),
                                make_float2(kRound, kRound));
    const float2 n = __fadd2_rn(m, make_float2(-kRound, -kRound));
    const float2 mn = make_float2(-n.x, -n.y);
    float2 r = __ffma2_rn(mn, make_float2(0.693145751953125f, 0.693145751953125f), x);
    r = __ffma2_rn(mn, make_float2(1.4286068e-06f, 1.4286068e-06f), r);
    float2 p = make_float2(1.984127e-04f, 1.984127e-04f);  // 1/7!, 1/6!, ..., 1, 1 in fp32
    p = __ffma2_rn(p, r, make_float2(1.3888889e-03f, 1.3888889e-03f));
    p = __ffma2_rn(p, r, make_float2(8.333334e-03f, 8.333334e-03f));
    p = __ffma2_rn(p, r, make_float2(4.1666668e-02f, 4.1666668e-02f));
    p = __ffma2_rn(p, r, make_float2(1.6666667e-01f, 1.6666667e-01f));
    p = __ffma2_rn(p, r, make_float2(0.5f, 0.5f));
    p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
    p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
    const int kx = int(__float_as_uint(m.x) - __float_as_uint(kRound));
    const int ky = int(__float_as_uint(m.y) - __float_as_uint(kRound));
    // k = a + b with a = floor(k/2), b = ceil(k/2), both in [-75, 64]; each
    // factor is built from k alone
    const float2 s1 = make_float2(__uint_as_float(uint32_t((kx >> 1) + 127) << 23),
                                  __uint_as_float(uint32_t((ky >> 1) + 127) << 23));
    const float2 s2 = make_float2(__uint_as_float(uint32_t(((kx + 1) >> 1) + 127) << 23),
                                  __uint_as_float(uint32_t(((ky + 1) >> 1) + 127) << 23));
    float2 e = __fmul2_rn(__fmul2_rn(p, s1), s2);
    const float inf = __uint_as_float(0x7F800000u);
    e.x = x.x > 88.8f ? inf : (x.x < -104.0f ? 0.0f : e.x);
    e.y = x.y > 88.8f ? inf : (x.y < -104.0f ? 0.0f : e.y);
    return e;
}

// x / d where only the bf16 rounding of the quotient is used: a reciprocal
// approximation times x. `redo` is raised when the result lies within w fp32
// ulps of a bf16 rounding midpoint, or d is huge (the reciprocal would leave
// the normal range); `zero` gives x's signed zero instead (no redo).
__device__ __forceinline__ float div_for_bf16(float x, float d, uint32_t w, bool zero, bool &redo) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(d));
    const float q = __fmul_rn(x, r);
    const uint32_t lo = __float_as_uint(q) & 0xFFFFu;
    if (zero) return __fmul_rn(x, 0.0f);
    redo = redo || (lo - (0x8000u - w) <= 2u * w) || (d > 1.0e36f);
    return q;
}

// The flag window of one value in fp32 ulps: 8 for silu (its exponent -x is
// exact); for gelu 8 + 4 |v|, the fp32 rounding of v = -2u amplified by e^v,
// counted where e^v is not negligible against 1 (|v| <= 83 there).
template <int kAct>
__device__ __forceinline__ uint32_t act_window(float e, float v) {
    if (kAct == kActSilu) return 8u;
    return 8u + (e >= 9.5367431640625e-07f && e <= 1.0e36f ? uint32_t(4.0f * fabsf(v)) : 0u);
}

// bf16x2 word -> activation of both values -> bf16x2 word (round to nearest
// even). `redo` is raised when a value needs the double-precision path; then
// act_bf16x2_exact gives the word.
__device__ __forceinline__ __nv_bfloat162 bf162_bits(uint32_t w) {
    return *reinterpret_cast<const __nv_bfloat162 *>(&w);
}
__device__ __forceinline__ uint32_t bits_bf162(__nv_bfloat162 v) {
    return *reinterpret_cast<const uint32_t *>(&v);
}

template <int kAct>
__device__ __forceinline__ uint32_t act_bf16x2(uint32_t w, bool &redo) {
    if (kAct == kActNone) return w;
    // relu: max(x, +0) of both halves in one instruction (max returns the
    // non-NaN operand, so NaN gives +0 as x > 0 ? x : 0 does; max(-0, +0)
    // is +0; every bf16 input is compared with the oracle through the test
    // hook)
    if (kAct == kActRelu) return bits_bf162(__hmax2(bf162_bits(w), bf162_bits(0u)));
    const float2 x = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    float2 a;
    if (kAct == kActRelu) {
        a = make_float2(x.x > 0.0f ? x.x : 0.0f, x.y > 0.0f ? x.y : 0.0f);
    } else {
        float2 v;
        if (kAct == kActSilu) {
            v = make_float2(-x.x, -x.y);
        } else {
            const float2 x3 = __fmul2_rn(__fmul2_rn(x, x), x);
            const float2 inner = __ffma2_rn(make_float2(0.044715f, 0.044715f), x3, x);
            const float2 u = __fmul2_rn(make_float2(7.978846e-01f, 7.978846e-01f), inner);
            v = __fmul2_rn(make_float2(-2.0f, -2.0f), u);
        }
        const float2 e = act_exp2(v);
        const float2 d = __fadd2_rn(make_float2(1.0f, 1.0f), e);
        // the signed-zero rule matters for gelu only (its v passes 182 below
        // x = -13.1; silu's only below x = -182, left to the double path)
        const bool gelu = kAct == kActGeluTanh;
        a = make_float2(div_for_bf16(x.x, d.x, act_window<kAct>(e.x, v.x), gelu && v.x > 182.0f, redo),
                        div_for_bf16(x.y, d.y, act_window<kAct>(e.y, v.y), gelu && v.y > 182.0f, redo));
    }
    const __nv_bfloat162 h = __floats2bfloat162_rn(a.x, a.y);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// One value in double precision, rounded once to bf16 (the bits).
template <int kAct>
__device__ __forceinline__ uint32_t act_bf16_double(float xf) {
    const double x = xf;
    double v;
    if (x != 0.0 && fabs(x) < 7.52316384526264e-37) {  // |x| < 2^-120
        // x/2 in units of the bf16 subnormal spacing 2^-133; a tie goes up
        const double t = x * 5.444517870735016e+39;  // 2^132
        const double lo = floor(t);
        const double q = (t - lo == 0.5) ? lo + 1.0 : rint(t);
        v = copysign(q * 9.183549615799121e-41, x);  // q * 2^-133
    } else if (kAct == kActSilu) {
        v = x / (1.0 + exp(-x));
    } else {
        const double u = 0.7978845608028654 * (x + 0.044715 * (x * x * x));  // sqrt(2/pi)
        v = x / (1.0 + exp(-2.0 * u));
    }
    const __nv_bfloat16 h = __double2bfloat16(v);
    return *reinterpret_cast<const uint16_t *>(&h);
}

template <int kAct>
__device__ __noinline__ uint32_t act_bf16x2_exact(uint32_t w) {
    return act_bf16_double<kAct>(__uint_as_float(w << 16)) |
           (act_bf16_double<kAct>(__uint_as_float(w & 0xFFFF0000u)) << 16);
}

template <int kAct>
__device__ __forceinline__ uint32_t act_bf16x2(uint32_t w) {
    bool redo = false;
    const uint32_t r = act_bf16x2<kAct>(w, redo);
    return redo ? act_bf16x2_exact<kAct>(w) : r;
}

// Lane t's 64 values of one block; base points at element 8t of the block.
template <int kAct = kActNone>
__device__ __forceinline__ void load_block(const uint16_t *base, float2 (&P)[kPairs]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(base + 32 * i));
        P[4 * i + 0] = widen_bf16x2(act_bf16x2<kAct>(u.x));
        P[4 * i + 1] = widen_bf16x2(act_bf16x2<kAct>(u.y));
        P[4 * i + 2] = widen_bf16x2(act_bf16x2<kAct>(u.z));
        P[4 * i + 3] = widen_bf16x2(act_bf16x2<kAct>(u.w));
    }
}

template <int kAct = kActNone>
__device__ __forceinline__ void load_block(const float *base, float2 (&P)[kPairs]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 a = __ldcs(reinterpret_cast<const float4 *>(base + 32 * i));
        const float4 b = __ldcs(reinterpret_cast<const float4 *>(base + 32 * i + 4));
        P[4 * i + 0] = make_float2(a.x, a.y);
        P[4 * i + 1] = make_float2(a.z, a.w);
        P[4 * i + 2] = make_float2(b.x, b.y);
        P[4 * i + 3] = make_float2(b.z, b.w);
    }
}

// Widening fused with the h = 1 butterfly for the two bf16 of one word:
// add.f32.bf16 / sub.f32.bf16 widen their bf16 operand exactly and round the
// fp32 sum once, giving fl(a + c) and fl(a - c) as the sequential definition
// does.
__device__ __forceinline__ float2 widen_stage1(uint32_t w) {
    float s, d;
    const float c = __uint_as_float(w & 0xFFFF0000u);
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %3;\n\tsub.rn.f32.bf16 %1, lo, %3;\n\t}"
        : "=f"(s), "=f"(d) : "r"(w), "f"(c));
    return make_float2(s, d);
}
// silu and tanh-form gelu through a table of exact results. Every bf16 input
// with |x| in [2^-9, 2^7) has its own entry, (|h| - 0x3B00) + 2048 sign for
// the bits h, filled by each CTA from act_bf16x2 (fast path with the
// double-precision redo, the same results bit for bit). Outside the table:
//  * |x| >= 2^7: x when x > 0, -0 when x < 0. The exact value differs from
//    those by x e^-x / (1 + e^-x) (silu; gelu's term is smaller still), far
//    below half a bf16 spacing of x, or is below 2^-134 in magnitude.
//  * 2^-125 <= |x| < 2^-9, and x = +-0: x / 2 (exact: x / 2 is a normal bf16
//    value). act(x) = x / 2 + c x^2 + O(x^3) with c = 1/4 (silu) or
//    sqrt(2/pi) / 2 (gelu), so the difference is below half a spacing of
//    x / 2 on either side for |x| < 2^-8.67.
//  * 0 < |x| < 2^-125 (where x / 2 leaves bf16's normal range), infinities
//    and NaN: `rare` is raised and the caller takes act_bf16x2_exact.
// Every bf16 input is checked against the CPU oracle through the test hook,
// which uses this same function.
constexpr uint32_t kActTabLo = 0x3B00u;  // 2^-9
constexpr int kActTabWords = 2048;       // 4096 entries of 16 bits

template <int kAct>
__device__ __forceinline__ void act_table_fill(uint32_t *tab, int tid, int nthreads) {
    for (int i = tid; i < kActTabWords; i += nthreads) {
        const uint32_t e = 2u * uint32_t(i);  // entries e, e + 1: same sign
        const uint32_t h = ((e & 0x800u) << 4) | (kActTabLo + (e & 0x7FFu));
        tab[i] = act_bf16x2<kAct>(h | ((h + 1u) << 16));
    }
}

template <int kAct>
__device__ __forceinline__ uint32_t act_word_tab(uint32_t w, const uint16_t *tab, bool &rare) {
    const uint32_t a2 = w & 0x7FFF7FFFu;
    const __nv_bfloat162 wb = bf162_bits(w);
    const __nv_bfloat162 ab = bf162_bits(a2);
    const uint32_t small = __hlt2_mask(ab, bf162_bits(0x3B003B00u));  // |x| < 2^-9
    const uint32_t inside = ~small & __hlt2_mask(ab, bf162_bits(0x43004300u));  // < 2^7
    const uint32_t half = bits_bf162(__hmul2(wb, bf162_bits(0x3F003F00u)));   // x * 0.5
    const uint32_t big = bits_bf162(__hmax2(wb, bf162_bits(0x80008000u)));    // max(x, -0)
    // both entries' indices at once: per half 0x8000 + |h| - 0x3B00 (no
    // borrow between the halves), its low 11 bits, then the sign as bit 11.
    // Every input gives an index inside the table; only the window's are used.
    const uint32_t i2 = (((w | 0x80008000u) - 0x3B003B00u) & 0x07FF07FFu) | ((w >> 4) & 0x08000800u);
    const uint32_t lo = tab[i2 & 0xFFFFu];
    const uint32_t hi = tab[i2 >> 16];
    const uint32_t t2 = lo | (hi << 16);
    const uint32_t rule = (half & small) | (big & ~small);
    const uint32_t tiny = __hlt2_mask(ab, bf162_bits(0x01000100u)) & ~__heq2_mask(ab, bf162_bits(0u));
    const uint32_t finite = __hlt2_mask(ab, bf162_bits(0x7F807F80u));
    rare = rare || ((tiny | ~finite) != 0u);
    return (t2 & inside) | (rule & ~inside);
}

// The input activation of one 16-byte chunk (4 words, 8 values): relu
// computed, silu and tanh-form gelu from the table; a word holding a value
// outside the table's reach is redone by act_bf16x2_exact.
template <int kAct>
__device__ __forceinline__ void act_chunk(const uint32_t (&w)[4], uint32_t (&a)[4],
                                          const uint16_t *tab) {
    bool rare[4] = {false, false, false, false};
#pragma unroll
    for (int q = 0; q < 4; ++q)
        a[q] = (kAct == kActSilu || kAct == kActGeluTanh) ? act_word_tab<kAct>(w[q], tab, rare[q])
                                                          : act_bf16x2<kAct>(w[q], rare[q]);
    if (rare[0] | rare[1] | rare[2] | rare[3]) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (rare[q]) a[q] = act_bf16x2_exact<kAct>(w[q]);
    }
}

// Applies the input activation in place to a lane's 64 bf16 values in
// shared memory (8 chunks of 16 bytes at saddr + 64 i), chunk by chunk with
// act_chunk, the function the staged quantiser applies to each loaded chunk.
template <int kAct>
__device__ __forceinline__ void act_in_smem(uint32_t saddr, const uint16_t *tab) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
        uint32_t w[4], a[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(saddr + 64u * i));
        act_chunk<kAct>(w, a, tab);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(saddr + 64u * i), "r"(a[0]),
                     "r"(a[1]), "r"(a[2]), "r"(a[3])
                     : "memory");
    }
}

// Test hook: the input activation exactly as the staged quantiser applies it
// (act_chunk on 16-byte chunks, the table filled per CTA as there); 8192
// values per CTA of 128 threads.
template <int kAct>
__global__ void __launch_bounds__(128)
input_act_kernel(const uint4 *__restrict__ X, uint4 *__restrict__ Y, int64_t n16) {
    __shared__ __align__(16) uint4 buf[1024];
    __shared__ uint32_t tab[kAct == kActSilu || kAct == kActGeluTanh ? kActTabWords : 1];
    const int t = threadIdx.x;
    const int64_t base = int64_t(blockIdx.x) * 1024;
    if (kAct == kActSilu || kAct == kActGeluTanh) act_table_fill<kAct>(tab, t, 128);
    for (int i = t; i < 1024; i += 128)
        buf[i] = base + i < n16 ? X[base + i] : make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    // lane l of quad q: chunks 32 q + l + 4 i (i = 0..7), 64 bytes apart
    act_in_smem<kAct>(smem_u32(&buf[32 * (t >> 2) + (t & 3)]),
                      reinterpret_cast<const uint16_t *>(tab));
    __syncthreads();
    for (int i = t; i < 1024; i += 128)
        if (base + i < n16) Y[base + i] = buf[i];
}

// Shared-memory loads of lane t's 64 staged values (the block's bf16 at
// saddr - 16 t; the lane's chunk i at saddr + 64 i). With sw5 = 1 the lane
// reads chunk i ^ 1 into register group i: two neighbouring blocks then read
// different 64-byte halves of the bank space in the same instruction, so the
// 8 lanes of a quarter-warp hit 8 different 16-byte bank groups. Register
// group i holds elements 8t + 32 (i ^ sw5) .. +7; the h = 32 stage and the
// stores take the swap into account. kStage1: widening fused with h = 1.
template <bool kStage1>
__device__ __forceinline__ void load_block_smem(uint32_t saddr, int sw5, float2 (&P)[kPairs]) {
    const uint32_t base[2] = {saddr + 64u * uint32_t(sw5), saddr - 64u * uint32_t(sw5)};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t w[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(base[i & 1] + 64u * i));
#pragma unroll
        for (int q = 0; q < 4; ++q) P[4 * i + q] = kStage1 ? widen_stage1(w[q]) : widen_bf16x2(w[q]);
    }
}

// load_block_smem with the input activation applied to each chunk as it
// arrives (act_chunk, as the test hook applies it).
template <bool kStage1, int kAct>
__device__ __forceinline__ void load_block_smem_act(uint32_t saddr, int sw5, float2 (&P)[kPairs],
                                                    const uint16_t *tab) {
    const uint32_t base[2] = {saddr + 64u * uint32_t(sw5), saddr - 64u * uint32_t(sw5)};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t w[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(base[i & 1] + 64u * i));
        uint32_t a[4];
        act_chunk<kAct>(w, a, tab);
#pragma unroll
        for (int q = 0; q < 4; ++q) P[4 * i + q] = kStage1 ? widen_stage1(a[q]) : widen_bf16x2(a[q]);
    }
}

template <int NP>
__device__ __forceinline__ void zero_block(float2 (&P)[NP]) {
#pragma unroll
    for (int j = 0; j < NP; ++j) P[j] = make_float2(0.0f, 0.0f);
}

// h = 1: the two halves of every pair.
template <int NP>
__device__ __forceinline__ void stage_in_pair(float2 (&P)[NP]) {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float a = P[j].x;
        const float c = P[j].y;
        P[j] = make_float2(__fadd_rn(a, c), __fsub_rn(a, c));
    }
}

// Pairs j and j + J (J a power of two): P[j] holds the element with the
// stage's bit clear (a), P[j + J] the one with it set (c).
template <int J, int NP>
__device__ __forceinline__ void stage_pairs(float2 (&P)[NP]) {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        if ((j & J) == 0) {
            const float2 a = P[j];
            const float2 c = P[j + J];
            P[j] = add2(a, c);
            P[j + J] = sub2(a, c);
        }
    }
}

// As stage_pairs, for a block whose two registers of each pair may hold the
// elements swapped (sg = -1: P[j] holds c, P[j + J] holds a). The element
// with the bit clear must receive a + c and the other a - c:
//   P[j]     <- fma(sg, P[j], P[j + J])   (a + c, or a - c when swapped)
//   P[j + J] <- fma(-sg, P[j + J], P[j])  (a - c, or a + c when swapped)
// fma(+-1, x, y) rounds the exact y +- x once, as the definition's add does.
template <int J, int NP>
__device__ __forceinline__ void stage_pairs_swz(float2 (&P)[NP], float2 sg, float2 nsg) {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        if ((j & J) == 0) {
            const float2 lo = P[j];
            const float2 hi = P[j + J];
            P[j] = __ffma2_rn(sg, lo, hi);
            P[j + J] = __ffma2_rn(nsg, hi, lo);
        }
    }
}

// Lanes t and t ^ L (L = 1, 2): the lane with the bit clear holds a and
// computes a + c; the other holds c and computes a - c = fma(-1, c, a).
template <int L, int NP>
__device__ __forceinline__ void stage_lanes(float2 (&P)[NP], int t) {
    const float s = (t & L) ? -1.0f : 1.0f;
    const float2 sg = make_float2(s, s);
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float2 p = make_float2(__shfl_xor_sync(0xFFFFFFFFu, P[j].x, L),
                                     __shfl_xor_sync(0xFFFFFFFFu, P[j].y, L));
        P[j] = __ffma2_rn(sg, P[j], p);
    }
}

// The 8 butterfly stages of ConvRot256, without the final * 1/16 (z = 16 y);
// kStage1Done when h = 1 was applied while loading; sw5 = 1 when the
// register groups of the h = 32 stage are swapped (staged kernel).
template <bool kStage1Done = false>
__device__ __forceinline__ void butterflies(float2 (&P)[kPairs], int t, int sw5 = 0) {
    if (!kStage1Done) stage_in_pair(P);    // h = 1
    stage_pairs<1>(P);   // h = 2
    stage_pairs<2>(P);   // h = 4
    stage_lanes<1>(P, t);  // h = 8
    stage_lanes<2>(P, t);  // h = 16
    const float s5 = sw5 ? -1.0f : 1.0f;
    stage_pairs_swz<4>(P, make_float2(s5, s5), make_float2(-s5, -s5));  // h = 32
    stage_pairs<8>(P);   // h = 64
    stage_pairs<16>(P);  // h = 128
}

// Largest |value| of the block, reduced over the kLanes lanes that hold it.
template <int kLanes = 4, int NP>
__device__ __forceinline__ float block_absmax(const float2 (&P)[NP]) {
    // four independent chains keep the reduction's dependency depth short
    float mm[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < NP; ++j) mm[j & 3] = max3(mm[j & 3], fabsf(P[j].x), fabsf(P[j].y));
    float m = fmaxf(max3(mm[0], mm[1], mm[2]), mm[3]);
#pragma unroll
    for (int l = 1; l < kLanes; l <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, l));
    return m;
}

// How a row is quantised, from its absmax (of z for rotated rows).
struct RowQuant {
    float s;      // the row scale to store (the definition's s)
    float div;    // divisor applied to the held values
    float rc;     // fl(1 / div) when fast
    bool fast;    // reciprocal path with the near-half-integer fallback
    bool scale16; // exact path must first form y = fl(z / 16)
    float qmax;   // codes lie in [-qmax, qmax]
};

// fl(a / kQ), the IEEE quotient, for kQ = 127 or 7 and finite a >= 2^-103,
// by one product and one fma with a two-word reciprocal hi + lo of 1 / kQ
// (hi = fl(1 / kQ), lo = fl(1 / kQ - hi); hi + lo is within 2^-56 (127) or
// 2^-51 (7) of 1 / kQ relative). The fma's exact sum a hi + fl(a lo) is
// within 2^-48 of a / kQ relative while fl(a lo) is a normal number; below
// that (a under about 2^-91 for 127, 2^-98.8 for 7) its absolute error, at
// most 2^-150, is below 2^-40 a / kQ. Why that suffices:
// with a = A 2^e (A a 24-bit integer) the bits of A / kQ beyond fp32's
// 24 repeat with period 7 (127 = 2^7 - 1) or 3 (7 = 2^3 - 1), so the part
// of a / kQ beyond the last kept bit is r / kQ of a unit in the last place
// for an integer r. It is therefore 0 (a / kQ exact) or at least 1 / 254
// (resp. 1 / 14) of a unit, about 2^-32 relative, away from the rounding
// midpoint, far more than 2^-40: the sum rounds as a / kQ does. Checked
// against the IEEE quotient for every fp32 significand by the test hook
// ck_test_row_quant_params.
template <int kQ>
__device__ __forceinline__ float div_by_q(float a) {
    static_assert(kQ == 127 || kQ == 7, "two-word reciprocal for 127 and 7 only");
    constexpr float hi = kQ == 127 ? 0x1.020408p-7f : 0x1.24924ap-3f;
    constexpr float lo = kQ == 127 ? 0x1.020408p-35f : -0x1.b6db6ep-28f;
    return __fmaf_rn(a, hi, __fmul_rn(a, lo));
}

// Reciprocal of a normal d within 2^-24 + 2^-43 relative (not necessarily
// the correctly rounded one): the hardware approximation r0 (relative error
// e0 <= 2^-22) and one Newton-Raphson step r0 + r0 (1 - d r0), whose
// relative error before the last rounding is at most e0^2 + 2^-24 e0.
__device__ __forceinline__ float rcp_newton(float d) {
    float r0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(d));
    const float e = __fmaf_rn(-d, r0, 1.0f);
    return __fmaf_rn(r0, e, r0);
}

// kQ = 127: INT8 codes; kQ = 7: signed INT4 codes (convrot_w4a4_linear).
// The fast path's reciprocal rc = rcp_newton(d) is within 2^-24 + 2^-43 of
// 1 / d relative, so for |z| <= amax the exact z rc lies within
// 127.00001 (2^-24 + 2^-43) + 2^-18 < 1.14e-5 of fl(z / d) (the second term: half
// a unit in the last place below 128). A value whose computed distance to
// the nearest integer is below 0.5 - 2^-16 (the distance itself rounded once,
// to within 2^-26) lies more than 2^-16 - 2^-26 = 1.52e-5 from every
// half-integer, so fl(z / d) rounds to the same integer. The bound holds a
// fortiori for |z / d| <= 7.
template <bool kRotate, int kQ = 127>
__device__ __forceinline__ RowQuant row_quant(float amax) {
    RowQuant r;
    const float qmax = float(kQ);
    r.qmax = qmax;
    if (kRotate) {
        if (amax >= kMinFoldAmax) {
            r.div = div_by_q<kQ>(amax);
            r.s = __fmul_rn(r.div, 0.0625f);
            r.fast = true;
            r.scale16 = false;
        } else {
            r.s = __fdiv_rn(__fmul_rn(amax, 0.0625f), qmax);
            r.div = r.s;
            r.fast = false;
            r.scale16 = true;
        }
    } else {
        r.s = __fdiv_rn(amax, qmax);
        r.div = r.s;
        r.fast = r.s >= kMinFastScale;
        r.scale16 = false;
    }
    r.rc = r.fast ? rcp_newton(r.div) : 0.0f;
    return r;
}

// Test hook: the divisor and the reciprocal that row_quant gives a rotated
// row of absmax amax[i] (grid-stride over n values).
template <int kQ>
__global__ void __launch_bounds__(256)
row_quant_params_kernel(const float *__restrict__ amax, int64_t n, float *__restrict__ div,
                        float *__restrict__ rc) {
    const int64_t step = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += step) {
        const RowQuant r = row_quant<true, kQ>(amax[i]);
        div[i] = r.div;
        rc[i] = r.rc;
    }
}

// Exact path for one value, as the definition states it; returns the bit
// pattern of 1.5 * 2^23 + q (low byte = q in two's complement).
__device__ __forceinline__ uint32_t code_exact(float z, const RowQuant &rq) {
    if (rq.div == 0.0f) return __float_as_uint(kMagic);
    const float y = rq.scale16 ? __fmul_rn(z, 0.0625f) : z;
    float q = rintf(__fdiv_rn(y, rq.div));
    q = fminf(fmaxf(q, -rq.qmax), rq.qmax);
    return __float_as_uint(__fadd_rn(q, kMagic));
}

// Fast path for two values (z) of a row with reciprocal rc = fl(1 / d):
// m = fl(z rc + 1.5 * 2^23) = 1.5 * 2^23 + rint(z rc), one rounding of the
// exact product-sum (|z rc| < 128, so the sum lies in [2^23, 2^24) where the
// spacing is 1); its low byte is the code. d = fl(rint(z rc) - z rc) is the
// (negated) distance to that integer; dmax tracks the largest |d|.
struct FastQuant {
    float2 rc2, nrc2, magic2, nmagic2;
    __device__ __forceinline__ explicit FastQuant(float rc)
        : rc2(make_float2(rc, rc)), nrc2(make_float2(-rc, -rc)),
          magic2(make_float2(kMagic, kMagic)), nmagic2(make_float2(-kMagic, -kMagic)) {}
    __device__ __forceinline__ float2 code2(float2 z, float &dmax) const {
        const float2 m = __ffma2_rn(z, rc2, magic2);
        const float2 rt = add2(m, nmagic2);
        const float2 d = __ffma2_rn(z, nrc2, rt);
        dmax = max3(dmax, fabsf(d.x), fabsf(d.y));
        return m;
    }
};

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t ab = __byte_perm(a, b, 0x0040);
    const uint32_t cd = __byte_perm(c, d, 0x0040);
    return __byte_perm(ab, cd, 0x5410);
}

// Where the codes of register group i go. In the staged kernel the group
// index is swizzled with bit 0 of the block index (sw5, see load_block_smem):
// register group i then holds elements 8t + 32 (i ^ sw5) .. +7, whose codes
// start at q[i & 1] + 32 i with q[0] = qbase + 32 sw5, q[1] = qbase - 32 sw5.
// Unswizzled callers pass sw5 = 0.
struct CodeDst {
    int8_t *q[2];
    __device__ __forceinline__ CodeDst(int8_t *qbase, int sw5)
        : q{qbase + 32 * sw5, qbase - 32 * sw5} {}
};

// Stores the 8 codes of group i: 8 int8 bytes at dst.q[i & 1] + 32 i, or
// (kPack4, unswizzled only) 8 signed nibbles in one 32-bit word at
// q + 16 i, element 2j in the low nibble of byte j. The destination already
// points at this lane's first element (or its packed byte).
template <bool kPack4>
__device__ __forceinline__ void store_group(const uint32_t (&u)[8], int i, const CodeDst &dst) {
    const uint32_t lo = pack4(u[0], u[1], u[2], u[3]);
    const uint32_t hi = pack4(u[4], u[5], u[6], u[7]);
    if (!kPack4) {
        *reinterpret_cast<uint2 *>(dst.q[i & 1] + 32 * i) = make_uint2(lo, hi);
    } else {
        const uint32_t a = lo & 0x0F0F0F0Fu, b = hi & 0x0F0F0F0Fu;
        const uint32_t a2 = a | (a >> 4), b2 = b | (b >> 4);  // byte pairs -> one byte each
        *reinterpret_cast<uint32_t *>(dst.q[0] + 16 * i) = __byte_perm(a2, b2, 0x6420);
    }
}

// The two rare paths of a group of 8 values out of line (each holds eight
// IEEE divisions), for the kernels whose unrolled loop body is largest (the
// activation table's); inline they timed faster in the plain quantiser.
struct Z8 {
    float v[8];
};
struct U8 {
    uint32_t v[8];
};
// Every value by the definition (rows too small for the fast path).
__device__ __noinline__ U8 codes8_exact(Z8 z, RowQuant rq) {
    U8 u;
#pragma unroll
    for (int k = 0; k < 8; ++k) u.v[k] = code_exact(z.v[k], rq);
    return u;
}
// A flagged group: the values near a half-integer by the definition, the
// others' fast codes recomputed.
__device__ __noinline__ U8 codes8_redo(Z8 z, RowQuant rq) {
    U8 u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float m = __fmaf_rn(z.v[k], rq.rc, kMagic);
        const float d = __fmaf_rn(z.v[k], -rq.rc, __fadd_rn(m, -kMagic));
        u.v[k] = fabsf(d) >= kNearHalf ? code_exact(z.v[k], rq) : __float_as_uint(m);
    }
    return u;
}

__device__ __forceinline__ Z8 group_values(const float2 (&P)[kPairs], int i) {
    Z8 z;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        z.v[2 * k] = P[4 * i + k].x;
        z.v[2 * k + 1] = P[4 * i + k].y;
    }
    return z;
}

template <bool kPack4>
__device__ __forceinline__ void store_group_u8(const U8 &u, int i, const CodeDst &dst) {
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = u.v[k];
    store_group<kPack4>(w, i, dst);
}

template <bool kPack4, bool kOutOfLine>
__device__ __forceinline__ void store_group_exact(const float2 (&P)[kPairs], int i,
                                                  const RowQuant &rq, const CodeDst &dst) {
    if (kOutOfLine) {
        store_group_u8<kPack4>(codes8_exact(group_values(P, i), rq), i, dst);
        return;
    }
    uint32_t u[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        u[2 * k] = code_exact(P[4 * i + k].x, rq);
        u[2 * k + 1] = code_exact(P[4 * i + k].y, rq);
    }
    store_group<kPack4>(u, i, dst);
}

// Quantise lane t's 64 values and store the codes: group i (pairs 4i..4i+3)
// holds 8 consecutive elements, stored as 8 contiguous bytes. The fast path
// stores every group without branching and records which groups hold a value
// near a half-integer; those (rare) groups are then recomputed exactly and
// stored again.
template <bool kPack4 = false, bool kOutOfLine = false>
__device__ __forceinline__ void quantize_store(const float2 (&P)[kPairs], const RowQuant &rq,
                                               int8_t *qbase, int sw5 = 0) {
    const CodeDst dst(qbase, sw5);
    if (!rq.fast) {
#pragma unroll
        for (int i = 0; i < 8; ++i) store_group_exact<kPack4, kOutOfLine>(P, i, rq, dst);
        return;
    }
    const FastQuant fq(rq.rc);
    uint32_t redo = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t u[8];
        float dmax = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 m = fq.code2(P[4 * i + k], dmax);
            u[2 * k] = __float_as_uint(m.x);
            u[2 * k + 1] = __float_as_uint(m.y);
        }
        redo |= uint32_t(dmax >= kNearHalf) << i;
        store_group<kPack4>(u, i, dst);
    }
    if (redo) {
        // In a flagged group only the values near a half-integer take the
        // exact path; the others keep their fast codes (recomputed).
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (!(redo & (1u << i))) continue;
            if (kOutOfLine) {
                store_group_u8<kPack4>(codes8_redo(group_values(P, i), rq), i, dst);
                continue;
            }
            uint32_t u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float z = (k & 1) ? P[4 * i + (k >> 1)].y : P[4 * i + (k >> 1)].x;
                const float m = __fmaf_rn(z, rq.rc, kMagic);
                const float d = __fmaf_rn(z, -rq.rc, __fadd_rn(m, -kMagic));
                u[k] = fabsf(d) >= kNearHalf ? code_exact(z, rq) : __float_as_uint(m);
            }
            store_group<kPack4>(u, i, dst);
        }
    }
}

// ------------------------------------------------------------------ kernels

// Single pass with direct loads: CTA = rows_per_cta rows x (K/256) quads.
template <bool kRotate, int kAct, int kQ, bool kPack4, typename TIn>
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
    // the lane's 8 chunks end at col0 + 232 (its last chunk starts 224 on)
    const bool in_row = CK_CHECK(!active || col0 + 232 <= K, kChkGlobalLoad | kChkGlobalStore);
    float2 P[kPairs];
    if (active && in_row)
        load_block<kAct>(X + row * ldx + col0, P);
    else
        zero_block(P);
    if (kRotate) butterflies(P, t);
    const float m = block_absmax(P);
    __syncthreads();  // s_amax initialised
    if (active && t == 0) atomicMax(&s_amax[row_local], __float_as_uint(m));
    __syncthreads();
    if (!active || !in_row) return;
    const RowQuant rq = row_quant<kRotate, kQ>(__uint_as_float(s_amax[row_local]));
    if (blk == 0 && t == 0) S[row] = rq.s;
    if (kPack4)
        quantize_store<true>(P, rq, Q + row * static_cast<int64_t>(K / 2) + col0 / 2);
    else
        quantize_store<false>(P, rq, Q + row * static_cast<int64_t>(K) + col0);
}

// Persistent single pass for BF16 rows: row groups are staged into shared
// memory with cp.async.bulk kBulkBufs groups ahead (one buffer each). One CTA
// barrier per group: after it, every thread has read its values out of the
// buffer (so the buffer can be refilled) and the row absmax is complete. The absmax slots are
// triple-buffered so a slot is cleared one full barrier before its next use.
template <bool kRotate, int kAct, int kQ>
__global__ void __launch_bounds__(kMaxThreads, 1)
quant_rows_bulk_kernel(const uint16_t *__restrict__ X, int64_t M, int K, int64_t ldx,
                       int rows_per_cta, int8_t *__restrict__ Q, float *__restrict__ S,
                       unsigned *err, uint64_t limit_ns) {
    extern __shared__ __align__(128) uint8_t stage_raw[];
    __shared__ unsigned s_amax[3][kMaxRowsPerCta];
    __shared__ __align__(8) uint64_t full[kBulkBufs];
    constexpr bool kTab = kAct == kActSilu || kAct == kActGeluTanh;
    __shared__ uint32_t act_tab[kTab ? kActTabWords : 1];
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int R = rows_per_cta;
    const int row_local = quad / nb;
    const int blk = quad - row_local * nb;
    const int col0 = blk * kBlock + 8 * t;
    const int sw5 = quad & 1;  // chunk swizzle of this lane (see load_block_smem)
    if (kTab) act_table_fill<kAct>(act_tab, tid, blockDim.x);
    const int64_t ngroups = (M + R - 1) / R;
    const uint32_t row_bytes = uint32_t(K) * 2u;
    const uint32_t buf0 = smem_u32(stage_raw);
    const uint32_t buf_bytes = uint32_t(R) * row_bytes;

    // The per-row work of a group (staging the row, clearing its absmax slot,
    // storing its scale) falls to the row's leader, lane t = 0 of its block
    // 0, so no one warp does all of it and reaches the CTA barrier late. A
    // buffer's mbarrier expects one arrival per row slot.
    const bool leader = row_local < R && blk == 0 && t == 0;
    if (tid == 0) {
        for (int j = 0; j < kBulkBufs; ++j) mbar_init(smem_u32(&full[j]), uint32_t(R));
        fence_mbar_init();
    }
    for (int i = tid; i < 3 * kMaxRowsPerCta; i += blockDim.x) (&s_amax[0][0])[i] = 0u;
    __syncthreads();

    // A leader: stage its row of group g into buffer b (past the last row it
    // only arrives).
    auto issue = [&](int64_t g, int b) {
        const int64_t r = g * R + row_local;
        const uint32_t bar = smem_u32(&full[b]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_expect_tx(bar, r < M ? row_bytes : 0u);
        if (r >= M) return;
        const uint32_t off = uint32_t(b) * buf_bytes + uint32_t(row_local) * row_bytes;
#ifdef CK_CHECKED
        if (!CK_CHECK(off + row_bytes <= dynamic_smem_bytes(), kChkBulkCopy))
            return;  // the wait on this group then runs out and reports the timeout
#endif
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
            ::"r"(buf0 + off),
            "l"(reinterpret_cast<uint64_t>(X + r * ldx)), "r"(row_bytes), "r"(bar)
            : "memory");
    };

    const int64_t g0 = blockIdx.x;
    const int64_t step = gridDim.x;
    if (leader)
        for (int j = 0; j < kBulkBufs; ++j)
            if (g0 + j * step < ngroups) issue(g0 + j * step, j);
    int slot = 0;  // i % 3
    int b = 0;     // i % kBulkBufs
    uint32_t par = 0;  // (i / kBulkBufs) & 1
    for (int i = 0; g0 + i * step < ngroups; ++i) {
        const int64_t g = g0 + i * step;
        const bool ok = mbar_wait_bounded(smem_u32(&full[b]), par, limit_ns, nullptr);
        const int64_t row = g * R + row_local;
        bool active = ok && row_local < R && row < M;
        float2 P[kPairs];
        const uint32_t sa = buf0 + uint32_t(b) * buf_bytes + uint32_t(row_local) * row_bytes +
                            uint32_t(col0) * 2u;
#ifdef CK_CHECKED
        // the lane reads [sa, sa + 464) of the buffer; its codes span col0 .. col0 + 232
        if (active && !CK_CHECK(sa - buf0 + 464u <= dynamic_smem_bytes() && col0 + 232 <= K,
                                kChkShared))
            active = false;
#endif
        if (active) {
            if (kAct != kActNone)
                load_block_smem_act<kRotate, kAct>(sa, sw5, P,
                                                   reinterpret_cast<const uint16_t *>(act_tab));
            else
                load_block_smem<kRotate>(sa, sw5, P);
        } else {
            zero_block(P);
        }
        if (kRotate) butterflies<true>(P, t, sw5);
        const float m = block_absmax(P);
        if (active && t == 0) atomicMax(&s_amax[slot][row_local], __float_as_uint(m));
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicMax(err, kDevErrTimeout);
            // let a late copy land before the CTA's shared memory is released
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000ull) {
            }
            break;
        }
        // Buffer b has been read by every thread: refill it kBulkBufs groups ahead.
        if (leader && g + kBulkBufs * step < ngroups) issue(g + kBulkBufs * step, b);
        const int clear = slot == 0 ? 2 : slot - 1;  // (i + 2) % 3
        if (leader) s_amax[clear][row_local] = 0u;
        if (active) {
            const RowQuant rq = row_quant<kRotate, kQ>(__uint_as_float(s_amax[slot][row_local]));
            if (blk == 0 && t == 0) S[row] = rq.s;
            quantize_store<false, kAct == kActSilu || kAct == kActGeluTanh>(
                P, rq, Q + row * static_cast<int64_t>(K) + col0, sw5);
        }
        slot = slot == 2 ? 0 : slot + 1;
        if (++b == kBulkBufs) {
            b = 0;
            par ^= 1u;
        }
    }
}

// ------------------------------------------------- input RMSNorm, fused
// int8_linear with its input RMSNorm and residual (comfy-kitchen 0.2.40,
// "Huawei Ascend backend"), the normalisation done inside the quantiser's
// staged load so the normalised rows never reach HBM:
//   h   = bf16_rne(x + r)  (h = x without a residual), written to Rout
//   y_k = the bf16 value nearest to h_k g_k / sqrt(mean(h^2) + eps)
//   then ConvRot256 and the per-row INT8 quantiser on y, as above.
// The residual add is one bf16x2 add: for two bf16 values the rounding of the
// exact sum equals the rounding of the fp32 sum (when the fp32 sum is inexact
// the smaller operand is below 2^-16 of the larger, far under half a bf16
// spacing, so both give the larger operand's neighbourhood the same way).
// The sum of squares runs in double (each h^2 exact): a lane's 64 values in
// order, the quad's four lanes by shuffles, then the row's block partials
// through shared memory in one fixed order (four interleaved chains, combined
// by shuffles), so one row gives one result. inv = 1 / sqrt(ss fl(1 / K) +
// eps) in double, inv32 its fp32 rounding. Fast path per value:
// hg = h g in fp32 (exact while the product is a normal fp32 number: 8-bit
// significands), then a = fl(hg fl(inv32 (1 - 2^-21))) and
// b = fl(hg fl(inv32 (1 + 2^-21))): four roundings of 2^-24 each and inv's
// own error (2^-24 + 2^-36) keep the exact value strictly between a and b.
// Rounding is monotonic, so when a and b round to the same bf16 word, that
// word is the exact value's rounding. A chunk of 8 values is redone in double
// precision (h g exact in double, one product with inv, one rounding to bf16)
// when some value's two words differ (it lies near a bf16 rounding midpoint)
// or its smallest |a| is below T = 2^-125 max(1, inv32): a subnormal h g or a
// shows up there (zeros included, which the double path gives exactly).
// |h inv| <= sqrt(K), so with G = max |g| < 2^16 (the weight vector is staged
// in shared memory when the CTA starts) no product overflows; weights of 2^16
// or more send every value through the double path.
constexpr float kNormLo = 0.99999952316284180f;  // 1 - 2^-21
constexpr float kNormHi = 1.00000047683715820f;  // 1 + 2^-21

struct NormArgs {
    const uint16_t *R;   // residual rows or nullptr
    int64_t ldr;
    uint16_t *Rout;      // residual output or nullptr (may alias X or R)
    int64_t ldo;
    const uint16_t *g;   // weight [K] or nullptr
    float eps;
};

// y of two values (h, g as bf16x2 words) in double precision.
__device__ __forceinline__ uint32_t norm_bf16x2_exact(uint32_t hw, uint32_t gw, double inv) {
    const double lo = double(__uint_as_float(hw << 16)) * double(__uint_as_float(gw << 16));
    const double hi =
        double(__uint_as_float(hw & 0xFFFF0000u)) * double(__uint_as_float(gw & 0xFFFF0000u));
    const __nv_bfloat16 a = __double2bfloat16(lo * inv), b = __double2bfloat16(hi * inv);
    return uint32_t(*reinterpret_cast<const uint16_t *>(&a)) |
           (uint32_t(*reinterpret_cast<const uint16_t *>(&b)) << 16);
}

// The two bf16 halves of a word as doubles (exact).
__device__ __forceinline__ void bf16x2_to_f64(uint32_t w, double &lo, double &hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f64.bf16 %0, l;\n\t"
        "cvt.f64.bf16 %1, h;\n\t}"
        : "=d"(lo), "=d"(hi)
        : "r"(w));
}

__device__ __forceinline__ float min3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Persistent, staged like quant_rows_bulk_kernel: x rows in two buffers
// (two groups ahead), the residual rows in one buffer refilled for the CTA's
// next group as soon as the current group's rows are in registers, then the
// weight vector. Two CTA barriers per group: one before the row's sum of
// squares is read (after it the staging buffers may be refilled), one before
// the row's absmax is read.
template <bool kResidual>
__global__ void __launch_bounds__(kMaxThreads, 1)
quant_norm_bulk_kernel(const uint16_t *__restrict__ X, int64_t M, int K, int64_t ldx,
                       int rows_per_cta, const NormArgs na, int8_t *__restrict__ Q,
                       float *__restrict__ S, unsigned *err, uint64_t limit_ns) {
    extern __shared__ __align__(128) uint8_t stage_raw[];
    __shared__ unsigned s_amax[3][kMaxRowsPerCta];
    __shared__ double s_ss[kMaxThreads / 4];
    __shared__ __align__(8) uint64_t full[3];  // x buffers 0 and 1, the residual buffer
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int R = rows_per_cta;
    const int row_local = quad / nb;
    const int blk = quad - row_local * nb;
    const int col0 = blk * kBlock + 8 * t;
    const int sw5 = quad & 1;
    const int64_t ngroups = (M + R - 1) / R;
    const uint32_t row_bytes = uint32_t(K) * 2u;
    const uint32_t buf0 = smem_u32(stage_raw);
    const uint32_t buf_bytes = uint32_t(R) * row_bytes;
    const uint32_t rbuf = buf0 + 2u * buf_bytes;  // residual rows (single buffer)

    // per-row work of a group falls to the row's leader (lane t = 0 of its
    // block 0), as in quant_rows_bulk_kernel; one arrival per row slot
    const bool leader = row_local < R && blk == 0 && t == 0;
    if (tid == 0) {
        mbar_init(smem_u32(&full[0]), uint32_t(R));
        mbar_init(smem_u32(&full[1]), uint32_t(R));
        mbar_init(smem_u32(&full[2]), uint32_t(R));
        fence_mbar_init();
    }
    for (int i = tid; i < 3 * kMaxRowsPerCta; i += blockDim.x) (&s_amax[0][0])[i] = 0u;
    // the weight vector (1 without one) staged once after the two staging
    // buffers, and G = max |g| (bf16 magnitude bits order like the values)
    __shared__ unsigned s_gmax;
    uint16_t *s_g = reinterpret_cast<uint16_t *>(stage_raw + (kResidual ? 3 : 2) * size_t(buf_bytes));
    const uint32_t sg0 = smem_u32(s_g);
    if (tid == 0) s_gmax = 0u;
    __syncthreads();
    {
        unsigned gm = 0u;
        for (int k = 8 * tid; k < K; k += 8 * blockDim.x) {
            uint4 v = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
            if (na.g) v = __ldg(reinterpret_cast<const uint4 *>(na.g + k));
            *reinterpret_cast<uint4 *>(s_g + k) = v;
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                gm = max(gm, max(w[q] & 0x7FFFu, (w[q] >> 16) & 0x7FFFu));
        }
        if (gm) atomicMax(&s_gmax, gm);
    }
    __syncthreads();

    // A leader: stage its row of group g (x, or the residual when res) into
    // the buffer at dst, completing on barrier `bar` (past the last row it
    // only arrives).
    auto issue = [&](int64_t g, bool res, uint32_t dst, uint32_t bar) {
        const int64_t r = g * R + row_local;
        const uint16_t *src = res ? na.R : X;
        const int64_t ld = res ? na.ldr : ldx;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_expect_tx(bar, r < M ? row_bytes : 0u);
        if (r >= M) return;
        const uint32_t d = dst + uint32_t(row_local) * row_bytes;
#ifdef CK_CHECKED
        if (!CK_CHECK(d + row_bytes - buf0 <= dynamic_smem_bytes(), kChkBulkCopy))
            return;  // the wait on this group then runs out and reports the timeout
#endif
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
            ::"r"(d), "l"(reinterpret_cast<uint64_t>(src + r * ld)), "r"(row_bytes), "r"(bar)
            : "memory");
    };

    const int64_t g0 = blockIdx.x;
    const int64_t step = gridDim.x;
    if (leader) {
        if (g0 < ngroups) {
            issue(g0, false, buf0, smem_u32(&full[0]));
            if (kResidual) issue(g0, true, rbuf, smem_u32(&full[2]));
        }
        if (g0 + step < ngroups) issue(g0 + step, false, buf0 + buf_bytes, smem_u32(&full[1]));
    }
    const double inv_k = 1.0 / double(K);  // mean = sum * fl(1 / K): within the bound
    int slot = 0;
    for (int i = 0; g0 + i * step < ngroups; ++i) {
        const int64_t g = g0 + i * step;
        const int b = i & 1;
        bool ok = mbar_wait_bounded(smem_u32(&full[b]), uint32_t(i >> 1) & 1u, limit_ns, nullptr);
        if (kResidual)
            ok = ok && mbar_wait_bounded(smem_u32(&full[2]), uint32_t(i) & 1u, limit_ns, nullptr);
        const int64_t row = g * R + row_local;
        bool active = ok && row_local < R && row < M;
        const uint32_t rowoff = uint32_t(row_local) * row_bytes + uint32_t(col0) * 2u;
#ifdef CK_CHECKED
        // x, the residual and the weight: [.. + rowoff, + 464) of their buffers;
        // the residual output and the codes: columns col0 .. col0 + 232 of the row
        if (active && !CK_CHECK((kResidual ? rbuf : buf0 + uint32_t(b) * buf_bytes) + rowoff + 464u -
                                        buf0 <= dynamic_smem_bytes() &&
                                    sg0 + 2u * uint32_t(col0) + 464u - buf0 <= dynamic_smem_bytes() &&
                                    col0 + 232 <= K,
                                kChkShared))
            active = false;
#endif
        const uint32_t sx = buf0 + uint32_t(b) * buf_bytes + rowoff;
        // h of this lane's 64 values (register group i = chunk i ^ sw5),
        // stored as the residual output, and its sum of squares (one
        // accumulator per chunk, combined in chunk order)
        uint32_t hw[kPairs];
        double acc[8];
        if (active) {
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8)
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(hw[4 * i8]), "=r"(hw[4 * i8 + 1]), "=r"(hw[4 * i8 + 2]),
                               "=r"(hw[4 * i8 + 3])
                             : "r"(sx + 64u * uint32_t(i8 ^ sw5)));
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8) {
                const int c = i8 ^ sw5;
                if (kResidual) {
                    uint32_t rw[4];
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(rw[0]), "=r"(rw[1]), "=r"(rw[2]), "=r"(rw[3])
                                 : "r"(rbuf + rowoff + 64u * uint32_t(c)));
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __nv_bfloat162 s2 =
                            __hadd2(*reinterpret_cast<const __nv_bfloat162 *>(&hw[4 * i8 + q]),
                                    *reinterpret_cast<const __nv_bfloat162 *>(&rw[q]));
                        hw[4 * i8 + q] = *reinterpret_cast<const uint32_t *>(&s2);
                    }
                }
                if (na.Rout)
                    *reinterpret_cast<uint4 *>(na.Rout + row * na.ldo + col0 + 32 * c) =
                        make_uint4(hw[4 * i8], hw[4 * i8 + 1], hw[4 * i8 + 2], hw[4 * i8 + 3]);
                double a = 0.0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    double lo, hi;
                    bf16x2_to_f64(hw[4 * i8 + q], lo, hi);
                    a = __fma_rn(lo, lo, a);
                    a = __fma_rn(hi, hi, a);
                }
                acc[i8] = a;
            }
        } else {
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8) acc[i8] = 0.0;
        }
        const double ss0 = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
        const double ss1 = __dadd_rn(__dadd_rn(acc[4], acc[5]), __dadd_rn(acc[6], acc[7]));
        double ss = __dadd_rn(ss0, ss1);
        ss = __dadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, 1));
        ss = __dadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, 2));
        if (active && t == 0) s_ss[quad] = ss;
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicMax(err, kDevErrTimeout);
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000ull) {
            }
            break;
        }
        // every thread has its values in registers: refill x buffer b two
        // groups ahead and the residual buffer for the next group
        if (leader) {
            if (g + 2 * step < ngroups) issue(g + 2 * step, false, buf0 + uint32_t(b) * buf_bytes,
                                              smem_u32(&full[b]));
            if (kResidual && g + step < ngroups) issue(g + step, true, rbuf, smem_u32(&full[2]));
        }
        const int clear = slot == 0 ? 2 : slot - 1;
        if (leader) s_amax[clear][row_local] = 0u;

        // the row's sum of squares from its blocks' partial sums: lane t of
        // each quad adds the partials t, t + 4, t + 8, ... in that order, and
        // the quad combines its four chains as (c0 + c1) + (c2 + c3). One
        // fixed order, so every quad of the row gets the same sum.
        double ssr = 0.0;
        if (active) {
            const double *part = &s_ss[row_local * nb];
            for (int q = t; q < nb; q += 4) ssr = __dadd_rn(ssr, part[q]);
        }
        ssr = __dadd_rn(ssr, __shfl_xor_sync(0xFFFFFFFFu, ssr, 1));
        ssr = __dadd_rn(ssr, __shfl_xor_sync(0xFFFFFFFFu, ssr, 2));

        float2 P[kPairs];
        if (active) {
            const double inv = rsqrt(__dmul_rn(ssr, inv_k) + double(na.eps));
            const float inv32 = __double2float_rn(inv);
            const float ilo = __fmul_rn(inv32, kNormLo), ihi = __fmul_rn(inv32, kNormHi);
            const float2 lo2 = make_float2(ilo, ilo), hi2 = make_float2(ihi, ihi);
            // T, or +inf (every chunk redone) when G >= 2^16 or not finite
            const float tiny = s_gmax < 0x4780u
                                   ? fmaxf(1.0f, inv32) * 2.3509887016445750e-38f
                                   : __uint_as_float(0x7F800000u);
            // per chunk: the fast path for its 4 words, the chunk again in
            // double when flagged, then the widening fused with h = 1
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8) {
                uint32_t gw[4];
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(gw[0]), "=r"(gw[1]), "=r"(gw[2]), "=r"(gw[3])
                             : "r"(sg0 + 2u * uint32_t(col0 + 32 * (i8 ^ sw5))));
                uint32_t yw[4];
                uint32_t diff = 0u;
                float amin = __uint_as_float(0x7F800000u);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 hg = __fmul2_rn(widen_bf16x2(hw[4 * i8 + q]), widen_bf16x2(gw[q]));
                    const float2 a = __fmul2_rn(hg, lo2), b = __fmul2_rn(hg, hi2);
                    const __nv_bfloat162 ra = __floats2bfloat162_rn(a.x, a.y);
                    const __nv_bfloat162 rb = __floats2bfloat162_rn(b.x, b.y);
                    const uint32_t wa = *reinterpret_cast<const uint32_t *>(&ra);
                    yw[q] = wa;
                    diff |= wa ^ *reinterpret_cast<const uint32_t *>(&rb);
                    amin = min3(amin, fabsf(a.x), fabsf(a.y));
                }
                if (diff != 0u || amin < tiny) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) yw[q] = norm_bf16x2_exact(hw[4 * i8 + q], gw[q], inv);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) P[4 * i8 + q] = widen_stage1(yw[q]);
            }
        } else {
            zero_block(P);
        }
        butterflies<true>(P, t, sw5);
        const float m = block_absmax(P);
        if (active && t == 0) atomicMax(&s_amax[slot][row_local], __float_as_uint(m));
        __syncthreads();
        if (active) {
            const RowQuant rq = row_quant<true, 127>(__uint_as_float(s_amax[slot][row_local]));
            if (blk == 0 && t == 0) S[row] = rq.s;
            quantize_store(P, rq, Q + row * static_cast<int64_t>(K) + col0, sw5);
        }
        slot = slot == 2 ? 0 : slot + 1;
    }
}

// Two passes for long rows (K > 32768): one CTA per row, 128 quads; pass 1
// rotates every block and reduces the absmax, pass 2 reloads (from L2),
// rotates again and quantises.
template <bool kRotate, int kAct, int kQ, bool kPack4, typename TIn>
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
        float2 P[kPairs];
        if (blk < nb && CK_CHECK(row < M && blk * kBlock + 8 * t + 232 <= K, kChkGlobalLoad))
            load_block<kAct>(xrow + blk * kBlock + 8 * t, P);
        else
            zero_block(P);
        if (kRotate) butterflies(P, t);
        m = fmaxf(m, block_absmax(P));
    }
    __syncthreads();
    if (t == 0) atomicMax(&s_amax, __float_as_uint(m));
    __syncthreads();
    const RowQuant rq = row_quant<kRotate, kQ>(__uint_as_float(s_amax));
    if (tid == 0) S[row] = rq.s;
    for (int b0 = 0; b0 < nb; b0 += kTwoPassQuads) {
        const int blk = b0 + quad;
        float2 P[kPairs];
        if (blk < nb && CK_CHECK(row < M && blk * kBlock + 8 * t + 232 <= K, kChkGlobalLoad))
            load_block<kAct>(xrow + blk * kBlock + 8 * t, P);
        else
            zero_block(P);
        if (kRotate) butterflies(P, t);
        if (blk < nb) {
            if (kPack4)
                quantize_store<true>(P, rq, Q + row * static_cast<int64_t>(K / 2) +
                                                (blk * kBlock + 8 * t) / 2);
            else
                quantize_store<false>(P, rq, Q + row * static_cast<int64_t>(K) + blk * kBlock + 8 * t);
        }
    }
}

// Rows per CTA: the CTA has lanes * nb * R useful threads rounded up to whole
// warps; pick the R with the fewest idle lanes, then the CTA size closest to
// `target` threads, with at most max_rows rows and max_threads threads.
int pick_rows_per_cta(int nb, int lanes, int max_rows, int max_threads, int target,
                      int *threads_out) {
    int best_r = 1, best_t = ((lanes * nb + 31) / 32) * 32;
    double best_waste = 2.0;
    int best_dist = 1 << 30;
    for (int r = 1; r <= max_rows && lanes * nb * r <= max_threads; ++r) {
        const int used = lanes * nb * r;
        const int threads = ((used + 31) / 32) * 32;
        if (threads > max_threads) break;
        const double waste = double(threads - used) / threads;
        const int dist = threads > target ? threads - target : target - threads;
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

std::mutex g_occ_mutex;
// (device, rotate, threads, smem) -> CTAs of the bulk kernel per SM
std::map<std::tuple<int, int, int, size_t>, int> g_bulk_occupancy;

template <bool kRotate, int kAct, int kQ>
cudaError_t bulk_blocks_per_sm(int dev, int threads, size_t smem, int *out) {
    std::lock_guard<std::mutex> lock(g_occ_mutex);
    const auto key = std::make_tuple(dev, (kRotate ? 1 : 0) + 2 * kAct + 16 * kQ, threads, smem);
    auto it = g_bulk_occupancy.find(key);
    if (it != g_bulk_occupancy.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(quant_rows_bulk_kernel<kRotate, kAct, kQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kBulkSmemBudget));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_rows_bulk_kernel<kRotate, kAct, kQ>,
                                                      threads, smem);
    if (e != cudaSuccess) return e;
    g_bulk_occupancy[key] = per_sm;
    *out = per_sm;
    return cudaSuccess;
}

template <bool kRotate, int kAct, int kQ>
cudaError_t launch_bulk(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, int8_t *Q, float *S,
                        unsigned *err, int num_sms, cudaStream_t stream, bool *launched) {
    *launched = false;
    const int nb = static_cast<int>(K / kBlock);
    const int max_rows = std::min(static_cast<int>(kBulkSmemBudget / (kBulkBufs * size_t(K) * 2)),
                                  kMaxRowsPerCta);
    if (max_rows < 1 || 4 * nb > kMaxThreads) return cudaSuccess;
    int threads = 0;
    const int rows = pick_rows_per_cta(nb, 4, max_rows, kMaxThreads, 256, &threads);
    const size_t smem = kBulkBufs * size_t(rows) * size_t(K) * 2;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = bulk_blocks_per_sm<kRotate, kAct, kQ>(dev, threads, smem, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaSuccess;
    const int64_t groups = (M + rows - 1) / rows;
    const int64_t cap = int64_t(per_sm) * num_sms;
    const unsigned grid = static_cast<unsigned>(groups < cap ? groups : cap);
    quant_rows_bulk_kernel<kRotate, kAct, kQ><<<grid, threads, smem, stream>>>(
        X, M, static_cast<int>(K), ldx, rows, Q, S, err, kDefaultWaitLimitNs);
    *launched = true;
    return cudaGetLastError();
}

template <bool kRotate, int kAct, int kQ, bool kPack4, typename TIn>
cudaError_t launch_direct(const TIn *X, int64_t M, int64_t K, int64_t ldx, int8_t *Q, float *S,
                          cudaStream_t stream) {
    const int nb = static_cast<int>(K / kBlock);
    if (4 * nb <= kMaxThreads) {
        int threads = 0;
        const int rows = pick_rows_per_cta(nb, 4, kMaxRowsPerCta, kMaxThreads, 256, &threads);
        const int64_t grid = (M + rows - 1) / rows;
        quant_rows_kernel<kRotate, kAct, kQ, kPack4, TIn><<<static_cast<unsigned>(grid), threads, 0, stream>>>(
            X, M, static_cast<int>(K), ldx, rows, Q, S);
    } else {
        quant_rows_two_pass_kernel<kRotate, kAct, kQ, kPack4, TIn>
            <<<static_cast<unsigned>(M), kTwoPassQuads * 4, 0, stream>>>(
                X, M, static_cast<int>(K), ldx, Q, S);
    }
    return cudaGetLastError();
}

template <bool kRotate, int kAct, int kQ = 127>
cudaError_t launch_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, int8_t *Q, float *S,
                        unsigned *err, int num_sms, cudaStream_t stream) {
    bool launched = false;
    cudaError_t e =
        launch_bulk<kRotate, kAct, kQ>(X, M, K, ldx, Q, S, err, num_sms, stream, &launched);
    if (e != cudaSuccess || launched) return e;
    return launch_direct<kRotate, kAct, kQ, false>(X, M, K, ldx, Q, S, stream);
}

// Packed signed INT4 [rows, K/2] -> int8 codes [rows, K]: 16 bytes in, 32 out
// per thread; nibbles sign-extended per byte ((x ^ 8) - 8, byte-wise SIMD).
__global__ void unpack_int4_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out,
                                   int64_t n16) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
         i += int64_t(gridDim.x) * blockDim.x) {
        const uint4 v = __ldcs(in + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo = __vsub4((w[j] & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
            const uint32_t hi = __vsub4(((w[j] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
            o[2 * j] = __byte_perm(lo, hi, 0x5140);
            o[2 * j + 1] = __byte_perm(lo, hi, 0x7362);
        }
        out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
        out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// ------------------------------------------------------------------ NVFP4
// ConvRot NVFP4 (ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix",
// section 5-1: FP4 E2M1 codes, one E4M3 scale per 16 values, the 128 x 4
// blocked scale layout, a per-tensor scale). On the ConvRot256-rotated rows:
//   s_t = amax(tensor) / 2688, b = E4M3_rne_sat((amax(block) / 6) / s_t),
//   d = float(b) * s_t, q = E2M1_rne_sat(y / d) (+0 when d == 0),
// two codes per byte with the lower element in the low nibble. The
// conversions use the hardware's round-to-nearest-even, saturating cvt (the
// E4M3 one gets the same value twice, so its result does not depend on which
// half of the packed pair an operand lands in).

__device__ __forceinline__ uint32_t e4m3_rne_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(v));
    return uint32_t(r) & 0xFFu;
}

// An E4M3 byte's value (sign clear, not NaN): its exponent and mantissa bits
// shifted into fp32's places (b << 20) read as 2^(e - 127) (1 + m / 8), or
// as the subnormal m 2^-129 when e = 0; the exact product with 2^120 gives
// 2^(e - 7) (1 + m / 8) and m 2^-9, E4M3's normal and subnormal values.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    return __fmul_rn(__uint_as_float(b << 20), 1.329227995784916e36f);  // 2^120
}

// Codes of 8 consecutive values y (one half of a 16-value scale block) with
// divisor d = float(b) * s_t, packed into 4 bytes (element 2j in the low
// nibble of byte j). The definition's code is E2M1_rne_sat(fl(y / d)).
// r = rcp.approx(d) is within a few units in the last place of 1 / d (taken
// as at most 2^-21 relative here; the instruction's documented bound is
// tighter), so u = fl(y r) lies within 2^-17.3 of fl(y / d) for |y / d| < 10
// (the block scale's rounding in E4M3's subnormal range leaves at most 1.5x
// headroom over 6). The E2M1 rounding boundaries 0.25, 0.75, ..., 5 are
// multiples of 1/4, so unless some u lies within 2^-16 of a multiple of 1/4,
// u converts to the same codes as the IEEE quotients; the values that are
// that close take the IEEE division. That includes y = +-0 (whose sign the
// code keeps) and, for all 8, a d in fp32's subnormal range (flushed by the
// approximation: r = inf).
// cvt.e2m1x2 puts its first source in the upper nibble; mov packs the four
// bytes low byte first.
// The rare path of nvfp4_encode8, kept out of line (it holds eight IEEE
// divisions): v[k] = fl(y[k] / d) for the values whose u lies within 2^-16
// of a multiple of 1/4 (all of them when r is not finite).
struct F8 {
    float v[8];
};
__device__ __noinline__ F8 nvfp4_encode8_redo(F8 y, F8 v, float r, float d) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float u = __fmul_rn(y.v[k], r);
        const float q = __fadd_rn(__fadd_rn(u, kMagic4), -kMagic4);
        if (!(fabsf(__fadd_rn(u, -q)) >= kNearQuarter)) v.v[k] = __fdiv_rn(y.v[k], d);
    }
    return v;
}

__device__ __forceinline__ uint32_t nvfp4_encode8(const float (&y)[8], float d) {
    if (d == 0.0f) return 0u;
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    const float2 rv = make_float2(r, r);
    const float2 mg = make_float2(kMagic4, kMagic4);
    const float2 nmg = make_float2(-kMagic4, -kMagic4);
    float v[8];
    float dmin = r <= 3.0e38f ? 1.0f : 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 u = __fmul2_rn(make_float2(y[2 * k], y[2 * k + 1]), rv);
        const float2 q = __fadd2_rn(__fadd2_rn(u, mg), nmg);  // nearest multiple of 1/4
        const float2 du = __ffma2_rn(q, make_float2(-1.0f, -1.0f), u);
        float m;
        asm("min.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(dmin), "f"(fabsf(du.x)), "f"(fabsf(du.y)));
        dmin = m;
        v[2 * k] = u.x;
        v[2 * k + 1] = u.y;
    }
    if (dmin < kNearQuarter) {
        // only the values near a multiple of 1/4 take the division (all of
        // them when r is not finite: |du| is then NaN)
        F8 yy, vv;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            yy.v[k] = y[k];
            vv.v[k] = v[k];
        }
        vv = nvfp4_encode8_redo(yy, vv, r, d);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = vv.v[k];
    }
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return out;
}

// fl(1 / fl(6 s_t)) for nvfp4_block_scale, or 0 when s_t is 0 or the
// reciprocal is not finite (every block then takes the exact divisions).
__device__ __forceinline__ float nvfp4_scale_rcp(float s_t) {
    if (!(s_t > 0.0f)) return 0.0f;
    const float c = __frcp_rn(__fmul_rn(6.0f, s_t));
    return c <= 3.0e38f ? c : 0.0f;
}

// Block scale b = E4M3_rne_sat(fl(fl(m / 6) / s_t)) of a block with absmax m.
// q = fl(m c6) is within 5 units in the last place of the two divisions'
// result (five roundings of relative size 2^-24 between them). In E4M3's
// normal range [2^-6, 448] the rounding keeps 3 of fp32's 23 mantissa bits,
// so q rounds as that result does unless its low 20 mantissa bits lie within
// 8 units of the half-way pattern 0x80000. Those blocks, values below 2^-6
// (E4M3's subnormal range, where the rounding position moves) and c6 = 0
// take the two IEEE divisions.
__device__ __noinline__ uint32_t nvfp4_block_scale_exact(float m, float s_t) {
    return e4m3_rne_sat(__fdiv_rn(__fdiv_rn(m, 6.0f), s_t));
}

__device__ __forceinline__ uint32_t nvfp4_block_scale(float m, float s_t, float c6) {
    if (!(s_t > 0.0f)) return 0u;
    const float q = __fmul_rn(m, c6);
    const uint32_t low = __float_as_uint(q) & 0xFFFFFu;
    if (q >= 0.0156265625f && low - 0x7FFF8u >= 16u) return e4m3_rne_sat(q);
    return nvfp4_block_scale_exact(m, s_t);
}

// Scale blocks of register groups c and c + 1 (c even) of a lane. The lanes
// t and t ^ 1 each hold 8 of a block's 16 values; the lane with t & 1 = 0
// computes the scale of group c's block and the other that of group c + 1's,
// and they swap the results. Returns the two packed code words (8 codes
// each); *b_own is the scale this lane computed, which it stores.
__device__ __forceinline__ uint2 nvfp4_codes_pair(const float2 (&P)[kPairs], int c, int t,
                                                  float s_t, float c6, uint32_t *b_own) {
    float y[2][8];
    float m8[2] = {0.0f, 0.0f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 z = __fmul2_rn(P[4 * (c + h) + k], make_float2(0.0625f, 0.0625f));
            y[h][2 * k] = z.x;
            y[h][2 * k + 1] = z.y;
            m8[h] = max3(m8[h], fabsf(z.x), fabsf(z.y));
        }
    }
    const float m0 = fmaxf(m8[0], __shfl_xor_sync(0xFFFFFFFFu, m8[0], 1));
    const float m1 = fmaxf(m8[1], __shfl_xor_sync(0xFFFFFFFFu, m8[1], 1));
    const bool odd = (t & 1) != 0;
    const uint32_t mine = nvfp4_block_scale(odd ? m1 : m0, s_t, c6);
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, mine, 1);
    const uint32_t b0 = odd ? other : mine;
    const uint32_t b1 = odd ? mine : other;
    *b_own = mine;
    return make_uint2(nvfp4_encode8(y[0], __fmul_rn(e4m3_to_f32(b0), s_t)),
                      nvfp4_encode8(y[1], __fmul_rn(e4m3_to_f32(b1), s_t)));
}

// Offset of the scale of row r, scale column c (of C) in the blocked layout:
// 512-byte tiles of 128 rows x 4 columns, column tiles fastest; rows r, r + 32,
// r + 64, r + 96 of a tile share the 16-byte line r % 32.
__device__ __forceinline__ bool nvfp4_sf_in_range(int64_t off, int64_t M, int C) {
    return CK_CHECK(off >= 0 && off < ((M + 127) / 128) * 128 * int64_t((C + 3) / 4 * 4),
                    kChkGlobalStore);
}

__device__ __forceinline__ int64_t nvfp4_sf_offset(int64_t r, int c, int C) {
    const int64_t tile = (r >> 7) * int64_t((C + 3) >> 2) + (c >> 2);
    return tile * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// Pass 1: absmax of the rotated tensor (of z = 16 y), as the bits of a
// non-negative float, atomicMax'ed into *amax_bits (zeroed before).
template <typename TIn>
__global__ void __launch_bounds__(kMaxThreads, 1)
nvfp4_amax_kernel(const TIn *__restrict__ X, int64_t M, int K, int64_t ldx, int rows_per_cta,
                  unsigned *amax_bits) {
    __shared__ unsigned s_max;
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int row_local = quad / nb;
    const int blk = quad - row_local * nb;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + row_local;
    const bool active = row_local < rows_per_cta && row < M &&
                        CK_CHECK(blk * kBlock + 8 * t + 232 <= K, kChkGlobalLoad);
    if (tid == 0) s_max = 0u;
    float2 P[kPairs];
    if (active)
        load_block<kActNone>(X + row * ldx + blk * kBlock + 8 * t, P);
    else
        zero_block(P);
    butterflies(P, t);
    const float m = block_absmax(P);
    __syncthreads();
    if (active && t == 0) atomicMax(&s_max, __float_as_uint(m));
    __syncthreads();
    if (tid == 0 && s_max != 0u) atomicMax(amax_bits, s_max);
}

// Pass 2: block scales and codes. Lane t of a quad holds elements
// 8t + 32i .. +7 of its 256-block (chunk i); a 16-value scale block is chunk
// i of lanes t and t ^ 1.
template <typename TIn>
__global__ void __launch_bounds__(kMaxThreads, 1)
nvfp4_quant_kernel(const TIn *__restrict__ X, int64_t M, int K, int64_t ldx, int rows_per_cta,
                   const unsigned *__restrict__ amax_bits, uint8_t *__restrict__ Q,
                   uint8_t *__restrict__ S) {
    const int tid = threadIdx.x;
    const int t = tid & 3;
    const int quad = tid >> 2;
    const int nb = K >> 8;
    const int row_local = quad / nb;
    const int blk = quad - row_local * nb;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + row_local;
    const int col0 = blk * kBlock + 8 * t;
    const bool active = row_local < rows_per_cta && row < M &&
                        CK_CHECK(col0 + 232 <= K, kChkGlobalLoad | kChkGlobalStore);
    float2 P[kPairs];
    if (active)
        load_block<kActNone>(X + row * ldx + col0, P);
    else
        zero_block(P);
    butterflies(P, t);
    const float amax = __fmul_rn(__uint_as_float(*amax_bits), 0.0625f);
    const float s_t = __fdiv_rn(amax, 2688.0f);
    const float c6 = nvfp4_scale_rcp(s_t);
    const int C = K >> 4;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        uint32_t b;
        const uint2 packed = nvfp4_codes_pair(P, i, t, s_t, c6, &b);
        if (active) {
            const int e0 = col0 + 32 * i;
            uint8_t *qr = Q + row * int64_t(K / 2);
            *reinterpret_cast<uint32_t *>(qr + e0 / 2) = packed.x;
            *reinterpret_cast<uint32_t *>(qr + (e0 + 32) / 2) = packed.y;
            const int64_t so = nvfp4_sf_offset(row, (e0 + 32 * (t & 1)) >> 4, C);
            if (nvfp4_sf_in_range(so, M, C)) S[so] = uint8_t(b);
        }
    }
}

// Staged, persistent variant of the two NVFP4 passes for bf16 rows, with
// staging private to each warp and no CTA barrier in the loop (the passes
// need no reduction over a row, so warps never wait for one another; a CTA
// barrier per row group, as the INT8 quantiser has, cost pass 2 more than
// two stalled warps per issued instruction). The row-major sequence of
// 256-blocks (block b = row nb + blk) is cut into units of 8 consecutive
// blocks; warp gw of the grid takes units gw, gw + W, gw + 2W, ... (W warps
// in the grid), and quad q of the warp takes block q of the unit. Each warp
// stages its units in kNvWarpBufs 4 KB buffers of its own (one
// cp.async.bulk per run of blocks within one row, completing on the
// buffer's mbarrier) and refills a buffer as soon as its own lanes have read
// it (__syncwarp). kPass 1: absmax of the rotated tensor into *amax_bits;
// kPass 2: codes and block scales (as nvfp4_quant_kernel).
constexpr int kNvWarpBufs = 3;
constexpr int kNvUnitBlocks = 8;
constexpr uint32_t kNvUnitBytes = kNvUnitBlocks * 512;
constexpr int kNvWarpThreads = 256;
constexpr int kNvWarpsPerCta = kNvWarpThreads / 32;

template <int kPass>
__global__ void __launch_bounds__(kNvWarpThreads, 2)
nvfp4_warp_kernel(const uint16_t *__restrict__ X, int64_t M, int K, int64_t ldx,
                  unsigned *amax_bits, uint8_t *__restrict__ Q, uint8_t *__restrict__ S,
                  unsigned *err, uint64_t limit_ns) {
    extern __shared__ __align__(128) uint8_t stage_raw[];
    __shared__ __align__(8) uint64_t full[kNvWarpsPerCta][kNvWarpBufs];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t = lane & 3;
    const int qw = lane >> 2;
    const int sw5 = qw & 1;  // chunk swizzle of this quad (see load_block_smem)
    const int nb = K >> 8;
    const int C = K >> 4;
    const int64_t nblocks = M * nb;
    const int64_t nunits = (nblocks + kNvUnitBlocks - 1) / kNvUnitBlocks;
    const int64_t gw = int64_t(blockIdx.x) * kNvWarpsPerCta + warp;
    const int64_t wstep = int64_t(gridDim.x) * kNvWarpsPerCta;
    const uint32_t wbuf = smem_u32(stage_raw) + uint32_t(warp) * kNvWarpBufs * kNvUnitBytes;

    if (lane == 0) {
        for (int j = 0; j < kNvWarpBufs; ++j) mbar_init(smem_u32(&full[warp][j]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    // Blocks advance by 8 wstep per unit of this warp: (row, blk) of a
    // unit's first block are kept incrementally (one division up front).
    const int64_t ustep = int64_t(kNvUnitBlocks) * wstep;
    const int64_t drow = ustep / nb;
    const int dblk = int(ustep - drow * nb);
    auto advance = [&](int64_t &row, int &blk) {
        row += drow;
        blk += dblk;
        if (blk >= nb) {
            blk -= nb;
            ++row;
        }
    };

    // Lane 0: stage unit u (first block at row, blk) into buffer b.
    auto issue = [&](int64_t u, int64_t row, int blk, int b) {
        const int64_t left = nblocks - u * kNvUnitBlocks;
        const int n = int(left < kNvUnitBlocks ? left : kNvUnitBlocks);
        const uint32_t bar = smem_u32(&full[warp][b]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_expect_tx(bar, uint32_t(n) * 512u);
        for (int i = 0; i < n;) {
            const int run = min(n - i, nb - blk);
#ifdef CK_CHECKED
            if (!CK_CHECK(row < M && blk + run <= nb &&
                              (wbuf - smem_u32(stage_raw)) + uint32_t(b) * kNvUnitBytes +
                                      uint32_t(i + run) * 512u <=
                                  dynamic_smem_bytes(),
                          kChkBulkCopy)) {
                i += run;  // the wait on this unit then runs out and reports the timeout
                continue;
            }
#endif
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                ::"r"(wbuf + uint32_t(b) * kNvUnitBytes + uint32_t(i) * 512u),
                "l"(reinterpret_cast<uint64_t>(X + row * ldx + int64_t(blk) * kBlock)),
                "r"(uint32_t(run) * 512u), "r"(bar)
                : "memory");
            i += run;
            blk += run;
            if (blk == nb) {
                blk = 0;
                ++row;
            }
        }
    };

    const int64_t b_first = gw * kNvUnitBlocks;
    int64_t row0 = b_first / nb;  // first block of this warp's current unit
    int blk0 = int(b_first - row0 * nb);
    int64_t irow = row0;           // first block of the next unit to stage
    int iblk = blk0;
    if (lane == 0) {
        for (int j = 0; j < kNvWarpBufs; ++j) {
            if (gw + j * wstep < nunits) issue(gw + j * wstep, irow, iblk, j);
            advance(irow, iblk);
        }
    }
    float s_t = 0.0f;
    if (kPass == 2) s_t = __fdiv_rn(__fmul_rn(__uint_as_float(*amax_bits), 0.0625f), 2688.0f);
    const float c6 = nvfp4_scale_rcp(s_t);
    float local_max = 0.0f;
    int b = 0;
    uint32_t par = 0;
    for (int64_t u = gw; u < nunits; u += wstep) {
        const bool ok = mbar_wait_bounded(smem_u32(&full[warp][b]), par, limit_ns, nullptr);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
            if (lane == 0) atomicMax(err, kDevErrTimeout);
            // let a late copy land before the CTA's shared memory is released
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000ull) {
            }
            break;
        }
        // this quad's block: qw blocks past the unit's first
        int64_t row = row0;
        int blk = blk0 + qw;
        while (blk >= nb) {
            blk -= nb;
            ++row;
        }
        bool active = u * kNvUnitBlocks + qw < nblocks;
#ifdef CK_CHECKED
        // the quad's block in the warp's buffer; the codes and scales of its row
        if (active &&
            !CK_CHECK(row < M && blk < nb &&
                          (wbuf - smem_u32(stage_raw)) + uint32_t(b) * kNvUnitBytes +
                                  uint32_t(qw + 1) * 512u <=
                              dynamic_smem_bytes(),
                      kChkShared))
            active = false;
#endif
        float2 P[kPairs];
        if (active)
            load_block_smem<true>(wbuf + uint32_t(b) * kNvUnitBytes + uint32_t(qw) * 512u +
                                      16u * uint32_t(t),
                                  sw5, P);
        else
            zero_block(P);
        __syncwarp();
        if (lane == 0 && u + kNvWarpBufs * wstep < nunits)
            issue(u + kNvWarpBufs * wstep, irow, iblk, b);
        if (lane == 0) advance(irow, iblk);
        advance(row0, blk0);
        butterflies<true>(P, t, sw5);
        if constexpr (kPass == 1) {
            // the lane's own maximum; the lanes are combined once, at the end
            local_max = fmaxf(local_max, block_absmax<1>(P));
        } else {
            // register group i holds chunk i ^ sw5: elements col0 + 32 (i ^ sw5) .. + 7
            const int col0 = blk * kBlock + 8 * t;
            uint8_t *qr = Q + row * int64_t(K / 2);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                uint32_t bsc;
                const uint2 packed = nvfp4_codes_pair(P, c, t, s_t, c6, &bsc);
                if (active) {
                    const int ea = col0 + 32 * (c + sw5);      // group c
                    const int eb = col0 + 32 * (c + 1 - sw5);  // group c + 1
                    *reinterpret_cast<uint32_t *>(qr + ea / 2) = packed.x;
                    *reinterpret_cast<uint32_t *>(qr + eb / 2) = packed.y;
                    const int64_t so = nvfp4_sf_offset(row, ((t & 1) ? eb : ea) >> 4, C);
                    if (nvfp4_sf_in_range(so, M, C)) S[so] = uint8_t(bsc);
                }
            }
        }
        if (++b == kNvWarpBufs) {
            b = 0;
            par ^= 1u;
        }
    }
    if (kPass == 1) {
        float m = local_max;
#pragma unroll
        for (int l = 1; l < 32; l <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, l));
        if (lane == 0 && m > 0.0f) atomicMax(amax_bits, __float_as_uint(m));
    }
}

// Turns the absmax bits of z into the per-tensor scale, in place.
__global__ void nvfp4_scale_kernel(float *s_t) {
    const float amax = __fmul_rn(__uint_as_float(*reinterpret_cast<unsigned *>(s_t)), 0.0625f);
    *s_t = __fdiv_rn(amax, 2688.0f);
}

// Decoding: value = e2m1(code) * (s_t * e4m3(scale)); 8 values per thread.
__global__ void nvfp4_dequant_kernel(const uint8_t *__restrict__ Q, const uint8_t *__restrict__ S,
                                     const float *__restrict__ s_t, int64_t rows, int K,
                                     int hi_first, float *__restrict__ out) {
    const int C = K >> 4;
    const int64_t groups = rows * int64_t(K / 8);
    const float st = *s_t;
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
         g += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = g / (K / 8);
        const int k0 = int(g - r * (K / 8)) * 8;
        const uint32_t w = *reinterpret_cast<const uint32_t *>(Q + r * int64_t(K / 2) + k0 / 2);
        const int64_t so = nvfp4_sf_offset(r, k0 >> 4, C);
        if (!CK_CHECK(so < ((rows + 127) / 128) * 128 * int64_t((C + 3) / 4 * 4), kChkGlobalLoad))
            continue;
        const float scale = __fmul_rn(st, e4m3_to_f32(S[so]));
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t byte = (w >> (8 * (j >> 1))) & 0xFFu;
            const bool high = ((j & 1) == 0) == (hi_first != 0);
            const uint32_t c = high ? (byte >> 4) : (byte & 15u);
            const uint32_t e = (c >> 1) & 3u, mbit = c & 1u;
            float mag = e == 0 ? 0.5f * float(mbit) : __uint_as_float((e + 126u) << 23) * (1.0f + 0.5f * float(mbit));
            v[j] = __fmul_rn((c & 8u) ? -mag : mag, scale);
        }
        float4 *o = reinterpret_cast<float4 *>(out + r * int64_t(K) + k0);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

}  // namespace

cudaError_t launch_quant_rows_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   bool rotate, int act, int qmax, int8_t *Q, float *S,
                                   unsigned *err, int num_sms, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    if (!rotate) return launch_bf16<false, kActNone>(X, M, K, ldx, Q, S, err, num_sms, stream);
    if (qmax == 7) return launch_bf16<true, kActNone, 7>(X, M, K, ldx, Q, S, err, num_sms, stream);
    switch (act) {
        case kActRelu: return launch_bf16<true, kActRelu>(X, M, K, ldx, Q, S, err, num_sms, stream);
        case kActSilu: return launch_bf16<true, kActSilu>(X, M, K, ldx, Q, S, err, num_sms, stream);
        case kActGeluTanh:
            return launch_bf16<true, kActGeluTanh>(X, M, K, ldx, Q, S, err, num_sms, stream);
        default: return launch_bf16<true, kActNone>(X, M, K, ldx, Q, S, err, num_sms, stream);
    }
}

template <bool kResidual>
cudaError_t launch_norm_bulk(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                             const NormArgs &na, int8_t *Q, float *S, unsigned *err, int num_sms,
                             cudaStream_t stream, bool *launched) {
    *launched = false;
    const int nb = static_cast<int>(K / kBlock);
    // per row: two x buffers (+ one residual buffer); then the weight vector
    const size_t per_row = 2 * size_t(K) * (kResidual ? 3 : 2);
    const int max_rows = std::min(static_cast<int>(kBulkSmemBudget / per_row), kMaxRowsPerCta);
    if (max_rows < 1 || 4 * nb > kMaxThreads) return cudaSuccess;
    int threads = 0;
    const int rows = pick_rows_per_cta(nb, 4, max_rows, kMaxThreads, 256, &threads);
    const size_t smem = size_t(rows) * per_row + 2 * size_t(K);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lock(g_occ_mutex);
        const auto key = std::make_tuple(dev, 1000 + (kResidual ? 1 : 0), threads, smem);
        auto it = g_bulk_occupancy.find(key);
        if (it != g_bulk_occupancy.end()) {
            per_sm = it->second;
        } else {
            e = cudaFuncSetAttribute(quant_norm_bulk_kernel<kResidual>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(kBulkSmemBudget + 2 * 14336));
            if (e != cudaSuccess) return e;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, quant_norm_bulk_kernel<kResidual>, threads, smem);
            if (e != cudaSuccess) return e;
            g_bulk_occupancy[key] = per_sm;
        }
    }
    if (per_sm < 1) return cudaSuccess;
    const int64_t groups = (M + rows - 1) / rows;
    const int64_t cap = int64_t(per_sm) * num_sms;
    const unsigned grid = static_cast<unsigned>(groups < cap ? groups : cap);
    quant_norm_bulk_kernel<kResidual><<<grid, threads, smem, stream>>>(
        X, M, static_cast<int>(K), ldx, rows, na, Q, S, err, kDefaultWaitLimitNs);
    *launched = true;
    return cudaGetLastError();
}

cudaError_t launch_quant_norm_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   const uint16_t *R, int64_t ldr, uint16_t *Rout, int64_t ldo,
                                   const uint16_t *g, float eps, int8_t *Q, float *S,
                                   unsigned *err, int num_sms, cudaStream_t stream,
                                   bool *launched) {
    *launched = false;
    if (M <= 0) {
        *launched = true;
        return cudaSuccess;
    }
    const NormArgs na{R, ldr, Rout, ldo, g, eps};
    if (R) return launch_norm_bulk<true>(X, M, K, ldx, na, Q, S, err, num_sms, stream, launched);
    return launch_norm_bulk<false>(X, M, K, ldx, na, Q, S, err, num_sms, stream, launched);
}

cudaError_t launch_test_row_quant_params(const float *amax, int64_t n, int q, float *div,
                                         float *rc, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const int64_t want = (n + 255) / 256;
    const unsigned grid = unsigned(want < 148 * 16 ? want : 148 * 16);
    if (q == 7)
        row_quant_params_kernel<7><<<grid, 256, 0, stream>>>(amax, n, div, rc);
    else
        row_quant_params_kernel<127><<<grid, 256, 0, stream>>>(amax, n, div, rc);
    return cudaGetLastError();
}

cudaError_t launch_test_input_act(const uint16_t *X, int64_t n, int act, uint16_t *Y,
                                  cudaStream_t stream) {
    const int64_t n16 = n / 8;  // n % 256 == 0: whole 16-byte chunks
    if (n16 <= 0) return cudaSuccess;
    const unsigned grid = unsigned((n16 + 1023) / 1024);
    const uint4 *x = reinterpret_cast<const uint4 *>(X);
    uint4 *y = reinterpret_cast<uint4 *>(Y);
    switch (act) {
        case kActRelu: input_act_kernel<kActRelu><<<grid, 128, 0, stream>>>(x, y, n16); break;
        case kActSilu: input_act_kernel<kActSilu><<<grid, 128, 0, stream>>>(x, y, n16); break;
        case kActGeluTanh:
            input_act_kernel<kActGeluTanh><<<grid, 128, 0, stream>>>(x, y, n16);
            break;
        default: input_act_kernel<kActNone><<<grid, 128, 0, stream>>>(x, y, n16); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_rows_f32(const float *W, int64_t N, int64_t K, bool int4_packed,
                                  int8_t *Q, float *S, cudaStream_t stream) {
    if (N <= 0) return cudaSuccess;
    if (int4_packed) return launch_direct<true, kActNone, 7, true>(W, N, K, K, Q, S, stream);
    return launch_direct<true, kActNone, 127, false>(W, N, K, K, Q, S, stream);
}

cudaError_t launch_unpack_int4(const uint8_t *Q4, int64_t rows, int64_t K, int8_t *Q8,
                               int num_sms, cudaStream_t stream) {
    const int64_t n16 = rows * (K / 2) / 16;  // K % 256 == 0: whole 16-byte chunks
    if (n16 <= 0) return cudaSuccess;
    const int64_t want = (n16 + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    unpack_int4_kernel<<<unsigned(want < cap ? want : cap), 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(Q4), reinterpret_cast<uint4 *>(Q8), n16);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_nvfp4_impl(const TIn *X, int64_t M, int64_t K, int64_t ldx, uint8_t *Q,
                              uint8_t *S, size_t s_bytes, float *s_t, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    const int nb = static_cast<int>(K / kBlock);
    if (4 * nb > kMaxThreads) return cudaErrorInvalidValue;
    int threads = 0;
    const int rows = pick_rows_per_cta(nb, 4, kMaxRowsPerCta, kMaxThreads, 256, &threads);
    const unsigned grid = static_cast<unsigned>((M + rows - 1) / rows);
    cudaError_t e = cudaMemsetAsync(s_t, 0, sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(S, 0, s_bytes, stream);
    if (e != cudaSuccess) return e;
    nvfp4_amax_kernel<TIn><<<grid, threads, 0, stream>>>(X, M, static_cast<int>(K), ldx, rows,
                                                       reinterpret_cast<unsigned *>(s_t));
    nvfp4_quant_kernel<TIn><<<grid, threads, 0, stream>>>(
        X, M, static_cast<int>(K), ldx, rows, reinterpret_cast<const unsigned *>(s_t), Q, S);
    nvfp4_scale_kernel<<<1, 1, 0, stream>>>(s_t);
    return cudaGetLastError();
}

cudaError_t launch_quant_nvfp4_bf16(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                    uint8_t *Q, uint8_t *S, size_t s_bytes, float *s_t,
                                    unsigned *err, int num_sms, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    const size_t smem = size_t(kNvWarpsPerCta) * kNvWarpBufs * kNvUnitBytes;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lock(g_occ_mutex);
        const auto key = std::make_tuple(dev, 3000, kNvWarpThreads, smem);
        auto it = g_bulk_occupancy.find(key);
        if (it != g_bulk_occupancy.end()) {
            per_sm = it->second;
        } else {
            for (auto *fn : {nvfp4_warp_kernel<1>, nvfp4_warp_kernel<2>}) {
                e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
                if (e != cudaSuccess) return e;
            }
            int p1 = 0, p2 = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p1, nvfp4_warp_kernel<1>, kNvWarpThreads, smem);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p2, nvfp4_warp_kernel<2>, kNvWarpThreads, smem);
            if (e != cudaSuccess) return e;
            per_sm = std::min(p1, p2);
            g_bulk_occupancy[key] = per_sm;
        }
    }
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t units = (M * (K / kBlock) + kNvUnitBlocks - 1) / kNvUnitBlocks;
    const int64_t ctas = (units + kNvWarpsPerCta - 1) / kNvWarpsPerCta;
    const unsigned grid = unsigned(std::min<int64_t>(ctas, int64_t(per_sm) * num_sms));
    e = cudaMemsetAsync(s_t, 0, sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(S, 0, s_bytes, stream);  // the layout's padding
    if (e != cudaSuccess) return e;
    unsigned *amax = reinterpret_cast<unsigned *>(s_t);
    nvfp4_warp_kernel<1><<<grid, kNvWarpThreads, smem, stream>>>(
        X, M, static_cast<int>(K), ldx, amax, Q, S, err, kDefaultWaitLimitNs);
    nvfp4_warp_kernel<2><<<grid, kNvWarpThreads, smem, stream>>>(
        X, M, static_cast<int>(K), ldx, amax, Q, S, err, kDefaultWaitLimitNs);
    nvfp4_scale_kernel<<<1, 1, 0, stream>>>(s_t);
    return cudaGetLastError();
}

cudaError_t launch_quant_nvfp4_f32(const float *W, int64_t N, int64_t K, uint8_t *Q, uint8_t *S,
                                   size_t s_bytes, float *s_t, cudaStream_t stream) {
    return launch_nvfp4_impl(W, N, K, K, Q, S, s_bytes, s_t, stream);
}

cudaError_t launch_dequant_nvfp4(const uint8_t *Q, const uint8_t *S, const float *s_t,
                                 int64_t rows, int64_t K, bool hi_first, float *out, int num_sms,
                                 cudaStream_t stream) {
    const int64_t groups = rows * (K / 8);
    if (groups <= 0) return cudaSuccess;
    const int64_t want = (groups + 255) / 256;
    const int64_t cap = int64_t(num_sms) * 8;
    nvfp4_dequant_kernel<<<unsigned(want < cap ? want : cap), 256, 0, stream>>>(
        Q, S, s_t, rows, static_cast<int>(K), hi_first ? 1 : 0, out);
    return cudaGetLastError();
}

namespace {
__global__ void checked_fire_kernel(int n) { CK_CHECK(int(threadIdx.x) >= n, kChkShared); }
}  // namespace

cudaError_t launch_test_checked_fire(cudaStream_t stream) {
    checked_fire_kernel<<<1, 1, 0, stream>>>(1);
    return cudaGetLastError();
}

CK_DEFINE_CHECK_READER(check_word_quant)

}  // namespace ck
