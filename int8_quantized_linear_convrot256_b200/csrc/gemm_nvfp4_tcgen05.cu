// Block-scaled NVFP4 GEMM on the sm_100a tensor cores (tcgen05.mma
// kind::mxf4nvf4, one E4M3 scale per 16 FP4 values) with the epilogue fused
// into the store.
//
// What is computed (ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix",
// section 5-1, nvfp4_gemm.py: FP4 E2M1 codes, block scales per 16 values in
// the 128 x 4 blocked layout, a per-tensor scale per operand, then
// a_dq @ w_dq.T + bias):
//   acc[m][n] = sum_k (e2m1(qa[m][k]) * e4m3(sa[m][k/16])) *
//                     (e2m1(qb[n][k]) * e4m3(sb[n][k/16]))     (fp32, tensor core)
//   Y[m][n]   = bf16_rne((acc * (s_ta * s_tb)) + float(bias[n]))
//
// Design:
//  * Persistent CTAs, one per SM, over 128 x 128 output tiles grouped by 16
//    M-tiles. Warp 0 loads (one lane), warp 1 issues the MMAs and owns TMEM,
//    warps 2-5 run the epilogue, warp 6 copies the scale tiles into TMEM.
//  * 5-stage ring. A stage holds one K-block of 256 values: A and B as
//    128 rows x 128 packed bytes (2-D TMA, 128-byte swizzle, zero fill past M
//    and N), plus the four 512-byte scale tiles of A and of B that cover the
//    block. The blocked layout keeps those tiles contiguous, so each is one
//    2 KB bulk copy.
//  * As soon as a stage's loads land, the copy warp's lane copies its scale
//    tiles into TMEM (tcgen05.cp 32x128b.warpx4) and commits them to the
//    stage's sf_ready barrier, which the MMA lane waits for; copies of later
//    stages are thereby queued while a stage's MMAs run. A tile's 32 lines of 16 bytes land in TMEM
//    lanes 0-31 and again in 32-63, 64-95 and 96-127, four columns wide.
//    Row r then finds its four scales in lane r, column r / 32, which is
//    where the MMA reads them.
//  * Four tcgen05.mma per stage (M128 N128 K64), each reading its own scale
//    tile's four columns. fp32 accumulators sit in TMEM, double-buffered
//    (2 x 128 columns). The scale columns of the five stages follow them.
//  * Every wait is bounded. On expiry the kernel records a timeout in the
//    device error word, lets in-flight copies and MMAs finish, frees TMEM and
//    returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

constexpr int BM = kNvfp4BM;
constexpr int BN = kNvfp4BN;
constexpr int BKB = kNvfp4BKBytes;
constexpr int kStages = 5;
constexpr int kABytes = BM * BKB;
constexpr int kBBytes = BN * BKB;
constexpr int kSfTileBytes = 512;           // 128 rows x 4 scales
constexpr int kSfBytes = 4 * kSfTileBytes;  // the 16 scales per row of one stage
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
constexpr int kAccBufs = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = uint32_t(kAccBufs * BN);
constexpr uint32_t kSfColsPerStage = 32;  // 16 for A, then 16 for B
constexpr int kThreads = 224;  // producer, MMA, 4 epilogue warps, scale copies
constexpr int kCopyWarp = 6;
constexpr int kEpilogueThreads = 128;
constexpr int kGroupM = 16;
constexpr int kMmaKBytes = 32;  // 64 FP4 values per tcgen05.mma

static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");

struct Control {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t sf_ready[kStages];  // the stage's scale copies have completed
    uint64_t tmem_full[kAccBufs];
    uint64_t tmem_empty[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + sizeof(Control);

// Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (format 1, bits
// 7-9 and 10-12), both K-major, N >> 3 at bits 17-22, E4M3 scales (bit 23 =
// 0), M >> 4 at bits 24-28; dense, K = 64, scale-factor IDs 0.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                            (uint32_t(BM >> 4) << 24);

// Operand descriptor: K-major rows of 128 bytes written by TMA with the
// 128-byte swizzle, 8-row atoms 1024 bytes apart, descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Source descriptor of a 512-byte scale tile for tcgen05.cp: 32 lines of 16
// bytes, no swizzle, 8-line core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
    return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(128 >> 4) << 32) | (uint64_t(1) << 46);
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void umma_nvfp4(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tile_of(int tile, int num_m, int num_n, int &mt, int &nt) {
    const int per_group = kGroupM * num_n;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int first_m = g * kGroupM;
    const int gsz = min(kGroupM, num_m - first_m);
    mt = first_m + r % gsz;
    nt = r / gsz;
}

__device__ __forceinline__ void raise_timeout(volatile int *abort, unsigned *err) {
    *abort = 1;
    atomicMax(err, kDevErrTimeout);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const Nvfp4GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Control *ctl = reinterpret_cast<Control *>(smem + size_t(kStages) * kStageBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (p.M + BM - 1) / BM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nk = p.K / (2 * BKB);
    const int sf_tiles_per_row_block = p.K / 64;  // (K / 16) scale columns / 4
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
            mbar_init(smem_u32(&ctl->sf_ready[s]), 1);
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(smem_u32(&ctl->tmem_full[a]), 1);
            mbar_init(smem_u32(&ctl->tmem_empty[a]), kEpilogueThreads);
        }
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int *abort = &ctl->abort;

    if (warp == 0) {
        // ------------------------------------------------ loads
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && !p.stall_producer && tile < num_tiles;
                 tile += gridDim.x) {
                int mt, nt;
                tile_of(tile, num_m, num_n, mt, nt);
                const uint8_t *sfa = p.sfa + int64_t(mt) * sf_tiles_per_row_block * kSfTileBytes;
                const uint8_t *sfb = p.sfb + int64_t(nt) * sf_tiles_per_row_block * kSfTileBytes;
                for (int kb = 0; kb < nk; ++kb) {
                    const uint32_t full = smem_u32(&ctl->full[stage]);
                    if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, limit,
                                           abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full, kStageBytes);
                    const uint32_t dst = smem_u32(smem + size_t(stage) * kStageBytes);
                    tma_load_2d(dst, &tmA, kb * BKB, mt * BM, full);
                    tma_load_2d(dst + kABytes, &tmB, kb * BKB, nt * BN, full);
                    bulk_load(dst + kABytes + kBBytes, sfa + int64_t(4 * kb) * kSfTileBytes,
                              kSfBytes, full);
                    bulk_load(dst + kABytes + kBBytes + kSfBytes,
                              sfb + int64_t(4 * kb) * kSfTileBytes, kSfBytes, full);
                    issued |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            // never leave a copy in flight into shared memory
            for (int s = 0; s < kStages; ++s)
                if (issued & (1u << s))
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), (last_parity >> s) & 1u, limit,
                                           nullptr))
                        raise_timeout(abort, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ scale copies + MMAs
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(smem_u32(&ctl->tmem_empty[acc]), acc_phase ^ 1u, limit,
                                       abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_bounded(smem_u32(&ctl->sf_ready[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_src = smem_u32(smem + size_t(stage) * kStageBytes);
                    const uint32_t tsfa = tmem_base + kSfCol0 + uint32_t(stage) * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    const uint64_t adesc = desc_sw128(a_src);
                    const uint64_t bdesc = desc_sw128(a_src + kABytes);
#pragma unroll
                    for (int k = 0; k < BKB / kMmaKBytes; ++k)
                        umma_nvfp4(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), kIdesc,
                                   tsfa + 4u * k, tsfb + 4u * k, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(smem_u32(&ctl->empty[stage]));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(smem_u32(&ctl->tmem_full[acc]));
                if (++acc == kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            umma_commit(smem_u32(&ctl->drain));
            if (!mbar_wait_bounded(smem_u32(&ctl->drain), 0u, limit, nullptr))
                raise_timeout(abort, p.err);
        }
    } else if (warp == kCopyWarp) {
        // ------------------------------------------------ scale tiles to TMEM
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                for (int kb = 0; kb < nk; ++kb) {
                    // the stage's loads have landed; the MMAs that last read its
                    // scale columns completed before the stage was refilled
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_src =
                        smem_u32(smem + size_t(stage) * kStageBytes) + kABytes + kBBytes;
                    const uint32_t sfb_src = sfa_src + kSfBytes;
                    const uint32_t tsfa = tmem_base + kSfCol0 + uint32_t(stage) * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tmem_cp_sf(tsfa + 4u * j, desc_sf(sfa_src + kSfTileBytes * j));
                        tmem_cp_sf(tsfb + 4u * j, desc_sf(sfb_src + kSfTileBytes * j));
                    }
                    umma_commit(smem_u32(&ctl->sf_ready[stage]));
                    issued |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            // every copy this thread issued completes before TMEM is freed
            for (int s = 0; s < kStages; ++s)
                if (issued & (1u << s))
                    if (!mbar_wait_bounded(smem_u32(&ctl->sf_ready[s]), (last_parity >> s) & 1u,
                                           limit, nullptr))
                        raise_timeout(abort, p.err);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2-5)
        const int quarter = warp & 3;
        const float alpha = __fmul_rn(*p.s_ta, *p.s_tb);
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            int mt, nt;
            tile_of(tile, num_m, num_n, mt, nt);
            if (!mbar_wait_bounded(smem_u32(&ctl->tmem_full[acc]), acc_phase, limit, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN);
            const int row = mt * BM + quarter * 32 + lane;
            const bool row_ok = row < p.M;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                __syncwarp();
                if (!CK_CHECK((tbase & 0xFFFFu) + uint32_t(c * 32) + 32u <= kTmemCols, kChkTmem))
                    continue;  // warp-uniform
                tmem_ld_32x32b_x32(tbase + uint32_t(c * 32), r);
                tmem_ld_wait();
                if (!row_ok) continue;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int n = nt * BN + c * 32 + 8 * g;
                    if (n >= p.N) break;
                    if (!CK_CHECK(n + 8 <= p.N, kChkGlobalStore | kChkGlobalLoad)) break;
                    float b[8];
                    if (p.bias) {
                        const uint4 bb = __ldg(reinterpret_cast<const uint4 *>(p.bias + n));
                        const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            b[2 * i] = __uint_as_float(bw[i] << 16);
                            b[2 * i + 1] = __uint_as_float(bw[i] & 0xFFFF0000u);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) b[i] = 0.0f;
                    }
                    float f[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        f[i] = __fadd_rn(__fmul_rn(__uint_as_float(r[8 * g + i]), alpha), b[i]);
                    uint4 out;
                    out.x = bf16x2_rn(f[0], f[1]);
                    out.y = bf16x2_rn(f[2], f[3]);
                    out.z = bf16x2_rn(f[4], f[5]);
                    out.w = bf16x2_rn(f[6], f[7]);
                    *reinterpret_cast<uint4 *>(p.Y + int64_t(row) * p.N + n) = out;
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl->tmem_empty[acc]));
            if (++acc == kAccBufs) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (!ok) raise_timeout(abort, p.err);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- 2-SM variant
// A cluster of 2 CTAs on the two SMs of a TPC computes 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (M = 256 split 128/128 over the pair, N = 256 with
// B split 128/128). Per K-block each CTA loads its own 128 rows of A and of
// B, the scale tiles of its own 128 A rows, and the scale tiles of all 256 B
// rows (its tensor core needs all of them). All loads are TMA loads whose
// completion bytes go to the even CTA's barrier. The even CTA copies the
// scale tiles into TMEM (tcgen05.cp.cta_group::2: each CTA's shared memory
// into its own TMEM) from a warp of its own, as soon as a stage's loads have
// landed, and signals each stage's copies on a barrier the MMA thread waits
// for; the copies for the next stages are thereby already queued while a
// stage's MMAs run. TMEM holds one 256-column fp32
// accumulator plus the scale columns of the 5 stages, so there is no room
// for a second accumulator. Instead 8 epilogue warps per CTA move the
// accumulator into registers (128 columns each) and release it before doing
// the math and the stores.
constexpr int kPairRowsN = 128;             // rows of A and of B per CTA
constexpr int kPairBMn = 2 * kPairRowsN;    // 256
constexpr int kPairBNn = 256;
constexpr int kPairSfaBytes = 4 * kSfTileBytes;       // own 128 A rows
constexpr int kPairSfbBytes = 2 * 4 * kSfTileBytes;   // all 256 B rows
constexpr int kPairStageBytesN = 2 * kPairRowsN * BKB + kPairSfaBytes + kPairSfbBytes;
constexpr int kPairStagesN = 5;
constexpr uint32_t kPairSfCol0 = 256;
constexpr uint32_t kPairSfColsPerStage = 48;  // 16 for A, 32 for B
constexpr int kPairThreadsN = 352;            // producer, MMA, 8 epilogue warps, scale copies
constexpr int kPairCopyWarpN = 10;
constexpr uint32_t kPairEpiWarpsN = 16;       // both CTAs
constexpr int kPairGroupNN = 32;  // N-tiles per raster group (21 timed 0.4 % slower, 63 3 %)

static_assert(kPairSfCol0 + kPairStagesN * kPairSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kPairStageBytesN % 1024 == 0, "stages keep the 1024-byte swizzle alignment");

struct PairControlN {
    uint64_t full[kPairStagesN];
    uint64_t empty[kPairStagesN];
    uint64_t sf_ready[kPairStagesN];  // the stage's scale copies have completed (even CTA)
    uint64_t tmem_full;
    uint64_t tmem_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kPairSmemBytesN =
    1024 + size_t(kPairStagesN) * kPairStageBytesN + sizeof(PairControlN);

constexpr uint32_t kPairIdescN = (1u << 7) | (1u << 10) | (uint32_t(kPairBNn >> 3) << 17) |
                                 (uint32_t(kPairBMn >> 4) << 24);

__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void umma_nvfp4_pair(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
}

__device__ __forceinline__ int ld_shared_cluster_s32_n(uint32_t cluster_addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}

// Raster by groups of kPairGroupNN N-tiles: inside a group N varies fastest,
// then M, so the group's B columns (weights and their scales) stay in L2
// while each M-tile of A is read from DRAM once per group.
__device__ __forceinline__ void tile_of_pair(int tile, int num_m, int num_n, int &mt, int &nt) {
    const int per_group = kPairGroupNN * num_m;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int first_n = g * kPairGroupNN;
    const int gsz = min(kPairGroupNN, num_n - first_n);
    nt = first_n + r % gsz;
    mt = r / gsz;
}

// tmSFA / tmSFB view the blocked scales as rows of 256 bytes; a box of 8 rows
// is 4 consecutive 512-byte tiles.
__global__ void __launch_bounds__(kPairThreadsN, 1)
gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSFA,
                       const __grid_constant__ CUtensorMap tmSFB, const Nvfp4GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairControlN *ctl =
        reinterpret_cast<PairControlN *>(smem + size_t(kPairStagesN) * kPairStageBytesN);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int num_m = (p.M + kPairBMn - 1) / kPairBMn;
    const int num_n = (p.N + kPairBNn - 1) / kPairBNn;
    const int num_tiles = num_m * num_n;
    const int nk = p.K / (2 * BKB);
    const int sf_rows_per_row_block = p.K / 32;  // 256-byte rows of one 128-row block
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStagesN; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
            mbar_init(smem_u32(&ctl->sf_ready[s]), 1);
        }
        mbar_init(smem_u32(&ctl->tmem_full), 1);
        mbar_init(smem_u32(&ctl->tmem_empty), kPairEpiWarpsN);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSFA);
        tma_prefetch_desc(&tmSFB);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&ctl->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int *abort = &ctl->abort;

    if (warp == 0) {
        // ------------------------------------------------ loads (both CTAs)
        if (lane == 0) {
            const uint32_t leader_full0 = mapa_shared(smem_u32(&ctl->full[0]), 0);
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            for (int tile = pair; ok && !p.stall_producer && tile < num_tiles;
                 tile += num_pairs) {
                int mt, nt;
                tile_of_pair(tile, num_m, num_n, mt, nt);
                const int a_row = mt * kPairBMn + int(rank) * kPairRowsN;
                const int b_row = nt * kPairBNn + int(rank) * kPairRowsN;
                const int sfa_row0 = (mt * 2 + int(rank)) * sf_rows_per_row_block;
                const int sfb_row0 = (nt * 2) * sf_rows_per_row_block;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, limit,
                                           abort)) {
                        ok = false;
                        break;
                    }
                    if (leader)
                        mbar_arrive_expect_tx(smem_u32(&ctl->full[stage]), 2 * kPairStageBytesN);
                    const uint32_t dst = smem_u32(smem + size_t(stage) * kPairStageBytesN);
                    const uint32_t bar = leader_full0 + uint32_t(8 * stage);
                    tma_load_2d_pair(dst, &tmA, kb * BKB, a_row, bar);
                    tma_load_2d_pair(dst + kPairRowsN * BKB, &tmB, kb * BKB, b_row, bar);
                    const uint32_t sf_dst = dst + 2 * kPairRowsN * BKB;
                    tma_load_2d_pair(sf_dst, &tmSFA, 0, sfa_row0 + 8 * kb, bar);
                    tma_load_2d_pair(sf_dst + kPairSfaBytes, &tmSFB, 0, sfb_row0 + 8 * kb, bar);
                    tma_load_2d_pair(sf_dst + kPairSfaBytes + 4 * kSfTileBytes, &tmSFB, 0,
                                     sfb_row0 + sf_rows_per_row_block + 8 * kb, bar);
                    issued |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kPairStagesN) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            if (leader)
                for (int s = 0; s < kPairStagesN; ++s)
                    if (issued & (1u << s))
                        if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), (last_parity >> s) & 1u,
                                               limit, nullptr))
                            raise_timeout(abort, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ scales to TMEM + MMAs (leader)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
                if (!mbar_wait_bounded(smem_u32(&ctl->tmem_empty), acc_phase ^ 1u, limit, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_bounded(smem_u32(&ctl->sf_ready[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_src = smem_u32(smem + size_t(stage) * kPairStageBytesN);
                    const uint32_t tsfa =
                        tmem_base + kPairSfCol0 + uint32_t(stage) * kPairSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    const uint64_t adesc = desc_sw128(a_src);
                    const uint64_t bdesc = desc_sw128(a_src + kPairRowsN * BKB);
#pragma unroll
                    for (int k = 0; k < BKB / kMmaKBytes; ++k)
                        umma_nvfp4_pair(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k),
                                        kPairIdescN, tsfa + 4u * k, tsfb + 8u * k,
                                        (kb | k) != 0 ? 1u : 0u);
                    umma_commit_pair_mc(smem_u32(&ctl->empty[stage]), 0x3);
                    if (++stage == kPairStagesN) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(smem_u32(&ctl->tmem_full), 0x3);
                acc_phase ^= 1u;
            }
            if (!ok) raise_timeout(abort, p.err);
            umma_commit_pair_mc(smem_u32(&ctl->drain), 0x1);
            if (!mbar_wait_bounded(smem_u32(&ctl->drain), 0u, limit, nullptr))
                raise_timeout(abort, p.err);
        }
    } else if (warp == kPairCopyWarpN) {
        // ------------------------------------------------ scale tiles to TMEM (leader)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
                for (int kb = 0; kb < nk; ++kb) {
                    // the stage's loads have landed; the MMAs that last read its
                    // scale columns completed before the stage was refilled
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_src =
                        smem_u32(smem + size_t(stage) * kPairStageBytesN) + 2 * kPairRowsN * BKB;
                    const uint32_t sfb_src = sfa_src + kPairSfaBytes;
                    const uint32_t tsfa =
                        tmem_base + kPairSfCol0 + uint32_t(stage) * kPairSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tmem_cp_sf_pair(tsfa + 4u * j, desc_sf(sfa_src + kSfTileBytes * j));
                        tmem_cp_sf_pair(tsfb + 8u * j, desc_sf(sfb_src + kSfTileBytes * j));
                        tmem_cp_sf_pair(tsfb + 8u * j + 4u,
                                        desc_sf(sfb_src + 4 * kSfTileBytes + kSfTileBytes * j));
                    }
                    umma_commit_pair_mc(smem_u32(&ctl->sf_ready[stage]), 0x1);
                    issued |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kPairStagesN) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            // every copy this thread issued completes before TMEM is freed
            for (int s = 0; s < kPairStagesN; ++s)
                if (issued & (1u << s))
                    if (!mbar_wait_bounded(smem_u32(&ctl->sf_ready[s]), (last_parity >> s) & 1u,
                                           limit, nullptr))
                        raise_timeout(abort, p.err);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2-9, both CTAs)
        const int quarter = warp & 3;      // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;  // columns [128 half, 128 half + 128)
        const uint32_t leader_tmem_empty = mapa_shared(smem_u32(&ctl->tmem_empty), 0);
        const float alpha = __fmul_rn(*p.s_ta, *p.s_tb);
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles; tile += num_pairs) {
            int mt, nt;
            tile_of_pair(tile, num_m, num_n, mt, nt);
            if (!mbar_wait_bounded(smem_u32(&ctl->tmem_full), acc_phase, limit, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(half * 128);
            uint32_t r[4][32];
            const bool cols_ok = CK_CHECK((tbase & 0xFFFFu) + 128u <= kTmemCols, kChkTmem);
            if (cols_ok) {  // warp-uniform
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + uint32_t(c * 32), r[c]);
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tmem_empty);
            acc_phase ^= 1u;
            const int row = mt * kPairBMn + int(rank) * kPairRowsN + quarter * 32 + lane;
            if (row < p.M && cols_ok) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int n = nt * kPairBNn + half * 128 + c * 32 + 8 * g;
                        if (n < p.N && CK_CHECK(n + 8 <= p.N, kChkGlobalStore | kChkGlobalLoad)) {
                            float b[8];
                            if (p.bias) {
                                const uint4 bb = __ldg(reinterpret_cast<const uint4 *>(p.bias + n));
                                const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    b[2 * i] = __uint_as_float(bw[i] << 16);
                                    b[2 * i + 1] = __uint_as_float(bw[i] & 0xFFFF0000u);
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < 8; ++i) b[i] = 0.0f;
                            }
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f[i] = __fadd_rn(__fmul_rn(__uint_as_float(r[c][8 * g + i]), alpha),
                                                 b[i]);
                            uint4 out;
                            out.x = bf16x2_rn(f[0], f[1]);
                            out.y = bf16x2_rn(f[2], f[3]);
                            out.z = bf16x2_rn(f[4], f[5]);
                            out.w = bf16x2_rn(f[6], f[7]);
                            *reinterpret_cast<uint4 *>(p.Y + int64_t(row) * p.N + n) = out;
                        }
                    }
                }
            }
        }
        if (!ok) raise_timeout(abort, p.err);
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    const int peer_abort =
        ld_shared_cluster_s32_n(mapa_shared(smem_u32(&ctl->abort), rank ^ 1u));
    if (*abort || peer_abort) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
    __syncwarp();
    cluster_sync_all();
}

std::mutex g_attr_mutex;
bool g_attr_set[64] = {};
int g_max_pairs[64] = {};

// The kernels' dynamic shared memory limits are raised once per device, and
// the number of co-resident 2-CTA clusters of the pair kernel is cached.
cudaError_t ensure_attributes(int *max_pairs) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (!g_attr_set[dev]) {
        e = cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kSmemBytes));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_nvfp4_pair_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kPairSmemBytesN));
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kPairThreadsN, 1, 1);
        cfg.dynamicSmemBytes = kPairSmemBytesN;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel, &cfg);
        if (e != cudaSuccess) return e;
        g_max_pairs[dev] = n;
        g_attr_set[dev] = true;
    }
    *max_pairs = g_max_pairs[dev];
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const CUtensorMap &tmA, const CUtensorMap &tmB,
                              const CUtensorMap &tmSFA, const CUtensorMap &tmSFB,
                              const Nvfp4GemmParams &p, int num_sms, bool allow_pair,
                              cudaStream_t stream) {
    if (p.M <= 0 || p.N <= 0) return cudaSuccess;
    int pairs = 0;
    cudaError_t e = ensure_attributes(&pairs);
    if (e != cudaSuccess) return e;
    if (allow_pair && p.M > BM && pairs > 0) {
        const int tiles = ((p.M + kPairBMn - 1) / kPairBMn) * ((p.N + kPairBNn - 1) / kPairBNn);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (tiles < pairs ? tiles : pairs), 1, 1);
        cfg.blockDim = dim3(kPairThreadsN, 1, 1);
        cfg.dynamicSmemBytes = kPairSmemBytesN;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, gemm_nvfp4_pair_kernel, tmA, tmB, tmSFA, tmSFB, p);
    }
    const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    gemm_nvfp4_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, p);
    return cudaGetLastError();
}

CK_DEFINE_CHECK_READER(check_word_gemm_nvfp4)

}  // namespace ck
