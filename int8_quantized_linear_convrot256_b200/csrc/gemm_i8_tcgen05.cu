// Dense INT8 x INT8 -> INT32 GEMM on the sm_100a tensor cores (tcgen05
// kind::i8) with the dequantisation epilogue fused into the store.
//
// What is computed (ComfyUI-AppleSilicon-FP8 README, "What it fixes" row 17:
// INT8 x INT8 -> INT32, then the per-row rescale and the bias in the store
// epilogue so the int32 product never reaches global memory; sglang PR "Tune
// Kitchen INT8 row splitting for SM120", Accuracy Test: INT8 weights, FP32
// row scales, BF16 bias and output):
//   acc[m][n] = sum_k Qx[m][k] * Qw[n][k]                      (exact, int32)
//   Y[m][n]   = bf16_rne(((float(acc) * s_x[m]) * s_w[n]) + float(bias[n]))
//
// Design:
//  * Persistent CTAs, one per SM (192 KB of shared memory each), walking
//    128 x 256 output tiles in groups of 16 M-tiles so that concurrently
//    running CTAs share the same A rows and B columns in L2.
//  * Warp roles: warp 0 = TMA producer (one lane), warp 1 = MMA issuer (one
//    lane; the warp also owns the TMEM allocation), warps 2-5 = epilogue.
//  * 4-stage shared-memory ring of K-blocks (128 int8 along K): A 128 x 128,
//    B 256 x 128, both K-major with the 128-byte swizzle, loaded by 2-D TMA.
//    Out-of-range rows (ragged M, ragged N) are zero-filled by TMA, so any M
//    runs in one launch.
//  * tcgen05.mma kind::i8, M = 128, N = 256, K = 32 per instruction, int32
//    accumulators in TMEM; two accumulator buffers (2 x 256 columns = all
//    512) so the epilogue of one tile overlaps the main loop of the next.
//  * Epilogue: tcgen05.ld 32 lanes x 32 columns per warp, fp32 math with
//    explicit _rn intrinsics in the definition's order, BF16 pack, 16-byte
//    stores clipped at M and N.
//  * Every wait is bounded; on expiry the kernel records a timeout in the
//    device error word, lets in-flight copies and MMAs finish, frees TMEM
//    and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ck_device.cuh"
#include "internal.h"

namespace ck {
namespace {

constexpr int BM = kGemmBM;
constexpr int BN = kGemmBN;
constexpr int BK = kGemmBK;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;
constexpr int kBBytes = BN * BK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccBufs = 2;
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 192;
constexpr int kEpilogueThreads = 128;
constexpr int kGroupM = 16;
constexpr int kUmmaK = 32;  // int8 elements (bytes) per tcgen05.mma

struct alignas(8) Control {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[kAccBufs];
    uint64_t tmem_empty[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + sizeof(Control);

// Instruction descriptor: D = S32 (bits 4-5 = 2), A and B signed 8-bit
// (bits 7-9 and 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at
// bits 24-28.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) |
                            (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major operand written by TMA with
// the 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart
// (stride byte offset), descriptor version 1, layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int &mt, int &nt,
                                            int group_m = kGroupM) {
    const int per_group = group_m * num_n;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int first_m = g * group_m;
    const int gsz = min(group_m, num_m - first_m);
    mt = first_m + r % gsz;
    nt = r / gsz;
}

// Raster by groups of group_n N-tiles: inside a group N varies fastest, then
// M, so the group's B columns (the weights) stay in L2 while each M-tile of
// A is read from DRAM once per group and used by the group's N-tiles while
// it is fresh.
__device__ __forceinline__ void tile_coords_n(int tile, int num_m, int num_n, int &mt, int &nt,
                                              int group_n) {
    const int per_group = group_n * num_m;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int first_n = g * group_n;
    const int gsz = min(group_n, num_n - first_n);
    nt = first_n + r % gsz;
    mt = r / gsz;
}

__device__ __forceinline__ void raise_timeout(volatile int *abort, unsigned *err) {
    *abort = 1;
    atomicMax(err, kDevErrTimeout);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <bool kRaw>
__device__ __forceinline__ void store_accumulators(const GemmParams &p, uint32_t tbase, int row,
                                                   int n_tile0);
__device__ __forceinline__ void store_accumulators_tma(const GemmParams &p,
                                                       const CUtensorMap *tmY, uint32_t tbase,
                                                       int row0, int lane, int n_tile0,
                                                       uint32_t stage_buf, int &chunk_count);

template <bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Control *ctl = reinterpret_cast<Control *>(smem + size_t(kStages) * kStageBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (p.M + BM - 1) / BM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nk = p.K / BK;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
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
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            if (!p.stall_producer) {
                for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                    int mt, nt;
                    tile_coords(tile, num_m, num_n, mt, nt);
                    for (int kb = 0; kb < nk; ++kb) {
                        const uint32_t empty = smem_u32(&ctl->empty[stage]);
                        const uint32_t full = smem_u32(&ctl->full[stage]);
                        if (!mbar_wait_bounded(empty, phase ^ 1u, limit, abort)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(full, kStageBytes);
                        const uint32_t a_dst = smem_u32(smem + size_t(stage) * kStageBytes);
                        tma_load_2d(a_dst, &tmA, kb * BK, mt * BM, full);
                        tma_load_2d(a_dst + kABytes, &tmB, kb * BK, nt * BN, full);
                        issued |= 1u << stage;
                        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            // Never leave a bulk copy in flight into shared memory: wait for
            // the last copy issued into every stage to land.
            for (int s = 0; s < kStages; ++s)
                if (issued & (1u << s))
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), (last_parity >> s) & 1u, limit,
                                           nullptr))
                        raise_timeout(abort, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
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
                    tc_fence_after();
                    const uint32_t a_src = smem_u32(smem + size_t(stage) * kStageBytes);
                    const uint64_t adesc = smem_desc_sw128(a_src);
                    const uint64_t bdesc = smem_desc_sw128(a_src + kABytes);
#pragma unroll
                    for (int k = 0; k < BK / kUmmaK; ++k) {
                        // advance the start address by k * 32 bytes (>> 4)
                        umma_i8(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), kIdesc,
                                (kb | k) != 0 ? 1u : 0u);
                    }
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
            // All MMAs issued by this thread complete before TMEM is freed.
            umma_commit(smem_u32(&ctl->drain));
            if (!mbar_wait_bounded(smem_u32(&ctl->drain), 0u, limit, nullptr))
                raise_timeout(abort, p.err);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2-5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            int mt, nt;
            tile_coords(tile, num_m, num_n, mt, nt);
            if (!mbar_wait_bounded(smem_u32(&ctl->tmem_full[acc]), acc_phase, limit, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN);
            store_accumulators<kRaw>(p, tbase, mt * BM + quarter * 32 + lane, nt * BN);
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
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- 2-SM variant
//
// A cluster of 2 CTAs on the two SMs of a TPC computes 256 x 256 output tiles
// with tcgen05.mma.cta_group::2 (M = 256 split 128/128 across the pair, N =
// 256 with B split 128/128). Each CTA loads only its own 128 rows of A and its
// 128 rows of B per K-block (32 KB per stage, 6 stages), so each SM streams
// 64 bytes of operands per MMA clock instead of 96. The even CTA (leader)
// issues the MMAs; the TMA loads of both CTAs complete on the leader's "full"
// barrier; the leader's commits arrive on "empty" and "tmem_full" barriers of
// both CTAs (tcgen05.commit multicast; no TMA multicast anywhere). Each CTA's
// epilogue drains its own TMEM (its 128 rows x 256 columns) and arrives on
// the leader's "tmem_empty" barrier.
constexpr int kPairRows = 128;
constexpr int kPairBM = 2 * kPairRows;
constexpr int kPairBN = 256;
constexpr int kPairStages = 6;
constexpr int kPairABytes = kPairRows * BK;
constexpr int kPairStageBytes = 2 * kPairRows * BK;
constexpr int kPairGroupN = 21;  // N-tiles per raster group (32 timed 1.3 % slower, 63 12 %)
constexpr uint32_t kPairEpilogueWarps = 8;  // 4 per CTA, one arrive each

struct alignas(8) PairControl {
    uint64_t full[kPairStages];
    uint64_t empty[kPairStages];
    uint64_t tmem_full[kAccBufs];
    uint64_t tmem_empty[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kEpiStageBytes = 4 * 2 * 2048;  // 4 epilogue warps x 2 buffers x 2 KB
constexpr size_t kPairSmemBytes =
    1024 + size_t(kPairStages) * kPairStageBytes + kEpiStageBytes + sizeof(PairControl);

constexpr uint32_t kPairIdesc = (2u << 4) | (1u << 7) | (1u << 10) |
                                (uint32_t(kPairBN >> 3) << 17) | (uint32_t(kPairBM >> 4) << 24);

__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t cluster_addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}

template <bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi_stage = smem + size_t(kPairStages) * kPairStageBytes;
    PairControl *ctl = reinterpret_cast<PairControl *>(epi_stage + kEpiStageBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int num_m = (p.M + kPairBM - 1) / kPairBM;
    const int num_n = (p.N + kPairBN - 1) / kPairBN;
    const int num_tiles = num_m * num_n;
    const int nk = p.K / BK;
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(smem_u32(&ctl->tmem_full[a]), 1);
            mbar_init(smem_u32(&ctl->tmem_empty[a]), kPairEpilogueWarps);
        }
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (!kRaw) tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&ctl->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM address written
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int *abort = &ctl->abort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint32_t leader_full0 = mapa_shared(smem_u32(&ctl->full[0]), 0);
            // the group's Qw columns serve every M-tile of the sweep: keep them
            // in L2 while A (used by one group's N-tiles) and Y (written
            // once) pass through
            const uint64_t keep = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_parity = 0;
            bool ok = true;
            if (!p.stall_producer) {
                for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
                    int mt, nt;
                    tile_coords_n(tile, num_m, num_n, mt, nt, kPairGroupN);
                    const int a_row = mt * kPairBM + int(rank) * kPairRows;
                    const int b_row = nt * kPairBN + int(rank) * kPairRows;
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, limit,
                                               abort)) {
                            ok = false;
                            break;
                        }
                        if (leader)
                            mbar_arrive_expect_tx(smem_u32(&ctl->full[stage]), 2 * kPairStageBytes);
                        const uint32_t dst = smem_u32(smem + size_t(stage) * kPairStageBytes);
                        const uint32_t bar = leader_full0 + uint32_t(8 * stage);
                        tma_load_2d_pair(dst, &tmA, kb * BK, a_row, bar);
                        tma_load_2d_pair_hint(dst + kPairABytes, &tmB, kb * BK, b_row, bar, keep);
                        issued |= 1u << stage;
                        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                        if (++stage == kPairStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            // The leader's full barriers count the bytes of both CTAs: once the
            // last phase of every used stage has completed, no copy of either
            // CTA is still in flight.
            if (leader)
                for (int s = 0; s < kPairStages; ++s)
                    if (issued & (1u << s))
                        if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), (last_parity >> s) & 1u,
                                               limit, nullptr))
                            raise_timeout(abort, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && leader) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
                if (!mbar_wait_bounded(smem_u32(&ctl->tmem_empty[acc]), acc_phase ^ 1u, limit,
                                       abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(acc * kPairBN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, limit, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_src = smem_u32(smem + size_t(stage) * kPairStageBytes);
                    const uint64_t adesc = smem_desc_sw128(a_src);
                    const uint64_t bdesc = smem_desc_sw128(a_src + kPairABytes);
#pragma unroll
                    for (int k = 0; k < BK / kUmmaK; ++k)
                        umma_i8_pair(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), kPairIdesc,
                                     (kb | k) != 0 ? 1u : 0u);
                    umma_commit_pair_mc(smem_u32(&ctl->empty[stage]), 0x3);
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(smem_u32(&ctl->tmem_full[acc]), 0x3);
                if (++acc == kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok) raise_timeout(abort, p.err);
            umma_commit_pair_mc(smem_u32(&ctl->drain), 0x1);
            if (!mbar_wait_bounded(smem_u32(&ctl->drain), 0u, limit, nullptr))
                raise_timeout(abort, p.err);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2-5, both CTAs)
        const int quarter = warp & 3;
        const uint32_t leader_tmem_empty0 = mapa_shared(smem_u32(&ctl->tmem_empty[0]), 0);
        const uint32_t stage_buf = smem_u32(epi_stage) + uint32_t(warp - 2) * 4096u;
        int chunk_count = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles; tile += num_pairs) {
            int mt, nt;
            tile_coords_n(tile, num_m, num_n, mt, nt, kPairGroupN);
            if (!mbar_wait_bounded(smem_u32(&ctl->tmem_full[acc]), acc_phase, limit, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * kPairBN);
            const int row0 = mt * kPairBM + int(rank) * kPairRows + quarter * 32;
            if (kRaw)
                store_accumulators<true>(p, tbase, row0 + lane, nt * kPairBN);
            else
                store_accumulators_tma(p, &tmY, tbase, row0, lane, nt * kPairBN, stage_buf,
                                       chunk_count);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tmem_empty0 + uint32_t(8 * acc));
            if (++acc == kAccBufs) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (!ok) raise_timeout(abort, p.err);
        // every bulk store issued by this warp has completed before exit
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    // After a timeout, give copies that may still be in flight (into this
    // CTA's shared memory, or onto the leader's barriers) time to land
    // before the pair's shared memory is released.
    const int peer_abort = ld_shared_cluster_s32(mapa_shared(smem_u32(&ctl->abort), rank ^ 1u));
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

// Epilogue of one 256-column accumulator row block written through shared
// memory and TMA stores: each 32-column chunk of the warp's 32 rows (2 KB of
// bf16) goes into one of two staging buffers of the warp, laid out as the
// TMA box {32 columns, 32 rows} with the 64-byte swizzle (16-byte piece k of
// row r sits at piece k ^ ((r >> 1) & 3)), which keeps the 32 lanes' shared
// stores free of bank conflicts; lane 0 then issues the bulk tensor store.
// The store clips rows past M and columns past N.
__device__ __forceinline__ void store_accumulators_tma(const GemmParams &p,
                                                       const CUtensorMap *tmY, uint32_t tbase,
                                                       int row0, int lane, int n_tile0,
                                                       uint32_t stage_buf, int &chunk_count) {
    const int row = row0 + lane;
    const bool row_ok = row < p.M;
    const bool warp_rows_ok = row0 < p.M;
    const float sx = row_ok ? p.s_x[row] : 0.0f;
    const uint32_t swz = uint32_t((lane >> 1) & 3);
#pragma unroll 1
    for (int c = 0; c < 256 / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        if (!CK_CHECK((tbase & 0xFFFFu) + uint32_t(c * 32) + 32u <= kTmemCols, kChkTmem))
            continue;  // warp-uniform
        tmem_ld_32x32b_x32(tbase + uint32_t(c * 32), r);
        tmem_ld_wait();
        const int n0 = n_tile0 + c * 32;
        if (!warp_rows_ok || n0 >= p.N) continue;  // warp-uniform
        const uint32_t buf = stage_buf + uint32_t(chunk_count & 1) * 2048u;
        // the bulk store that last read this buffer (two chunks ago) is done
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int n = n0 + 8 * g;
            uint4 out = make_uint4(0u, 0u, 0u, 0u);
            if (n < p.N && CK_CHECK(n + 8 <= p.N, kChkGlobalLoad)) {
                const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.s_w + n));
                const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.s_w + n + 4));
                const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
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
                for (int i = 0; i < 8; ++i) {
                    float v = __int2float_rn(int(r[8 * g + i]));
                    v = __fmul_rn(v, sx);
                    v = __fmul_rn(v, sw[i]);
                    f[i] = __fadd_rn(v, b[i]);
                }
                out.x = bf16x2_rn(f[0], f[1]);
                out.y = bf16x2_rn(f[2], f[3]);
                out.z = bf16x2_rn(f[4], f[5]);
                out.w = bf16x2_rn(f[6], f[7]);
            }
            const uint32_t dst = buf + uint32_t(lane) * 64u + ((uint32_t(g) ^ swz) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(out.x),
                         "r"(out.y), "r"(out.z), "r"(out.w)
                         : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d_hint(tmY, n0, row0, buf, l2_policy_evict_first());
            bulk_commit_group();
        }
        ++chunk_count;
    }
}

// Epilogue of one 256-column accumulator row block: this warp's 32 TMEM lanes
// (rows), 8 chunks of 32 columns. tcgen05.ld is warp-collective, so every
// lane takes part even when its row is past M; stores are clipped at M and N.
template <bool kRaw>
__device__ __forceinline__ void store_accumulators(const GemmParams &p, uint32_t tbase, int row,
                                                   int n_tile0) {
    const bool row_ok = row < p.M;
    float sx = 0.0f;
    if (!kRaw && row_ok) sx = p.s_x[row];
#pragma unroll 1
    for (int c = 0; c < 256 / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        if (!CK_CHECK((tbase & 0xFFFFu) + uint32_t(c * 32) + 32u <= kTmemCols, kChkTmem))
            continue;  // warp-uniform
        tmem_ld_32x32b_x32(tbase + uint32_t(c * 32), r);
        tmem_ld_wait();
        const int n0 = n_tile0 + c * 32;
        if (!row_ok) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int n = n0 + 8 * g;
            if (n >= p.N) break;
            if (!CK_CHECK(n + 8 <= p.N, kChkGlobalStore | kChkGlobalLoad)) break;
            if (kRaw) {
                int4 *dst = reinterpret_cast<int4 *>(p.acc + int64_t(row) * p.N + n);
                dst[0] = make_int4(int(r[8 * g + 0]), int(r[8 * g + 1]), int(r[8 * g + 2]),
                                   int(r[8 * g + 3]));
                dst[1] = make_int4(int(r[8 * g + 4]), int(r[8 * g + 5]), int(r[8 * g + 6]),
                                   int(r[8 * g + 7]));
            } else {
                const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.s_w + n));
                const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.s_w + n + 4));
                const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
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
                for (int i = 0; i < 8; ++i) {
                    float v = __int2float_rn(int(r[8 * g + i]));
                    v = __fmul_rn(v, sx);
                    v = __fmul_rn(v, sw[i]);
                    f[i] = __fadd_rn(v, b[i]);
                }
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

// ---------------------------------------------------------------- peak probe
//
// The INT8 tensor-core ceiling of this device, measured: every CTA pair
// issues `mmas` back-to-back tcgen05.mma.cta_group::2.kind::i8 of the GEMM's
// shape (M 256, N 256, K 32, int32 accumulators in TMEM) on operands that sit
// in shared memory (their values do not matter), with no global-memory
// traffic and no epilogue. 2 * 256 * 256 * 32 operations per instruction.
constexpr int kProbeThreads = 128;
constexpr size_t kProbeSmemBytes = 1024 + 2 * size_t(kPairABytes) + 64;

__global__ void __launch_bounds__(kProbeThreads, 1)
i8_mma_peak_kernel(int64_t mmas, unsigned *err, uint64_t limit_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *done = reinterpret_cast<uint64_t *>(smem + 2 * kPairABytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    const int warp = threadIdx.x >> 5;
    const bool leader = cluster_ctarank() == 0;

    for (int i = threadIdx.x; i < 2 * kPairABytes / 16; i += kProbeThreads)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(done), 1);
        fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zeros visible to the MMA
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), kPairBN);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (leader && threadIdx.x == 32) {
        const uint32_t a = smem_u32(smem);
        const uint64_t adesc = smem_desc_sw128(a);
        const uint64_t bdesc = smem_desc_sw128(a + kPairABytes);
        for (int64_t i = 0; i < mmas; ++i) {
            const uint64_t k = uint64_t(2 * (i & 3));  // the four K steps of a 128-byte K-block
            umma_i8_pair(tmem, adesc + k, bdesc + k, kPairIdesc, i != 0 ? 1u : 0u);
        }
        umma_commit_pair_mc(smem_u32(done), 0x3);
    }
    if (threadIdx.x == 0 && !mbar_wait_bounded(smem_u32(done), 0u, limit_ns, nullptr))
        atomicMax(err, kDevErrTimeout);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kPairBN);
    }
}

}  // namespace

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_plan_mutex;
int g_max_pairs[kMaxDevices];  // co-resident clusters of the pair kernel; 0 = not queried
bool g_attrs_set[kMaxDevices];

cudaError_t set_attributes() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(gemm_i8_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(kSmemBytes))) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(gemm_i8_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(kSmemBytes))) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(gemm_i8_pair_kernel<false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(kPairSmemBytes))) != cudaSuccess)
        return e;
    return cudaFuncSetAttribute(gemm_i8_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kPairSmemBytes));
}

// Number of 2-CTA clusters of the pair kernel that fit on the device at once.
cudaError_t max_active_pairs(int dev, int *out) {
    std::lock_guard<std::mutex> lock(g_plan_mutex);
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!g_attrs_set[dev]) {
        cudaError_t e = set_attributes();
        if (e != cudaSuccess) return e;
        g_attrs_set[dev] = true;
    }
    if (g_max_pairs[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kPairSmemBytes;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_i8_pair_kernel<false>, &cfg);
        if (e != cudaSuccess) return e;
        g_max_pairs[dev] = n > 0 ? n : -1;
    }
    *out = g_max_pairs[dev] > 0 ? g_max_pairs[dev] : 0;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_i8_mma_peak(int64_t mmas, unsigned *err, uint64_t limit_ns, int *pairs_out,
                               cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int pairs = 0;
    e = max_active_pairs(dev, &pairs);  // one probe pair per pair of SMs the GEMM uses
    if (e != cudaSuccess) return e;
    if (pairs <= 0) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(i8_mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kProbeSmemBytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kProbeThreads, 1, 1);
    cfg.dynamicSmemBytes = kProbeSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    *pairs_out = pairs;
    return cudaLaunchKernelEx(&cfg, i8_mma_peak_kernel, mmas, err, limit_ns);
}

cudaError_t plan_gemm(int M, int N, int num_sms, GemmPlan *plan) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int pairs = 0;
    e = max_active_pairs(dev, &pairs);
    if (e != cudaSuccess) return e;
    plan->pair = M > kGemmBM && pairs > 0;
    if (plan->pair) {
        const int tiles = ((M + kPairBM - 1) / kPairBM) * ((N + kPairBN - 1) / kPairBN);
        plan->b_box_rows = kPairRows;
        plan->grid = 2 * (tiles < pairs ? tiles : pairs);
    } else {
        const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
        plan->b_box_rows = BN;
        plan->grid = tiles < num_sms ? tiles : num_sms;
    }
    return cudaSuccess;
}

cudaError_t launch_gemm_i8(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmY,
                           const GemmParams &p, bool raw_i32, const GemmPlan &plan,
                           cudaStream_t stream) {
    if (p.M <= 0 || p.N <= 0) return cudaSuccess;
    if (!plan.pair) {
        if (raw_i32)
            gemm_i8_kernel<true><<<plan.grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, p);
        else
            gemm_i8_kernel<false><<<plan.grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, p);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(plan.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (raw_i32) return cudaLaunchKernelEx(&cfg, gemm_i8_pair_kernel<true>, tmA, tmB, tmY, p);
    return cudaLaunchKernelEx(&cfg, gemm_i8_pair_kernel<false>, tmA, tmB, tmY, p);
}

CK_DEFINE_CHECK_READER(check_word_gemm_i8)

}  // namespace ck
