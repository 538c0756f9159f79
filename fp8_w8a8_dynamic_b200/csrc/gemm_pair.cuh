// gemm_pair.cuh — prefill-sized FP8 GEMM on CTA pairs (tcgen05 cta_group::2):
//     Y[m, n] = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
//
// A cluster of two CTAs computes 256 x BN output tiles (BN = 256, or 128
// when that fills the GPU in fewer rounds) with one MMA stream:
//   - each CTA loads, with plain TMA (no multicast), its own 128 rows of the
//     X8 tile and its own BN/2 rows of the W8 tile into the same shared-memory
//     offsets; the loads of both CTAs count their bytes on the even CTA's
//     "full" barrier;
//   - one thread of the even CTA issues tcgen05.mma.cta_group::2 (M = 256,
//     N = BN, K = 32 per instruction); the hardware reads the A rows and the
//     B columns of both CTAs, and each CTA's TMEM receives its 128 rows of D;
//   - tcgen05.commit with a two-CTA mask frees the ring slot in both CTAs and
//     hands each CTA its finished accumulator;
//   - each CTA's four epilogue warps scale their 128 rows, stage 32 x 32
//     bf16 blocks in shared memory and store them with TMA (coalesced,
//     asynchronous), and report back to the even CTA, which then reuses
//     that accumulator.
// With BN = 256, per CTA and k-block the ring takes 32 KB for 128 x 256 x 128
// MACs, two thirds of the bytes a single-CTA 128 x 256 tile needs, so a
// six-deep ring fits and L2 -> SM traffic drops by a third.  Two fp32
// accumulators (2 x BN TMEM columns) overlap the epilogue of one tile with the
// main loop of the next.  Tiles are walked n-fastest.
//
// Every wait is bounded (see gemm_tiled.cuh); both CTAs meet on a cluster
// barrier before either leaves, so neither exits while the other may still
// touch its shared memory or TMEM.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {
namespace pair {

constexpr int BM = 256;        // rows of the pair's tile (128 per CTA)
constexpr int HALF = 128;
constexpr int BK = 128;
constexpr int MMA_K = 32;
constexpr int kThreads = 192;

// BN: columns of the pair's tile (BN/2 W8 rows per CTA), 256 or 128.
template <int BN, int STAGES>
struct Layout {
    static_assert(BN == 256 || BN == 128, "pair tile width");
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int A_BYTES = HALF * BK;       // this CTA's rows of X8
    static constexpr int B_BYTES = (BN / 2) * BK;   // this CTA's rows of W8
    static constexpr int CTA_STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = STAGES * A_BYTES;
    static constexpr int STG_OFF = STAGES * CTA_STAGE_BYTES;     // epilogue staging: 4 warps x 2 x 2 KB
    static constexpr int BAR_OFF = STG_OFF + 4 * 4096;
    static constexpr int NUM_BARS = 2 * STAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmY, const float* __restrict__ s_a, const float* __restrict__ s_w,
                 __nv_bfloat16* __restrict__ Y, int M, int N, int K) {
    using L = Layout<BN, STAGES>;
    constexpr int TMEM_COLS = L::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sA = sbase + L::A_OFF;
    const uint32_t sB = sbase + L::B_OFF;
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const uint32_t cr = cluster_ctarank();  // 0: issues the MMAs, 1: its partner
    const int pair_id = int(blockIdx.x >> 1);
    const int num_pairs = int(gridDim.x >> 1);
    const int m_tiles = (M + BM - 1) / BM;
    const int n_tiles = (N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int kb_count = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);  // four epilogue warps in each CTA
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_arrive_release();
    cluster_wait_acquire();  // both CTAs' barriers exist before any cross-CTA signal
    const uint32_t tmem_base = *tmem_holder;

    // The next call's quantize kernel may start launching; it waits for this
    // grid to finish before it touches memory.
    grid_launch_dependents();
    grid_dependency_wait();  // X8 and s_a may come from the kernel launched just before

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint64_t policy_x = l2_policy_evict_normal();
            const uint64_t policy_w = l2_policy_evict_last();
            for (int tile = pair_id; tile < num_tiles && !*abort_flag; tile += num_pairs) {
                const int tm = tile / n_tiles, tn = tile % n_tiles;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                    const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
                    if (cr == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * L::CTA_STAGE_BYTES);
                    tma_load_2d_pair(sA + stage * L::A_BYTES, &tmX, leader_full, kb * BK, tm * BM + int(cr) * HALF,
                                     policy_x);
                    tma_load_2d_pair(sB + stage * L::B_BYTES, &tmW, leader_full, kb * BK, tn * BN + int(cr) * (BN / 2),
                                     policy_w);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && cr == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool issued_any = false;
            int local = 0;
            for (int tile = pair_id; tile < num_tiles; tile += num_pairs, ++local) {
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                bool ok = true;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = sA + stage * L::A_BYTES;
                    const uint32_t b0 = sB + stage * L::B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / MMA_K; ++kk)
                        mma_f8_pair(d_tmem, sw128_kmajor_desc(a0 + kk * MMA_K), sw128_kmajor_desc(b0 + kk * MMA_K),
                                    idesc, (kb | kk) != 0);
                    issued_any = true;
                    mma_commit_pair_mc(empty_bar(stage), 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit_pair_mc(tfull_bar(acc), 0x3);
            }
            if (*abort_flag && issued_any) {
                volatile int no_abort = 0;
                mma_commit_pair_mc(drain_bar, 0x1);
                mbar_wait(drain_bar, 0, &no_abort, 10000000ull);
            }
        }
    } else {
        const uint32_t q = warp & 3u;
        const uint32_t leader_tempty0 = mapa_shared(tempty_bar(0), 0);
        const uint32_t leader_tempty1 = mapa_shared(tempty_bar(1), 0);
        TmaEpilogue ep{&tmY, sbase + uint32_t(L::STG_OFF) + q * 4096u};
        int local = 0;
        for (int tile = pair_id; tile < num_tiles; tile += num_pairs, ++local) {
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) break;
            tc_fence_after();
            const int tm = tile / n_tiles, tn = tile % n_tiles;
            const int row0 = tm * BM + int(cr) * HALF + int(q * 32);
            const int row = row0 + int(lane);
            const float sa = row < M ? __ldcg(s_a + row) : 0.0f;  // written by the previous kernel
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + uint32_t(acc * BN + c * 32), r);
                tmem_wait_ld();
                ep.put(r, sa, s_w, tn * BN + c * 32, row0, M, N, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0);
        }
        ep.drain(lane);
    }

    tc_fence_before();
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace pair
}  // namespace mfp8
