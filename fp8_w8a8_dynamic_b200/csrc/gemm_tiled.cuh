// gemm_tiled.cuh — persistent, warp-specialised tcgen05 FP8 GEMM for
// prefill-sized M:
//     Y[m, n] = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
// X8 [M, K] and W8 [N, K] are both K-major ("TN"), which is what the 8-bit
// tcgen05.mma operand path takes without a transpose.
//
// Structure (one CTA per SM, 6 warps):
//   warp 0     TMA producer: 128 x 128-byte tiles of X8 and BN x 128-byte
//              tiles of W8 into a STAGES-deep shared-memory ring (128-byte
//              swizzle), completion tracked by transaction-count mbarriers;
//   warp 1     TMEM allocator and MMA issuer: one thread issues
//              tcgen05.mma.kind::f8f6f4 (128 x BN x 32 per instruction) into
//              one of two fp32 TMEM accumulators (2 x BN columns), and
//              tcgen05.commit releases ring slots and hands finished
//              accumulators to the epilogue;
//   warps 2-5  epilogue: tcgen05.ld of their 32-lane quarter of the
//              accumulator, scale by s_a[m] * s_w[n], round to bf16, stage
//              32 x 32 blocks in shared memory and store them with TMA.
// The two accumulators let the epilogue of tile i overlap the main loop of
// tile i+1.  Tiles are walked n-fastest so that one wave of CTAs shares
// a few X8 row panels and the whole W8 stays L2-resident.
//
// Every wait is bounded (mbar_wait): on timeout the kernel records
// MFP8_ERR_TIMEOUT, drains what it has in flight and frees its TMEM.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {
namespace tiled {

constexpr int BM = 128;          // rows of X8 per tile (MMA M)
constexpr int BK = 128;          // bytes (= e4m3 elements) of K per ring slot
constexpr int MMA_K = 32;        // K of one tcgen05.mma for 8-bit operands
constexpr int kThreads = 192;

template <int BN, int STAGES>
struct Layout {
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = STAGES * A_BYTES;
    static constexpr int STG_OFF = STAGES * STAGE_BYTES;  // epilogue staging: 4 warps x 2 x 2 KB
    static constexpr int BAR_OFF = STG_OFF + 4 * 4096;
    // full[S], empty[S], tfull[2], tempty[2], drain
    static constexpr int NUM_BARS = 2 * STAGES + 5;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // tmem base, abort flag
    static constexpr int USED = MISC_OFF + 16;
    static constexpr int SMEM_BYTES = USED + 1024;  // slack for 1024-byte alignment
    static constexpr int TMEM_COLS = 2 * BN;
    static_assert(TMEM_COLS <= 512, "two accumulators must fit in TMEM");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "MMA N for M=128");
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tiled_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const __grid_constant__ CUtensorMap tmY,
                  const float* __restrict__ s_a, const float* __restrict__ s_w,
                  __nv_bfloat16* __restrict__ Y, int M, int N, int K) {
    using L = Layout<BN, STAGES>;
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
            mbar_init(tempty_bar(b), 4);  // one arrival per epilogue warp
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // The next call's quantize kernel may start launching; it waits for this
    // grid to finish before it touches memory.
    grid_launch_dependents();
    // X8 and s_a may come from the quantize kernel launched just before.
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            const uint64_t policy_w = l2_policy_evict_last();
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                const int tm = tile / n_tiles, tn = tile % n_tiles;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                    mbar_arrive_expect_tx(full_bar(stage), L::STAGE_BYTES);
                    tma_load_2d(sA + stage * L::A_BYTES, &tmX, full_bar(stage), kb * BK, tm * BM);
                    tma_load_2d_hint(sB + stage * L::B_BYTES, &tmW, full_bar(stage), kb * BK, tn * BN, policy_w);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (*abort_flag) {
                // Let every copy still in flight land before the CTA exits.
                volatile int no_abort = 0;
                for (int s = 0; s < STAGES; ++s)
                    if (issued_mask & (1u << s))
                        mbar_wait(full_bar(s), (issued_parity >> s) & 1u, &no_abort, 10000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool issued_any = false;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
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
                    for (int kk = 0; kk < BK / MMA_K; ++kk) {
                        mma_f8(d_tmem, sw128_kmajor_desc(a0 + kk * MMA_K), sw128_kmajor_desc(b0 + kk * MMA_K),
                               idesc, (kb | kk) != 0);
                    }
                    issued_any = true;
                    mma_commit(empty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(tfull_bar(acc));
            }
            if (*abort_flag && issued_any) {
                // Wait for the tensor cores to finish before TMEM is freed.
                volatile int no_abort = 0;
                mma_commit(drain_bar);
                mbar_wait(drain_bar, 0, &no_abort, 10000000ull);
            }
        }
    } else {
        // Epilogue: warp w may read TMEM lanes [32*(w%4), 32*(w%4)+32); the
        // rows go out through shared memory and TMA stores (TmaEpilogue).
        const uint32_t q = warp & 3u;
        TmaEpilogue ep{&tmY, sbase + uint32_t(L::STG_OFF) + q * 4096u};
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) break;
            tc_fence_after();
            const int tm = tile / n_tiles, tn = tile % n_tiles;
            const int row0 = tm * BM + int(q * 32);
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
            if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        ep.drain(lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

}  // namespace tiled
}  // namespace mfp8
