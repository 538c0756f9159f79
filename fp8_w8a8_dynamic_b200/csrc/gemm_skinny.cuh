// gemm_skinny.cuh — decode-sized FP8 GEMM (M <= 128 tokens) without
// clusters: split-K over the whole GPU with a last-arriver reduction.
//
//   Y[m, n] = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
//
// At decode sizes the Linear is a stream of W8 through the SMs, and what
// bounds a tcgen05 kernel is how many weight bytes one MMA instruction
// consumes: a tcgen05.mma takes about the same time whether its N is 16 or
// 256, so the weights are the MMA's B operand (N = 256 output channels per
// instruction, 8 KB of W8) and the tokens its A operand (M = 128 rows, of
// which only the first M are real; the TMA load fills the rest with zeros
// and reads nothing for them).
//
// Grid: tiles (256 channels each) x splits (K ranges), at most one CTA per
// SM, no clusters.  Each CTA
//   1. streams its W8 K-range into a 4-stage TMA ring straight away (the
//      weights do not depend on the kernel before it when declared static);
//   2. waits for the activation codes of the quantize kernel launched just
//      before (programmatic dependent launch), and loads them per stage;
//   3. issues 4 MMAs per 128-byte k-block into one fp32 TMEM accumulator;
//   4. writes rows 0..M-1 of the accumulator (fp32) to the workspace
//      ([tile][split][M][256]),
//      fences, and counts itself on the tile's counter;
//   5. the last CTA of a tile to arrive sums the split partials in split
//      order (deterministic), applies s_a[m] * s_w[n] and writes BF16.
// The tile counters live in the workspace and are zeroed by the quantize
// kernel of the same call, so no state carries over between calls.
//
// Every wait is bounded; see gemm_tiled.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {
namespace skinny {

constexpr int BM = 128;       // MMA M: token rows (real ones first)
constexpr int BN = 256;       // MMA N: output channels per tile
constexpr int BK = 128;
constexpr int MMA_K = 32;
constexpr int kThreads = 192;
constexpr int kMaxM = 128;    // all four epilogue warps read their TMEM lanes

template <int STAGES>
struct Layout {
    static constexpr int A_BYTES = BM * BK;   // 16 KB of codes (M real rows)
    static constexpr int B_BYTES = BN * BK;   // 32 KB of weights
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = STAGES * A_BYTES;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2;  // full, empty, tfull, drain
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // tmem holder, abort, last flag
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    static constexpr int TMEM_COLS = BN;
};

// A stage's transaction count is the whole box, rows filled with zeros
// included.
template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const float* __restrict__ s_a, const float* __restrict__ s_w,
                   __nv_bfloat16* __restrict__ Y, float* __restrict__ partial, unsigned int* __restrict__ counters,
                   int M, int N, int K, int weights_static) {
    using L = Layout<STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sA = sbase + L::A_OFF;
    const uint32_t sB = sbase + L::B_OFF;
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const int splits = int(gridDim.x);
    const int split = int(blockIdx.x);
    const int tile = int(blockIdx.y);
    const int n0 = tile * BN;
    const int kb_total = (K + BK - 1) / BK;
    const int kb_begin = int((int64_t(kb_total) * split) / splits);
    const int kb_end = int((int64_t(kb_total) * (split + 1)) / splits);
    const int nkb = kb_end - kb_begin;  // >= 1 (host keeps splits <= kb_total)

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        *last_flag = 0;
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

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t policy_w = l2_policy_evict_first();
            uint32_t issued_mask = 0, issued_parity = 0;
            const int prologue = nkb < STAGES ? nkb : STAGES;
            // Weights first: they do not depend on the previous kernel when
            // the caller declared them static.
            if (!weights_static) grid_dependency_wait();
            for (int i = 0; i < prologue; ++i) {
                mbar_arrive_expect_tx(full_bar(i), L::STAGE_BYTES);
                tma_load_2d_hint(sB + i * L::B_BYTES, &tmW, full_bar(i), (kb_begin + i) * BK, n0, policy_w);
            }
            grid_dependency_wait();  // the codes come from the quantize kernel
            for (int i = 0; i < prologue; ++i) {
                tma_load_2d(sA + i * L::A_BYTES, &tmX, full_bar(i), (kb_begin + i) * BK, 0);
                issued_mask |= 1u << i;
            }
            int stage = prologue % STAGES;
            uint32_t phase = prologue == STAGES ? 1u : 0u;
            for (int i = prologue; i < nkb; ++i) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(full_bar(stage), L::STAGE_BYTES);
                tma_load_2d_hint(sB + stage * L::B_BYTES, &tmW, full_bar(stage), (kb_begin + i) * BK, n0, policy_w);
                tma_load_2d(sA + stage * L::A_BYTES, &tmX, full_bar(stage), (kb_begin + i) * BK, 0);
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (*abort_flag) {
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
            bool ok = true, issued_any = false;
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = sA + stage * L::A_BYTES;
                const uint32_t b0 = sB + stage * L::B_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / MMA_K; ++kk)
                    mma_f8(tmem_base, sw128_kmajor_desc(a0 + kk * MMA_K), sw128_kmajor_desc(b0 + kk * MMA_K), idesc,
                           (i | kk) != 0);
                issued_any = true;
                mma_commit(empty_bar(stage));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) {
                mma_commit(tfull_bar);
            } else if (issued_any) {
                volatile int no_abort = 0;
                mma_commit(drain_bar);
                mbar_wait(drain_bar, 0, &no_abort, 10000000ull);
            }
        }
    } else {
        // Warp w reads TMEM lanes [32 (w % 4), 32 (w % 4) + 32): token rows.
        const uint32_t q = warp & 3u;
        const int m = int(q * 32 + lane);
        if (int(q * 32) < M && mbar_wait(tfull_bar, 0, abort_flag)) {
            tc_fence_after();
            float* dst = partial + ((int64_t(tile) * splits + split) * M + m) * BN;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + uint32_t(c), r);
                tmem_wait_ld();
                if (m < M) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        __stcg(reinterpret_cast<float4*>(dst + c + j),
                               make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                           __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])));
                }
            }
            __threadfence();  // partial visible GPU-wide before this split is counted
        }
        tc_fence_before();
    }

    // Count this split in; the last one of the tile reduces.
    __syncthreads();
    if (threadIdx.x == 0 && !*abort_flag) {
        __threadfence();
        const unsigned int prev = atomicAdd(counters + tile, 1u);
        *last_flag = (prev == unsigned(splits - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag) {
        __threadfence();
        grid_dependency_wait();  // s_a comes from the quantize kernel
        const int cols = min(BN, N - n0);
        for (int e = int(threadIdx.x); e < M * cols; e += kThreads) {
            const int m = e / cols;
            const int c = e % cols;
            const float* src = partial + (int64_t(tile) * splits * M + m) * BN + c;
            float acc = 0.0f;
            for (int p = 0; p < splits; ++p) acc += __ldcg(src + int64_t(p) * M * BN);
            const int n = n0 + c;
            Y[int64_t(m) * N + n] = __float2bfloat16_rn(acc * __ldcg(s_a + m) * __ldg(s_w + n));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

}  // namespace skinny
}  // namespace mfp8
