// gemm_skinny.cuh — decode-sized FP8_DYNAMIC GEMM (M <= 128 tokens) without
// clusters: split-K over the whole GPU with a last-arriver reduction.
//
//   Y[m, n] = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
//
// At decode sizes the Linear is a stream of W8 through the SMs, and what
// bounds a tcgen05 kernel is how many weight bytes one MMA instruction
// consumes: the weights are the MMA's B operand (N = 256 output channels
// per instruction, 8 KB of W8) and the tokens its A operand (M = 128 rows,
// of which only the first M are real; the rest are zeros).
//
// Grid: tiles (256 channels each) x splits (K ranges), at most one CTA per
// SM, no clusters.  Each CTA
//   1. streams its W8 K-range into a 4-stage TMA ring straight away (the
//      weights do not depend on the kernel before it when declared static);
//   2. loads the activation codes of its K-range, per stage, from the codes
//      the quantize kernel launched just before wrote (TMA; rows >= M are
//      filled with zeros and cost no reads);
//   3. issues 4 MMAs per 128-byte k-block into one fp32 TMEM accumulator;
//   4. writes rows 0..M-1 of the accumulator (fp32) to the workspace
//      ([tile][split][M][256]), fences, and counts itself on the tile's
//      counter (atomicInc with wrap-around: the last arrival puts it back to
//      zero, so the counters stay zero between calls);
//   5. the last CTA of a tile to arrive pulls the tile's partials into its
//      (by then idle) ring with bulk copies, one round trip for all splits,
//      sums them in split order (deterministic), applies s_a[m] * s_w[n]
//      (staged in shared memory while the weights streamed) and writes BF16.
//
// Every wait is bounded; see gemm_tiled.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace mfp8 {
namespace skinny {

constexpr int BM = 128;       // MMA M: token rows (real ones first)
constexpr int BN = 256;       // MMA N: output channels per tile
constexpr int BK = 128;
constexpr int MMA_K = 32;
constexpr int kThreads = 192;
constexpr int kMaxM = 128;    // all four epilogue warps read their TMEM lanes
constexpr int kMaxSplits = 16;

template <int STAGES>
struct Layout {
    static constexpr int A_BYTES = BM * BK;   // 16 KB of codes (M real rows)
    static constexpr int B_BYTES = BN * BK;   // 32 KB of weights
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = STAGES * A_BYTES;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 3;  // full, empty, tfull, drain, reduce
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // tmem holder, abort, last flag
    static constexpr int SW_OFF = (MISC_OFF + 16 + 15) / 16 * 16;  // s_w of the tile [BN], read as float4
    static constexpr int SA_OFF = SW_OFF + BN * 4;                                 // s_a [kMaxM]
    static constexpr int SMEM_BYTES = SA_OFF + kMaxM * 4 + 1024;
    static_assert(SW_OFF % 16 == 0 && BAR_OFF % 8 == 0 && RING_BYTES % 1024 == 0, "shared-memory alignment");
    static constexpr int TMEM_COLS = BN;
};

struct Args {
    const float* s_a;        // activation scales from the quantize kernel
    const float* s_w;
    __nv_bfloat16* Y;
    float* partial;
    unsigned int* counters;
    int M, N, K;
    int weights_static;
};

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const Args args) {
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
    const uint32_t red_bar = bar0 + 8u * (2 * STAGES + 2);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
    float* sw_sm = reinterpret_cast<float*>(smem + L::SW_OFF);
    float* sa_sm = reinterpret_cast<float*>(smem + L::SA_OFF);

    const int M = args.M, N = args.N, K = args.K;
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
    const int prologue = nkb < STAGES ? nkb : STAGES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(drain_bar, 1);
        mbar_init(red_bar, 1);
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
    // The next call's quantize kernel may start launching; it waits for this
    // grid to finish before it touches memory.
    grid_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t policy_w = l2_policy_evict_first();
            uint32_t issued_parity = 0;
            if (!args.weights_static) grid_dependency_wait();
            for (int i = 0; i < prologue; ++i) {
                mbar_arrive_expect_tx(full_bar(i), L::STAGE_BYTES);
                tma_load_2d_hint(sB + i * L::B_BYTES, &tmW, full_bar(i), (kb_begin + i) * BK, n0, policy_w);
            }
            grid_dependency_wait();  // the codes come from the quantize kernel
            for (int i = 0; i < prologue; ++i)
                tma_load_2d(sA + i * L::A_BYTES, &tmX, full_bar(i), (kb_begin + i) * BK, 0);
            uint32_t issued_mask = (1u << prologue) - 1u;
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
                // Only the weight copies' bytes are outstanding; a slot whose
                // code writers gave up simply never completes its phase.
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
        const uint32_t q = warp & 3u;
        {
            // The scales the last arriver applies, staged while the weights
            // stream (s_a comes from the quantize kernel: wait for it).
            grid_dependency_wait();
            const int t = int(threadIdx.x) - 64;  // 0..127
            for (int c = t; c < BN; c += 128) sw_sm[c] = (n0 + c < N) ? __ldcg(args.s_w + n0 + c) : 0.f;
            for (int m = t; m < M; m += 128) sa_sm[m] = __ldcg(args.s_a + m);
        }
        // Warp w reads TMEM lanes [32 (w % 4), 32 (w % 4) + 32): token rows.
        const int m = int(q * 32 + lane);
        if (int(q * 32) < M && mbar_wait(tfull_bar, 0, abort_flag)) {
            tc_fence_after();
            float* dst = args.partial + ((int64_t(tile) * splits + split) * M + m) * BN;
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
        // Wraps back to zero on the last arrival.
        const unsigned int prev = atomicInc(args.counters + tile, unsigned(splits - 1));
        *last_flag = (prev == unsigned(splits - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag) {
        __threadfence();  // the other splits' partials, published before their count
        // The tile's partials [splits][M][BN] go into the ring (every MMA
        // has completed, so it is idle), rows_per rows of every split per
        // round: normally one round, one copy per split.
        const int cols = min(BN, N - n0);  // a multiple of 8
        const int c4 = cols / 4;
        const int rows_per = min(M, (L::RING_BYTES / (BN * 4)) / splits);
        const float* tile_part = args.partial + int64_t(tile) * splits * M * BN;
        uint32_t red_phase = 0;
        for (int r0 = 0; r0 < M; r0 += rows_per) {
            const int rows = min(rows_per, M - r0);
            const uint32_t bytes = uint32_t(rows) * BN * 4;
            if (threadIdx.x == 0) {
                fence_proxy_async_global();  // partials: generic stores -> bulk-copy reads
                mbar_arrive_expect_tx(red_bar, bytes * uint32_t(splits));
                for (int j = 0; j < splits; ++j)
                    bulk_load(sbase + uint32_t(j) * bytes, tile_part + (int64_t(j) * M + r0) * BN, bytes, red_bar);
            }
            // One decision for the whole CTA, so that every thread meets the
            // same barriers even when a wait gives up.
            if (!__syncthreads_and(mbar_wait(red_bar, red_phase, abort_flag))) {
                if (threadIdx.x == 0) {
                    // Let the copies in flight land before the CTA exits.
                    volatile int no_abort = 0;
                    mbar_wait(red_bar, red_phase, &no_abort, 10000000ull);
                }
                break;
            }
            red_phase ^= 1u;
            const int items = rows * c4;
            for (int e = int(threadIdx.x); e < items; e += kThreads) {
                const int mr = e / c4, c = (e % c4) * 4;
                const float* src = reinterpret_cast<const float*>(smem) + mr * BN + c;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int j = 0; j < splits; ++j) {
                    const float4 v = *reinterpret_cast<const float4*>(src + j * (bytes / 4));
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                const int m = r0 + mr;
                const float sa = sa_sm[m];
                const float4 sw = *reinterpret_cast<const float4*>(sw_sm + c);
                __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * sa * sw.x, acc.y * sa * sw.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * sa * sw.z, acc.w * sa * sw.w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t*>(&lo);
                pk.y = *reinterpret_cast<uint32_t*>(&hi);
                *reinterpret_cast<uint2*>(args.Y + int64_t(m) * N + n0 + c) = pk;
            }
            fence_proxy_async_smem();  // ring: these generic reads -> the next round's bulk-copy writes
            __syncthreads();
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
