// gemm_splitk.cuh — weight-streaming tcgen05 FP8 GEMM for decode-sized M.
//
// At M <= 128 the Linear is bound by reading W8 from HBM, so the kernel is
// shaped around the weight stream rather than around the output tile:
//   - operands are swapped: a 128-row tile of W8 is the MMA's A operand
//     (M = 128) and the M tokens, padded to MP (16..128), are its N, so the
//     accumulator is D^T [128 output channels x MP tokens] in TMEM;
//   - K is split across the CTAs of a thread-block cluster (S CTAs, one
//     K-slice each, S chosen so that the grid covers every SM), each with a
//     deep TMA ring so that enough weight bytes are in flight per SM;
//   - the S partial accumulators are reduced through distributed shared
//     memory in a fixed rank order (deterministic, no workspace, no atomics),
//     each CTA reducing 128/S of the output channels, then scaled by
//     s_a[m] * s_w[n] and written as bf16.
//
// Every wait is bounded; see gemm_tiled.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {
namespace splitk {

constexpr int BW = 128;   // weight rows per tile (MMA M)
constexpr int BK = 128;   // bytes of K per ring slot
constexpr int MMA_K = 32;
constexpr int kThreads = 192;
constexpr int kMaxCluster = 8;

template <int MP, int STAGES>
struct Layout {
    static constexpr int W_BYTES = BW * BK;   // 16 KB
    static constexpr int X_BYTES = MP * BK;
    static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = STAGES * W_BYTES;
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
    // fp32 partial D^T, row = output channel, padded against bank conflicts.
    // It reuses the ring once the main loop is over.
    static constexpr int RED_LD = MP + 4;
    static constexpr int RED_BYTES = BW * RED_LD * 4;
    static_assert(RED_BYTES <= RING_BYTES, "partial tile must fit in the ring");
    static constexpr int BAR_OFF = RING_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2;  // full, empty, tfull, drain
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int USED = MISC_OFF + 16;
    static constexpr int SMEM_BYTES = USED + 1024;
    static constexpr int TMEM_COLS = MP < 32 ? 32 : MP;
    static_assert(MP % 16 == 0 && MP >= 16 && MP <= 256, "MMA N for M=128");
};

template <int MP, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const float* __restrict__ s_a, const float* __restrict__ s_w,
                   __nv_bfloat16* __restrict__ Y, int M, int N, int K) {
    using L = Layout<MP, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sW = sbase + L::W_OFF;
    const uint32_t sX = sbase + L::X_OFF;
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    float* red = reinterpret_cast<float*>(smem);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const uint32_t S = gridDim.x;  // cluster spans the whole x dimension
    const int n0 = blockIdx.y * BW;
    const int kb_total = (K + BK - 1) / BK;
    const int kb_begin = int((int64_t(kb_total) * rank) / S);
    const int kb_end = int((int64_t(kb_total) * (rank + 1)) / S);
    const int nkb = kb_end - kb_begin;  // >= 1: the host keeps S <= kb_total

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
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
            int stage = 0;
            uint32_t phase = 0;
            // The weight tiles do not depend on the previous kernel: start
            // streaming them first, then wait for X8 before its first load.
            const int prologue = nkb < STAGES ? nkb : STAGES;
            for (int i = 0; i < prologue; ++i) {
                mbar_arrive_expect_tx(full_bar(i), L::STAGE_BYTES);
                tma_load_2d_hint(sW + i * L::W_BYTES, &tmW, full_bar(i), (kb_begin + i) * BK, n0, policy_w);
            }
            grid_dependency_wait();
            for (int i = 0; i < prologue; ++i) {
                tma_load_2d(sX + i * L::X_BYTES, &tmX, full_bar(i), (kb_begin + i) * BK, 0);
                issued_mask |= 1u << i;
            }
            stage = prologue % STAGES;
            phase = prologue == STAGES ? 1u : 0u;
            for (int i = prologue; i < nkb; ++i) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(full_bar(stage), L::STAGE_BYTES);
                tma_load_2d_hint(sW + stage * L::W_BYTES, &tmW, full_bar(stage), (kb_begin + i) * BK, n0, policy_w);
                tma_load_2d(sX + stage * L::X_BYTES, &tmX, full_bar(stage), (kb_begin + i) * BK, 0);
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
            constexpr uint32_t idesc = idesc_e4m3_f32(BW, MP);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued_any = false;
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t w0 = sW + stage * L::W_BYTES;
                const uint32_t x0 = sX + stage * L::X_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / MMA_K; ++kk)
                    mma_f8(tmem_base, sw128_kmajor_desc(w0 + kk * MMA_K), sw128_kmajor_desc(x0 + kk * MMA_K),
                           idesc, (i | kk) != 0);
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
        // Epilogue warps: accumulator lanes -> fp32 partial tile in shared memory.
        const uint32_t q = warp & 3u;
        const int nl = int(q * 32 + lane);  // output channel within the tile
        if (mbar_wait(tfull_bar, 0, abort_flag)) {
            tc_fence_after();
            float* dst = red + nl * L::RED_LD;
#pragma unroll
            for (int c = 0; c < MP; c += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem_base + ((q * 32u) << 16) + uint32_t(c), r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(dst + c + j) =
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                    __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            }
        }
        tc_fence_before();
    }

    // Every partial tile of the cluster is in shared memory after this.
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();

    if (!*abort_flag) {
        grid_dependency_wait();  // s_a may come from the kernel launched just before
        // This CTA reduces output channels [c0, c1) of the tile over the S
        // partials, in rank order, then applies the scales.
        const int c0 = int((BW * rank) / S);
        const int c1 = int((BW * (rank + 1)) / S);
        const int rows = c1 - c0;
        const int mcount = M < MP ? M : MP;
        const uint32_t red_base = smem_u32(red);
        for (int e = threadIdx.x; e < rows * mcount; e += kThreads) {
            const int m = e / rows;
            const int nl = c0 + e % rows;
            const int n = n0 + nl;
            const uint32_t off = uint32_t((nl * L::RED_LD + m) * 4);
            float acc = 0.0f;
            for (uint32_t p = 0; p < S; ++p) {
                float v;
                asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(mapa_shared(red_base + off, p)) : "memory");
                acc += v;
            }
            if (n < N) Y[int64_t(m) * N + n] = __float2bfloat16_rn(acc * __ldcg(s_a + m) * __ldg(s_w + n));
        }
    }

    // Keep this CTA's shared memory alive until every peer has read it.
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

}  // namespace splitk
}  // namespace mfp8
