// gemm_cluster.cuh — the FP8 GEMM for small and middle M (up to 256 token
// rows) on activation codes already quantized (the quantize pass of
// mfp8_linear, or the caller's codes in mfp8_gemm):
//
//   Y[m, n] = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
//
// Source of the rule: "MOSS-VL quantization README", FP8-Dynamic recipe
// (float8_e4m3fn weights with one static scale per output channel, FP8
// per-token dynamic activations).
//
// At these sizes the Linear still streams N*K weight bytes and little else,
// and a tcgen05.mma costs about the same up to N = 64 however few columns it
// has.  So the weights are the MMA's 128-row A operand (4 KB per
// instruction) and the tokens its N = MP columns (M rounded up to 16): the
// whole batch in one accumulator of MP TMEM columns.  The layout is the one
// of the decode kernel (gemm_stream.cuh) with the codes loaded by TMA:
//   - a cluster of S CTAs (S in 1, 2, 4, 8) owns one tile of 128 output
//     channels and splits K; each CTA streams its weight K blocks and the
//     matching code blocks (MP rows x 128 bytes) through one TMA ring, the
//     weights before the dependency wait when they are static;
//   - one thread issues 4 MMAs per K block;
//   - with S > 1, once every CTA of the cluster has its accumulator (a
//     cluster barrier), the partial rows are exchanged in rounds of TC
//     token columns: each CTA copies its accumulator columns from TMEM into
//     its own ring (free by then), one slot per owning rank (rank r owns
//     128/S of the channels), and one thread sends each slot to its owner
//     with a single bulk shared-memory copy across the cluster, counted on
//     the owner's barrier; the owner adds the S partials in rank order
//     (deterministic), scales and stores BF16; a cluster barrier ends the
//     round, after which the slots are reused.  With S = 1 the epilogue
//     stores directly.
// About 98 KB of shared memory and at most 256 TMEM columns, so two CTAs
// fit on an SM and the next kernel's CTAs can start alongside.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 2-5 epilogue (warp w reads TMEM lanes 32 (w % 4) .. +31,
// one output channel per thread).  Every wait is bounded; on a timeout the
// kernel records MFP8_ERR_TIMEOUT, drains what it has in flight and frees
// its TMEM.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {
namespace cluster {

constexpr int kThreads = 192;
constexpr int TILE = 128;                   // output channels per cluster (MMA M)
constexpr int SUB = 128;                    // K bytes per block: swizzle atom, TMA box width
constexpr int MMA_K = 32;
constexpr int kMaxM = 256;                  // token rows (MMA N up to 256)
constexpr int kMaxCluster = 8;
constexpr int kMaxStages = 8;
constexpr int kWBlockBytes = TILE * SUB;    // one weight K block of the tile: 16 KB
constexpr int kRingBytes = 96 * 1024;       // weight + code ring; later the partial-row receive area
constexpr int kRingBig = 192 * 1024;        // the ring when the grid has at most one CTA per SM
constexpr int kMinStages = 2;
static_assert(SUB / MMA_K == 4, "a K block is four MMAs");

// Launch geometry, computed on the host (cluster_geometry in mfp8.cu).
struct Geometry {
    int S;       // CTAs per cluster (K split)
    int mp;      // token columns of the MMA: M rounded up to 16
    int stages;  // ring depth; a stage is a weight block and a code block
    int tc;      // token columns per exchange round (S > 1): a multiple of 16, <= mp
    int ring;    // ring bytes: kRingBytes (two CTAs fit on an SM) or kRingBig (grids of at most one CTA per SM)
};

__host__ __device__ constexpr int stage_bytes(int mp) { return kWBlockBytes + mp * SUB; }

__host__ __device__ constexpr uint32_t tmem_cols(int mp) {
    return mp <= 32 ? 32u : mp <= 64 ? 64u : mp <= 128 ? 128u : 256u;
}

// Ring bytes one exchange round of tc token columns takes (S > 1): the
// receive slots [S][tc][128/S] fp32 of the channels this CTA owns, then the
// send slots [S-1][tc][128/S] fp32 of the channels the other ranks own.
__host__ __device__ constexpr int exchange_bytes(int S, int tc) {
    return (TILE * tc * 4 / S) * (2 * S - 1);
}

// Shared memory, from a 1024-byte aligned base:
//   [ring] g.ring bytes: stage s at s * stage_bytes(mp) (weights, then
//          codes); with S > 1 it later holds the exchange slots
//          (exchange_bytes)
//   then, at offset g.ring: [sa] [256] f32, [sw] [128] f32, barriers, TMEM
//          base and abort flag
struct Smem {
    static constexpr int SA_OFF = 0;  // from the end of the ring
    static constexpr int SW_OFF = SA_OFF + kMaxM * 4;
    static constexpr int BAR_OFF = SW_OFF + TILE * 4;
    // full[8], empty[8], tfull, rbar, drain, (pad)
    static constexpr int NUM_BARS = 2 * kMaxStages + 4;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int USED = MISC_OFF + 16;
    static constexpr int bytes(int ring) { return ring + USED + 1024; }  // + alignment slack
    static constexpr int MAX_BYTES = kRingBig + USED + 1024;
    static_assert(exchange_bytes(2, 16) <= kRingBytes, "one round of the narrowest exchange fits in the ring");
    static_assert(kMinStages * stage_bytes(kMaxM) <= kRingBytes, "ring room");
    static_assert(MAX_BYTES <= 227 * 1024, "shared memory of one CTA");
};

struct Args {
    const float* s_a;  // [M]
    const float* s_w;  // [N]
    __nv_bfloat16* Y;  // [M, N]
    int M, N, K;
    int weights_static;
    Geometry g;
};

__global__ void __launch_bounds__(kThreads, 2)
gemm_cluster_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const Args args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int M = args.M, N = args.N, K = args.K;
    const int S = args.g.S, MP = args.g.mp, STAGES = args.g.stages;
    const int SB = stage_bytes(MP);
    uint8_t* fixed = smem + args.g.ring;  // scales, barriers and flags follow the ring
    const uint32_t bar0 = smem_u32(fixed) + Smem::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * kMaxStages);  // accumulator complete
    const uint32_t rbar = tfull_bar + 8u;                     // all partials of my channels received
    const uint32_t drain_bar = tfull_bar + 16u;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fixed + Smem::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(fixed + Smem::MISC_OFF + 4);
    float* sa_sm = reinterpret_cast<float*>(fixed + Smem::SA_OFF);
    float* sw_sm = reinterpret_cast<float*>(fixed + Smem::SW_OFF);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const int rank = S > 1 ? int(cluster_ctarank()) : 0;
    const int tile = int(blockIdx.x) / S;
    const int n0 = tile * TILE;
    const int KB = (K + SUB - 1) / SUB;
    const int kb0 = int((int64_t(KB) * rank) / S);
    const int kb1 = int((int64_t(KB) * (rank + 1)) / S);
    const int nkb = kb1 - kb0;  // >= 1 (the host keeps S <= KB)
    const int CPR = TILE / S;   // channels each rank owns in the reduction
    const uint32_t tcols = tmem_cols(MP);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        // (S > 1) each round, the S - 1 slots sent to this CTA: one arrival
        // (this thread's, below and at the end of each round) and the bytes
        mbar_init(rbar, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (S > 1) mbar_arrive_expect_tx(rbar, uint32_t((S - 1) * CPR * args.g.tc * 4));
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    if (S > 1) {
        // Every CTA's barriers are initialised before any remote store.
        cluster_arrive_release();
        cluster_wait_acquire();
    } else {
        __syncthreads();
    }
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // The next kernel on the stream may start launching now: before its own
    // dependency wait it only sets itself up and fetches static weights.
    grid_launch_dependents();

    bool have_acc = false;
    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer --
            // Weight blocks may go before the dependency wait (static
            // weights); code blocks only after it: the codes come from the
            // quantize pass just before this kernel.
            const uint64_t policy = l2_policy_evict_first();
            const int first = nkb < STAGES ? nkb : STAGES;
            bool waited = false;
            if (!args.weights_static) {
                grid_dependency_wait();
                waited = true;
            }
            for (int e = 0; e < first; ++e) {
                const uint32_t st = sbase + uint32_t(e * SB);
                mbar_arrive_expect_tx(full_bar(e), uint32_t(SB));
                tma_load_2d_hint(st, &tmW, full_bar(e), (kb0 + e) * SUB, n0, policy);
            }
            for (int e = first; e < nkb; ++e) prefetch_tile_l2(&tmW, (kb0 + e) * SUB, n0);
            if (!waited) grid_dependency_wait();
            for (int e = 0; e < first; ++e)
                tma_load_2d(sbase + uint32_t(e * SB + kWBlockBytes), &tmX, full_bar(e), (kb0 + e) * SUB, 0);
            int stage = first == STAGES ? 0 : first;
            uint32_t phase = first == STAGES ? 1u : 0u;
            uint32_t issued_mask = (1u << first) - 1u, issued_parity = 0;
            for (int e = first; e < nkb; ++e) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                const uint32_t st = sbase + uint32_t(stage * SB);
                mbar_arrive_expect_tx(full_bar(stage), uint32_t(SB));
                tma_load_2d_hint(st, &tmW, full_bar(stage), (kb0 + e) * SUB, n0, policy);
                tma_load_2d(st + uint32_t(kWBlockBytes), &tmX, full_bar(stage), (kb0 + e) * SUB, 0);
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
            // ----------------------------------------------- MMA issuer --
            // One wait per K block and four straight MMAs: at these N the
            // issuing thread's own latency sets the pace.
            const uint32_t idesc = idesc_e4m3_f32(TILE, uint32_t(MP));
            constexpr uint64_t kStep = MMA_K >> 4;  // descriptor units (16 bytes) per 32-byte K step
            const uint64_t d0 = sw128_kmajor_desc(sbase);
            const uint64_t dX = uint64_t(kWBlockBytes) >> 4;
            const uint64_t dS = uint64_t(SB) >> 4;
            const int refill = nkb - STAGES;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued_any = false;
            for (int e = 0; e < nkb; ++e) {
                if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                if (e == 0) tc_fence_after();
                issued_any = true;
                const uint64_t dA = d0 + uint64_t(stage) * dS;
                const uint64_t dB = dA + dX;
                mma_f8(tmem_base, dA, dB, idesc, e != 0);
                mma_f8(tmem_base, dA + kStep, dB + kStep, idesc, 1u);
                mma_f8(tmem_base, dA + 2 * kStep, dB + 2 * kStep, idesc, 1u);
                mma_f8(tmem_base, dA + 3 * kStep, dB + 3 * kStep, idesc, 1u);
                if (e < refill) mma_commit(empty_bar(stage));  // the producer refills this slot
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
        // -------------------------------------------- epilogue, part 1 --
        const int t = int(threadIdx.x) - 64;  // 0..127
        sw_sm[t] = (n0 + t < N) ? __ldg(args.s_w + n0 + t) : 0.f;
        grid_dependency_wait();  // s_a comes from the quantize pass
        for (int m = t; m < kMaxM; m += 128) sa_sm[m] = m < M ? __ldg(args.s_a + m) : 0.f;
        have_acc = mbar_wait(tfull_bar, 0, abort_flag);
        named_bar_sync(1, 128);  // sa_sm, sw_sm complete
    }

    // With S > 1 every CTA of the cluster has its accumulator before any
    // partial row lands in a ring: the rings are free from here on.
    __syncwarp();
    if (S > 1) {
        tc_fence_before();
        cluster_arrive_release();
        cluster_wait_acquire();
        tc_fence_after();
    }

    if (S == 1) {
        if (warp >= 2) {
            // -------------------------------------- epilogue, one CTA --
            const int q = int(warp & 3u);       // TMEM lane quarter of this warp
            const int c = q * 32 + int(lane);  // channel within the tile
            if (have_acc) tc_fence_after();
            for (int c0 = 0; c0 < MP && have_acc; c0 += 16) {
                uint32_t acc[16];
                tmem_ld_32x32b_x16(tmem_base + ((uint32_t(q) * 32u) << 16) + uint32_t(c0), acc);
                tmem_wait_ld();
                if (n0 + c < N) {
                    // scales read before the stores (see ld_shared_f4)
                    const float sw = ld_shared_f32(smem_u32(sw_sm + c));
                    float sa[16];
#pragma unroll
                    for (int mm = 0; mm < 16; mm += 4) {
                        const float4 v = ld_shared_f4(smem_u32(sa_sm + c0 + mm));
                        sa[mm] = v.x;
                        sa[mm + 1] = v.y;
                        sa[mm + 2] = v.z;
                        sa[mm + 3] = v.w;
                    }
#pragma unroll
                    for (int mm = 0; mm < 16; ++mm)
                        if (c0 + mm < M)
                            args.Y[int64_t(c0 + mm) * N + n0 + c] =
                                __float2bfloat16_rn(__uint_as_float(acc[mm]) * sa[mm] * sw);
                }
            }
        }
    } else {
        // ---------------------------------- partial-row exchange, S > 1 --
        // Rounds of TC token columns.  Slot layout (fp32, token-major):
        // receive slot s = partials from rank s of the 128/S channels this
        // CTA owns, at s * SLOT; send slot of owner o != rank at (S + o') *
        // SLOT, o' = o or o - 1 (this rank's own slot is written straight
        // into receive slot `rank`).  Row r of a slot is token tok0 + r, its
        // 128/S channels contiguous.  Every warp takes part in the round's
        // closing cluster barrier.
        const int TC = args.g.tc;
        const int rounds = (MP + TC - 1) / TC;
        const uint32_t row_bytes = uint32_t(CPR * 4);
        const uint32_t SLOT = row_bytes * uint32_t(TC);
        for (int j = 0; j < rounds; ++j) {
            const int tok0 = j * TC;
            const int tcj = MP - tok0 < TC ? MP - tok0 : TC;  // columns this round (a multiple of 16)
            if (warp >= 2) {
                const int t = int(threadIdx.x) - 64;
                const int q = int(warp & 3u);
                const int c = q * 32 + int(lane);
                const int o = c / CPR, cl = c % CPR;
                const uint32_t slot = o == rank ? uint32_t(rank) * SLOT : uint32_t(S + (o < rank ? o : o - 1)) * SLOT;
                // This thread's channel in every row of its slot: the 32 lanes
                // of a warp write consecutive words of a row.
                const uint32_t col = sbase + slot + uint32_t(cl) * 4u;
                if (have_acc) {
                    if (j == 0) tc_fence_after();
                    const uint32_t taddr = tmem_base + ((uint32_t(q) * 32u) << 16) + uint32_t(tok0);
                    int c0 = 0;
                    for (; c0 + 32 <= tcj; c0 += 32) {
                        uint32_t acc[32];
                        tmem_ld_32x32b_x32(taddr + uint32_t(c0), acc);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            asm volatile("st.shared.b32 [%0], %1;" ::"r"(col + uint32_t(c0 + i) * row_bytes), "r"(acc[i])
                                         : "memory");
                    }
                    if (c0 < tcj) {  // a last 16 columns
                        uint32_t acc[16];
                        tmem_ld_32x32b_x16(taddr + uint32_t(c0), acc);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            asm volatile("st.shared.b32 [%0], %1;" ::"r"(col + uint32_t(c0 + i) * row_bytes), "r"(acc[i])
                                         : "memory");
                    }
                }
                fence_proxy_async_smem();  // slot writes -> the bulk copies' reads
                named_bar_sync(1, 128);
                if (t == 0 && have_acc) {
                    for (int o2 = 0; o2 < S; ++o2) {
                        if (o2 == rank) continue;
                        const uint32_t src = sbase + uint32_t(S + (o2 < rank ? o2 : o2 - 1)) * SLOT;
                        bulk_copy_to_cluster(mapa_shared(sbase + uint32_t(rank) * SLOT, uint32_t(o2)), src, SLOT,
                                             mapa_shared(rbar, uint32_t(o2)));
                    }
                }
                // Sum the S partials of the channels this rank owns, in rank
                // order, for this round's token columns.
                const bool have_partials = mbar_wait_cluster(rbar, uint32_t(j & 1), abort_flag);
                if (!have_partials && t == 0) {
                    volatile int no_abort = 0;
                    mbar_wait_cluster(rbar, uint32_t(j & 1), &no_abort, 20000000ull);
                }
                // Rows of this round that exist: M - tok0 (when positive).
                const int mj = M - tok0 < tcj ? M - tok0 : tcj;
                if (have_partials && mj > 0) {
                    // One thread per (token row, group of 4 channels): a
                    // 16-byte read per rank (all S issued together; the warp
                    // reads 512 contiguous bytes), the rescale, and one 8-byte
                    // store of 4 bf16 (the warp's stores cover whole row
                    // segments).  Shared memory is read by shared-space
                    // address (ld_shared_*) so that the reads are not ordered
                    // behind the Y stores.
                    const int GPR = CPR / 4;  // 4-channel groups per row
                    const uint32_t sa_base = smem_u32(sa_sm + tok0);
                    const uint32_t sw_base = smem_u32(sw_sm + rank * CPR);
                    for (int e = t; e < mj * GPR; e += 128) {
                        const int r = e / GPR, g4 = e % GPR;
                        const int n = n0 + rank * CPR + 4 * g4;
                        if (n >= N) continue;  // N % 8 == 0: a group of 4 is all in or all out
                        const uint32_t off = uint32_t(r) * row_bytes + uint32_t(16 * g4);
                        float4 p[kMaxCluster];
#pragma unroll
                        for (int i = 0; i < kMaxCluster; ++i)
                            if (i < S) p[i] = ld_shared_f4(sbase + uint32_t(i) * SLOT + off);
                        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < kMaxCluster; ++i)
                            if (i < S) {
                                sum.x += p[i].x;
                                sum.y += p[i].y;
                                sum.z += p[i].z;
                                sum.w += p[i].w;
                            }
                        const float sa = ld_shared_f32(sa_base + uint32_t(4 * r));
                        const float4 sw = ld_shared_f4(sw_base + uint32_t(16 * g4));
                        const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x * sa * sw.x, sum.y * sa * sw.y);
                        const __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z * sa * sw.z, sum.w * sa * sw.w);
                        uint2 packed;
                        packed.x = *reinterpret_cast<const uint32_t*>(&lo);
                        packed.y = *reinterpret_cast<const uint32_t*>(&hi);
                        *reinterpret_cast<uint2*>(args.Y + int64_t(tok0 + r) * N + n) = packed;
                    }
                }
                // Arm the barrier for the next round's slots before any rank
                // can send them (they go only after the cluster barrier below).
                if (t == 0 && j + 1 < rounds) mbar_arrive_expect_tx(rbar, (uint32_t(S) - 1u) * SLOT);
            }
            // Every slot sent this round has landed (each owner waited for its
            // own) and been summed: the slots are free, and after the last
            // round no copy is in flight from or into this CTA.
            __syncwarp();
            cluster_arrive_release();
            cluster_wait_acquire();
        }
    }

    // With S > 1 a CTA receives bulk copies only into its own ring, after the
    // cluster barrier above, and every copy from or into it completed before
    // the last round's cluster barrier.  After a timeout the waiting thread
    // gave the late bytes a second bounded wait.
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tcols);
    }
}

}  // namespace cluster
}  // namespace mfp8
