// gemm_decode.cuh — the decode-sized Linear (M <= 64 tokens) in one kernel:
// per-token activation quantization fused into a weight-streaming split-K
// tcgen05 GEMM, with all cross-CTA traffic pushed through distributed shared
// memory so that no CTA ever waits on a full cluster barrier after start-up.
//
// Work split: a 128-row tile of W8 (output channels n0..n0+127) is the MMA's
// A operand; the tokens, padded to MP, are its N; K is split over the S CTAs
// of a cluster (rank r owns k-blocks [r*KB/S, (r+1)*KB/S)).
//
// Per CTA:
//   0. init barriers, allocate TMEM, arrive on the cluster barrier;
//   1. thread 0 starts the W8 stream into a STAGES-deep TMA ring (before
//      waiting on the previous kernel when the caller declared the weights
//      static);
//   2. every thread loads its share of this CTA's K-slice of X (BF16) into
//      registers (a large slice's remainder is read again in step 4) and
//      folds it into a per-row absmax in shared memory;
//   3. the per-row slice maxima are pushed to every CTA of the cluster with
//      st.async (remote store + transaction count on the receiver's
//      mbarrier); each CTA then holds all S maxima of every row, takes the
//      row absmax and forms the per-token scale (IEEE divide, as the
//      standalone quantizer);
//   4. the registers are quantized to e4m3 and written into shared memory in
//      the 128-byte-swizzled K-major layout the MMA reads (rows >= M and
//      columns >= K are zero);
//   5. one thread issues the MMAs as W8 stages land (fp32 accumulator
//      D^T[128 x MP] in TMEM);
//   6. the epilogue warps read their 32 accumulator rows (output channels)
//      and push each row, with st.async, to the CTA of the cluster that owns
//      that channel (rank r owns channels [128r/S, 128(r+1)/S));
//   7. each CTA waits for the S partial rows of its channels, sums them in
//      rank order (deterministic), scales by s_a[m] * s_w[n] and stores BF16.
// The codes and scales are bit-identical to mfp8_quantize_act; the first
// cluster can write them out for checking.
//
// Every wait is bounded; see gemm_tiled.cuh.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace mfp8 {
namespace decode {

constexpr int BW = 128;
constexpr int BK = 128;
constexpr int MMA_K = 32;
constexpr int kThreads = 192;
constexpr int kMaxCluster = 8;
constexpr int kGroupsPerBlock = BK / 8;  // 8-element groups per k-block row

__device__ __forceinline__ void st_async_u32(uint32_t remote_addr, uint32_t v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];"
                 ::"r"(remote_addr), "r"(v), "r"(remote_bar) : "memory");
}

__device__ __forceinline__ void st_async_v4(uint32_t remote_addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(remote_addr), "r"(a), "r"(b), "r"(c), "r"(d), "r"(remote_bar) : "memory");
}

// Shared-memory layout (byte offsets from the 1024-aligned base).
template <int MP, int STAGES>
struct Layout {
    static constexpr int W_BYTES = BW * BK;
    static constexpr int RING = 0;
    static constexpr int RING_BYTES = STAGES * W_BYTES;
    static constexpr int X_TILE = MP * BK;  // codes of one k-block, multiple of 1024
    static_assert(X_TILE % 1024 == 0, "code tiles keep the 1024-byte swizzle alignment");
    static constexpr int TMEM_COLS = MP < 32 ? 32 : MP;
    static constexpr int NUM_BARS = 2 * STAGES + 4;  // full, empty, tfull, drain, xbar, rbar
    // [X tiles: nkb_cap * X_TILE][recv: 128 rows * MP floats][pmax_all: kMaxCluster * MP]
    // [pmax_local: MP][sa: MP][1/sa: MP][s_w of my channels: 128][bars][tmem holder, abort flag]
    __host__ __device__ static int x_off() { return RING_BYTES; }
    __host__ __device__ static int recv_off(int nkb_cap) { return x_off() + nkb_cap * X_TILE; }
    // S * ceil(128 / S) <= 128 + S rows of partials
    __host__ __device__ static int pmax_all_off(int nkb_cap) { return recv_off(nkb_cap) + (BW + kMaxCluster) * MP * 4; }
    __host__ __device__ static int pmax_off(int nkb_cap) { return pmax_all_off(nkb_cap) + kMaxCluster * MP * 4; }
    __host__ __device__ static int sa_off(int nkb_cap) { return pmax_off(nkb_cap) + MP * 4; }
    __host__ __device__ static int sw_off(int nkb_cap) { return sa_off(nkb_cap) + 2 * MP * 4; }
    __host__ __device__ static int bar_off(int nkb_cap) { return (sw_off(nkb_cap) + BW * 4 + 7) & ~7; }
    __host__ __device__ static int misc_off(int nkb_cap) { return bar_off(nkb_cap) + NUM_BARS * 8; }
    __host__ __device__ static int smem_bytes(int nkb_cap) { return misc_off(nkb_cap) + 16 + 1024; }
};

// ITEMS: 8-element groups of X a thread keeps in registers between the
// absmax pass and the codes pass; groups beyond ITEMS * 192 are read twice.
template <int MP, int STAGES, int ITEMS>
__global__ void __launch_bounds__(kThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __nv_bfloat16* __restrict__ X,
                   const float* __restrict__ s_w, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
                   int nkb_cap, int weights_static, uint8_t* __restrict__ x8_out, float* __restrict__ sa_out) {
    using L = Layout<MP, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sW = sbase + L::RING;
    const uint32_t sX = sbase + L::x_off();
    uint8_t* xtiles = smem + L::x_off();
    float* recv = reinterpret_cast<float*>(smem + L::recv_off(nkb_cap));         // [S][rows][MP] packed
    uint32_t* pmax_all = reinterpret_cast<uint32_t*>(smem + L::pmax_all_off(nkb_cap));  // [S][MP]
    uint32_t* pmax = reinterpret_cast<uint32_t*>(smem + L::pmax_off(nkb_cap));          // [MP]
    float* sa_sm = reinterpret_cast<float*>(smem + L::sa_off(nkb_cap));                  // [MP]
    float* ra_sm = sa_sm + MP;                                                            // [MP] 1/s
    float* sw_sm = reinterpret_cast<float*>(smem + L::sw_off(nkb_cap));                  // [my_rows]
    const uint32_t bar0 = sbase + L::bar_off(nkb_cap);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 1);
    const uint32_t xbar = bar0 + 8u * (2 * STAGES + 2);  // all S slice maxima received
    const uint32_t rbar = bar0 + 8u * (2 * STAGES + 3);  // all S partials of my channels received
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::misc_off(nkb_cap));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc_off(nkb_cap) + 4);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const uint32_t S = gridDim.x;
    const int n0 = blockIdx.y * BW;
    const int kb_total = (K + BK - 1) / BK;
    const int kb_begin = int((int64_t(kb_total) * rank) / S);
    const int kb_end = int((int64_t(kb_total) * (rank + 1)) / S);
    const int nkb = kb_end - kb_begin;  // 1 <= nkb <= nkb_cap (host)
    const int k_lo = kb_begin * BK;
    // Output channels this CTA reduces.
    const int c0 = int((BW * rank) / S);
    const int c1 = int((BW * (rank + 1)) / S);
    const int my_rows = c1 - c0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(drain_bar, 1);
        mbar_init(xbar, 1);
        mbar_init(rbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // Bytes this CTA will receive: S slice maxima per row, and S partial
        // rows of MP floats for each of its channels.
        mbar_arrive_expect_tx(xbar, S * MP * 4u);
        mbar_arrive_expect_tx(rbar, S * uint32_t(my_rows) * MP * 4u);
        tma_prefetch_desc(&tmW);
    }
    if (threadIdx.x < MP) pmax[threadIdx.x] = 0;
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Peers may push into this CTA once they pass the matching wait.
    cluster_arrive_release();
    const uint32_t tmem_base = *tmem_holder;

    // 1. The weight stream.
    const int prologue = nkb < STAGES ? nkb : STAGES;
    uint64_t policy_w = 0;
    if (threadIdx.x == 0) {
        policy_w = l2_policy_evict_first();
        if (!weights_static) grid_dependency_wait();
        for (int i = 0; i < prologue; ++i) {
            mbar_arrive_expect_tx(full_bar(i), L::W_BYTES);
            tma_load_2d_hint(sW + i * L::W_BYTES, &tmW, full_bar(i), (kb_begin + i) * BK, n0, policy_w);
        }
    }
    // The channel scales this CTA applies, fetched while the rest proceeds.
    if (weights_static && threadIdx.x >= 64 && threadIdx.x < 64 + my_rows) {
        const int n = n0 + c0 + int(threadIdx.x) - 64;
        sw_sm[threadIdx.x - 64] = n < N ? __ldg(s_w + n) : 0.0f;
    }
    grid_dependency_wait();  // X comes from earlier work on the stream
    grid_launch_dependents();
    if (!weights_static && threadIdx.x >= 64 && threadIdx.x < 64 + my_rows) {
        const int n = n0 + c0 + int(threadIdx.x) - 64;
        sw_sm[threadIdx.x - 64] = n < N ? __ldg(s_w + n) : 0.0f;
    }

    // 2. This CTA's K-slice of X into registers; per-row slice absmax.
    const int groups_per_row = nkb * kGroupsPerBlock;
    const int items = M * groups_per_row;  // rows >= M are padding
    uint4 xv[ITEMS];
    {
        uint32_t run_max = 0;
        int run_row = -1;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int e = int(threadIdx.x) + i * kThreads;
            xv[i] = make_uint4(0u, 0u, 0u, 0u);
            if (e < items) {
                const int m = e / groups_per_row;
                const int k = k_lo + (e % groups_per_row) * 8;
                if (k < K) {
                    xv[i] = __ldg(reinterpret_cast<const uint4*>(X + int64_t(m) * K + k));
                    const uint32_t a = absmax_bits_u4(xv[i], 0u);
                    const uint32_t a16 = max(a & 0xffffu, a >> 16);
                    if (m != run_row) {
                        if (run_row >= 0) atomicMax(pmax + run_row, run_max);
                        run_row = m;
                        run_max = 0;
                    }
                    run_max = max(run_max, a16);
                }
            }
        }
        // Items beyond the register cache (large slices): max only; the
        // codes pass reads them again (L2-resident by then).
        for (int e = int(threadIdx.x) + ITEMS * kThreads; e < items; e += kThreads) {
            const int m = e / groups_per_row;
            const int k = k_lo + (e % groups_per_row) * 8;
            if (k < K) {
                const uint32_t a = absmax_bits_u4(__ldg(reinterpret_cast<const uint4*>(X + int64_t(m) * K + k)), 0u);
                const uint32_t a16 = max(a & 0xffffu, a >> 16);
                if (m != run_row) {
                    if (run_row >= 0) atomicMax(pmax + run_row, run_max);
                    run_row = m;
                    run_max = 0;
                }
                run_max = max(run_max, a16);
            }
        }
        if (run_row >= 0) atomicMax(pmax + run_row, run_max);
    }
    __syncthreads();
    cluster_wait_acquire();  // every CTA of the cluster has initialised its barriers

    // 3. Push this slice's maxima to every CTA; collect the S maxima of every row.
    if (threadIdx.x < MP) {
        const int m = int(threadIdx.x);
        const uint32_t slot = smem_u32(pmax_all + rank * MP + m);
        for (uint32_t p = 0; p < S; ++p)
            st_async_u32(mapa_shared(slot, p), pmax[m], mapa_shared(xbar, p));
    }
    if (mbar_wait(xbar, 0, abort_flag)) {
        if (threadIdx.x < MP) {
            const int m = int(threadIdx.x);
            uint32_t amax = 0;
            for (uint32_t p = 0; p < S; ++p) amax = max(amax, pmax_all[p * MP + m]);
            const float s = scale_from_absmax_bits(amax);
            sa_sm[m] = s;
            ra_sm[m] = __frcp_rn(s);
            if (sa_out && blockIdx.y == 0 && rank == 0 && m < M) sa_out[m] = s;
        }
    }
    __syncthreads();

    // 4. Codes into the swizzled tiles (zeros for padding rows and columns).
    for (int e = items + int(threadIdx.x); e < MP * groups_per_row; e += kThreads) {
        const int m = e / groups_per_row;
        const int g = e % groups_per_row;
        const int kc = (g % kGroupsPerBlock) * 8;
        const int chunk = (kc >> 4) ^ (m & 7);
        *reinterpret_cast<uint2*>(xtiles + (g / kGroupsPerBlock) * L::X_TILE + m * BK + chunk * 16 + (kc & 15)) =
            make_uint2(0u, 0u);
    }
    {
        const bool write_out = x8_out != nullptr && blockIdx.y == 0;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int e = int(threadIdx.x) + i * kThreads;
            if (e < items) {
                const int m = e / groups_per_row;
                const int g = e % groups_per_row;
                const int kb_local = g / kGroupsPerBlock;
                const int kc = (g % kGroupsPerBlock) * 8;
                const int k = k_lo + g * 8;
                uint2 q = make_uint2(0u, 0u);
                if (k < K) {
                    q = quantize8(xv[i], sa_sm[m], ra_sm[m]);
                    if (write_out) *reinterpret_cast<uint2*>(x8_out + int64_t(m) * K + k) = q;
                }
                const int chunk = (kc >> 4) ^ (m & 7);
                *reinterpret_cast<uint2*>(xtiles + kb_local * L::X_TILE + m * BK + chunk * 16 + (kc & 15)) = q;
            }
        }
        for (int e = int(threadIdx.x) + ITEMS * kThreads; e < items; e += kThreads) {
            const int m = e / groups_per_row;
            const int g = e % groups_per_row;
            const int kc = (g % kGroupsPerBlock) * 8;
            const int k = k_lo + g * 8;
            uint2 q = make_uint2(0u, 0u);
            if (k < K) {
                q = quantize8(__ldg(reinterpret_cast<const uint4*>(X + int64_t(m) * K + k)), sa_sm[m], ra_sm[m]);
                if (write_out) *reinterpret_cast<uint2*>(x8_out + int64_t(m) * K + k) = q;
            }
            const int chunk = (kc >> 4) ^ (m & 7);
            *reinterpret_cast<uint2*>(xtiles + (g / kGroupsPerBlock) * L::X_TILE + m * BK + chunk * 16 + (kc & 15)) = q;
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // codes -> tensor-core reads
    __syncthreads();

    // 5. Ring refills and MMAs.
    if (warp == 0) {
        if (lane == 0) {
            uint32_t issued_mask = (1u << prologue) - 1u, issued_parity = 0;
            int stage = prologue % STAGES;
            uint32_t phase = prologue == STAGES ? 1u : 0u;
            for (int i = prologue; i < nkb && !*abort_flag; ++i) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(full_bar(stage), L::W_BYTES);
                tma_load_2d_hint(sW + stage * L::W_BYTES, &tmW, full_bar(stage), (kb_begin + i) * BK, n0, policy_w);
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
            bool ok = !*abort_flag, issued_any = false;
            for (int i = 0; i < nkb && ok; ++i) {
                if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t w0 = sW + stage * L::W_BYTES;
                const uint32_t x0 = sX + i * L::X_TILE;
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
        // 6. Accumulator rows -> the owning CTA.  Row nl (output channel
        //    n0 + nl) belongs to rank p with c0(p) <= nl < c1(p).
        const uint32_t q = warp & 3u;
        const int nl = int(q * 32 + lane);
        if (mbar_wait(tfull_bar, 0, abort_flag)) {
            tc_fence_after();
            uint32_t p = uint32_t((nl * int(S)) / BW);
            while (p + 1 < S && nl >= int((BW * (p + 1)) / S)) ++p;
            while (p > 0 && nl < int((BW * p) / S)) --p;
            const int pc0 = int((BW * p) / S);
            const int prow = int((BW * (p + 1)) / S) - pc0;
            // recv layout of the owner: [src rank][its rows][MP]
            const uint32_t dst = mapa_shared(smem_u32(recv) + uint32_t(((rank * prow) + (nl - pc0)) * MP * 4), p);
            const uint32_t dbar = mapa_shared(rbar, p);
#pragma unroll
            for (int c = 0; c < MP; c += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem_base + ((q * 32u) << 16) + uint32_t(c), r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 4) st_async_v4(dst + (c + j) * 4, r[j], r[j + 1], r[j + 2], r[j + 3], dbar);
            }
        }
        tc_fence_before();
    }

    // 7. Reduce this CTA's channels over the S partials, in rank order.
    if (mbar_wait(rbar, 0, abort_flag)) {
        for (int e = threadIdx.x; e < my_rows * M; e += kThreads) {
            const int m = e / my_rows;
            const int r = e % my_rows;
            const int n = n0 + c0 + r;
            float acc = 0.0f;
            for (uint32_t p = 0; p < S; ++p) acc += recv[(p * my_rows + r) * MP + m];
            if (n < N) Y[int64_t(m) * N + n] = __float2bfloat16_rn(acc * sa_sm[m] * sw_sm[r]);
        }
    } else {
        // Give partials still on their way a bounded chance to land before
        // this CTA's shared memory goes away.
        volatile int no_abort = 0;
        mbar_wait(rbar, 0, &no_abort, 10000000ull);
        mbar_wait(xbar, 0, &no_abort, 10000000ull);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

}  // namespace decode
}  // namespace mfp8
