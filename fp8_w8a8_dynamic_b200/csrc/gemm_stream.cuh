// gemm_stream.cuh — the whole FP8_DYNAMIC Linear for decode-sized M
// (M <= 16 tokens) in one kernel: per-token quantization of X, the e4m3 GEMM
// on tcgen05 tensor cores, the scale epilogue and the BF16 store.
//
//   s_a[m]   = fl32(max_k |X[m,k]| / 448)            (raised to FLT_MIN)
//   X8[m,k]  = e4m3_rn_satfinite(fl32(X[m,k] / s_a[m]))
//   Y[m, n]  = bf16( (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n] )
//
// Source of the rule: "MOSS-VL quantization README", FP8-Dynamic recipe
// (float8_e4m3fn weights with one static scale per output channel, FP8
// per-token dynamic activations), and the "MOSS-VL-Realtime-FP8
// mixed-precision strategy" article, section "252 个主力 Linear 层为什么用
// FP8 E4M3" (decode speed is set by how fast the weights are read).
//
// At these sizes the Linear is a stream of N*K weight bytes through the SMs.
// A tcgen05.mma costs at least about 48 cycles however small it is, so each
// instruction should carry as many weight bytes as it can: the weights are
// the A operand (M = 128 output channels x 32 bytes of K = 4 KB per
// instruction) and the tokens the B operand (N = 16, the first M real).
//
// Work split: a cluster of S CTAs (S in 1, 2, 4, 8) owns one tile of 128
// output channels; CTA r of the cluster owns the r-th of S contiguous
// ranges of K blocks.  S is chosen so that the grid is about one CTA per
// SM.  Per CTA:
//   1. start the tile's weights of its K range streaming through a TMA ring
//      (before waiting on the previous kernel when the weights are static);
//      the MMA thread moves the first K blocks from the ring into TMEM
//      (tcgen05.cp) as they land, so up to 7 more blocks than the ring
//      holds are on chip before X exists, and L2 is asked to prefetch the
//      rest;
//   2. the quantizer warps load this CTA's K slice of X (BF16) and take
//      each token's absmax over the slice; the slice maxima go to every CTA
//      of the cluster with st.async (a remote shared-memory store counted on
//      the receiver's mbarrier), so every CTA ends up with the row absmax
//      over all of K and the same scale;
//   3. they quantize the slice (the codes and scales are bit-identical to
//      mfp8_quantize_act) into shared memory in the 128-byte-swizzled
//      K-major layout the MMA reads;
//   4. one thread issues 4 MMAs per 128-byte K block into an fp32 TMEM
//      accumulator D[128 channels][16 tokens], with the weight operand read
//      from TMEM for the parked blocks and from the ring for the others;
//   5. with S > 1, each channel's partial row is pushed with st.async to
//      the CTA of the cluster that owns the channel (rank r owns 128/S of
//      them), which adds the S partials in rank order (deterministic),
//      scales by s_a[m] * s_w[n] and stores BF16.  With S = 1 the epilogue
//      stores directly.
// Shared memory stays near 109 KB and TMEM at most 256 columns (the
// accumulator plus 7 parked K blocks of 32 columns), so two CTAs fit on an
// SM: the kernel lets its dependent launch start at once
// (programmatic dependent launch), and the next Linear's CTAs become
// resident and stream their weights while this one finishes.
//
// Warp roles (64 + 32 QW threads): warp 0 TMA producer, warp 1 TMEM owner
// and MMA issuer, warps 2 .. QW + 1 quantizers and epilogue (warp w reads
// TMEM lanes 32 (w % 4) .. +31 and 64 / QW token columns).  Every wait is bounded; on a timeout the kernel records
// MFP8_ERR_TIMEOUT, drains what it has in flight and frees its TMEM.  A CTA
// leaves only after every remote store addressed to it has landed.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace mfp8 {
namespace stream {

// The kernel is instantiated for 4 or 8 quantizer/epilogue warps (QW): 8
// hide each other's latency when each CTA has many tokens to quantize
// (M > 8), 4 cost less in set-up and barriers below that.
template <int QW>
struct Warps {
    static constexpr int kThreads = 64 + 32 * QW;      // + producer and MMA warps
    static constexpr int kQuantThreads = 32 * QW;
    static constexpr int kRegItems = 64 / QW;          // X vectors a quantizer thread keeps in registers
    static constexpr int kCols = 64 / QW;              // token columns per epilogue warp
    static_assert(QW == 4 || QW == 8, "4 or 8 quantizer warps");
};
constexpr int TILE = 128;                 // output channels per cluster (MMA M)
constexpr int MMA_N = 16;                 // token columns of the MMA (first M real)
constexpr int MMA_K = 32;
constexpr int SUB = 128;                  // K bytes per block: swizzle atom, TMA box width
constexpr int kMaxM = 16;
constexpr int kMaxCluster = 8;
constexpr int kMaxStages = 8;
constexpr int kWStageBytes = TILE * SUB;  // one K block of the tile: 16 KB
constexpr int kShared = 96 * 1024;        // code store + weight ring
constexpr int kMaxCodeBytes = 64 * 1024;
constexpr int kMinStages = 2;
constexpr int kMaxChunks = 16;            // code barriers: 64 or 128 vectors of every row each
constexpr int kAccCols = 32;              // TMEM columns set aside for the accumulator (16 used)
constexpr int kBlockCols = SUB / 4;       // TMEM columns of one weight K block (128 lanes x 128 bytes)
constexpr int kMaxTmemBlocks = (256 - kAccCols) / kBlockCols;  // weight K blocks parked in TMEM: 7
static_assert(SUB / MMA_K == 4 && MMA_K / 4 == 8, "a K block is four MMAs of 8 TMEM columns each");

// Launch geometry, computed on the host (stream_geometry in mfp8.cu).
struct Geometry {
    int S;           // CTAs per cluster (K split)
    int mpad;        // code rows per K block in shared memory: 8 (M <= 8) or 16
    int code_bytes;  // (largest K range in blocks) * mpad * 128, rounded up to 1 KB
    int stages;      // weight ring depth
    int tm_blocks;   // weight K blocks a CTA may park in TMEM (0 .. kMaxTmemBlocks)
};

// TMEM columns a CTA allocates: the accumulator, then tm_blocks weight
// blocks, rounded up to a power of two.  Two CTAs per SM fit in the 512.
__host__ __device__ constexpr uint32_t tmem_cols(int tm_blocks) {
    const int need = kAccCols + (tm_blocks > 0 ? tm_blocks : 0) * kBlockCols;
    return need <= 32 ? 32u : need <= 64 ? 64u : need <= 128 ? 128u : 256u;
}

// Shared memory, from a 1024-byte aligned base:
//   [code store | weight ring]  kShared bytes (the ring starts at code_bytes)
//   [recv] partial rows this CTA owns: [S][128/S][16] fp32 = 8 KB
//   [amax_all] [kMaxCluster][16] u32, [amax_local] [16] u32, [sa] [16] f32
//   [s_w] [128] f32, barriers, TMEM base and abort flag
struct Smem {
    static constexpr int RECV_OFF = kShared;
    static constexpr int RECV_BYTES = TILE * MMA_N * 4;
    static constexpr int AMAX_ALL_OFF = RECV_OFF + RECV_BYTES;
    static constexpr int AMAX_OFF = AMAX_ALL_OFF + kMaxCluster * kMaxM * 4;
    static constexpr int SA_OFF = AMAX_OFF + kMaxM * 4;
    static constexpr int SW_OFF = SA_OFF + kMaxM * 4;
    static constexpr int BAR_OFF = SW_OFF + TILE * 4;
    // wfull[8], wempty[8], chunk[16], xbar, tfull, rbar, drain, tcopy, (pad)
    static constexpr int NUM_BARS = 2 * kMaxStages + kMaxChunks + 6;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int USED = MISC_OFF + 16;
    static constexpr int BYTES = USED + 1024;  // alignment slack
    static_assert(AMAX_ALL_OFF % 16 == 0 && RECV_OFF % 1024 == 0, "st.async targets are 16-byte aligned");
    static_assert(kShared - kMaxCodeBytes >= kMinStages * kWStageBytes, "ring room");
};

struct Args {
    const __nv_bfloat16* X;  // [M, K]
    const float* s_w;        // [N]
    __nv_bfloat16* Y;        // [M, N]
    uint8_t* x8_out;         // optional copy of the codes [M, K] (tile 0's cluster writes it)
    float* sa_out;           // optional copy of the scales [M]
    int M, N, K;
    int weights_static;
    Geometry g;
};

// Position of 16-byte token group g of a partial row in the receive slot
// of channel cl: g ^ recv_swz(cl).  Eight consecutive channels then cover
// all 32 banks when one group is read across them.
__device__ __forceinline__ int recv_swz(int cl) { return (cl >> 1) & 3; }

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint2 v) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y));
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

template <int QW>
__global__ void __launch_bounds__(Warps<QW>::kThreads, 2)
gemm_stream_kernel(const __grid_constant__ CUtensorMap tmW, const Args args) {
    constexpr int kQuantThreads = Warps<QW>::kQuantThreads;
    constexpr int kRegItems = Warps<QW>::kRegItems;
    constexpr int kCols = Warps<QW>::kCols;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int M = args.M, N = args.N, K = args.K;
    const int S = args.g.S, MPAD = args.g.mpad, STAGES = args.g.stages;
    const uint32_t sCode = sbase;
    const uint32_t sW = sbase + uint32_t(args.g.code_bytes);
    const uint32_t bar0 = sbase + Smem::BAR_OFF;
    auto wfull_bar = [&](int s) { return bar0 + 8u * s; };
    auto wempty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
    auto chunk_bar = [&](int c) { return bar0 + 8u * (2 * kMaxStages + c); };  // codes of one chunk written
    const uint32_t xbar = bar0 + 8u * (2 * kMaxStages + kMaxChunks);  // all S slice maxima received
    const uint32_t tfull_bar = xbar + 8u;                              // accumulator complete
    const uint32_t rbar = xbar + 16u;                                  // all partials of my channels received
    const uint32_t drain_bar = xbar + 24u;
    const uint32_t tcopy_bar = xbar + 32u;                             // weight blocks copied into TMEM
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Smem::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::MISC_OFF + 4);
    uint32_t* amax_all = reinterpret_cast<uint32_t*>(smem + Smem::AMAX_ALL_OFF);
    uint32_t* amax_loc = reinterpret_cast<uint32_t*>(smem + Smem::AMAX_OFF);
    float* sa_sm = reinterpret_cast<float*>(smem + Smem::SA_OFF);
    float* sw_sm = reinterpret_cast<float*>(smem + Smem::SW_OFF);

    const uint32_t warp = warp_id_sync();
    const uint32_t lane = lane_id();
    const int rank = S > 1 ? int(cluster_ctarank()) : 0;
    const int tile = int(blockIdx.x) / S;
    const int n0 = tile * TILE;
    const int KB = (K + SUB - 1) / SUB;
    const int kb0 = int((int64_t(KB) * rank) / S);
    const int kb1 = int((int64_t(KB) * (rank + 1)) / S);
    const int nkb = kb1 - kb0;  // >= 1 (the host keeps S <= KB)
    const int k0 = kb0 * SUB;
    const int k1 = min(kb1 * SUB, K);
    const int CPR = TILE / S;   // channels each rank owns in the reduction
    // Quantizer layout (see there): TPR threads per token row, and a code
    // barrier per CV vectors (16 per K block) of every row.
    int mp2 = 1;
    while (mp2 < M) mp2 <<= 1;
    const int TPR = kQuantThreads / mp2;
    const int CV = TPR > 64 ? TPR : 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(wfull_bar(s), 1);
            mbar_init(wempty_bar(s), 1);
        }
        mbar_init(xbar, 1);
        for (int c = 0; c < kMaxChunks; ++c)
            mbar_init(chunk_bar(c), kQuantThreads / 32);  // one arrival per quantizer warp
        mbar_init(tfull_bar, 1);
        mbar_init(rbar, 1);
        mbar_init(drain_bar, 1);
        mbar_init(tcopy_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // The remote bytes this CTA will receive: S slices of 16 maxima, and
        // (S > 1) the S partial rows of each of its 128/S channels.
        if (S > 1) {
            mbar_arrive_expect_tx(xbar, uint32_t(S * kMaxM * 4));
            // 128 channel rows of ceil(M / 4) * 4 fp32 each
            mbar_arrive_expect_tx(rbar, uint32_t(TILE * ((M + 3) / 4) * 16));
        }
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), tmem_cols(args.g.tm_blocks));
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

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer --
            if (!args.weights_static) grid_dependency_wait();
            const uint64_t policy = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            for (int i = 0; i < nkb; ++i) {
                if (i >= STAGES && !mbar_wait(wempty_bar(stage), phase ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(wfull_bar(stage), uint32_t(kWStageBytes));
                tma_load_2d_hint(sW + uint32_t(stage * kWStageBytes), &tmW, wfull_bar(stage), (kb0 + i) * SUB, n0,
                                 policy);
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                if (i + 1 == STAGES)  // the ring is full: L2 fetches the rest meanwhile
                    for (int jb = STAGES; jb < nkb; ++jb) prefetch_tile_l2(&tmW, (kb0 + jb) * SUB, n0);
            }
            if (*abort_flag) {
                volatile int no_abort = 0;
                for (int s = 0; s < STAGES; ++s)
                    if (issued_mask & (1u << s))
                        mbar_wait(wfull_bar(s), (issued_parity >> s) & 1u, &no_abort, 10000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ----------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_e4m3_f32(TILE, MMA_N);
            // K blocks 0 .. T-1 move from the ring into TMEM as soon as they
            // land (before the dependency wait when the weights are static),
            // which frees their slots for blocks STAGES .. STAGES+T-1: the
            // CTA then holds T + STAGES blocks of its slice before X exists.
            const int spare = nkb - STAGES;
            const int T = spare <= 0 ? 0 : (spare < args.g.tm_blocks ? spare : args.g.tm_blocks);
            const uint32_t tmem_w = tmem_base + uint32_t(kAccCols);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued_any = false;
            for (int i = 0; i < T; ++i) {
                if (!mbar_wait(wfull_bar(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = sW + uint32_t(stage * kWStageBytes);
#pragma unroll
                for (int kk = 0; kk < SUB / MMA_K; ++kk)
                    tmem_cp_128x256b(tmem_w + uint32_t(i * kBlockCols + kk * (MMA_K / 4)),
                                     sw128_kmajor_desc(a0 + kk * MMA_K));
                issued_any = true;
                if (i + STAGES < nkb) mma_commit(wempty_bar(stage));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok && T > 0) mma_commit(tcopy_bar);
            // One thread issues every MMA, and at N = 16 its own instruction
            // latency, not the tensor core, sets the pace: an mbarrier test
            // that succeeds at once costs about 200 cycles and per-block
            // bookkeeping as much again, against about 50 cycles per MMA.
            // So the ring blocks already in flight are waited for here,
            // while the quantizers work; the loop then waits once per code
            // chunk (BPC K blocks) and once per block only for blocks still
            // streaming in, and runs straight 4-MMA groups in between, with
            // descriptors advanced by addition.
            const int pre = nkb < T + STAGES ? nkb : T + STAGES;
            {
                int st = stage;
                uint32_t ph = phase;
                for (int i = T; i < pre && ok; ++i) {
                    if (!mbar_wait(wfull_bar(st), ph, abort_flag)) ok = false;
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
            }
            const uint64_t dA0 = sw128_kmajor_desc(sW);
            const uint64_t dB0 = sw128_kmajor_desc(sCode);
            constexpr uint64_t kStep = MMA_K >> 4;        // descriptor units (16 bytes) per 32-byte K step
            constexpr uint64_t kStageStep = kWStageBytes >> 4;
            const uint64_t kBlockStepB = uint64_t(MPAD * SUB) >> 4;
            const int BPC = CV / (SUB / 8);                // K blocks per code chunk: 4 or 8
            const int refill = nkb - STAGES;
            // The four 32-byte K steps of one block, weights from the ring.
            auto mma4 = [&](uint64_t dA, uint64_t dB, uint32_t accf) {
                mma_f8(tmem_base, dA, dB, idesc, accf);
                mma_f8(tmem_base, dA + kStep, dB + kStep, idesc, 1u);
                mma_f8(tmem_base, dA + 2 * kStep, dB + 2 * kStep, idesc, 1u);
                mma_f8(tmem_base, dA + 3 * kStep, dB + 3 * kStep, idesc, 1u);
            };
            int i = 0;
            for (int c = 0; i < nkb && ok; ++c) {
                if (!mbar_wait(chunk_bar(c), 0, abort_flag)) { ok = false; break; }
                if (c == 0 && T > 0 && !mbar_wait(tcopy_bar, 0, abort_flag)) { ok = false; break; }
                tc_fence_after();
                issued_any = true;
                const int iend = nkb < i + BPC ? nkb : i + BPC;
                uint64_t dB = dB0 + uint64_t(i) * kBlockStepB;
                for (; i < iend && i < T; ++i, dB += kBlockStepB) {  // weights parked in TMEM
                    const uint32_t aT = tmem_w + uint32_t(i * kBlockCols);
                    mma_f8_tmem_a(tmem_base, aT, dB, idesc, i != 0);
                    mma_f8_tmem_a(tmem_base, aT + 8u, dB + kStep, idesc, 1u);
                    mma_f8_tmem_a(tmem_base, aT + 16u, dB + 2 * kStep, idesc, 1u);
                    mma_f8_tmem_a(tmem_base, aT + 24u, dB + 3 * kStep, idesc, 1u);
                }
                // Weights in the ring.  A block below `refill` releases its
                // slot for the producer; the blocks from `pre` on are still
                // streaming in and are waited for one by one.
                for (; i < iend && i < pre && i < refill; ++i, dB += kBlockStepB) {
                    const uint64_t dA = dA0 + uint64_t(stage) * kStageStep;
                    mma4(dA, dB, i != 0);
                    mma_commit(wempty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                for (; i < iend && i < pre; ++i, dB += kBlockStepB) {
                    mma4(dA0 + uint64_t(stage) * kStageStep, dB, i != 0);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                for (; i < iend; ++i, dB += kBlockStepB) {
                    if (!mbar_wait(wfull_bar(stage), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    mma4(dA0 + uint64_t(stage) * kStageStep, dB, i != 0);
                    if (i < refill) mma_commit(wempty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
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
        // ------------------------------------------ quantizers, epilogue --
        const int t = int(threadIdx.x) - 64;     // 0 .. kQuantThreads - 1
        const int q = int(warp & 3u);            // TMEM lane quarter of this warp
        const int half = (int(warp) - 2) >> 2;   // and its token columns: kCols * half .. + kCols - 1
        // s_w of the tile (static weights: no need to wait).
        if (!args.weights_static) grid_dependency_wait();
        if (t < TILE) sw_sm[t] = (n0 + t < N) ? __ldg(args.s_w + n0 + t) : 0.f;
        if (t < kMaxM) amax_loc[t] = 0u;
        // Ask L2 for this CTA's slice of X (M rows of (k1 - k0) * 2 bytes)
        // while the previous kernel finishes.  A prefetch returns nothing
        // to the thread: the values used are read after the wait below, so
        // X may still be the previous kernel's output.
        if (t < M) {
            const __nv_bfloat16* p = args.X + int64_t(t) * K + k0;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                         ::"l"(reinterpret_cast<uint64_t>(p)), "r"(uint32_t(k1 - k0) * 2u) : "memory");
        }
        // X may be the previous kernel's output.
        grid_dependency_wait();

        // Rows are spread over the kQuantThreads threads: TPR threads per row (a power
        // of two), thread t takes row t / TPR and the vectors j, j + TPR, ...
        // of the slice (j = t % TPR).  Item u of every thread lies in chunk
        // u / IPC (CV = IPC * TPR vectors of the row per chunk).
        const int m = t / TPR;
        const int j = t % TPR;
        const bool real = m < M;
        const int nv = (k1 - k0) / 8;             // vectors of the slice in a row
        const int nvp = nkb * (SUB / 8);          // ... padded to whole K blocks
        const int items = (nvp + TPR - 1) / TPR;  // per thread
        const bool in_regs = items <= kRegItems;
        const uint4* xrow = reinterpret_cast<const uint4*>(args.X + int64_t(real ? m : 0) * K + k0);
        named_bar_sync(1, kQuantThreads);  // amax_loc cleared

        uint4 buf[kRegItems];
        uint32_t amax = 0;
        for (int u0 = 0; u0 < items; u0 += kRegItems) {
#pragma unroll
            for (int u = 0; u < kRegItems; ++u) {
                const int v = j + (u0 + u) * TPR;
                buf[u] = (real && u0 + u < items && v < nv) ? ldg_nc(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kRegItems; ++u) amax = absmax_bits_u4(buf[u], amax);
        }
        amax = max(amax & 0xffffu, amax >> 16);
        for (int off = 1; off < min(TPR, 32); off <<= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (real && (j & 31) == 0) atomicMax(amax_loc + m, amax);
        named_bar_sync(1, kQuantThreads);
        // With S > 1 this slice's maxima go to every CTA of the cluster (into
        // slot `rank`), and every CTA takes the max over the S slots.
        if (S > 1 && t < S) {
            const uint32_t dst = mapa_shared(smem_u32(amax_all + rank * kMaxM), uint32_t(t));
            const uint32_t bar = mapa_shared(xbar, uint32_t(t));
#pragma unroll
            for (int i = 0; i < kMaxM; i += 4)
                st_async_v4(dst + 4u * i, make_uint4(amax_loc[i], amax_loc[i + 1], amax_loc[i + 2], amax_loc[i + 3]),
                            bar);
        }
        float s = 1.f, r = 1.f;
        const bool have_scale = S == 1 || mbar_wait(xbar, 0, abort_flag);
        if (!have_scale && t == 0) {
            volatile int no_abort = 0;
            mbar_wait(xbar, 0, &no_abort, 20000000ull);
        }
        if (have_scale) {
            if (real) {
                uint32_t a = S == 1 ? amax_loc[m] : 0u;
                for (int i = 0; i < S && S > 1; ++i) a = max(a, amax_all[i * kMaxM + m]);
                s = scale_from_absmax_bits(a);
                r = __frcp_rn(s);
                if (j == 0) {
                    sa_sm[m] = s;
                    if (args.sa_out && tile == 0 && rank == 0) args.sa_out[m] = s;
                }
            }
            // Codes of the slice, K block b of row m at b * MPAD * 128 + m * 128,
            // 16-byte chunks swizzled by (m & 7).  Vectors past K (a ragged
            // last block) are zero codes.  Rows whose scale is below
            // kFmaMinScale take the divide, one vector at a time.
            const bool write_out = args.x8_out != nullptr && tile == 0;
            const uint32_t code_row = sCode + uint32_t(m * SUB);
            auto put = [&](int v, uint2 code) {
                const int blk = v >> 4, c16 = (v & 15) >> 1;
                st_shared_v2(code_row + uint32_t(blk * MPAD * SUB + ((c16 ^ (m & 7)) << 4) + ((v & 1) << 3)), code);
                if (write_out && v < nv)
                    *reinterpret_cast<uint2*>(args.x8_out + int64_t(m) * K + k0 + int64_t(v) * 8) = code;
            };
            const bool fast = s >= kFmaMinScale;
            const int IPC = CV / TPR;
            const int nchunks = (nvp + CV - 1) / CV;
            int chunks_done = 0;
            for (int u0 = 0; u0 < items; u0 += kRegItems) {
                if (!in_regs && real) {
#pragma unroll
                    for (int u = 0; u < kRegItems; ++u) {
                        const int v = j + (u0 + u) * TPR;
                        buf[u] = (u0 + u < items && v < nv) ? ldg_nc(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                // Four vectors at a time with no branch between them, so their
                // arithmetic overlaps; a chunk's barrier is arrived on as soon
                // as every thread is past it.
#pragma unroll
                for (int g = 0; g < kRegItems; g += 4) {
                    if (u0 + g < items) {
                        if (real) {
                            uint2 code[4];
                            if (fast) {
#pragma unroll
                                for (int u = 0; u < 4; ++u) code[u] = quantize8_fast(buf[g + u], s, r);
                            } else {
#pragma unroll
                                for (int u = 0; u < 4; ++u) code[u] = quantize8_div_call(buf[g + u], s);
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int v = j + (u0 + g + u) * TPR;
                                if (u0 + g + u < items && v < nvp) put(v, v < nv ? code[u] : make_uint2(0u, 0u));
                            }
                        }
                        const int done = min(u0 + g + 4, items);
                        const int ready = done >= items ? nchunks : done / IPC;
                        if (ready > chunks_done) {
                            fence_proxy_async_smem();  // codes: generic stores -> tensor-core reads
                            __syncwarp();
                            if (lane == 0)
                                for (int cc = chunks_done; cc < ready; ++cc) mbar_arrive(chunk_bar(cc));
                            chunks_done = ready;
                        }
                    }
                }
            }
        }
        named_bar_sync(1, kQuantThreads);  // sa_sm complete

        // Epilogue: this warp's 32 channels, kCols token columns each.
        const int c = q * 32 + int(lane);  // channel within the tile
        const int m0 = kCols * half;       // first token column of this warp
        uint32_t acc[kCols];
        const bool have_acc = have_scale && mbar_wait(tfull_bar, 0, abort_flag);
        if (have_acc && m0 < M) {
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t(q) * 32u) << 16) + uint32_t(m0);
            if constexpr (kCols == 16)
                tmem_ld_32x32b_x16(ta, acc);
            else
                tmem_ld_32x32b_x8(ta, acc);
            tmem_wait_ld();
        }
        if (S == 1) {
            if (have_acc && m0 < M && n0 + c < N) {
                // The scales are read before the stores, by shared-space
                // address: a generic read after a global store waits for it.
                const float sw = ld_shared_f32(smem_u32(sw_sm + c));
                float sa[kCols];
#pragma unroll
                for (int mm = 0; mm < kCols; mm += 4) {
                    const float4 v = ld_shared_f4(smem_u32(sa_sm + m0 + mm));
                    sa[mm] = v.x;
                    sa[mm + 1] = v.y;
                    sa[mm + 2] = v.z;
                    sa[mm + 3] = v.w;
                }
#pragma unroll
                for (int mm = 0; mm < kCols; ++mm)
                    if (m0 + mm < M)
                        args.Y[int64_t(m0 + mm) * N + n0 + c] =
                            __float2bfloat16_rn(__uint_as_float(acc[mm]) * sa[mm] * sw);
            }
        } else {
            // Partial row of channel c to its owner: slot [rank][c % CPR],
            // 16 token columns in four 16-byte groups, group g stored at
            // position g ^ swz(c % CPR) so that the owner's reads of one
            // group across consecutive channels hit distinct banks.  This
            // warp sends the groups of its kCols token columns.
            if (have_acc && m0 < M) {
                const int owner = c / CPR;
                const int cl = c % CPR;
                const uint32_t local = sbase + uint32_t(Smem::RECV_OFF + ((rank * CPR + cl) * MMA_N) * 4);
                const uint32_t dst = mapa_shared(local, uint32_t(owner));
                const uint32_t bar = mapa_shared(rbar, uint32_t(owner));
#pragma unroll
                for (int h = 0; h < kCols / 4; ++h) {
                    const int g = m0 / 4 + h;
                    if (4 * g < M)  // the token columns that exist, in groups of 4
                        st_async_v4(dst + 16u * uint32_t(g ^ recv_swz(cl)),
                                    make_uint4(acc[4 * h], acc[4 * h + 1], acc[4 * h + 2], acc[4 * h + 3]), bar);
                }
            }
            // Sum the S partials of the channels this rank owns, in rank order.
            const bool have_partials = mbar_wait(rbar, 0, abort_flag);
            if (!have_partials && t == 0) {
                volatile int no_abort = 0;
                mbar_wait(rbar, 0, &no_abort, 20000000ull);
            }
            if (have_partials) {
                // One thread per (channel, group of 4 tokens): a 16-byte read
                // per rank (all issued together), consecutive channels across
                // the warp, so the Y stores of each token row are contiguous.
                // Shared memory is read by shared-space address: a generic
                // read after a global store would wait for the store.
                const int G = (M + 3) / 4;
                const uint32_t recv_base = sbase + uint32_t(Smem::RECV_OFF);
                for (int e = t; e < CPR * G; e += kQuantThreads) {
                    const int cl = e % CPR, g = e / CPR;
                    const int n = n0 + rank * CPR + cl;
                    const uint32_t slot = recv_base + uint32_t((cl * MMA_N + 4 * (g ^ recv_swz(cl))) * 4);
                    float4 p[kMaxCluster];
#pragma unroll
                    for (int i = 0; i < kMaxCluster; ++i)
                        if (i < S) p[i] = ld_shared_f4(slot + uint32_t(i * CPR * MMA_N * 4));
                    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < kMaxCluster; ++i)
                        if (i < S) {
                            sum.x += p[i].x;
                            sum.y += p[i].y;
                            sum.z += p[i].z;
                            sum.w += p[i].w;
                        }
                    if (n < N) {
                        const float sw = ld_shared_f32(smem_u32(sw_sm + rank * CPR + cl));
                        const float4 sa = ld_shared_f4(smem_u32(sa_sm + 4 * g));
                        const float v[4] = {sum.x * sa.x, sum.y * sa.y, sum.z * sa.z, sum.w * sa.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (4 * g + j < M) args.Y[int64_t(4 * g + j) * N + n] = __float2bfloat16_rn(v[j] * sw);
                    }
                }
            }
        }
        tc_fence_before();
    }

    // A CTA receives remote stores only into its maxima and partial-row
    // slots, and has waited for all of them (xbar, rbar) before it gets
    // here, so it can leave without a cluster barrier.  After a timeout the
    // waiting thread gave the late bytes a second bounded wait.
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols(args.g.tm_blocks));
    }
}

}  // namespace stream
}  // namespace mfp8
