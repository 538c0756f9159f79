// mfp8.cu — the C ABI declared in include/mfp8.h: argument checks, kernel
// choice, TMA descriptor set-up and launches.  The whole library is this
// one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "../../include/mfp8.h"
#include "status.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "gemm_tiled.cuh"
#include "gemm_pair.cuh"
#include "gemm_stream.cuh"
#include "gemm_cluster.cuh"
#include "producer.cuh"
#include "kv8.cuh"

namespace mfp8 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = int64_t(1) << 30;  // rows / columns accepted per dimension

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int sm_count = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

mfp8_status current_device(int* dev_out, DeviceInfo* info_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return MFP8_ERR_CUDA;
        }
        d.supported = (major == 10 && minor == 0);
        d.sm_count = sms;
        d.ready = true;
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr) {
            cudaGetLastError();
            return MFP8_ERR_CUDA;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!d.supported) return MFP8_ERR_DEVICE;
    *dev_out = dev;
    *info_out = d;
    return MFP8_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [rows, cols] row-major 8-bit matrix, tiles of box_rows x 128 bytes with
// the 128-byte swizzle.
mfp8_status make_map_u8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(cols)};
    cuuint32_t box[2] = {128u, cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MFP8_OK : MFP8_ERR_CUDA;
}

// Y [rows, cols] bf16 for the TMA-store epilogue: 32 x 32 boxes, 64-byte
// rows with the 64-byte swizzle (cols % 8 == 0, so rows are 16-byte aligned).
mfp8_status make_map_y(CUtensorMap* map, void* base, int64_t rows, int64_t cols) {
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MFP8_OK : MFP8_ERR_CUDA;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

mfp8_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? MFP8_OK : MFP8_ERR_CUDA;
}

// ------------------------------------------------------------- quantize --

template <class Kern>
mfp8_status launch_quant(Kern kern, bool dependent, int64_t R, const uint4* x, int64_t K, uint2* q, float* S,
                         cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(R));  // one block per row
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, x, K, q, S) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

// The warp-per-row kernel: `blocks` blocks of 8 rows, R rows in all.
template <class Kern>
mfp8_status launch_quant(Kern kern, bool dependent, int64_t blocks, int64_t R, const uint4* x, int64_t K, uint2* q,
                         float* S, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, x, R, K, q, S) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

template <bool EARLY_TRIGGER>
mfp8_status quantize_rows_t(const void* X, int64_t R, int64_t K, void* Q, float* S, cudaStream_t stream) {
    if (R == 0) return MFP8_OK;
    const int64_t nvec = K / 8;
    const uint4* x = static_cast<const uint4*>(X);
    uint2* q = static_cast<uint2*>(Q);
    // Many rows: 1, 2 or 4 warps per row (8 warps per block) while a row
    // fits in their registers; longer rows get more warps.
    auto blocks = [&](int wpr) { return (R * wpr + kQuantThreads / 32 - 1) / (kQuantThreads / 32); };
    if (R >= 256 && nvec <= 32 * 16 * 4 && blocks(4) <= INT32_MAX) {
        if (nvec <= 32 * 4)
            return launch_quant(quant_rows_warp_kernel<4, 1, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(1), R, x, K, q, S,
                                stream);
        if (nvec <= 32 * 8)
            return launch_quant(quant_rows_warp_kernel<8, 1, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(1), R, x, K, q, S,
                                stream);
        if (nvec <= 32 * 8 * 2)
            return launch_quant(quant_rows_warp_kernel<8, 2, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(2), R, x, K, q, S,
                                stream);
        if (nvec <= 32 * 8 * 4)
            return launch_quant(quant_rows_warp_kernel<8, 4, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(4), R, x, K, q, S,
                                stream);
        if (nvec <= 32 * 12 * 4)
            return launch_quant(quant_rows_warp_kernel<12, 4, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(4), R, x, K, q, S,
                                stream);
        return launch_quant(quant_rows_warp_kernel<16, 4, EARLY_TRIGGER>, EARLY_TRIGGER, blocks(4), R, x, K, q, S,
                            stream);
    }
    if (nvec <= 256) return launch_quant(quant_rows_reg_kernel<1, EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
    if (nvec <= 512) return launch_quant(quant_rows_reg_kernel<2, EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
    if (nvec <= 1024) return launch_quant(quant_rows_reg_kernel<4, EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
    if (nvec <= 1536) return launch_quant(quant_rows_reg_kernel<6, EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
    if (nvec <= 2048) return launch_quant(quant_rows_reg_kernel<8, EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
    return launch_quant(quant_rows_loop_kernel<EARLY_TRIGGER>, EARLY_TRIGGER, R, x, K, q, S, stream);
}

// Activations: the GEMM launched next may start its prologue early.
mfp8_status quantize_act_rows(const void* X, int64_t R, int64_t K, void* Q, float* S, cudaStream_t stream) {
    return quantize_rows_t<true>(X, R, K, Q, S, stream);
}

// Weights: no early start for whatever follows.
mfp8_status quantize_weight_rows(const void* X, int64_t R, int64_t K, void* Q, float* S, cudaStream_t stream) {
    return quantize_rows_t<false>(X, R, K, Q, S, stream);
}

mfp8_status check_quant_args(const void* X, int64_t R, int64_t K, const void* Q, const float* S) {
    if (R < 0 || K < 0) return MFP8_ERR_INVALID_ARG;
    if (K == 0 || K % 16 != 0 || K > kMaxDim || R > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (R == 0) return MFP8_OK;
    if (!X || !Q || !S) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Q) || !aligned16(S)) return MFP8_ERR_MISALIGNED;
    if (ranges_overlap(X, size_t(R * K * 2), Q, size_t(R * K)) ||
        ranges_overlap(X, size_t(R * K * 2), S, size_t(R * 4)) ||
        ranges_overlap(Q, size_t(R * K), S, size_t(R * 4)))
        return MFP8_ERR_INVALID_ARG;
    return MFP8_OK;
}

// ----------------------------------------------------------------- GEMM --


template <class Kern>
mfp8_status set_smem(Kern kern, int bytes, int dev, bool* done) {
    if (done[dev]) return MFP8_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    done[dev] = true;
    return MFP8_OK;
}

template <int BN, int STAGES>
mfp8_status launch_tiled_bn(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8,
                            const float* s_w, int64_t N, int64_t w_rows, void* Y, bool dependent, int dev,
                            const DeviceInfo& info,
                            cudaStream_t stream) {
    using L = tiled::Layout<BN, STAGES>;
    auto kern = tiled::gemm_tiled_kernel<BN, STAGES>;
    static bool attr_done[kMaxDevices] = {};
    mfp8_status st = set_smem(kern, L::SMEM_BYTES, dev, attr_done);
    if (st != MFP8_OK) return st;
    CUtensorMap tmX, tmW, tmY;
    if ((st = make_map_u8(&tmX, X8, M, K, tiled::BM)) != MFP8_OK) return st;
    if ((st = make_map_u8(&tmW, W8, w_rows, K, BN)) != MFP8_OK) return st;
    if ((st = make_map_y(&tmY, Y, M, N)) != MFP8_OK) return st;
    const int64_t tiles = ((M + tiled::BM - 1) / tiled::BM) * ((N + BN - 1) / BN);
    const unsigned grid = static_cast<unsigned>(tiles < info.sm_count ? tiles : info.sm_count);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(tiled::kThreads);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmX, tmW, tmY, s_a, s_w, static_cast<__nv_bfloat16*>(Y), int(M), int(N),
                           int(K)) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

// The 1-CTA kernel's tile width: 256 when that already gives a CTA to most
// SMs, else the widest of 128, 64, 32 that does (narrower tiles re-read the
// X8 row panel more often from L2, but a mid-sized M with 256-wide tiles
// leaves most SMs idle: M = 128, N = 4096 is 16 tiles).
int tiled_tile_width(int64_t M, int64_t N, const DeviceInfo& info) {
    const int64_t mt = (M + tiled::BM - 1) / tiled::BM;
    for (int bn : {256, 128, 64})
        if (mt * ((N + bn - 1) / bn) * 4 >= int64_t(info.sm_count) * 3) return bn;
    return 32;
}

mfp8_status launch_tiled(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8,
                         const float* s_w, int64_t N, int64_t w_rows, void* Y, bool dependent, int dev,
                         const DeviceInfo& info,
                         cudaStream_t stream) {
    switch (tiled_tile_width(M, N, info)) {
        case 256: return launch_tiled_bn<256, 4>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
        case 128: return launch_tiled_bn<128, 6>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
        case 64: return launch_tiled_bn<64, 8>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
        default: return launch_tiled_bn<32, 10>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
    }
}

// Clusters of `S` CTAs of `kern` (with `smem` bytes each) that the device
// keeps resident at once.  Clusters are placed inside one GPC, so this can be
// below (SMs x CTAs per SM) / S.  Cached per device and kernel.
template <class Kern>
int max_active_clusters(Kern kern, int S, int smem, int threads, int dev) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, int, int>, int> cache;
    const auto key = std::make_tuple(dev, reinterpret_cast<const void*>(kern), S, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(S));
    cfg.blockDim = dim3(unsigned(threads));
    cfg.dynamicSmemBytes = size_t(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}

template <int BN, int STAGES>
mfp8_status launch_pair_bn(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8, const float* s_w,
                           int64_t N, int64_t w_rows, void* Y, bool dependent, int dev, const DeviceInfo& info,
                           cudaStream_t stream) {
    using L = pair::Layout<BN, STAGES>;
    auto kern = pair::gemm_pair_kernel<BN, STAGES>;
    static bool attr_done[kMaxDevices] = {};
    mfp8_status st = set_smem(kern, L::SMEM_BYTES, dev, attr_done);
    if (st != MFP8_OK) return st;
    CUtensorMap tmX, tmW, tmY;
    if ((st = make_map_u8(&tmX, X8, M, K, pair::HALF)) != MFP8_OK) return st;
    if ((st = make_map_u8(&tmW, W8, w_rows, K, BN / 2)) != MFP8_OK) return st;
    if ((st = make_map_y(&tmY, Y, M, N)) != MFP8_OK) return st;
    const int64_t tiles = ((M + pair::BM - 1) / pair::BM) * ((N + BN - 1) / BN);
    // The grid is persistent: only as many pairs as can be resident at once.
    int64_t max_pairs = max_active_clusters(kern, 2, L::SMEM_BYTES, pair::kThreads, dev);
    if (max_pairs <= 0 || max_pairs > info.sm_count / 2) max_pairs = info.sm_count / 2;
    const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(2 * pairs));
    cfg.blockDim = dim3(pair::kThreads);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tmX, tmW, tmY, s_a, s_w, static_cast<__nv_bfloat16*>(Y), int(M), int(N),
                           int(K)) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

// Tile width for the pair kernel: the one that finishes sooner, counting
// rounds of tiles over the CTA pairs times the time of one tile.  A
// 256 x 128 tile moves 3/4 of the bytes of a 256 x 256 tile for half the
// MACs and measured about 1.45x slower per MAC, so it is chosen only when it
// saves rounds (narrow N, e.g. the k/v projections at M = 2048).
int pair_tile_width(int64_t M, int64_t N, const DeviceInfo& info) {
    const int64_t pairs = info.sm_count / 2;
    const int64_t mt = (M + pair::BM - 1) / pair::BM;
    const int64_t r256 = (mt * ((N + 255) / 256) + pairs - 1) / pairs;
    const int64_t r128 = (mt * ((N + 127) / 128) + pairs - 1) / pairs;
    return double(r128) * 128.0 * 1.45 < double(r256) * 256.0 ? 128 : 256;
}

mfp8_status launch_pair(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8, const float* s_w,
                        int64_t N, int64_t w_rows, void* Y, bool dependent, int dev, const DeviceInfo& info,
                        cudaStream_t stream) {
    if (pair_tile_width(M, N, info) == 128)
        return launch_pair_bn<128, 8>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
    return launch_pair_bn<256, 6>(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
}

constexpr int64_t kStreamMaxM = stream::kMaxM;
constexpr int64_t kClusterMaxM = cluster::kMaxM;

int sm_count_for_sizing();

int choose_path(int64_t M, int64_t N, int64_t K) {
    (void)K;
    if (M <= kStreamMaxM) return MFP8_PATH_FUSED;
    // The cluster split-K kernel up to 128 rows (measured ahead of the
    // 128-row tiles there on the layer's shapes); above, its stages of a
    // weight block and up to 256 code rows leave too shallow a ring and the
    // tiles are faster.
    if (M <= 128) return MFP8_PATH_SPLITK;
    if (M < 256) return MFP8_PATH_TILED;
    // Too few 256 x 256 pair tiles to occupy half the CTA pairs (the k/v
    // projections at M = 2048 make 32): narrower single-CTA tiles fill the
    // GPU instead.
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    if (pair_tiles * 4 < sm_count_for_sizing()) return MFP8_PATH_TILED;
    return MFP8_PATH_PAIR;
}

mfp8_status check_gemm_args(int64_t M, int64_t N, int64_t K, const void* W8, const float* s_w, const void* Y) {
    if (M < 0 || N < 0 || K < 0) return MFP8_ERR_INVALID_ARG;
    if (K == 0 || K % 16 != 0 || N == 0 || K > kMaxDim || N > kMaxDim || M > kMaxDim)
        return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (M > 0 && M * (K > N ? K : N) > (int64_t(1) << 40)) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (!W8 || !s_w || (M > 0 && !Y)) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(W8) || !aligned16(s_w) || !aligned16(Y)) return MFP8_ERR_MISALIGNED;
    if (M > 0 && (ranges_overlap(Y, size_t(M * N * 2), W8, size_t(N * K)) ||
                  ranges_overlap(Y, size_t(M * N * 2), s_w, size_t(N * 4))))
        return MFP8_ERR_INVALID_ARG;
    return MFP8_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// How one call uses the caller's workspace: the activation codes X8 [M, K]
// and scales s_a [M] of the quantize pass, each 256-byte aligned.  Nothing
// in it outlives the call.
struct Plan {
    size_t x8_off = 0, sa_off = 0, total = 0;
};

Plan make_plan(int64_t M, int64_t K, bool codes) {
    Plan p;
    if (!codes) return p;  // nothing to keep: no workspace needed
    p.x8_off = 0;
    p.sa_off = round_up(size_t(M) * size_t(K), 256);
    p.total = p.sa_off + round_up(size_t(M) * 4, 256);
    return p;
}

// N not a multiple of 8: rows of Y are not 16-byte aligned, which the
// kernels' vector stores and the TMA store maps need.  The kernels then run
// on N8 = N rounded up to 8 channels: the weight tensor map keeps N rows
// (rows N .. N8-1 read as zeros), the channel scales are copied into a
// zero-padded [N8] array and the output goes to an [M, N8] scratch, whose
// first N columns a copy kernel writes into Y.  Both scratch arrays follow
// the codes in the workspace.
struct PadPlan {
    int64_t n8 = 0;
    size_t sw_off = 0, y_off = 0, total = 0;
};

PadPlan make_pad_plan(int64_t M, int64_t N, size_t start) {
    PadPlan p;
    p.n8 = N;
    p.total = start;
    if (N % 8 == 0) return p;
    p.n8 = (N + 7) / 8 * 8;
    p.sw_off = round_up(start, 256);
    p.y_off = round_up(p.sw_off + size_t(p.n8) * 4, 256);
    p.total = round_up(p.y_off + size_t(M) * size_t(p.n8) * 2, 256);
    return p;
}

__global__ void pad_scales_kernel(const float* __restrict__ s_w, int64_t N, float* __restrict__ sw8, int64_t N8) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < N8; i += int64_t(gridDim.x) * blockDim.x)
        sw8[i] = i < N ? s_w[i] : 0.0f;
}

__global__ void crop_rows_kernel(const uint16_t* __restrict__ Y8, int64_t N8, uint16_t* __restrict__ Y, int64_t M,
                                 int64_t N) {
    const int64_t n = M * N;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t m = i / N;
        Y[i] = Y8[m * N8 + (i - m * N)];
    }
}


// ------------------------------------------- decode: one-kernel Linear --

// Cluster size S (K split) of the one-kernel decode path: the largest power
// of two up to 8 that keeps tiles * S within 1.5 CTAs per SM (two fit on an
// SM; more CTAs keep more weight copies in flight), no more
// than the K blocks, and raised (up to 8) until the codes of one CTA's K
// range fit its code store.  Weight ring: what is left of the shared region.
// Returns false when no S fits (K too long for this path).
bool stream_geometry(int64_t M, int64_t N, int64_t K, int sm_count, stream::Geometry* g) {
    const int64_t tiles = (N + stream::TILE - 1) / stream::TILE;
    const int64_t kb = (K + stream::SUB - 1) / stream::SUB;
    const int mpad = M <= 8 ? 8 : 16;
    // The K split doubles while the grid stays within 1.5 CTAs per SM, and
    // on up to 2 per SM while every CTA keeps at least 8 K blocks (long-K
    // Linears such as down_proj, where more CTAs in flight stream faster).
    int S = 1;
    auto grow = [&](int s) {
        if (s >= stream::kMaxCluster || s * 2 > kb) return false;
        const int64_t ctas = tiles * s * 2;
        return ctas <= sm_count * 3 / 2 || (ctas <= int64_t(sm_count) * 2 && kb / (s * 2) >= 8);
    };
    while (grow(S)) S *= 2;
    auto code_bytes = [&](int s_) {
        const int64_t kbs = (kb + s_ - 1) / s_;
        return (kbs * mpad * stream::SUB + 1023) / 1024 * 1024;
    };
    while (code_bytes(S) > stream::kMaxCodeBytes && S < stream::kMaxCluster && S * 2 <= kb) S *= 2;
    if (code_bytes(S) > stream::kMaxCodeBytes) return false;
    g->S = S;
    g->mpad = mpad;
    g->code_bytes = int(code_bytes(S));
    const int st = (stream::kShared - g->code_bytes) / stream::kWStageBytes;
    g->stages = st > stream::kMaxStages ? stream::kMaxStages : st;
    // K blocks beyond the ring wait in TMEM (up to 7 per CTA).
    const int64_t spare = (kb + S - 1) / S - g->stages;
    g->tm_blocks = spare <= 0 ? 0 : int(spare < stream::kMaxTmemBlocks ? spare : stream::kMaxTmemBlocks);
    return g->stages >= stream::kMinStages;
}

mfp8_status launch_stream(const void* X, int64_t M, int64_t K, const void* W8, const float* s_w, int64_t N,
                          int64_t w_rows,
                          void* Y, bool weights_static, bool dependent, void* x8_out, float* sa_out, int dev,
                          const DeviceInfo& info, cudaStream_t stream) {
    if (M < 1 || M > kStreamMaxM || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
        return MFP8_ERR_UNSUPPORTED_SHAPE;
    stream::Geometry g;
    if (!stream_geometry(M, N, K, info.sm_count, &g)) return MFP8_ERR_UNSUPPORTED_SHAPE;
    // Eight quantizer warps pay off once a CTA has more than 8 token rows.
    const bool wide = M > 8;
    auto kern = wide ? stream::gemm_stream_kernel<8> : stream::gemm_stream_kernel<4>;
    static bool attr_done4[kMaxDevices] = {}, attr_done8[kMaxDevices] = {};
    mfp8_status st = set_smem(kern, stream::Smem::BYTES, dev, wide ? attr_done8 : attr_done4);
    if (st != MFP8_OK) return st;
    const int64_t tiles = (N + stream::TILE - 1) / stream::TILE;
    const int64_t grid = tiles * g.S;
    if (grid > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap tmW;
    if ((st = make_map_u8(&tmW, W8, w_rows, K, stream::TILE)) != MFP8_OK) return st;

    stream::Args args;
    args.X = static_cast<const __nv_bfloat16*>(X);
    args.s_w = s_w;
    args.Y = static_cast<__nv_bfloat16*>(Y);
    args.x8_out = static_cast<uint8_t*>(x8_out);
    args.sa_out = sa_out;
    args.M = int(M);
    args.N = int(N);
    args.K = int(K);
    args.weights_static = weights_static ? 1 : 0;
    args.g = g;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(unsigned(wide ? stream::Warps<8>::kThreads : stream::Warps<4>::kThreads));
    cfg.dynamicSmemBytes = stream::Smem::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(g.S);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tmW, args) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

// ------------------------------ small / middle M: cluster split-K on codes --

// Cluster size S (K split) of the split-K path: the decode kernel's rule (up
// to 1.5 CTAs per SM, or 2 while each CTA keeps 8+ K blocks).  Ring: as many
// weight + code stages as fit.
bool cluster_geometry(int64_t M, int64_t N, int64_t K, int sm_count, cluster::Geometry* g) {
    if (M < 1 || M > cluster::kMaxM) return false;
    const int64_t tiles = (N + cluster::TILE - 1) / cluster::TILE;
    const int64_t kb = (K + cluster::SUB - 1) / cluster::SUB;
    int S = 1;
    auto grow = [&](int s) {
        if (s >= cluster::kMaxCluster || s * 2 > kb) return false;
        const int64_t ctas = tiles * s * 2;
        return ctas <= sm_count * 3 / 2 || (ctas <= int64_t(sm_count) * 2 && kb / (s * 2) >= 8);
    };
    while (grow(S)) S *= 2;
    g->S = S;
    g->mp = int((M + 15) / 16 * 16);
    // A grid of at most one CTA per SM takes the deeper ring (more bytes in
    // flight per CTA, fewer exchange rounds); larger grids keep two CTAs per
    // SM resident.
    g->ring = tiles * S <= sm_count ? cluster::kRingBig : cluster::kRingBytes;
    const int st = g->ring / cluster::stage_bytes(g->mp);
    g->stages = st > cluster::kMaxStages ? cluster::kMaxStages : st;
    // Exchange rounds: as few as the ring allows, of equal width (a multiple
    // of 32 token columns where the round is that wide, else of 16: whole
    // 32-column TMEM loads).
    g->tc = g->mp;
    if (S > 1) {
        int rounds = 1;
        auto width = [&](int r) {
            const int w = (g->mp + r - 1) / r;
            return w > 16 ? (w + 31) / 32 * 32 : 16;
        };
        while (cluster::exchange_bytes(S, width(rounds)) > g->ring) ++rounds;
        g->tc = width(rounds) < g->mp ? width(rounds) : g->mp;
    }
    return g->stages >= cluster::kMinStages;
}

mfp8_status launch_cluster(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8, const float* s_w,
                           int64_t N, int64_t w_rows, void* Y, bool weights_static, bool dependent, int dev,
                           const DeviceInfo& info,
                           cudaStream_t stream) {
    cluster::Geometry g;
    if (!cluster_geometry(M, N, K, info.sm_count, &g)) return MFP8_ERR_UNSUPPORTED_SHAPE;
    auto kern = cluster::gemm_cluster_kernel;
    static bool attr_done[kMaxDevices] = {};
    mfp8_status st = set_smem(kern, cluster::Smem::MAX_BYTES, dev, attr_done);
    if (st != MFP8_OK) return st;
    const int64_t tiles = (N + cluster::TILE - 1) / cluster::TILE;
    const int64_t grid = tiles * g.S;
    if (grid > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap tmX, tmW;
    if ((st = make_map_u8(&tmW, W8, w_rows, K, cluster::TILE)) != MFP8_OK) return st;
    if ((st = make_map_u8(&tmX, X8, M, K, g.mp)) != MFP8_OK) return st;

    cluster::Args args;
    args.s_a = s_a;
    args.s_w = s_w;
    args.Y = static_cast<__nv_bfloat16*>(Y);
    args.M = int(M);
    args.N = int(N);
    args.K = int(K);
    args.weights_static = weights_static ? 1 : 0;
    args.g = g;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(cluster::kThreads);
    cfg.dynamicSmemBytes = size_t(cluster::Smem::bytes(g.ring));
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(g.S);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tmX, tmW, args) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

// The GEMM on codes already in memory (tiled, pair, or split-K).
mfp8_status run_gemm(const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8, const float* s_w,
                     int64_t N, int64_t w_rows, void* Y, int path, bool weights_static, bool dependent, int dev,
                     const DeviceInfo& info, cudaStream_t stream) {
    // The kernels take M, N, K as 32-bit.
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (path == MFP8_PATH_TILED) return launch_tiled(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
    if (path == MFP8_PATH_PAIR) return launch_pair(X8, s_a, M, K, W8, s_w, N, w_rows, Y, dependent, dev, info, stream);
    if (path == MFP8_PATH_SPLITK)
        return launch_cluster(X8, s_a, M, K, W8, s_w, N, w_rows, Y, weights_static, dependent, dev, info, stream);
    return MFP8_ERR_INVALID_ARG;
}

int sm_count_for_sizing() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        return sms;
    cudaGetLastError();
    return 148;  // B200
}

// Scratch of mfp8_linear_noalloc: one fixed array per device, part of the
// module's own global memory, so that entry point allocates nothing.  It is
// for callers that cannot call an allocator where they call the Linear: a C
// host with no device allocator of its own, or one whose memory is planned
// in full up front (a fixed budget per GPU).  Every call on a device uses
// the same bytes, so two calls that can be in flight at once race.
constexpr size_t kStaticWsBytes = MFP8_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

// The array's device address, looked up once per device and context.  In
// host code `g_static_ws` names a host-side stand-in, not device memory; the
// address kernels need comes from cudaGetSymbolAddress with the device
// current.  It is cached together with the context's unique ID: a context
// that was destroyed and created again (cudaDeviceReset) reloads the module,
// which may place the array elsewhere, and the new ID forces a new lookup.
struct StaticWs {
    unsigned long long ctx_id = 0;
    void* ptr = nullptr;
};
StaticWs g_static_ws_cache[kMaxDevices];
PFN_cuCtxGetCurrent_v4000 g_ctx_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_get_id = nullptr;

// Unique ID of the calling thread's current context (0 when none is bound).
mfp8_status current_context_id(unsigned long long* id) {
    if (!g_ctx_get_current || !g_ctx_get_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2) {
            cudaGetLastError();
            return MFP8_ERR_CUDA;
        }
        g_ctx_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return MFP8_ERR_CUDA;
    *id = 0;
    if (ctx && g_ctx_get_id(ctx, id) != CUDA_SUCCESS) return MFP8_ERR_CUDA;
    return MFP8_OK;
}

mfp8_status static_workspace(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long id = 0;
    mfp8_status st = current_context_id(&id);
    if (st != MFP8_OK) return st;
    StaticWs& c = g_static_ws_cache[dev];
    if (id == 0 || c.ptr == nullptr || c.ctx_id != id) {
        // cudaGetSymbolAddress also binds the device's primary context to
        // this thread if none was bound yet; the ID is read after it.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MFP8_ERR_CUDA;
        }
        if ((st = current_context_id(&id)) != MFP8_OK) return st;
        c.ptr = p;
        c.ctx_id = id;
    }
    *out = c.ptr;
    return MFP8_OK;
}

__global__ void bounded_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing ever arrives on this barrier: the wait must give up.
        mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
    }
}

// Launch of a fused producer kernel: one block per row, VPT vectors of 8
// values per thread (rows up to 16384 values), as a programmatic dependent.
template <template <int> class Pick, class... A>
mfp8_status launch_producer(int64_t nvec, int64_t M, cudaStream_t stream, A... args) {
    auto launch = [&](auto kern) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(M));
        cfg.blockDim = dim3(producer::kThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) {
            cudaGetLastError();
            return MFP8_ERR_CUDA;
        }
        return MFP8_OK;
    };
    if (nvec <= 256) return launch(Pick<1>::kern());
    if (nvec <= 512) return launch(Pick<2>::kern());
    if (nvec <= 1024) return launch(Pick<4>::kern());
    if (nvec <= 1536) return launch(Pick<6>::kern());
    if (nvec <= 2048) return launch(Pick<8>::kern());
    return MFP8_ERR_UNSUPPORTED_SHAPE;
}

// A launch that may begin while the previous kernel on the stream drains
// (programmatic dependent launch); the kernel waits for that kernel's
// results with griddepcontrol.wait before its first global load.
template <typename... KArgs, typename... A>
mfp8_status launch_pdl(void (*kern)(KArgs...), dim3 grid, int threads, cudaStream_t stream, int smem_bytes,
                       A... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = size_t(smem_bytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return MFP8_OK;
}

template <int VPT>
struct PickRmsnorm {
    static auto kern() { return producer::rmsnorm_quant_kernel<producer::kThreads, VPT>; }
};
constexpr int64_t kSiluWideFrom = 1024;  // rows above this many 8-value vectors take 512 threads

template <int VPT>
struct PickSiluMul {
    static auto kern() { return producer::silu_mul_quant_kernel<producer::kThreads, VPT>; }
};

// The padded run: scales padded, X quantized (unless FUSED), the kernels on
// N8 channels into the scratch, then the crop.  Every launch here is a plain
// stream-ordered launch, so the scratch scales are complete before any
// kernel reads them.
mfp8_status run_padded(const void* X_bf16, const void* X8, const float* s_a, int64_t M, int64_t K, const void* W8,
                       const float* s_w, int64_t N, void* Y, const PadPlan& pad, uint8_t* base, int path,
                       void* X_fp8_out, float* x_scale_out, int dev, const DeviceInfo& info, cudaStream_t stream) {
    float* sw8 = reinterpret_cast<float*>(base + pad.sw_off);
    void* y8 = base + pad.y_off;
    const int64_t cap = int64_t(info.sm_count) * 8;
    pad_scales_kernel<<<unsigned((pad.n8 + 255) / 256 < cap ? (pad.n8 + 255) / 256 : cap), 256, 0, stream>>>(
        s_w, N, sw8, pad.n8);
    mfp8_status st = launch_status();
    if (st != MFP8_OK) return st;
    if (path == MFP8_PATH_FUSED) {
        st = launch_stream(X_bf16, M, K, W8, sw8, pad.n8, N, y8, /*weights_static=*/false, /*dependent=*/false,
                           X_fp8_out, x_scale_out, dev, info, stream);
    } else {
        // the per-row quantizer without the early trigger: the same codes as
        // mfp8_quantize_act, launched in plain stream order
        if (X_bf16 && (st = quantize_weight_rows(X_bf16, M, K, const_cast<void*>(X8), const_cast<float*>(s_a),
                                                 stream)) != MFP8_OK)
            return st;
        st = run_gemm(X8, s_a, M, K, W8, sw8, pad.n8, N, y8, path, /*weights_static=*/false, /*dependent=*/false,
                      dev, info, stream);
    }
    if (st != MFP8_OK) return st;
    const int64_t nb = (M * N + 255) / 256;
    crop_rows_kernel<<<unsigned(nb < cap ? nb : cap), 256, 0, stream>>>(static_cast<const uint16_t*>(y8), pad.n8,
                                                                        static_cast<uint16_t*>(Y), M, N);
    return launch_status();
}

}  // namespace
}  // namespace mfp8

using namespace mfp8;

extern "C" {

mfp8_status mfp8_quantize_weight(const void* W_bf16, int64_t N, int64_t K, void* W_fp8, float* w_scale,
                                 void* stream) {
    mfp8_status st = check_quant_args(W_bf16, N, K, W_fp8, w_scale);
    if (st != MFP8_OK || N == 0) return st;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    return quantize_weight_rows(W_bf16, N, K, W_fp8, w_scale, static_cast<cudaStream_t>(stream));
}

mfp8_status mfp8_quantize_act(const void* X_bf16, int64_t M, int64_t K, void* X_fp8, float* x_scale,
                              void* stream) {
    mfp8_status st = check_quant_args(X_bf16, M, K, X_fp8, x_scale);
    if (st != MFP8_OK || M == 0) return st;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    return quantize_act_rows(X_bf16, M, K, X_fp8, x_scale, static_cast<cudaStream_t>(stream));
}

size_t mfp8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return 0;
    return make_pad_plan(M, N, make_plan(M, K, true).total).total;
}

mfp8_status mfp8_linear_ex(const void* X_bf16, int64_t M, int64_t K, const void* W_fp8, const float* w_scale,
                           int64_t N, void* Y_bf16, void* workspace, size_t workspace_bytes_given, int path,
                           int flags, void* X_fp8_out, float* x_scale_out, void* stream) {
    mfp8_status st = check_gemm_args(M, N, K, W_fp8, w_scale, Y_bf16);
    if (st != MFP8_OK) return st;
    if (path < MFP8_PATH_AUTO || path > MFP8_PATH_FUSED) return MFP8_ERR_INVALID_ARG;
    if ((flags & ~MFP8_FLAG_STATIC_WEIGHTS) != 0) return MFP8_ERR_INVALID_ARG;
    if (path == MFP8_PATH_SPLITK && M > kClusterMaxM) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (path == MFP8_PATH_FUSED && M > kStreamMaxM) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return MFP8_OK;
    if (!X_bf16) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(X_bf16)) return MFP8_ERR_MISALIGNED;
    if ((X_fp8_out == nullptr) != (x_scale_out == nullptr)) return MFP8_ERR_INVALID_ARG;
    if (ranges_overlap(X_bf16, size_t(M * K * 2), Y_bf16, size_t(M * N * 2))) return MFP8_ERR_INVALID_ARG;
    if (X_fp8_out) {
        if (!aligned16(X_fp8_out) || !aligned16(x_scale_out)) return MFP8_ERR_MISALIGNED;
        if ((st = check_quant_args(X_bf16, M, K, X_fp8_out, x_scale_out)) != MFP8_OK) return st;
        if (ranges_overlap(X_fp8_out, size_t(M * K), Y_bf16, size_t(M * N * 2)) ||
            ranges_overlap(x_scale_out, size_t(M * 4), Y_bf16, size_t(M * N * 2)))
            return MFP8_ERR_INVALID_ARG;
    }
    if (path == MFP8_PATH_AUTO) path = choose_path(M, (N + 7) / 8 * 8, K);
    const bool weights_static = (flags & MFP8_FLAG_STATIC_WEIGHTS) != 0;
    // FUSED (M <= 16): one kernel quantizes X on chip and streams the
    // weights; it keeps nothing in the workspace.
    const bool fused = path == MFP8_PATH_FUSED;
    const Plan plan = fused ? Plan() : make_plan(M, K, X_fp8_out == nullptr);
    const PadPlan pad = make_pad_plan(M, N, plan.total);
    if (pad.total > 0) {
        if (!workspace || workspace_bytes_given < pad.total) return MFP8_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MFP8_ERR_MISALIGNED;
        if (ranges_overlap(workspace, pad.total, Y_bf16, size_t(M * N * 2)) ||
            ranges_overlap(workspace, pad.total, X_bf16, size_t(M * K * 2)) ||
            (X_fp8_out && (ranges_overlap(workspace, pad.total, X_fp8_out, size_t(M * K)) ||
                           ranges_overlap(workspace, pad.total, x_scale_out, size_t(M * 4)))))
            return MFP8_ERR_INVALID_ARG;
    }

    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    if (pad.n8 != N) {
        const void* X8 = fused ? nullptr : (X_fp8_out ? X_fp8_out : base + plan.x8_off);
        const float* s_a = fused ? nullptr : (x_scale_out ? x_scale_out : reinterpret_cast<float*>(base + plan.sa_off));
        return run_padded(X_bf16, X8, s_a, M, K, W_fp8, w_scale, N, Y_bf16, pad, base, path, X_fp8_out, x_scale_out,
                          dev, info, s);
    }
    if (fused)
        return launch_stream(X_bf16, M, K, W_fp8, w_scale, N, N, Y_bf16, weights_static, /*dependent=*/true,
                             X_fp8_out, x_scale_out, dev, info, s);
    void* X8 = X_fp8_out ? X_fp8_out : base + plan.x8_off;
    float* s_a = x_scale_out ? x_scale_out : reinterpret_cast<float*>(base + plan.sa_off);
    if ((st = quantize_act_rows(X_bf16, M, K, X8, s_a, s)) != MFP8_OK) return st;
    return run_gemm(X8, s_a, M, K, W_fp8, w_scale, N, N, Y_bf16, path, weights_static,
                    /*dependent=*/true, dev, info, s);
}

mfp8_status mfp8_linear(const void* X_bf16, int64_t M, int64_t K, const void* W_fp8, const float* w_scale,
                        int64_t N, void* Y_bf16, void* workspace, size_t workspace_bytes_given, void* stream) {
    return mfp8_linear_ex(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes_given,
                          MFP8_PATH_AUTO, 0, nullptr, nullptr, stream);
}

mfp8_status mfp8_linear_noalloc(const void* X_bf16, int64_t M, int64_t K, const void* W_fp8, const float* w_scale,
                               int64_t N, void* Y_bf16, void* stream) {
    mfp8_status st = check_gemm_args(M, N, K, W_fp8, w_scale, Y_bf16);
    if (st != MFP8_OK || M == 0) return st;
    if (mfp8_linear_workspace_bytes(M, N, K) > kStaticWsBytes) return MFP8_ERR_WORKSPACE;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    void* ws = nullptr;
    if ((st = static_workspace(dev, &ws)) != MFP8_OK) return st;
    return mfp8_linear_ex(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, ws, kStaticWsBytes, MFP8_PATH_AUTO, 0,
                          nullptr, nullptr, stream);
}

int mfp8_choose_path(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return MFP8_PATH_AUTO;
    return choose_path(M, N, K);
}

size_t mfp8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return 0;
    return make_pad_plan(M, N, 0).total;  // only N % 8 != 0 needs scratch
}

mfp8_status mfp8_gemm(const void* X_fp8, const float* x_scale, int64_t M, int64_t K, const void* W_fp8,
                      const float* w_scale, int64_t N, void* Y_bf16, void* workspace, size_t workspace_bytes_given,
                      int path, void* stream) {
    mfp8_status st = check_gemm_args(M, N, K, W_fp8, w_scale, Y_bf16);
    if (st != MFP8_OK) return st;
    if (path < MFP8_PATH_AUTO || path > MFP8_PATH_PAIR) return MFP8_ERR_INVALID_ARG;
    if (path == MFP8_PATH_SPLITK && M > kClusterMaxM) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return MFP8_OK;
    if (!X_fp8 || !x_scale) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(X_fp8) || !aligned16(x_scale)) return MFP8_ERR_MISALIGNED;
    if (ranges_overlap(X_fp8, size_t(M * K), Y_bf16, size_t(M * N * 2)) ||
        ranges_overlap(x_scale, size_t(M * 4), Y_bf16, size_t(M * N * 2)))
        return MFP8_ERR_INVALID_ARG;
    const PadPlan pad = make_pad_plan(M, N, 0);
    if (path == MFP8_PATH_AUTO) path = choose_path(M, pad.n8, K);
    if (path == MFP8_PATH_FUSED) path = MFP8_PATH_SPLITK;  // codes given: the split-K kernel streams them
    if (pad.total > 0) {
        if (!workspace || workspace_bytes_given < pad.total) return MFP8_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MFP8_ERR_MISALIGNED;
        if (ranges_overlap(workspace, pad.total, Y_bf16, size_t(M * N * 2)) ||
            ranges_overlap(workspace, pad.total, X_fp8, size_t(M * K)) ||
            ranges_overlap(workspace, pad.total, x_scale, size_t(M * 4)))
            return MFP8_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pad.n8 != N)
        return run_padded(nullptr, X_fp8, x_scale, M, K, W_fp8, w_scale, N, Y_bf16, pad,
                          static_cast<uint8_t*>(workspace), path, nullptr, nullptr, dev, info, s);
    return run_gemm(X_fp8, x_scale, M, K, W_fp8, w_scale, N, N, Y_bf16, path, /*weights_static=*/false,
                    /*dependent=*/false, dev, info, s);
}

mfp8_status mfp8_rmsnorm_quantize(const void* X_bf16, const void* gamma_bf16, float eps, int64_t M, int64_t K,
                                  void* Y_bf16, void* X_fp8, float* x_scale, void* stream) {
    mfp8_status st = check_quant_args(X_bf16, M, K, X_fp8, x_scale);
    if (st != MFP8_OK) return st;
    if (K > 16384) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (!(eps >= 0.0f) || eps > 1.0f) return MFP8_ERR_INVALID_ARG;
    if (M == 0) return MFP8_OK;
    if (!gamma_bf16) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(gamma_bf16) || !aligned16(Y_bf16)) return MFP8_ERR_MISALIGNED;
    if (Y_bf16 && (ranges_overlap(Y_bf16, size_t(M * K * 2), X_bf16, size_t(M * K * 2)) ||
                   ranges_overlap(Y_bf16, size_t(M * K * 2), X_fp8, size_t(M * K)) ||
                   ranges_overlap(Y_bf16, size_t(M * K * 2), x_scale, size_t(M * 4))))
        return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    const int64_t nvec = K / 8;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint4* xv = static_cast<const uint4*>(X_bf16);
    const uint4* gv = static_cast<const uint4*>(gamma_bf16);
    uint4* yv = static_cast<uint4*>(Y_bf16);
    uint2* qv = static_cast<uint2*>(X_fp8);
    // Rows up to 4096 values: 128 threads per row.
    if (nvec <= 128)
        return launch_pdl(producer::rmsnorm_quant_kernel<128, 1>, dim3(unsigned(M)), 128, s, 0, xv, gv, K, eps, yv,
                          qv, x_scale);
    if (nvec <= 256)
        return launch_pdl(producer::rmsnorm_quant_kernel<128, 2>, dim3(unsigned(M)), 128, s, 0, xv, gv, K, eps, yv,
                          qv, x_scale);
    if (nvec <= 512)
        return launch_pdl(producer::rmsnorm_quant_kernel<128, 4>, dim3(unsigned(M)), 128, s, 0, xv, gv, K, eps, yv,
                          qv, x_scale);
    return launch_producer<PickRmsnorm>(nvec, M, s, xv, gv, K, eps, yv, qv, x_scale);
}

mfp8_status mfp8_silu_mul_quantize(const void* GU_bf16, int64_t M, int64_t I, void* Y_bf16, void* X_fp8,
                                   float* x_scale, void* stream) {
    if (M < 0 || I < 0) return MFP8_ERR_INVALID_ARG;
    if (I == 0 || I % 16 != 0 || I > 16384 || M > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return MFP8_OK;
    if (!GU_bf16 || !X_fp8 || !x_scale) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(GU_bf16) || !aligned16(X_fp8) || !aligned16(x_scale) || !aligned16(Y_bf16))
        return MFP8_ERR_MISALIGNED;
    const size_t in_bytes = size_t(M) * size_t(2 * I) * 2;
    if (ranges_overlap(GU_bf16, in_bytes, X_fp8, size_t(M * I)) ||
        ranges_overlap(GU_bf16, in_bytes, x_scale, size_t(M * 4)) ||
        ranges_overlap(X_fp8, size_t(M * I), x_scale, size_t(M * 4)) ||
        (Y_bf16 && (ranges_overlap(Y_bf16, size_t(M * I * 2), GU_bf16, in_bytes) ||
                    ranges_overlap(Y_bf16, size_t(M * I * 2), X_fp8, size_t(M * I)) ||
                    ranges_overlap(Y_bf16, size_t(M * I * 2), x_scale, size_t(M * 4)))))
        return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    const int64_t nvec = I / 8;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint4* gu = static_cast<const uint4*>(GU_bf16);
    uint4* yv = static_cast<uint4*>(Y_bf16);
    uint2* qv = static_cast<uint2*>(X_fp8);
    // Long rows: 512 threads per row (more warps resident per SM to hide the
    // loads behind the arithmetic).
    if (nvec > kSiluWideFrom && nvec <= 1536)
        return launch_pdl(producer::silu_mul_quant_kernel<512, 3>, dim3(unsigned(M)), 512, s, 0, gu, I, yv, qv, x_scale);
    if (nvec > kSiluWideFrom && nvec <= 2048)
        return launch_pdl(producer::silu_mul_quant_kernel<512, 4>, dim3(unsigned(M)), 512, s, 0, gu, I, yv, qv, x_scale);
    return launch_producer<PickSiluMul>(nvec, M, s, gu, I, yv, qv, x_scale);
}

mfp8_status mfp8_kv_quantize(const void* KV_bf16, int64_t T, int64_t H, int64_t D, void* KV_fp8, float* kv_scale,
                             void* stream) {
    if (T < 0 || H < 0 || D < 0) return MFP8_ERR_INVALID_ARG;
    if (H == 0 || D == 0 || D % 16 != 0 || D > kMaxDim || H > kMaxDim || T > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    const int64_t R = T * H;
    if (R > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    mfp8_status st = check_quant_args(KV_bf16, R, D, KV_fp8, kv_scale);
    if (st != MFP8_OK || R == 0) return st;
    int dev;
    DeviceInfo info;
    if ((st = current_device(&dev, &info)) != MFP8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D > 256) return quantize_weight_rows(KV_bf16, R, D, KV_fp8, kv_scale, s);  // long rows: the row kernels
    const int vpr = int(D / 8);
    const int lpr = vpr <= 2 ? 2 : vpr <= 4 ? 4 : vpr <= 8 ? 8 : vpr <= 16 ? 16 : 32;
    const int64_t rows_per_block = int64_t(kQuantThreads / 32) * (32 / lpr) * kSmallRowItems;
    const int64_t blocks = (R + rows_per_block - 1) / rows_per_block;
    if (blocks > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    const uint4* x = static_cast<const uint4*>(KV_bf16);
    uint2* q = static_cast<uint2*>(KV_fp8);
    const dim3 grid{static_cast<unsigned>(blocks)};
    switch (lpr) {
        case 2: return launch_pdl(quant_small_rows_kernel<2>, grid, kQuantThreads, s, 0, x, R, int(D), q, kv_scale);
        case 4: return launch_pdl(quant_small_rows_kernel<4>, grid, kQuantThreads, s, 0, x, R, int(D), q, kv_scale);
        case 8: return launch_pdl(quant_small_rows_kernel<8>, grid, kQuantThreads, s, 0, x, R, int(D), q, kv_scale);
        case 16: return launch_pdl(quant_small_rows_kernel<16>, grid, kQuantThreads, s, 0, x, R, int(D), q, kv_scale);
        default: return launch_pdl(quant_small_rows_kernel<32>, grid, kQuantThreads, s, 0, x, R, int(D), q, kv_scale);
    }
}

mfp8_status mfp8_kv_dequantize(const void* KV_fp8, const float* kv_scale, int64_t T, int64_t H, int64_t D,
                               void* KV_bf16, void* stream) {
    if (T < 0 || H < 0 || D < 0) return MFP8_ERR_INVALID_ARG;
    if (H == 0 || D == 0 || D % 16 != 0 || D > kMaxDim || H > kMaxDim || T > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    const int64_t R = T * H;
    if (R > kMaxDim) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (R == 0) return MFP8_OK;
    if (!KV_fp8 || !kv_scale || !KV_bf16) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(KV_fp8) || !aligned16(kv_scale) || !aligned16(KV_bf16)) return MFP8_ERR_MISALIGNED;
    if (ranges_overlap(KV_bf16, size_t(R * D * 2), KV_fp8, size_t(R * D)) ||
        ranges_overlap(KV_bf16, size_t(R * D * 2), kv_scale, size_t(R * 4)))
        return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    const int64_t n8 = R * D / 8;
    const int64_t blocks = (n8 + kQuantThreads * kDequantItems - 1) / (kQuantThreads * kDequantItems);
    if (blocks > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    return launch_pdl(kv_dequant_kernel, dim3(unsigned(blocks)), kQuantThreads, static_cast<cudaStream_t>(stream), 0,
                      static_cast<const uint2*>(KV_fp8), kv_scale, n8, int(D), static_cast<uint4*>(KV_bf16));
}

mfp8_status mfp8_kv8_quantize(const void* KV_bf16, int64_t T, int64_t H, int64_t D, void* KV_u8, float* kv_scale,
                              float* kv_zero, void* stream) {
    if (T < 0 || H < 0 || D < 0) return MFP8_ERR_INVALID_ARG;
    if (H == 0 || D == 0 || D % 16 != 0 || T % kv8::kGroup != 0 || D > kMaxDim || H > kMaxDim || T > kMaxDim)
        return MFP8_ERR_UNSUPPORTED_SHAPE;
    const int64_t C = H * D;
    if (C > kMaxDim || (T > 0 && C > (int64_t(1) << 40) / T)) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MFP8_OK;
    if (!KV_bf16 || !KV_u8 || !kv_scale || !kv_zero) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(KV_bf16) || !aligned16(KV_u8) || !aligned16(kv_scale) || !aligned16(kv_zero))
        return MFP8_ERR_MISALIGNED;
    const int64_t G = T / kv8::kGroup;
    const size_t nin = size_t(T * C) * 2, nq = size_t(T * C), nf = size_t(G * C) * 4;
    if (ranges_overlap(KV_bf16, nin, KV_u8, nq) || ranges_overlap(KV_bf16, nin, kv_scale, nf) ||
        ranges_overlap(KV_bf16, nin, kv_zero, nf) || ranges_overlap(KV_u8, nq, kv_scale, nf) ||
        ranges_overlap(KV_u8, nq, kv_zero, nf) || ranges_overlap(kv_scale, nf, kv_zero, nf))
        return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    const int64_t tiles_per_group = (C + kv8::kTileCols - 1) / kv8::kTileCols;
    const int64_t blocks = G * tiles_per_group;
    if (blocks > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    return launch_pdl(kv8::quant_kernel, dim3(unsigned(blocks)), kv8::kQuantThreads, static_cast<cudaStream_t>(stream), 0,
                      static_cast<const uint4*>(KV_bf16), C / 8, tiles_per_group, static_cast<uint2*>(KV_u8), kv_scale,
                      kv_zero);
}

mfp8_status mfp8_kv8_read(const void* KV_u8, const float* kv_scale, const float* kv_zero, int64_t Tq,
                          const void* tail_bf16, int64_t Tr, int64_t H, int64_t D, void* out_bf16, void* stream) {
    if (Tq < 0 || Tr < 0 || H < 0 || D < 0) return MFP8_ERR_INVALID_ARG;
    if (H == 0 || D == 0 || D % 16 != 0 || Tq % kv8::kGroup != 0 || D > kMaxDim || H > kMaxDim || Tq > kMaxDim ||
        Tr > kMaxDim)
        return MFP8_ERR_UNSUPPORTED_SHAPE;
    const int64_t C = H * D, T = Tq + Tr;
    if (C > kMaxDim || (T > 0 && C > (int64_t(1) << 40) / T)) return MFP8_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MFP8_OK;
    if (!out_bf16 || (Tq > 0 && (!KV_u8 || !kv_scale || !kv_zero)) || (Tr > 0 && !tail_bf16))
        return MFP8_ERR_INVALID_ARG;
    if (!aligned16(out_bf16) || !aligned16(KV_u8) || !aligned16(kv_scale) || !aligned16(kv_zero) ||
        !aligned16(tail_bf16))
        return MFP8_ERR_MISALIGNED;
    const size_t nout = size_t(T * C) * 2, nq = size_t(Tq * C), nf = size_t(Tq / kv8::kGroup * C) * 4,
                 nt = size_t(Tr * C) * 2;
    if ((Tq > 0 && (ranges_overlap(out_bf16, nout, KV_u8, nq) || ranges_overlap(out_bf16, nout, kv_scale, nf) ||
                    ranges_overlap(out_bf16, nout, kv_zero, nf))) ||
        (Tr > 0 && ranges_overlap(out_bf16, nout, tail_bf16, nt)))
        return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    const int64_t C8 = C / 8, n_tail16 = Tr * C / 8;
    const int64_t items = Tq / kv8::kReadRows * C8 + n_tail16;
    const int64_t blocks = (items + kv8::kReadThreads - 1) / kv8::kReadThreads;
    if (blocks > INT32_MAX) return MFP8_ERR_UNSUPPORTED_SHAPE;
    return launch_pdl(kv8::read_kernel, dim3(unsigned(blocks)), kv8::kReadThreads, static_cast<cudaStream_t>(stream), 0,
                      static_cast<const uint2*>(KV_u8), reinterpret_cast<const float4*>(kv_scale),
                      reinterpret_cast<const float4*>(kv_zero), Tq, C8, static_cast<const uint4*>(tail_bf16),
                      n_tail16, static_cast<uint4*>(out_bf16));
}

int64_t mfp8_kv8_history_tokens(int64_t T) {
    if (T < 0) return -1;
    return T < 128 ? 0 : kv8::kGroup * ((T - 128) / kv8::kGroup);
}

mfp8_status mfp8_debug_kv8_code_check(void* out_u64x2, int64_t n_scale_pairs, uint32_t seed, void* stream) {
    if (!out_u64x2 || n_scale_pairs <= 0 || n_scale_pairs > INT32_MAX) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(out_u64x2)) return MFP8_ERR_MISALIGNED;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(out_u64x2, 0, 16, s) != cudaSuccess) return MFP8_ERR_CUDA;
    kv8::code_check_kernel<<<unsigned(n_scale_pairs), 256, 0, s>>>(static_cast<unsigned long long*>(out_u64x2), seed);
    return launch_status();
}

mfp8_status mfp8_e4m3_encode_f32(const float* in, int64_t n, uint8_t* out, void* stream) {
    if (n < 0) return MFP8_ERR_INVALID_ARG;
    if (n == 0) return MFP8_OK;
    if (!in || !out) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(in) || !aligned16(out)) return MFP8_ERR_MISALIGNED;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    const int64_t pairs = (n + 1) / 2;
    int64_t blocks = (pairs + 255) / 256;
    const int64_t cap = int64_t(info.sm_count) * 16;
    if (blocks > cap) blocks = cap;
    e4m3_encode_kernel<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(in, n, out);
    return launch_status();
}

mfp8_status mfp8_debug_quantize_check(void* out_u64x2, void* stream) {
    if (!out_u64x2) return MFP8_ERR_INVALID_ARG;
    if (!aligned16(out_u64x2)) return MFP8_ERR_MISALIGNED;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(out_u64x2, 0, 16, s) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    quantize_check_kernel<<<0x7f80u, 256, 0, s>>>(static_cast<unsigned long long*>(out_u64x2));
    return launch_status();
}

mfp8_status mfp8_debug_bounded_wait(int64_t timeout_us, void* stream) {
    if (timeout_us < 1 || timeout_us > 100000) return MFP8_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(timeout_us) * 1000u);
    return launch_status();
}

mfp8_status mfp8_get_device_status(void* stream) {
    int dev;
    DeviceInfo info;
    mfp8_status st = current_device(&dev, &info);
    if (st != MFP8_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    int word = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_status, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return MFP8_ERR_CUDA;
    }
    return static_cast<mfp8_status>(word);
}

const char* mfp8_status_string(mfp8_status status) {
    switch (status) {
        case MFP8_OK: return "ok";
        case MFP8_ERR_INVALID_ARG: return "invalid argument";
        case MFP8_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case MFP8_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (K must be a positive multiple of 16, N of 8)";
        case MFP8_ERR_WORKSPACE: return "workspace missing or too small";
        case MFP8_ERR_CUDA: return "CUDA runtime error";
        case MFP8_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
        case MFP8_ERR_DEVICE: return "device is not compute capability 10.0 (B200)";
    }
    return "unknown status";
}

int mfp8_version(void) { return 100; }

}  // extern "C"
