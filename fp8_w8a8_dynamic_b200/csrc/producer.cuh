// producer.cuh — the per-token activation quantization fused into the
// kernels that produce the quantized Linears' inputs, so the activations are
// read once and leave as e4m3 codes and scales:
//
//   RMSNorm (before q/k/v and gate/up): y = bf16(x * r * g),
//       r = 1 / sqrt(mean_k(x^2) + eps)
//   gated MLP activation (before down), on the packed gate_up output:
//       y = bf16(silu(gate) * up),  silu(v) = v / (1 + e^-v) (computed as
//       v e^v / (1 + e^v) for v < 0, which cannot overflow)
//   then, per token, s = fl32(max|y| / 448) and q = e4m3(fl32(y / s)), the
//   codes of mfp8_quantize_act applied to the bf16 y.
//
// Sources: the "MOSS-VL-Realtime-FP8 mixed-precision strategy" article keeps
// the norms in high precision in front of the FP8 Linears; the "MOSS-VL
// quantization README" FP8-Dynamic recipe quantizes the Linears' inputs per
// token at run time and packs gate/up into one Linear.  The pages name
// neither eps nor the MLP activation: SiLU(gate) * up is a reading.
//
// One block per token row, the row in registers (VPT 16-byte vectors of 8
// bf16 per thread).  Every fp32 reduction runs in a fixed order (lanes by
// shuffle, then warps in warp order), so results are deterministic.  The
// kernels are programmatic dependents: the GEMM launched next may start its
// prologue at once and waits for the codes.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace mfp8 {
namespace producer {

constexpr int kThreads = 256;  // block size of the SiLU kernel and of RMSNorm on long rows

// Sum over the block, the same order on every run.
template <int kWarps>
__device__ __forceinline__ float block_sum(float v, float* red /* [kWarps] */) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) s += red[i];
    return s;
}

// Max of a bf16 magnitude (as bits) over the block.
template <int kWarps>
__device__ __forceinline__ uint32_t block_max(uint32_t v, uint32_t* red /* [kWarps] */) {
    v = __reduce_max_sync(0xffffffffu, v);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    uint32_t r = red[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) r = max(r, red[i]);
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// The row's codes and scale from its bf16 values y (held as VPT vectors):
// the quantizer of quant.cuh on the same bits.
template <int THREADS, int VPT>
__device__ __forceinline__ void quantize_row(const uint4 (&y)[VPT], int64_t nvec, int64_t row, uint2* __restrict__ Q,
                                             float* __restrict__ S, uint32_t* red) {
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) acc = absmax_bits_u4(y[i], acc);
    const uint32_t amax = block_max<THREADS / 32>(max(acc & 0xffffu, acc >> 16), red);
    const float s = scale_from_absmax_bits(amax);
    const float r = __frcp_rn(s);
    if (threadIdx.x == 0) S[row] = s;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * THREADS;
        if (j < nvec) Q[row * nvec + j] = quantize8(y[i], s, r);
    }
}

// RMSNorm + quantize.  X [M, K], gain G [K], bf16; Y [M, K] bf16 (optional),
// Q [M, K] codes, S [M] scales.  K / 8 <= VPT * THREADS.  Rows up to 4096
// values take 128 threads (fewer warps per reduction, more rows resident
// per SM), longer rows 256.
template <int THREADS, int VPT>
__global__ void __launch_bounds__(THREADS)
rmsnorm_quant_kernel(const uint4* __restrict__ X, const uint4* __restrict__ G, int64_t K, float eps,
                     uint4* __restrict__ Y, uint2* __restrict__ Q, float* __restrict__ S) {
    constexpr int kWarps = THREADS / 32;
    grid_launch_dependents();
    grid_dependency_wait();  // X may be the previous kernel's output
    __shared__ float red_f[kWarps];
    __shared__ uint32_t red_u[kWarps];
    const int64_t row = blockIdx.x;
    const int64_t nvec = K >> 3;
    uint4 x[VPT];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * THREADS;
        x[i] = j < nvec ? __ldg(X + row * nvec + j) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float lo = bf16_lo(w[t]), hi = bf16_hi(w[t]);
            ss = __fmaf_rn(lo, lo, ss);
            ss = __fmaf_rn(hi, hi, ss);
        }
    }
    const float total = block_sum<kWarps>(ss, red_f);
    const float r = 1.0f / sqrtf(total / float(K) + eps);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * THREADS;
        const uint4 g = j < nvec ? __ldg(G + j) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            o[t] = pack_bf16x2(__fmul_rn(__fmul_rn(bf16_lo(w[t]), r), bf16_lo(gw[t])),
                               __fmul_rn(__fmul_rn(bf16_hi(w[t]), r), bf16_hi(gw[t])));
        x[i] = make_uint4(o[0], o[1], o[2], o[3]);  // now y
        if (Y != nullptr && j < nvec) Y[row * nvec + j] = x[i];
    }
    quantize_row<THREADS, VPT>(x, nvec, row, Q, S, red_u);
}

// silu(v) * u in fp32 with CUDA's fast exponential and division intrinsics
// (__expf, __fdividef: errors of a few fp32 units, up to about a hundred
// for |v| near 88, far below half a bf16 unit, 2^-9 relative), in a form that
// cannot overflow: v / (1 + e^-v) for v >= 0 and v e^v / (1 + e^v) below
// (for v < -88, e^-v overflows and the first form would return 0 where the
// value is still a normal number).
__device__ __forceinline__ float silu_mul(float v, float u) {
    const float e = __expf(-fabsf(v));  // in (0, 1]
    const float num = v >= 0.0f ? v : v * e;
    return __fdividef(num, 1.0f + e) * u;
}

// SiLU(gate) * up + quantize, on the packed gate_up output GU [M, 2I] (gate
// in columns 0 .. I-1, up in I .. 2I-1); Y [M, I] bf16 (optional), Q [M, I]
// codes, S [M] scales.  I / 8 <= VPT * THREADS.
template <int THREADS, int VPT>
__global__ void __launch_bounds__(THREADS)
silu_mul_quant_kernel(const uint4* __restrict__ GU, int64_t I, uint4* __restrict__ Y, uint2* __restrict__ Q,
                      float* __restrict__ S) {
    grid_launch_dependents();
    grid_dependency_wait();  // GU may be the previous kernel's output
    __shared__ uint32_t red_u[THREADS / 32];
    const int64_t row = blockIdx.x;
    const int64_t nvec = I >> 3;
    const uint4* gate = GU + row * 2 * nvec;
    const uint4* up = gate + nvec;
    uint4 y[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * THREADS;
        uint4 gv = make_uint4(0u, 0u, 0u, 0u), uv = gv;
        if (j < nvec) {
            gv = __ldg(gate + j);
            uv = __ldg(up + j);
        }
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            o[t] = pack_bf16x2(silu_mul(bf16_lo(gw[t]), bf16_lo(uw[t])), silu_mul(bf16_hi(gw[t]), bf16_hi(uw[t])));
        y[i] = make_uint4(o[0], o[1], o[2], o[3]);
        if (Y != nullptr && j < nvec) Y[row * nvec + j] = y[i];
    }
    quantize_row<THREADS, VPT>(y, nvec, row, Q, S, red_u);
}

}  // namespace producer
}  // namespace mfp8
