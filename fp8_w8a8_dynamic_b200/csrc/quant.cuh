// quant.cuh — per-row (per-token / per-output-channel) e4m3 quantization.
//
// Source of the rule: "MOSS-VL quantization README", FP8-Dynamic recipe
// section (weights float8_e4m3fn channel-wise static; activations FP8
// per-token dynamic) and the "MOSS-VL-Realtime-FP8 mixed-precision strategy"
// article, section "252 个主力 Linear 层为什么用 FP8 E4M3".  One rule serves
// both: a weight row is an output channel, an activation row is a token.
//   s    = fl32(max_k |x_k| / 448), raised to FLT_MIN when smaller
//   q_k  = e4m3_rn_satfinite(fl32(x_k / s))
// The codes are those of an IEEE round-to-nearest division x / s, so they
// are bit-identical to the CPU oracle's; quantize8 reaches them with one
// multiply per element and an exact divide only near e4m3 rounding
// boundaries (see there).
//
// Memory-bound: each row is read once (16-byte loads, 8 bf16 per load),
// held in registers while the block reduces its absmax, then converted and
// stored as packed 8-byte groups of codes.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mfp8 {

constexpr float kFltMin = 1.17549435082228750797e-38f;  // 2^-126
constexpr float kE4m3Max = 448.0f;

// Two fp32 values -> two e4m3 codes, `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    // The first source operand lands in the upper byte.
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// |x| of a bf16 orders like its 15 low bits read as an unsigned integer, so
// the absmax is an integer max (exact, and NaN-free inputs assumed).
__device__ __forceinline__ uint32_t absmax_bits_u4(uint4 v, uint32_t acc) {
    const uint32_t m = 0x7fff7fffu;
    acc = __vmaxu2(acc, v.x & m);
    acc = __vmaxu2(acc, v.y & m);
    acc = __vmaxu2(acc, v.z & m);
    acc = __vmaxu2(acc, v.w & m);
    return acc;
}

__device__ __forceinline__ float scale_from_absmax_bits(uint32_t amax16) {
    const float amax = __uint_as_float(amax16 << 16);
    float s = __fdiv_rn(amax, kE4m3Max);
    return s < kFltMin ? kFltMin : s;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Exact quantization without a divide per element.
//
// The code of x is e4m3(fl32(x / s)).  With r = fl32(1 / s) (one correctly
// rounded reciprocal per row), q = fl32(x * r) differs from x / s by at most
// 2^-23 |x / s|, so from fl32(x / s) by at most about 3 units in the last
// place of q.  e4m3 rounding is a step function of its input whose steps
// sit at the midpoints between neighbouring codes; if q is more than 8 ulps
// away from every such midpoint, q and fl32(x / s) lie on the same step and
// encode to the same code.  Only values closer than that (rare) are divided
// exactly.  The midpoints in fp32 bits:
//   - |q| >= 432 encodes to 448 whatever the rounding (saturation above
//     464), so nothing from 440 up needs a check;
//   - e4m3 normals (|q| >= 2^-6): 3 mantissa bits, so a midpoint is an fp32
//     whose low 20 mantissa bits are exactly 1 << 19;
//   - e4m3 subnormals (|q| < 2^-6): steps of 2^-9, midpoints at odd
//     multiples of 2^-10; in fixed point with 2^-34 units (exact for
//     |q| >= 2^-11) a midpoint is 2^24 modulo 2^25.  Below 2^-11 everything
//     encodes to zero (the first midpoint is 2^-10).
__device__ __forceinline__ bool near_e4m3_midpoint(float q) {
    const uint32_t b = __float_as_uint(q) & 0x7fffffffu;
    if (b >= 0x43dc0000u) return false;                    // |q| >= 440
    if (b >= 0x3c800000u) {                                // |q| >= 2^-6
        const int32_t d = int32_t(b & 0xfffffu) - 0x80000;
        return d >= -8 && d <= 8;
    }
    if (b < 0x3a000000u) return false;                     // |q| < 2^-11
    const uint32_t a = uint32_t(__uint_as_float(b) * 17179869184.0f);  // |q| * 2^34, exact
    const int32_t d = int32_t(a & 0x1ffffffu) - 0x1000000;
    return d >= -128 && d <= 128;                          // 8 ulps of the largest binade here
}

// 8 bf16 values -> 8 e4m3 codes (byte i = value i).  r must be fl32(1 / s).
__device__ __forceinline__ uint2 quantize8(uint4 v, float s, float r) {
    float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float q[8];
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[i] = x[i] * r;
        slow |= near_e4m3_midpoint(q[i]);
    }
    if (slow) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], s);
    }
    uint2 out;
    out.x = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
    out.y = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
    return out;
}

// The reference form: one IEEE divide per element.
__device__ __forceinline__ uint2 quantize8_div(uint4 v, float s) {
    uint2 q;
    q.x = e4m3x2(__fdiv_rn(bf16_lo(v.x), s), __fdiv_rn(bf16_hi(v.x), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(v.y), s), __fdiv_rn(bf16_hi(v.y), s)) << 16);
    q.y = e4m3x2(__fdiv_rn(bf16_lo(v.z), s), __fdiv_rn(bf16_hi(v.z), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(v.w), s), __fdiv_rn(bf16_hi(v.w), s)) << 16);
    return q;
}

constexpr int kQuantThreads = 256;

// Block-wide max of a 16-bit magnitude held by every thread.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red /* [8] */) {
    v = __reduce_max_sync(0xffffffffu, v);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    uint32_t r = red[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) r = max(r, red[w]);
    return r;
}

// One block per row; the row (K/8 16-byte vectors) lives in registers,
// VPT vectors per thread.  Requires K/8 <= VPT * 256.
// EARLY_TRIGGER (activation quantization) is the programmatic-dependent
// form: the kernel lets the GEMM that follows begin its prologue at once
// (that GEMM waits for the codes before reading them), then waits for the
// grid before it.  The weight quantizer leaves it off, so nothing that
// follows starts before the weight codes are complete.
// Block 0 also clears `nzero` words at `zero` (the split-K counters of the
// GEMM that follows in the same call).
template <int VPT, bool EARLY_TRIGGER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_reg_kernel(const uint4* __restrict__ X, int64_t K, uint2* __restrict__ Q,
                      float* __restrict__ S, unsigned int* __restrict__ zero, int nzero) {
    // Launched as a programmatic dependent of the previous kernel.  The GEMM
    // that follows may start launching at once: before its own wait it only
    // sets itself up and (static weights) reads W, and one of its CTAs and
    // one of these always fit on an SM together.  This kernel then waits for
    // the previous one (X may be its output, and it may still read this
    // call's buffers) before touching memory.
    if (EARLY_TRIGGER) {
        grid_launch_dependents();
        grid_dependency_wait();
    }
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += kQuantThreads) zero[i] = 0u;
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t row = blockIdx.x;
    const int64_t nvec = K >> 3;
    const uint4* xr = X + row * nvec;
    uint4 v[VPT];
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * kQuantThreads;
        if (j < nvec) {
            v[i] = __ldg(xr + j);
            acc = absmax_bits_u4(v[i], acc);
        } else {
            v[i] = make_uint4(0, 0, 0, 0);
        }
    }
    const uint32_t amax = block_max_u32(max(acc & 0xffffu, acc >> 16), red);
    const float s = scale_from_absmax_bits(amax);
    const float r = __frcp_rn(s);
    if (threadIdx.x == 0) S[row] = s;
    uint2* qr = Q + row * nvec;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j = threadIdx.x + int64_t(i) * kQuantThreads;
        if (j < nvec) qr[j] = quantize8(v[i], s, r);
    }
}

// Any K: two passes over the row (the second one is served by L2).
template <bool EARLY_TRIGGER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_loop_kernel(const uint4* __restrict__ X, int64_t K, uint2* __restrict__ Q,
                       float* __restrict__ S, unsigned int* __restrict__ zero, int nzero) {
    if (EARLY_TRIGGER) {  // as in quant_rows_reg_kernel
        grid_launch_dependents();
        grid_dependency_wait();
    }
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += kQuantThreads) zero[i] = 0u;
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t row = blockIdx.x;
    const int64_t nvec = K >> 3;
    const uint4* xr = X + row * nvec;
    uint32_t acc = 0;
    for (int64_t j = threadIdx.x; j < nvec; j += kQuantThreads) acc = absmax_bits_u4(__ldg(xr + j), acc);
    const uint32_t amax = block_max_u32(max(acc & 0xffffu, acc >> 16), red);
    const float s = scale_from_absmax_bits(amax);
    const float r = __frcp_rn(s);
    if (threadIdx.x == 0) S[row] = s;
    uint2* qr = Q + row * nvec;
    for (int64_t j = threadIdx.x; j < nvec; j += kQuantThreads) qr[j] = quantize8(__ldg(xr + j), s, r);
}

// Diagnostic: the e4m3 conversion alone, on arbitrary fp32 values.
__global__ void e4m3_encode_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ out) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t p = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; 2 * p < n; p += stride) {
        const int64_t i = 2 * p;
        if (i + 1 < n) {
            const uint32_t c = e4m3x2(in[i], in[i + 1]);
            out[i] = uint8_t(c & 0xff);
            out[i + 1] = uint8_t(c >> 8);
        } else {
            out[i] = uint8_t(e4m3x2(in[i], 0.0f) & 0xff);
        }
    }
}

}  // namespace mfp8
