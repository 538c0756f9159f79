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
// are bit-identical to the CPU oracle's; quantize8 reaches them with a
// multiply by the reciprocal and two fused multiply-adds per element (see
// div_rn_by_recip), checked against the divide on every bf16 pair.
//
// Memory-bound: each row is read once (16-byte loads, 8 bf16 per load),
// held in registers while the block reduces its absmax, then converted and
// stored as packed 8-byte groups of codes.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

__device__ __forceinline__ float scale_from_absmax_bits_div(uint32_t amax16) {
    const float amax = __uint_as_float(amax16 << 16);
    float s = __fdiv_rn(amax, kE4m3Max);
    return s < kFltMin ? kFltMin : s;
}

// The same scale without a divide.  448 = 7 * 2^6, so fl32(a / 448) is
// fl32(a / 7) * 2^-6 (scaling by a power of two is exact while the result
// is normal; below FLT_MIN both forms are raised to FLT_MIN).  fl32(a / 7)
// is Markstein's corrected quotient with the correctly rounded reciprocal
// 1/7 = 0x3E124925.  Checked against the divide for every bf16 absmax
// (mfp8_debug_quantize_check).
__device__ __forceinline__ float scale_from_absmax_bits(uint32_t amax16) {
    const float a = __uint_as_float(amax16 << 16);
    const float r7 = __uint_as_float(0x3E124925u);
    const float q0 = __fmul_rn(a, r7);
    const float e = __fmaf_rn(-q0, 7.0f, a);
    const float s = __fmul_rn(__fmaf_rn(e, r7, q0), 0.015625f);
    return s < kFltMin ? kFltMin : s;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// The reference form: one IEEE divide per element.
__device__ __forceinline__ uint2 quantize8_div(uint4 v, float s) {
    uint2 q;
    q.x = e4m3x2(__fdiv_rn(bf16_lo(v.x), s), __fdiv_rn(bf16_hi(v.x), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(v.y), s), __fdiv_rn(bf16_hi(v.y), s)) << 16);
    q.y = e4m3x2(__fdiv_rn(bf16_lo(v.z), s), __fdiv_rn(bf16_hi(v.z), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(v.w), s), __fdiv_rn(bf16_hi(v.w), s)) << 16);
    return q;
}

// fl32(a / s) without a divide: r = fl32(1 / s) (correctly rounded),
// q0 = fl32(a * r) is within one unit in the last place of a / s, the
// residual a - q0 * s is exact in one fused multiply-add, and one more fused
// multiply-add q0 + (a - q0 s) * r rounds to the correctly rounded quotient
// (Markstein's theorem on division by reciprocal with a corrected quotient).
// Every step rounds to nearest, which is odd-symmetric, so -a gives exactly
// the negated result; the one exception is a = -0, for which the residual
// step returns +0.  Checked against the IEEE divide on every pair of bf16
// values with |x| <= absmax, both signs (mfp8_debug_quantize_check).
__device__ __forceinline__ float div_rn_by_recip(float a, float s, float r) {
    const float q0 = __fmul_rn(a, r);
    const float e = __fmaf_rn(-q0, s, a);
    return __fmaf_rn(e, r, q0);
}

// Two bf16 values (one 32-bit word) -> two e4m3 codes (16 bits, low value in
// the low byte).
// The quotients carry x's sign except for x = -0 (see div_rn_by_recip), so
// the sign bits of x are OR-ed into the codes: a no-op for every other x.
// Both values go through div_rn_by_recip's three steps at once in paired
// fp32 arithmetic (ns2 = (-s, -s), r2 = (r, r)): each lane rounds exactly as
// the scalar steps do, and x - q0 s is q0 * (-s) + x in one fused
// multiply-add.
__device__ __forceinline__ uint32_t quantize2_fma(uint32_t w, uint64_t ns2, uint64_t r2) {
    const uint64_t x = pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    const uint64_t q0 = mul2(x, r2);
    float lo, hi;
    unpack2(fma2(fma2(q0, ns2, x), r2, q0), lo, hi);
    return e4m3x2(lo, hi) | (__byte_perm(w, 0u, 0x4431u) & 0x8080u);  // bits 15, 31 of w -> 7, 15
}

// 8 bf16 values -> 8 e4m3 codes, same codes as quantize8_div.  The
// corrected quotient needs an exact residual a - q0 s; when s is tiny that
// residual falls below the normal fp32 range and loses bits, so rows with
// s < 2^-64 (absmax below about 2.4e-17) take the divide.
constexpr float kFmaMinScale = 5.42101086242752217004e-20f;  // 2^-64

// For s >= kFmaMinScale only (callers that check the scale once per row).
__device__ __forceinline__ uint2 quantize8_fast(uint4 v, float s, float r) {
    uint2 out;
    const uint64_t ns2 = pack2(-s, -s), r2 = pack2(r, r);
    out.x = quantize2_fma(v.x, ns2, r2) | (quantize2_fma(v.y, ns2, r2) << 16);
    out.y = quantize2_fma(v.z, ns2, r2) | (quantize2_fma(v.w, ns2, r2) << 16);
    return out;
}

// The divide form out of line, for the rare rows with a tiny scale inside
// unrolled loops.
__device__ __noinline__ uint2 quantize8_div_call(uint4 v, float s) { return quantize8_div(v, s); }

__device__ __forceinline__ uint2 quantize8(uint4 v, float s, float r) {
    return s < kFmaMinScale ? quantize8_div(v, s) : quantize8_fast(v, s, r);
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
template <int VPT, bool EARLY_TRIGGER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_reg_kernel(const uint4* __restrict__ X, int64_t K, uint2* __restrict__ Q,
                      float* __restrict__ S) {
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

// WPR warps per row (1, 2 or 4), 8 / WPR rows per block, for rows of at
// most 32 * VPL * WPR 16-byte vectors: the row stays in registers, each warp
// holds a contiguous share of it, the absmax is a warp reduction (and, with
// WPR > 1, a max over the row's warps through shared memory), and each warp
// then quantizes and stores its own share.  Loads and stores are
// lane-contiguous (512 and 256 bytes per instruction).  More warps per row
// give the SM more loads in flight and shorten each warp's serial chain.
// EARLY_TRIGGER as in quant_rows_reg_kernel.
template <int VPL, int WPR, bool EARLY_TRIGGER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_warp_kernel(const uint4* __restrict__ X, int64_t R, int64_t K, uint2* __restrict__ Q,
                       float* __restrict__ S) {
    static_assert(WPR == 1 || WPR == 2 || WPR == 4, "1, 2 or 4 warps per row");
    constexpr int kRowsPerBlock = kQuantThreads / 32 / WPR;
    if (EARLY_TRIGGER) {
        grid_launch_dependents();
        grid_dependency_wait();
    }
    const int w = threadIdx.x >> 5;
    const int part = w % WPR;
    const int64_t row = int64_t(blockIdx.x) * kRowsPerBlock + w / WPR;
    const bool live = row < R;
    const int lane = threadIdx.x & 31;
    const int64_t nvec = K >> 3;
    const uint4* xr = X + (live ? row : 0) * nvec;
    uint4 v[VPL];
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int64_t j = int64_t(part * VPL + i) * 32 + lane;
        v[i] = (live && j < nvec) ? __ldg(xr + j) : make_uint4(0, 0, 0, 0);
        acc = absmax_bits_u4(v[i], acc);
    }
    uint32_t amax = __reduce_max_sync(0xffffffffu, max(acc & 0xffffu, acc >> 16));
    if (WPR > 1) {
        __shared__ uint32_t red[kQuantThreads / 32];
        if (lane == 0) red[w] = amax;
        __syncthreads();
#pragma unroll
        for (int p = 0; p < WPR; ++p) amax = max(amax, red[(w / WPR) * WPR + p]);
    }
    if (!live) return;
    const float s = scale_from_absmax_bits(amax);
    const float r = __frcp_rn(s);
    if (part == 0 && lane == 0) S[row] = s;
    uint2* qr = Q + row * nvec;
    if (s < kFmaMinScale) {
        for (int i = 0; i < VPL; ++i) {
            const int64_t j = int64_t(part * VPL + i) * 32 + lane;
            if (j < nvec) qr[j] = quantize8_div_call(v[i], s);
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int64_t j = int64_t(part * VPL + i) * 32 + lane;
        if (j < nvec) qr[j] = quantize8_fast(v[i], s, r);
    }
}

// Any K: two passes over the row (the second one is served by L2).
template <bool EARLY_TRIGGER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_loop_kernel(const uint4* __restrict__ X, int64_t K, uint2* __restrict__ Q,
                       float* __restrict__ S) {
    if (EARLY_TRIGGER) {  // as in quant_rows_reg_kernel
        grid_launch_dependents();
        grid_dependency_wait();
    }
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

// ------------------------------------------------------- FP8 KV cache --
// "MOSS-VL quantization README", SGLang paragraph (--kv-cache-dtype
// fp8_e4m3; the pages give only the flag).  A K or V tensor [T, H, D] in
// bf16 gets one scale per (token, head) row of D values, by the activation
// rule above; dequantize is bf16(fl32(dec(q) * s)).

// Rows of D <= 256 values (D % 16 == 0): LPR lanes per row (a power of two
// >= D / 8), each holding one 16-byte vector of 8 values, 32 / LPR rows per
// warp and kSmallRowItems such row groups per warp, all loads issued first;
// a warp's loads and stores are contiguous.  The absmax is a shuffle
// reduction over the row's lanes.
constexpr int kSmallRowItems = 4;

template <int LPR>
__global__ void __launch_bounds__(kQuantThreads)
quant_small_rows_kernel(const uint4* __restrict__ X, int64_t R, int D, uint2* __restrict__ Q,
                        float* __restrict__ S) {
    grid_launch_dependents();
    grid_dependency_wait();  // X may be the previous kernel's output
    constexpr int kRowsPerWarp = 32 / LPR;
    const int lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t(blockIdx.x) * (kQuantThreads / 32) + (threadIdx.x >> 5)) * kRowsPerWarp *
                             kSmallRowItems + lane / LPR;
    const int v = lane % LPR;
    const int vpr = D >> 3;  // vectors per row
    uint4 x[kSmallRowItems];
#pragma unroll
    for (int k = 0; k < kSmallRowItems; ++k) {
        const int64_t row = row0 + k * kRowsPerWarp;
        x[k] = row < R && v < vpr ? __ldg(X + row * vpr + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kSmallRowItems; ++k) {
        const int64_t row = row0 + k * kRowsPerWarp;
        const uint32_t acc = absmax_bits_u4(x[k], 0u);
        uint32_t amax = max(acc & 0xffffu, acc >> 16);
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (row < R && v < vpr) {
            const float s = scale_from_absmax_bits(amax);
            if (v == 0) S[row] = s;
            Q[row * vpr + v] = quantize8(x[k], s, __frcp_rn(s));
        }
    }
}

// Dequantize: each thread turns 16 codes (16 bytes) into 16 bf16 (32 bytes).
// e4m3 -> f16 is exact, f16 -> f32 is exact, the product with the row scale
// rounds once to fp32 and the cast to bf16 rounds to nearest even.
__device__ __forceinline__ uint32_t dequant2(uint16_t codes2, float s) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes2));
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    const float2 f = __half22float2(h);
    const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(f.x, s), __fmul_rn(f.y, s));
    return *reinterpret_cast<const uint32_t*>(&b);
}

// Dequantize: each thread takes kDequantItems items of 8 codes (an 8-byte
// load) -> 8 bf16 (one 16-byte store), items blockDim.x apart, so a warp's
// store covers 512 contiguous bytes, whole sectors; all of a thread's loads
// are issued before its arithmetic.  n8 = R * D / 8.  A programmatic
// dependent: the codes may be the previous kernel's output.
constexpr int kDequantItems = 4;

__global__ void __launch_bounds__(kQuantThreads)
kv_dequant_kernel(const uint2* __restrict__ Q, const float* __restrict__ S, int64_t n8, int D,
                  uint4* __restrict__ out) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int g8 = D >> 3;  // 8-code groups per row
    const int64_t base = int64_t(blockIdx.x) * (kQuantThreads * kDequantItems) + threadIdx.x;
    uint2 q[kDequantItems];
    float s[kDequantItems];
#pragma unroll
    for (int k = 0; k < kDequantItems; ++k) {
        const int64_t i = base + k * kQuantThreads;
        q[k] = i < n8 ? __ldcs(Q + i) : make_uint2(0u, 0u);
        s[k] = i < n8 ? __ldg(S + i / g8) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kDequantItems; ++k) {
        const int64_t i = base + k * kQuantThreads;
        if (i < n8)
            __stcs(out + i, make_uint4(dequant2(uint16_t(q[k].x & 0xffffu), s[k]), dequant2(uint16_t(q[k].x >> 16), s[k]),
                                       dequant2(uint16_t(q[k].y & 0xffffu), s[k]), dequant2(uint16_t(q[k].y >> 16), s[k])));
    }
}

// Diagnostic: for every absmax a (a positive finite bf16, or zero) the
// divide-free scale against fl32(a / 448), and for every bf16 x with
// |x| <= a the codes of quantize8 against those of the IEEE-divide form.  Block b takes absmax bits b; out[0] counts mismatching
// values, out[1] keeps one of them as (a << 16) | x.
__global__ void quantize_check_kernel(unsigned long long* __restrict__ out) {
    const uint32_t a = blockIdx.x;  // 0 .. 0x7f7f
    const float s = scale_from_absmax_bits(a);
    const float r = __frcp_rn(s);
    unsigned long long bad = 0;
    uint32_t witness = 0;
    if (threadIdx.x == 0 && __float_as_uint(s) != __float_as_uint(scale_from_absmax_bits_div(a))) {
        ++bad;  // the scale itself differs from the divide's
        witness = (a << 16) | 0xffffu;
    }
    // x magnitudes 0..a, both signs: 2 (a + 1) values, 8 per step
    const uint32_t n = 2u * (a + 1u);
    for (uint32_t base = threadIdx.x * 8u; base < n; base += blockDim.x * 8u) {
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t j = base + uint32_t(i);
            const uint32_t mag = j < n ? (j >> 1) : 0u;
            h[i] = mag | ((j & 1u) << 15);
        }
        const uint4 v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                   h[6] | (h[7] << 16));
        const uint2 f = quantize8(v, s, r);
        const uint2 d = quantize8_div(v, s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t cf = ((i < 4 ? f.x : f.y) >> (8 * (i & 3))) & 0xffu;
            const uint32_t cd = ((i < 4 ? d.x : d.y) >> (8 * (i & 3))) & 0xffu;
            if (base + uint32_t(i) < n && cf != cd) {
                ++bad;
                witness = (a << 16) | h[i];
            }
        }
    }
    if (bad) {
        atomicAdd(out, bad);
        atomicExch(out + 1, (unsigned long long)witness);
    }
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
