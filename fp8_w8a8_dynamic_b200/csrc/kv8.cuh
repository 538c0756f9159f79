// kv8.cuh — the INT8 KV cache: the history of a K or V tensor quantized to
// 8-bit codes in groups of 64 tokens, the latest positions kept in bf16, and
// the read that dequantizes the history and appends the bf16 tail.
//
// Source: "MOSS-VL quantization README", KV8 section.  generation_config.json
// carries a quantized cache with the hqq backend, nbits 8, axis_key and
// axis_value 0, q_group_size 64 and residual_length 128; older positions live
// quantized and a short bf16 tail is appended when the history is read back.
// The section does not give HQQ's optimizer.  Readings:
//  - a tensor is [T tokens][H heads][D], C = H * D columns; axis 0 is the
//    token axis, so a group is 64 consecutive tokens of one column, with one
//    scale and one zero point per (group, column): [T / 64][C] fp32 each;
//  - the fit is the asymmetric min-max one with an integer zero point, fp32,
//    each step rounded to nearest even:
//      range = max - min;  s = max(range / 255, FLT_MIN) when range > 0,
//      s = max(|min|, FLT_MIN) for a constant group;  z = rint(-min / s) + 0
//      q = min(255, max(0, rint(x / s + z)))
//  - dequantize: bf16((q - z) * s), q - z exact.
// Inputs must be finite with max - min finite in fp32; then |z| <= 255 *
// 2^9 (a non-constant group of bf16 values has range >= 2^-9 max|x|, so
// |min| / s <= 255 * 2^9), far below 2^23.
//
// Layout in HBM: codes [T][C] u8 (the input's layout, one byte per value),
// scale and zero [T / 64][C] fp32.  Both kernels are bound by HBM: quantize
// moves 2 + 1 bytes per value and 8 per group and column, the read 1 + 2
// per history value, 8 per group and column, and 2 + 2 per tail value.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "quant.cuh"

namespace mfp8 {
namespace kv8 {

constexpr int kGroup = 64;
constexpr int kQuantThreads = 256;  // 8 warps; warp w takes tokens 8w .. 8w + 7 of the group
constexpr int kTileCols = 256;      // columns per quantize tile: 32 chunks of 8
constexpr int kSliceRows = kGroup / (kQuantThreads / 32);
constexpr int kReadThreads = 256;
constexpr int kReadRows = 8;  // tokens per thread in the read

// The group's scale and zero point.
__device__ __forceinline__ void fit(float mn, float mx, float& s, float& z) {
    const float range = __fsub_rn(mx, mn);
    s = range > 0.0f ? __fdiv_rn(range, 255.0f) : fabsf(mn);
    s = s < kFltMin ? kFltMin : s;
    z = __fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.0f);  // -0 -> +0
}

// One code by the IEEE divide (for scales below kFmaMinScale).  The
// float-to-unsigned conversion rounds to nearest even and clamps below at 0
// (NaN -> 0); the min clamps above at 255.
__device__ __forceinline__ uint32_t code_div(float x, float s, float z) {
    const uint32_t c = __float2uint_rn(__fadd_rn(__fdiv_rn(x, s), z));
    return c < 255u ? c : 255u;
}

// Two codes for one word of two bf16 values (lanes = its two columns).
// x / s is the corrected quotient: q0 = x r with r = fl32(1/s), the residual
// x - q0 s in one fused multiply-add (ns = -s), and q0 + residual * r
// rounded once: the correctly rounded quotient whenever the residual is
// exact (Markstein's theorem), which holds for |x| >= 2^-103 (the residual,
// about 2^-23 |x|, stays normal).  Smaller x with s >= kFmaMinScale = 2^-64
// give |x / s| < 2^-39, and then t = q + z rounds to z or to within 2^-39 of
// 0 whatever the quotient's last bits, so the code is the divide's.
// code_check_kernel compares the two forms on random groups.
// Within a group t = fl32(q + z) lies in [-1/2, 256]: z - fl32(-min / s) is
// in [-1/2, 1/2] exactly and q is monotone in x.  So no lower clamp is
// needed: t is clamped to 255 from above, and adding 1.5 * 2^23 rounds it to
// the nearest integer (ties to even) into the low mantissa byte (-1/2 gives
// 0).  Returns the two codes in bytes 0 and 1; bytes 2 and 3 are not
// defined.
__device__ __forceinline__ uint32_t codes2(uint32_t w, uint64_t ns, uint64_t r, uint64_t z) {
    const uint64_t x = pack2(bf16_lo(w), bf16_hi(w));
    const uint64_t q0 = mul2(x, r);
    const uint64_t t = add2(fma2(fma2(q0, ns, x), r, q0), z);
    float a, b;
    unpack2(t, a, b);
    unpack2(add2(pack2(fminf(a, 255.0f), fminf(b, 255.0f)), pack2(12582912.0f, 12582912.0f)), a, b);
    return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040u);
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t w) {
    __nv_bfloat162 b;
    memcpy(&b, &w, sizeof b);
    return b;
}

__device__ __forceinline__ uint32_t bits_of(__nv_bfloat162 b) {
    uint32_t w;
    memcpy(&w, &b, sizeof w);
    return w;
}

// Diagnostic: the codes of codes2 against the divide form, on groups.
// Block b draws two groups from a hash of (seed, b): each a random finite
// bf16 minimum and a maximum that is either another random finite bf16 or a
// few bf16 steps above the minimum (narrow groups far from zero).  Each
// group is fitted as the quantize kernel fits it; groups with a scale below
// kFmaMinScale (coded by the divide there) are skipped.  Every finite bf16
// x in [min, max] is coded both ways (lane 0: first group, lane 1: second).
// out[0] += mismatches, out[1] = one of them as (scale bits << 32) | x bits.
__device__ __forceinline__ uint32_t mix32(uint32_t h) {
    h ^= h >> 16;
    h *= 0x7feb352du;
    h ^= h >> 15;
    h *= 0x846ca68bu;
    h ^= h >> 16;
    return h;
}

__device__ __forceinline__ uint32_t finite_bf16(uint32_t h) {
    const uint32_t b = h & 0xffffu;
    return (b & 0x7f80u) == 0x7f80u ? (b & 0x807fu) : b;  // inf / NaN exponents -> zero exponent
}

__device__ __forceinline__ float bf16_val(uint32_t b) { return __uint_as_float(b << 16); }

__global__ void code_check_kernel(unsigned long long* __restrict__ out, uint32_t seed) {
    float mn[2], mx[2], s[2], z[2], r[2];
    bool live[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t h = mix32(seed * 0x9e3779b9u + blockIdx.x * 2u + k), h2 = mix32(h ^ 0x632be5abu);
        const uint32_t a = finite_bf16(h);
        uint32_t b = finite_bf16(h2);
        if (h2 & 0x10000u) {  // narrow: up to 63 bf16 steps above a, same sign, finite
            const uint32_t mag = a & 0x7fffu, step = (h2 >> 17) & 63u;
            b = (a & 0x8000u) ? ((mag > step ? mag - step : 0u) | 0x8000u) : (mag + step < 0x7f80u ? mag + step : mag);
        }
        const float fa = bf16_val(a), fb = bf16_val(b);
        mn[k] = fminf(fa, fb);
        mx[k] = fmaxf(fa, fb);
        fit(mn[k], mx[k], s[k], z[k]);
        r[k] = __frcp_rn(s[k]);
        live[k] = s[k] >= kFmaMinScale && isfinite(__fsub_rn(mx[k], mn[k]));
    }
    const uint64_t ns = pack2(-s[0], -s[1]), r2 = pack2(r[0], r[1]), z2 = pack2(z[0], z[1]);
    unsigned long long bad = 0;
    uint32_t witness = 0;
    for (uint32_t x16 = threadIdx.x; x16 < 65536u; x16 += blockDim.x) {
        if ((x16 & 0x7f80u) == 0x7f80u) continue;  // inf, NaN
        const float x = bf16_val(x16);
        const bool in0 = live[0] && x >= mn[0] && x <= mx[0], in1 = live[1] && x >= mn[1] && x <= mx[1];
        if (!in0 && !in1) continue;
        const uint32_t w = x16 | (x16 << 16);
        const uint32_t c = codes2(w, ns, r2, z2);
        if (in0 && (c & 0xffu) != code_div(x, s[0], z[0])) {
            ++bad;
            witness = x16;
        }
        if (in1 && ((c >> 8) & 0xffu) != code_div(x, s[1], z[1])) {
            ++bad;
            witness = x16 | 0x10000u;
        }
    }
    if (bad) {
        atomicAdd(out, bad);
        out[1] = (static_cast<unsigned long long>(__float_as_uint(s[0])) << 32) | witness;
    }
}

// The divide form of one thread's 8 rows x 8 columns, for the rare tiles
// with a scale below kFmaMinScale; it reads its rows again (from L2).
__device__ __noinline__ void codes_div_rows(const uint4* src, int64_t C8, uint2* dst, const float* s_sm,
                                            const float* z_sm) {
    for (int i = 0; i < kSliceRows; ++i) {
        const uint4 v = src[i * C8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t c[8];
        for (int q = 0; q < 4; ++q) {
            c[2 * q] = code_div(bf16_lo(w[q]), s_sm[2 * q], z_sm[2 * q]);
            c[2 * q + 1] = code_div(bf16_hi(w[q]), s_sm[2 * q + 1], z_sm[2 * q + 1]);
        }
        dst[i * C8] = make_uint2(c[0] | c[1] << 8 | c[2] << 16 | c[3] << 24,
                                 c[4] | c[5] << 8 | c[6] << 16 | c[7] << 24);
    }
}

// Quantize: KV [T][C8] as 16-byte vectors of 8 bf16 (C8 = C / 8), T = 64 G.
// Block b takes tile (group g, 256 columns ct).  Lane l of warp w loads the
// 8 columns 8 l .. 8 l + 7 of the tile for the 8 tokens 8w .. 8w + 7 (each
// warp load: 512 contiguous bytes of one token) and keeps them in registers;
// the warps' partial minima and maxima meet in shared memory, thread j fits
// column j and writes its scale and zero point, and every thread then
// writes its 8 x 8 codes (8-byte stores, 256 contiguous bytes per warp).
// The input crosses HBM once.
__global__ void __launch_bounds__(kQuantThreads, 4)
quant_kernel(const uint4* __restrict__ KV, int64_t C8, int64_t tiles_per_group, uint2* __restrict__ Q,
             float* __restrict__ S, float* __restrict__ Z) {
    __shared__ uint4 red_mn[kQuantThreads / 32][32], red_mx[kQuantThreads / 32][32];
    __shared__ __align__(16) float s_sm[kTileCols];
    __shared__ __align__(16) float r_sm[kTileCols];
    __shared__ __align__(16) float z_sm[kTileCols];
    grid_launch_dependents();
    grid_dependency_wait();  // KV may be the previous kernel's output
    const int64_t g = blockIdx.x / tiles_per_group, ct = blockIdx.x % tiles_per_group;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c8 = ct * 32 + lane;
    const bool valid = c8 < C8;
    const int64_t row0 = g * kGroup + warp * kSliceRows;
    const uint4* src = KV + row0 * C8 + c8;
    uint4 v[kSliceRows];
#pragma unroll
    for (int i = 0; i < kSliceRows; ++i) v[i] = valid ? __ldcs(src + i * C8) : make_uint4(0u, 0u, 0u, 0u);
    {
        __nv_bfloat162 mn[4] = {as_bf162(v[0].x), as_bf162(v[0].y), as_bf162(v[0].z), as_bf162(v[0].w)};
        __nv_bfloat162 mx[4] = {mn[0], mn[1], mn[2], mn[3]};
#pragma unroll
        for (int i = 1; i < kSliceRows; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                mn[q] = __hmin2(mn[q], as_bf162(w[q]));
                mx[q] = __hmax2(mx[q], as_bf162(w[q]));
            }
        }
        red_mn[warp][lane] = make_uint4(bits_of(mn[0]), bits_of(mn[1]), bits_of(mn[2]), bits_of(mn[3]));
        red_mx[warp][lane] = make_uint4(bits_of(mx[0]), bits_of(mx[1]), bits_of(mx[2]), bits_of(mx[3]));
    }
    __syncthreads();
    {
        const int j = threadIdx.x, chunk = j >> 3, word = (j & 7) >> 1;
        const uint32_t* pmn = reinterpret_cast<const uint32_t*>(&red_mn[0][chunk]) + word;
        const uint32_t* pmx = reinterpret_cast<const uint32_t*>(&red_mx[0][chunk]) + word;
        __nv_bfloat162 mn = as_bf162(pmn[0]), mx = as_bf162(pmx[0]);
#pragma unroll
        for (int w = 1; w < kQuantThreads / 32; ++w) {
            mn = __hmin2(mn, as_bf162(pmn[w * 32 * 4]));
            mx = __hmax2(mx, as_bf162(pmx[w * 32 * 4]));
        }
        const bool hi = j & 1;
        float sc, zp;
        fit(hi ? bf16_hi(bits_of(mn)) : bf16_lo(bits_of(mn)), hi ? bf16_hi(bits_of(mx)) : bf16_lo(bits_of(mx)), sc,
            zp);
        s_sm[j] = sc;
        r_sm[j] = __frcp_rn(sc);
        z_sm[j] = zp;
        const int64_t col = ct * kTileCols + j;
        if (col < C8 * 8) {
            S[g * C8 * 8 + col] = sc;
            Z[g * C8 * 8 + col] = zp;
        }
    }
    __syncthreads();
    if (!valid) return;
    const float* fs = s_sm + lane * 8;
    bool fast = true;
    uint64_t ns[4], r[4], z[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 s2 = *reinterpret_cast<const float2*>(fs + 2 * q);
        fast = fast && s2.x >= kFmaMinScale && s2.y >= kFmaMinScale;
        ns[q] = pack2(-s2.x, -s2.y);
        const float2 r2 = *reinterpret_cast<const float2*>(r_sm + lane * 8 + 2 * q);
        const float2 z2 = *reinterpret_cast<const float2*>(z_sm + lane * 8 + 2 * q);
        r[q] = pack2(r2.x, r2.y);
        z[q] = pack2(z2.x, z2.y);
    }
    uint2* dst = Q + row0 * C8 + c8;
    if (fast) {
#pragma unroll
        for (int i = 0; i < kSliceRows; ++i) {
            const uint32_t c01 = codes2(v[i].x, ns[0], r[0], z[0]), c23 = codes2(v[i].y, ns[1], r[1], z[1]);
            const uint32_t c45 = codes2(v[i].z, ns[2], r[2], z[2]), c67 = codes2(v[i].w, ns[3], r[3], z[3]);
            __stcs(dst + i * C8, make_uint2(__byte_perm(c01, c23, 0x5410u), __byte_perm(c45, c67, 0x5410u)));
        }
    } else {
        codes_div_rows(src, C8, dst, fs, z_sm + lane * 8);
    }
}

// Four codes of one 32-bit word -> four bf16 (two words).  2^23 + q is built
// by placing the code in the low mantissa byte of 2^23; subtracting
// zz = 2^23 + z (exact, |z| < 2^22) leaves q - z exactly, and one product
// by s rounds it to fp32.  Lanes are columns 4k .. 4k + 3 in pairs.
__device__ __forceinline__ uint2 dequant4(uint32_t w, const uint64_t* s, const uint64_t* zz) {
    const uint64_t b01 = pack2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u)),
                               __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7541u)));
    const uint64_t b23 = pack2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7542u)),
                               __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7543u)));
    float v0, v1, v2, v3;
    unpack2(mul2(sub2(b01, zz[0]), s[0]), v0, v1);
    unpack2(mul2(sub2(b23, zz[1]), s[1]), v2, v3);
    return make_uint2(bits_of(__floats2bfloat162_rn(v0, v1)), bits_of(__floats2bfloat162_rn(v2, v3)));
}

// The read: out [Tq + Tr][C] bf16 = the Tq history tokens dequantized, then
// the Tr tail tokens copied.  C8 = C / 8.  Threads below nA each take 8
// columns (an 8-byte load of codes, one 16-byte store per token, so a
// warp's store covers 512 contiguous bytes: whole sectors) of kReadRows
// tokens of one group, with the 8 scales and zero points in registers; all
// of the thread's loads are issued before any arithmetic.  The threads after
// them copy the tail, 16 bytes each.
__global__ void __launch_bounds__(kReadThreads)
read_kernel(const uint2* __restrict__ Q, const float4* __restrict__ S, const float4* __restrict__ Z, int64_t Tq,
            int64_t C8, const uint4* __restrict__ tail, int64_t n_tail16, uint4* __restrict__ out) {
    grid_launch_dependents();
    grid_dependency_wait();  // the cache may be the previous kernel's output
    const int64_t i = int64_t(blockIdx.x) * kReadThreads + threadIdx.x;
    const int64_t nA = (Tq / kReadRows) * C8;
    if (i < nA) {
        const int64_t rb = i / C8, c = i - rb * C8;
        const int64_t t0 = rb * kReadRows, g = t0 / kGroup;
        uint2 q[kReadRows];
#pragma unroll
        for (int t = 0; t < kReadRows; ++t) q[t] = __ldcs(Q + (t0 + t) * C8 + c);
        uint64_t s[4], zz[4];
        const uint64_t big = pack2(8388608.0f, 8388608.0f);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float4 a = __ldg(S + (g * C8 + c) * 2 + j);
            const float4 b = __ldg(Z + (g * C8 + c) * 2 + j);
            s[2 * j] = pack2(a.x, a.y), s[2 * j + 1] = pack2(a.z, a.w);
            zz[2 * j] = add2(pack2(b.x, b.y), big), zz[2 * j + 1] = add2(pack2(b.z, b.w), big);
        }
#pragma unroll
        for (int t = 0; t < kReadRows; ++t) {
            const uint2 a = dequant4(q[t].x, s, zz), b = dequant4(q[t].y, s + 2, zz + 2);
            __stcs(out + (t0 + t) * C8 + c, make_uint4(a.x, a.y, b.x, b.y));
        }
    } else if (i - nA < n_tail16) {
        const int64_t j = i - nA;
        __stcs(out + Tq * C8 + j, __ldcs(tail + j));
    }
}

}  // namespace kv8
}  // namespace mfp8
