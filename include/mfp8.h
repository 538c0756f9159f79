/*
 * mfp8.h — C ABI of the B200 (sm_100a) FP8_DYNAMIC quantized Linear.
 *
 * The method (stated by the "MOSS-VL quantization README", github OpenMOSS/
 * MOSS-VL quantization/, FP8-Dynamic recipe section, and by the
 * "MOSS-VL-Realtime-FP8 mixed-precision strategy" article, section
 * "252 个主力 Linear 层为什么用 FP8 E4M3"):
 *   - weights are float8_e4m3fn with one static scale per output channel,
 *     computed once, offline;
 *   - the input activations of the quantized kernels are float8_e4m3fn with
 *     one scale per token, computed at run time;
 *   - the product of the two is rescaled and written back as BF16 (the
 *     recipe runs the model in bfloat16).
 * Readings taken where the pages are silent (the same in the CPU oracle):
 *   scale      s = fl32(max|row| / 448), raised to FLT_MIN (2^-126) if smaller;
 *   code       e4m3(fl32(x / s)) with an IEEE round-to-nearest fp32 divide,
 *              then round-to-nearest-even to e4m3, saturating to +-448;
 *   product    fp32 accumulation of the e4m3 x e4m3 products on the tensor
 *              cores, then y = bf16_rn(acc * s_a[m] * s_w[n]); no bias.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated; the caller allocates and
 *     owns every buffer, including any workspace.  Nothing here allocates
 *     device memory or keeps a pointer after the call returns.
 *   - Matrices are row-major and contiguous.  X is [M, K] (one row per
 *     token), W is [N, K] (one row per output channel: the Linear's
 *     (out_features, in_features) layout), Y is [M, N].  BF16 buffers hold
 *     IEEE bfloat16 bit patterns; FP8 buffers hold float8_e4m3fn codes, one
 *     byte each; scales are fp32.
 *   - Every pointer must be 16-byte aligned.  K must be a positive multiple
 *     of 16, N >= 1, M >= 0 (M == 0 is a no-op).  When N is not a multiple
 *     of 8 (rows of Y not 16-byte aligned) the Linear runs its kernels on N
 *     rounded up to 8 channels into scratch taken from the workspace (the
 *     workspace-size functions count it), then copies the first N columns
 *     into Y: two small extra launches, and MFP8_FLAG_STATIC_WEIGHTS has no
 *     effect.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued on it; no call blocks the host except mfp8_get_device_status.
 *     The calls do not synchronise and may be captured in a CUDA graph.
 *   - Argument errors are returned before anything is enqueued.  Errors that
 *     arise on the device (a bounded wait that ran out) are recorded in a
 *     per-device status word that mfp8_get_device_status reads and clears.
 *     Nothing is thrown across this boundary.
 *   - Inputs holding Inf or NaN are outside the contract: the kernels still
 *     terminate, but the outputs are unspecified.
 */
#ifndef MFP8_H
#define MFP8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MFP8_API __attribute__((visibility("default")))
#else
#define MFP8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MFP8_OK = 0,
    MFP8_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, overlapping in/out */
    MFP8_ERR_MISALIGNED = 2,        /* a pointer is not 16-byte aligned */
    MFP8_ERR_UNSUPPORTED_SHAPE = 3, /* K not a positive multiple of 16, N < 1, too large */
    MFP8_ERR_WORKSPACE = 4,         /* workspace missing or smaller than mfp8_linear_workspace_bytes */
    MFP8_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    MFP8_ERR_TIMEOUT = 6,           /* a kernel's bounded wait ran out (device status) */
    MFP8_ERR_DEVICE = 7             /* the current device is not compute capability 10.0 */
} mfp8_status;

/* Per-channel weight quantization (one-time, offline).
 * Source: README FP8-Dynamic section, "float8_e4m3fn channel-wise static";
 * Realtime-FP8 article: per-channel scales computed once, zero run-time cost.
 *   W_bf16  [N, K] bf16, read only.
 *   W_fp8   [N, K] e4m3 codes, written.      w_scale [N] fp32, written.
 *   W_fp8[n,k] = e4m3(fl32(W[n,k] / w_scale[n])), w_scale[n] = fl32(max_k |W[n,k]| / 448).
 * Bit-exact with the CPU oracle. */
MFP8_API mfp8_status mfp8_quantize_weight(const void* W_bf16, int64_t N, int64_t K,
                                 void* W_fp8, float* w_scale, void* stream);

/* Per-token activation quantization (every call).
 * Source: README FP8-Dynamic section, "FP8 per-token dynamic"; Realtime-FP8
 * article: the scale is computed for each token at run time.
 *   X_bf16 [M, K] bf16, read only.
 *   X_fp8  [M, K] e4m3 codes, written.       x_scale [M] fp32, written.
 * Same rule as mfp8_quantize_weight, one scale per row of X. */
MFP8_API mfp8_status mfp8_quantize_act(const void* X_bf16, int64_t M, int64_t K,
                              void* X_fp8, float* x_scale, void* stream);

/* Bytes of device workspace that are enough for mfp8_linear and for every
 * kernel choice of mfp8_linear_ex at these sizes: the activation codes
 * [M, K] and scales [M] of the quantize pass, each rounded up to 256 bytes.
 * Never fails; returns 0 for invalid sizes (mfp8_linear then reports the
 * error). */
MFP8_API size_t mfp8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* The FP8_DYNAMIC Linear: Y = bf16(  (Xq . Wq^T) * x_scale (x) w_scale  ).
 * Source: README FP8-Dynamic section (FP8 weights, per-token FP8 inputs to
 * "the quantized kernels", model in bfloat16).
 *   X_bf16   [M, K] bf16 activations, read only.
 *   W_fp8    [N, K] e4m3 weight codes and w_scale [N] fp32, both from
 *            mfp8_quantize_weight, read only.
 *   Y_bf16   [M, N] bf16, written.  Must not overlap any input.
 *   workspace / workspace_bytes: device scratch of at least
 *            mfp8_linear_workspace_bytes(M, N, K) bytes, 16-byte aligned,
 *            any contents.  It holds the activation codes and scales between
 *            the quantize pass and the GEMM of this call; nothing in it
 *            outlives the call.  Calls that may run at the same time need
 *            separate workspaces.  The one-kernel decode path (M <= 16) does
 *            not touch it.
 * The activation quantization (per-token scale + e4m3 codes) happens inside
 * this call: its codes and scales are bit-identical to mfp8_quantize_act.
 * Outputs are within |y - y_ref| <= 2^-7 |y_ref| + 1e-5 * sum_k |a_k w_k| s_a s_w
 * of the exact rescaled product y_ref. */
MFP8_API mfp8_status mfp8_linear(const void* X_bf16, int64_t M, int64_t K,
                        const void* W_fp8, const float* w_scale, int64_t N,
                        void* Y_bf16, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Kernel choice for mfp8_linear_ex. */
typedef enum {
    MFP8_PATH_AUTO = 0,   /* what mfp8_linear does: chosen from M, N, K */
    MFP8_PATH_TILED = 1,  /* quantize pass, then the persistent 128-row-tile tcgen05 GEMM */
    MFP8_PATH_SPLITK = 2, /* quantize pass, then the split-K GEMM on CTA clusters, partials summed on chip (M <= 256) */
    MFP8_PATH_PAIR = 3,   /* quantize pass, then the 256-row-tile GEMM on CTA pairs (tcgen05 cta_group::2) */
    MFP8_PATH_FUSED = 4   /* one kernel: quantizes X on chip and streams the weights, K split over a CTA cluster (M <= 16) */
} mfp8_path;

/* The kernel MFP8_PATH_AUTO takes at these sizes (FUSED for M <= 16, SPLITK
 * up to 128, TILED below 256, PAIR above); MFP8_PATH_AUTO itself for sizes
 * no kernel takes. */
MFP8_API int mfp8_choose_path(int64_t M, int64_t N, int64_t K);

/* Flags for mfp8_linear_ex. */
#define MFP8_FLAG_STATIC_WEIGHTS 1
/* The caller promises that W_fp8 and w_scale are not written by any work
 * still pending on `stream` (they are a model's static weights, quantized
 * once).  The decode-sized kernel may then start streaming the weights while
 * the previous kernel on the stream is still finishing (programmatic
 * dependent launch); the activations are still read only after that kernel
 * has completed.  Without the flag every input is read after it. */

/* mfp8_linear with an explicit kernel choice, flags, and optional copies of
 * the activation codes and scales it computed (X_fp8_out [M, K] and
 * x_scale_out [M]; pass NULL for none).  Used to test each kernel on the
 * same shapes, to check that the activation bytes of every path are
 * bit-identical to mfp8_quantize_act, and by callers with static weights.
 * MFP8_PATH_FUSED is one launch that quantizes X on chip (the CTAs of a
 * cluster share their slice maxima, so each has the full row scales) and
 * sums the K-split partial rows in the cluster's shared memory, so it keeps
 * nothing in the workspace (it may be NULL with 0 bytes) unless N % 8 != 0
 * (the padded scratch of the conventions).  When
 * X_fp8_out is given, the codes are written there as well (the quantize
 * pass writes them there instead of the workspace).  Returns MFP8_ERR_UNSUPPORTED_SHAPE if the chosen kernel
 * cannot take these sizes, MFP8_ERR_INVALID_ARG for an unknown path or flag. */
MFP8_API mfp8_status mfp8_linear_ex(const void* X_bf16, int64_t M, int64_t K,
                           const void* W_fp8, const float* w_scale, int64_t N,
                           void* Y_bf16, void* workspace, size_t workspace_bytes,
                           int path, int flags, void* X_fp8_out, float* x_scale_out,
                           void* stream);

/* Size of the library's own scratch for mfp8_linear_noalloc: 16 MiB per device. */
#define MFP8_STATIC_WORKSPACE_BYTES (16u << 20)

/* mfp8_linear without a caller workspace: the scratch is a fixed array of
 * MFP8_STATIC_WORKSPACE_BYTES in the library's device memory, one per
 * device.  The pages describe no counterpart: this serves callers that
 * cannot allocate at the call site (a C host without its own device
 * allocator, or one that plans all device memory up front).  The call
 * allocates no memory.
 *   Arguments, results and tolerance: as mfp8_linear (kernel choice AUTO).
 *   Sizes whose mfp8_linear_workspace_bytes(M, N, K) exceeds
 *   MFP8_STATIC_WORKSPACE_BYTES are rejected with MFP8_ERR_WORKSPACE before
 *   any device work (the quantized activations need about M * K bytes:
 *   every projection up to K = 12288 fits for M <= 1300).
 *   Set-up: the first call on each device (and again after the device's
 *   context was reset) looks up the array's address; that first call should
 *   come before any stream capture.
 *   Concurrency: every call on a device shares the one scratch array.  Calls
 *   that may be in flight at the same time (different streams, or host
 *   threads) race and give wrong results; serialise them, e.g. on one stream. */
MFP8_API mfp8_status mfp8_linear_noalloc(const void* X_bf16, int64_t M, int64_t K,
                                const void* W_fp8, const float* w_scale, int64_t N,
                                void* Y_bf16, void* stream);

/* Workspace bytes mfp8_gemm needs: 0 when N is a multiple of 8 (no GEMM
 * kernel keeps anything in one; the workspace may then be NULL), else the
 * padded scratch of the conventions above: the [N8] scales and the [M, N8]
 * bf16 output, N8 = N rounded up to 8. */
MFP8_API size_t mfp8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* The contraction and epilogue alone, on activations already quantized by
 * mfp8_quantize_act: Y = bf16((X_fp8 . W_fp8^T) * x_scale (x) w_scale).
 * Lets the GEMM be timed and checked without the quantize pass.  path is
 * AUTO, TILED, SPLITK or PAIR (FUSED is taken as SPLITK: the codes are
 * given).  `workspace` (mfp8_gemm_workspace_bytes(M, N, K) bytes) is used
 * only when N % 8 != 0; otherwise it may be NULL with 0 bytes. */
MFP8_API mfp8_status mfp8_gemm(const void* X_fp8, const float* x_scale, int64_t M, int64_t K,
                      const void* W_fp8, const float* w_scale, int64_t N,
                      void* Y_bf16, void* workspace, size_t workspace_bytes,
                      int path, void* stream);

/* The activation quantization fused into its producer: RMSNorm, the
 * producer of the q/k/v and gate/up inputs ("MOSS-VL-Realtime-FP8
 * mixed-precision strategy" article: the norms stay in high precision and
 * feed the FP8 Linears).  Per token row of X [M, K] (bf16):
 *   y = bf16(x * r * gamma),  r = 1 / sqrt(mean(x^2) + eps)   (fp32)
 *   x_scale[m], X_fp8[m, :] = the mfp8_quantize_act codes of the bf16 y
 * so the codes and scales are bit-identical to mfp8_quantize_act on the
 * bf16 y that Y_bf16 receives (Y_bf16 may be NULL when only the codes are
 * wanted).  The codes feed mfp8_gemm.  The pages fix neither eps nor the
 * norm's rounding; y is within one bf16 unit of the exact value.
 *   gamma_bf16 [K]; X_fp8 [M, K] u8; x_scale [M] fp32; caller-owned,
 *   16-byte aligned, outputs not overlapping inputs.  K % 16 == 0 and
 *   K <= 16384 (else MFP8_ERR_UNSUPPORTED_SHAPE); 0 <= eps <= 1
 *   (else MFP8_ERR_INVALID_ARG); M == 0 is a no-op. */
MFP8_API mfp8_status mfp8_rmsnorm_quantize(const void* X_bf16, const void* gamma_bf16, float eps,
                                  int64_t M, int64_t K, void* Y_bf16, void* X_fp8, float* x_scale,
                                  void* stream);

/* The same for the gated MLP activation before down_proj, on the packed
 * gate_up_proj output ("MOSS-VL quantization README", packed modules):
 * GU_bf16 [M, 2I] holds gate in columns 0 .. I-1 and up in I .. 2I-1;
 *   y = bf16(silu(gate) * up),  silu(v) = v / (1 + e^-v)   (fp32; for
 *   v < 0 as v e^v / (1 + e^v), which cannot overflow)
 * and X_fp8 [M, I], x_scale [M] are the mfp8_quantize_act codes and scales of
 * y.  The pages do not name the activation: SiLU(gate) * up is this
 * library's reading.  Y_bf16 [M, I] optional; I % 16 == 0, I <= 16384. */
MFP8_API mfp8_status mfp8_silu_mul_quantize(const void* GU_bf16, int64_t M, int64_t I, void* Y_bf16,
                                   void* X_fp8, float* x_scale, void* stream);

/* FP8 e4m3 KV cache.  "MOSS-VL quantization README", SGLang paragraph
 * (--kv-cache-dtype fp8_e4m3); the pages give only the flag, so the scale
 * rule is this library's reading: a K or V tensor [T tokens][H heads][D]
 * (bf16, row-major, contiguous) gets one fp32 scale per (token, head) row of
 * D values, s = fl32(max |x| / 448) raised to FLT_MIN, and codes
 * e4m3(fl32(x / s)) with round-to-nearest-even and saturation: the
 * activation rule of mfp8_quantize_act, so the bytes are identical to
 * mfp8_quantize_act on the [T*H, D] view.
 *   KV_fp8 [T][H][D] u8 and kv_scale [T][H] fp32 are written; caller-owned,
 *   16-byte aligned, not overlapping the input.  D % 16 == 0 (else
 *   MFP8_ERR_UNSUPPORTED_SHAPE); T == 0 is a no-op. */
MFP8_API mfp8_status mfp8_kv_quantize(const void* KV_bf16, int64_t T, int64_t H, int64_t D,
                             void* KV_fp8, float* kv_scale, void* stream);

/* The inverse of mfp8_kv_quantize for reading the cache:
 * KV_bf16[t][h][d] = bf16(fl32(dec(KV_fp8[t][h][d]) * kv_scale[t][h])), the
 * product rounded to fp32, then to bf16 (round to nearest even).  Same
 * shapes, alignment and errors as mfp8_kv_quantize; KV_bf16 must not overlap
 * the codes or scales. */
MFP8_API mfp8_status mfp8_kv_dequantize(const void* KV_fp8, const float* kv_scale, int64_t T, int64_t H,
                               int64_t D, void* KV_bf16, void* stream);

/* ------------------------------------------------------ INT8 KV cache -- */

/* The INT8 KV cache ("MOSS-VL quantization README", KV8 section: the hqq
 * backend with nbits 8, axis_key = axis_value = 0, q_group_size 64 and
 * residual_length 128; the history lives quantized and the bf16 tail of the
 * latest positions is appended when it is read).  The section gives these
 * settings, not HQQ's optimizer; the readings below are this library's.
 *
 * A K or V tensor of one layer is [T tokens][H heads][D] bf16, C = H * D
 * columns.  A group is 64 consecutive tokens of one column (axis 0 = the
 * token axis); each group has one scale s and one zero point z, fp32, from
 * the asymmetric min-max fit, every step rounded to nearest even:
 *   range = max - min;  s = max(range / 255, FLT_MIN) if range > 0, else
 *   max(|min|, FLT_MIN);  z = rint(-min / s) (+0 for zero);
 *   q = min(255, max(0, rint(x / s + z)));
 *   dequantized value = bf16((q - z) * s).
 * Values must be finite and max - min finite in fp32.  The latest 128
 * positions stay bf16; older ones are quantized in whole groups
 * (mfp8_kv8_history_tokens). */

/* Quantize T tokens (T a multiple of 64) into codes and fits.
 * KV_bf16 [T][H][D] device bf16; KV_u8 [T][H][D] device u8 codes (written);
 * kv_scale, kv_zero [T/64][H][D] device fp32 (written).  To append to a
 * history of Tq tokens pass KV_u8 + Tq*H*D, kv_scale + (Tq/64)*H*D and
 * kv_zero + (Tq/64)*H*D.  Asynchronous on `stream`; the caller owns every
 * buffer.  Errors: MFP8_ERR_INVALID_ARG (negative size, null pointer,
 * overlapping buffers), MFP8_ERR_UNSUPPORTED_SHAPE (T % 64 != 0, H or D
 * zero, D % 16 != 0, a size above 2^31 - 1 or T*H*D above 2^40),
 * MFP8_ERR_MISALIGNED (a pointer not 16-byte aligned).  T = 0 is a no-op. */
MFP8_API mfp8_status mfp8_kv8_quantize(const void* KV_bf16, int64_t T, int64_t H, int64_t D, void* KV_u8,
                                       float* kv_scale, float* kv_zero, void* stream);

/* Read the cache back: out [Tq + Tr][H][D] device bf16 (written) holds the
 * Tq history tokens (Tq a multiple of 64) dequantized, then the Tr tail
 * tokens tail_bf16 [Tr][H][D] copied unchanged.  KV_u8, kv_scale, kv_zero
 * as written by mfp8_kv8_quantize (may be null when Tq = 0; tail_bf16 may be
 * null when Tr = 0).  out must not overlap the inputs.  Same errors as
 * mfp8_kv8_quantize, with Tq % 64 != 0 unsupported.  Tq + Tr = 0 is a
 * no-op. */
MFP8_API mfp8_status mfp8_kv8_read(const void* KV_u8, const float* kv_scale, const float* kv_zero, int64_t Tq,
                                   const void* tail_bf16, int64_t Tr, int64_t H, int64_t D, void* out_bf16,
                                   void* stream);

/* Host only: how many of a cache's T positions are held quantized.  The
 * latest 128 stay bf16 and older ones are quantized in whole groups of 64:
 * 64 * floor((T - 128) / 64) for T >= 128, 0 for 0 <= T < 128, -1 for
 * T < 0.  After appending n positions to a cache of T, the oldest
 * mfp8_kv8_history_tokens(T + n) - mfp8_kv8_history_tokens(T) tail
 * positions move into the history. */
MFP8_API int64_t mfp8_kv8_history_tokens(int64_t T);

/* Diagnostic: checks the quantizer's divide-free arithmetic against IEEE
 * divides.  The scale fl32(absmax / 448) of every absmax (0 and each positive
 * finite bf16) is computed as a corrected quotient by 7 times 2^-6, and each
 * code rounds x / s with one multiply by the correctly rounded reciprocal,
 * one fused multiply-add for the residual and one for the corrected quotient;
 * both are compared with the divide for every bf16 x with |x| <= absmax,
 * both signs.  out_u64x2 [2] device uint64, written: [0] the number of
 * scales and codes that differ (0 when the arithmetic is exact), [1] one of
 * them as (absmax_bits << 16) | x_bits (x_bits 0xffff: the scale).  Read it
 * after synchronising `stream`. */
MFP8_API mfp8_status mfp8_debug_quantize_check(void* out_u64x2, void* stream);

/* Diagnostic: checks the INT8 KV cache's divide-free codes against IEEE
 * divides.  Each of n_scale_pairs blocks draws two groups from a hash of
 * (seed, block): a random finite bf16 minimum and a maximum that is either
 * another random finite bf16 or a few bf16 steps above it.  Each group is
 * fitted as mfp8_kv8_quantize fits it, and every finite bf16 x between its
 * minimum and maximum is coded both ways, q = min(255, max(0, rint(x / s +
 * z))); groups whose scale is below 2^-64 (coded by the divide in the
 * kernel) are skipped.  out_u64x2 [2] device uint64, zeroed then written:
 * [0] the number of codes that differ, [1] one of them as (scale_bits << 32)
 * | x_bits.  n_scale_pairs in [1, 2^31 - 1].  Read it after synchronising
 * `stream`. */
MFP8_API mfp8_status mfp8_debug_kv8_code_check(void* out_u64x2, int64_t n_scale_pairs, uint32_t seed, void* stream);

/* Diagnostic: encode n fp32 values with the device's e4m3 conversion (the
 * one the quantize kernels use).  in [n] fp32, out [n] codes.  Used to check
 * the hardware conversion against the oracle on every fp32 bit pattern. */
MFP8_API mfp8_status mfp8_e4m3_encode_f32(const float* in, int64_t n, uint8_t* out, void* stream);

/* Diagnostic: one kernel waits on a barrier that nothing releases, with a
 * bound of `timeout_us` microseconds (at most 100000), then records
 * MFP8_ERR_TIMEOUT in the status word and returns.  Exercises the
 * device-error path without faulting or hanging the GPU. */
MFP8_API mfp8_status mfp8_debug_bounded_wait(int64_t timeout_us, void* stream);

/* Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns MFP8_OK, MFP8_ERR_TIMEOUT, or MFP8_ERR_CUDA if the
 * synchronisation itself failed. */
MFP8_API mfp8_status mfp8_get_device_status(void* stream);

/* Static description of a status code (never NULL). */
MFP8_API const char* mfp8_status_string(mfp8_status status);

/* Library version, as major * 10000 + minor * 100 + patch. */
MFP8_API int mfp8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MFP8_H */
