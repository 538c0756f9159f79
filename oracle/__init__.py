"""CPU oracle for the FP8_DYNAMIC quantized Linear.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the CUDA library and its Python binding) never imports it, and this
package never imports the product.

The arithmetic lives in ``mfp8_oracle.c`` (plain C, fp64/int64, OpenMP); this
module only marshals numpy arrays into it.  What each function follows:

* ``e4m3_encode`` / ``e4m3_decode`` - the float8_e4m3fn format named by the
  "MOSS-VL quantization README", FP8-Dynamic recipe section, and described as
  "4 exponent bits, 3 mantissa bits" in the "MOSS-VL-Realtime-FP8
  mixed-precision strategy" article, section "252 个主力 Linear 层为什么用
  FP8 E4M3".  Rounding (nearest-even) and saturation to 448 are this
  project's reading; the pages state neither.
* ``quantize_rows`` - one scale per row: per output channel for weights
  ("channel-wise static"), per token for activations ("per-token dynamic"),
  same README section.  Scale = fl32(absmax / 448), floored at FLT_MIN
  (reading; the pages give no formula).
* ``linear_ref`` - exact fp64 contraction of the decoded codes, rescaled by
  s_a[m] * s_w[n]; ``dot_int64`` is the same contraction in integers.
* ``within_tolerance`` - the acceptance rule for BF16 outputs:
  |y - y_ref| <= 2^-7 |y_ref| + 1e-5 * s_abs.
* ``kv_quantize`` / ``kv_dequantize`` - the FP8 e4m3 KV cache that the
  README's SGLang paragraph turns on with --kv-cache-dtype fp8_e4m3 (the
  pages give only the flag).  Reading: one scale per (token, head) row of a
  [T, H, D] tensor by the activation rule; dequantize = bf16(fl32(dec * s)).
  ``f32_to_bf16`` is round-to-nearest-even on the dropped 16 bits.
* ``kv8_quantize`` / ``kv8_read`` / ``kv8_history_tokens`` - the INT8 KV
  cache of the README's KV8 section (hqq backend, nbits 8, q_group_size 64,
  axis 0, residual_length 128; the pages do not give HQQ's optimizer).
  Readings: groups of 64 consecutive tokens per (head, channel) column of a
  [T, H, D] tensor; the asymmetric min-max fit with an integer zero point in
  fp32 (each rounding stated in the C source); the read dequantizes the
  history and appends the bf16 tail; the latest 128 positions stay bf16 and
  older ones are quantized in whole groups of 64.
* ``rmsnorm`` / ``silu_mul`` - the producers of the quantized Linears'
  inputs, exactly in fp64: RMSNorm before q/k/v and gate/up (named by the
  "MOSS-VL-Realtime-FP8 mixed-precision strategy" article, norms kept in high
  precision), and SiLU(gate) * up on the packed gate_up output before down
  (the activation is not named on the pages: a reading).
"""
import ctypes

import numpy as np

from . import build as _build


class Oracle:
    """ctypes view of one build of ``mfp8_oracle.c`` (the default build, or a
    copy compiled by a test that plants a mistake in it)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode_array.argtypes = [P, i64, P]
        L.orc_e4m3_decode_array.argtypes = [P, i64, P]
        L.orc_e4m3_encode_bits_range.argtypes = [ctypes.c_uint64, ctypes.c_uint64, P]
        L.orc_row_scale.restype = ctypes.c_float
        L.orc_row_scale.argtypes = [P, i64]
        L.orc_quantize_rows.argtypes = [P, i64, i64, P, P]
        L.orc_linear_ref.argtypes = [P, P, i64, P, P, i64, i64, P, P]
        L.orc_dot_int64.argtypes = [P, i64, P, i64, i64, P]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_kv_quantize.argtypes = [P, i64, i64, i64, P, P]
        L.orc_kv_dequantize.argtypes = [P, P, i64, i64, i64, P]
        L.orc_rmsnorm.argtypes = [P, P, i64, i64, ctypes.c_double, P]
        L.orc_kv8_quantize.argtypes = [P, i64, i64, i64, P, P, P]
        L.orc_kv8_read.argtypes = [P, P, P, i64, P, i64, i64, i64, P]
        L.orc_kv8_history_tokens.restype = i64
        L.orc_kv8_history_tokens.argtypes = [i64]
        L.orc_silu_mul.argtypes = [P, i64, i64, P]
        self.L = L
        self.path = path

    def num_threads(self) -> int:
        return int(self.L.orc_num_threads())

    def e4m3_decode(self, codes):
        codes = _c(codes, np.uint8)
        out = np.empty(codes.shape, dtype=np.float64)
        self.L.orc_e4m3_decode_array(_ptr(codes), codes.size, _ptr(out))
        return out

    def e4m3_encode(self, values):
        values = _c(values, np.float32)
        out = np.empty(values.shape, dtype=np.uint8)
        self.L.orc_e4m3_encode_array(_ptr(values), values.size, _ptr(out))
        return out

    def e4m3_encode_bits_range(self, lo: int, hi: int):
        """Codes of every fp32 bit pattern in [lo, hi)."""
        out = np.empty(hi - lo, dtype=np.uint8)
        self.L.orc_e4m3_encode_bits_range(ctypes.c_uint64(lo), ctypes.c_uint64(hi), _ptr(out))
        return out

    def row_scale(self, row_bits) -> np.float32:
        row_bits = _c(row_bits, np.uint16)
        return np.float32(self.L.orc_row_scale(_ptr(row_bits), row_bits.size))

    def quantize_rows(self, x_bits):
        """x_bits: uint16 [R, K] holding bf16 bit patterns.
        Returns (codes uint8 [R, K], scales float32 [R])."""
        x_bits = _c(x_bits, np.uint16)
        R, K = x_bits.shape
        q = np.empty((R, K), dtype=np.uint8)
        s = np.empty((R,), dtype=np.float32)
        self.L.orc_quantize_rows(_ptr(x_bits), R, K, _ptr(q), _ptr(s))
        return q, s

    def linear_ref(self, x8, s_a, w8, s_w, want_abs: bool = True):
        """Exact reference of the rescaled FP8 contraction.
        x8 uint8 [M,K], s_a f32 [M], w8 uint8 [N,K], s_w f32 [N].
        Returns (y_ref f64 [M,N], s_abs f64 [M,N] or None)."""
        x8 = _c(x8, np.uint8)
        w8 = _c(w8, np.uint8)
        s_a = _c(s_a, np.float32)
        s_w = _c(s_w, np.float32)
        M, K = x8.shape
        N, K2 = w8.shape
        assert K == K2 and s_a.shape == (M,) and s_w.shape == (N,)
        y = np.empty((M, N), dtype=np.float64)
        sa = np.empty((M, N), dtype=np.float64) if want_abs else None
        self.L.orc_linear_ref(_ptr(x8), _ptr(s_a), M, _ptr(w8), _ptr(s_w), N, K,
                              _ptr(y), _ptr(sa) if want_abs else None)
        return y, sa

    def f32_to_bf16(self, values):
        """bf16 bit patterns of fp32 values (round to nearest even)."""
        values = _c(values, np.float32)
        return np.array([self.L.orc_f32_to_bf16(float(v)) for v in values.ravel()],
                        dtype=np.uint16).reshape(values.shape)

    def kv_quantize(self, kv_bits):
        """kv_bits: uint16 bf16 patterns [T, H, D] -> (codes u8 [T, H, D], scales f32 [T, H])."""
        kv_bits = _c(kv_bits, np.uint16)
        T, H, D = kv_bits.shape
        q = np.empty((T, H, D), dtype=np.uint8)
        s = np.empty((T, H), dtype=np.float32)
        self.L.orc_kv_quantize(_ptr(kv_bits), T, H, D, _ptr(q), _ptr(s))
        return q, s

    def kv_dequantize(self, codes, scales):
        """codes u8 [T, H, D], scales f32 [T, H] -> bf16 bit patterns [T, H, D]."""
        codes = _c(codes, np.uint8)
        scales = _c(scales, np.float32)
        T, H, D = codes.shape
        out = np.empty((T, H, D), dtype=np.uint16)
        self.L.orc_kv_dequantize(_ptr(codes), _ptr(scales), T, H, D, _ptr(out))
        return out

    def kv8_quantize(self, kv_bits):
        """kv_bits uint16 [T, H, D], T % 64 == 0 -> (codes u8 [T, H, D],
        scale f32 [T/64, H, D], zero f32 [T/64, H, D])."""
        kv_bits = _c(kv_bits, np.uint16)
        T, H, D = kv_bits.shape
        if T % 64:
            raise ValueError("kv8_quantize: T must be a multiple of 64")
        q = np.empty((T, H, D), dtype=np.uint8)
        sc = np.empty((T // 64, H, D), dtype=np.float32)
        z = np.empty((T // 64, H, D), dtype=np.float32)
        self.L.orc_kv8_quantize(_ptr(kv_bits), T, H, D, _ptr(q), _ptr(sc), _ptr(z))
        return q, sc, z

    def kv8_read(self, codes, scale, zero, resid_bits):
        """Dequantized codes [Tq, H, D] followed by the bf16 residual [Tr, H, D] -> bf16 bits [Tq + Tr, H, D]."""
        codes, scale, zero = _c(codes, np.uint8), _c(scale, np.float32), _c(zero, np.float32)
        resid_bits = _c(resid_bits, np.uint16)
        Tq, H, D = codes.shape
        Tr = resid_bits.shape[0]
        out = np.empty((Tq + Tr, H, D), dtype=np.uint16)
        self.L.orc_kv8_read(_ptr(codes), _ptr(scale), _ptr(zero), Tq, _ptr(resid_bits), Tr, H, D, _ptr(out))
        return out

    def kv8_history_tokens(self, T):
        return int(self.L.orc_kv8_history_tokens(int(T)))

    def rmsnorm(self, x_bits, g_bits, eps):
        """x_bits uint16 [M, K], g_bits uint16 [K] -> fp64 [M, K], exact."""
        x_bits = _c(x_bits, np.uint16)
        g_bits = _c(g_bits, np.uint16)
        M, K = x_bits.shape
        y = np.empty((M, K), dtype=np.float64)
        self.L.orc_rmsnorm(_ptr(x_bits), _ptr(g_bits), M, K, float(eps), _ptr(y))
        return y

    def silu_mul(self, gu_bits):
        """gu_bits uint16 [M, 2I] (gate, then up) -> fp64 [M, I], exact."""
        gu_bits = _c(gu_bits, np.uint16)
        M, I2 = gu_bits.shape
        y = np.empty((M, I2 // 2), dtype=np.float64)
        self.L.orc_silu_mul(_ptr(gu_bits), M, I2 // 2, _ptr(y))
        return y

    def dot_int64(self, x8, w8):
        """Integer form of the contraction: sum_k (2^9 dec(x)) * (2^9 dec(w))."""
        x8 = _c(x8, np.uint8)
        w8 = _c(w8, np.uint8)
        M, K = x8.shape
        N, _ = w8.shape
        out = np.empty((M, N), dtype=np.int64)
        self.L.orc_dot_int64(_ptr(x8), M, _ptr(w8), N, K, _ptr(out))
        return out


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def e4m3_decode(codes):
    return default().e4m3_decode(codes)


def e4m3_encode(values):
    return default().e4m3_encode(values)


def e4m3_encode_bits_range(lo: int, hi: int):
    return default().e4m3_encode_bits_range(lo, hi)


def row_scale(row_bits):
    return default().row_scale(row_bits)


def quantize_rows(x_bits):
    return default().quantize_rows(x_bits)


def linear_ref(x8, s_a, w8, s_w, want_abs: bool = True):
    return default().linear_ref(x8, s_a, w8, s_w, want_abs)


def kv_quantize(kv_bits):
    return default().kv_quantize(kv_bits)


def kv_dequantize(codes, scales):
    return default().kv_dequantize(codes, scales)


def f32_to_bf16(values):
    return default().f32_to_bf16(values)


def rmsnorm(x_bits, g_bits, eps):
    return default().rmsnorm(x_bits, g_bits, eps)


def kv8_quantize(kv_bits):
    return default().kv8_quantize(kv_bits)


def kv8_read(codes, scale, zero, resid_bits):
    return default().kv8_read(codes, scale, zero, resid_bits)


def kv8_history_tokens(T):
    return default().kv8_history_tokens(T)


def silu_mul(gu_bits):
    return default().silu_mul(gu_bits)


def dot_int64(x8, w8):
    return default().dot_int64(x8, w8)


def bf16_bits_to_f32(bits):
    bits = _c(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


TOL_REL = 2.0 ** -7
TOL_ABS_FRAC = 1e-5


def tolerance(y_ref, s_abs):
    return TOL_REL * np.abs(y_ref) + TOL_ABS_FRAC * s_abs


def within_tolerance(y, y_ref, s_abs):
    """Element mask of |y - y_ref| <= 2^-7 |y_ref| + 1e-5 s_abs."""
    y = np.asarray(y, dtype=np.float64)
    return np.abs(y - y_ref) <= tolerance(y_ref, s_abs)
