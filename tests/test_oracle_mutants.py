"""Plant a mistake in a copy of the CPU oracle and check that a pin catches it.

Each mutant is a textual edit of ``oracle/mfp8_oracle.c`` compiled into a
temporary library; the real oracle is untouched.  A mutant that every pin
accepts would mean the pins cannot see that class of mistake.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins as P
from oracle import build as obuild

MUTANTS = {
    # rounding: truncate instead of nearest-even
    "truncate": ("double steps = nearbyint(ldexp(a, -q));", "double steps = trunc(ldexp(a, -q));"),
    # rounding: ties away from zero instead of ties to even
    "ties_away": ("double steps = nearbyint(ldexp(a, -q));", "double steps = round(ldexp(a, -q));"),
    # exponent bias off by one in the decoder
    "bias": ("else mag = ldexp(1.0 + m / 8.0, e - 7);", "else mag = ldexp(1.0 + m / 8.0, e - 8);"),
    # scale constant wrong
    "scale_240": ("float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    # multiply instead of divide when quantizing
    "mul_not_div": ("float q = orc_bf16_to_f32(row[k]) / sr;", "float q = orc_bf16_to_f32(row[k]) * sr;"),
    # quotient by reciprocal multiplication: fl32(x * fl32(1/s)) rounds
    # differently from fl32(x / s) for some x
    "recip_mul": ("float q = orc_bf16_to_f32(row[k]) / sr;", "float q = orc_bf16_to_f32(row[k]) * (1.0f / sr);"),
    # scale by reciprocal multiplication: fl32(a * fl32(1/448)) != fl32(a / 448)
    # for about half the bf16 absmax values
    "scale_recip": ("float s = amax / 448.0f;", "float s = amax * (1.0f / 448.0f);"),
    # sign of zero dropped
    "zero_sign": ("if (r == 0.0) return sign;", "if (r == 0.0) return 0;"),
    # transposed output index
    "transpose_out": ("if (y_ref) y_ref[m * N + n] = dot * sc;", "if (y_ref) y_ref[n * M + m] = dot * sc;"),
    # a dropped term in the dot product
    "dropped_term": ("for (k = 0; k < K; ++k) {\n                    double p", "for (k = 1; k < K; ++k) {\n                    double p"),
    # the activation scale is not applied
    "no_sa": ("double sc = (double)s_a[m] * (double)s_w[n];", "double sc = (double)s_w[n];"),
    # bf16 by truncation instead of round-to-nearest-even
    "bf16_truncate": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;",
                      "if (lower > 0xFFFFu) upper += 1u;"),
    # bf16 ties away from zero
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;",
                       "if (lower >= 0x8000u) upper += 1u;"),
    # KV dequantize without the scale
    "kv_no_scale": ("float v = (float)orc_e4m3_decode(Q[r * D + k]) * s[r];",
                    "float v = (float)orc_e4m3_decode(Q[r * D + k]);"),
    # RMSNorm over the sum instead of the mean
    "rms_sum": ("double r = 1.0 / sqrt(ss / (double)K + eps);", "double r = 1.0 / sqrt(ss + eps);"),
    # RMSNorm without the gain
    "rms_no_gain": ("y[m * K + k] = (double)orc_bf16_to_f32(row[k]) * r * (double)orc_bf16_to_f32(g[k]);",
                    "y[m * K + k] = (double)orc_bf16_to_f32(row[k]) * r;"),
    # SiLU with the wrong sign in the exponent
    "silu_sign": ("y[m * I + k] = gv / (1.0 + exp(-gv)) * uv;", "y[m * I + k] = gv / (1.0 + exp(gv)) * uv;"),
    # gate and up swapped
    "silu_swap": ("double gv = (double)orc_bf16_to_f32(GU[m * 2 * I + k]);",
                  "double gv = (double)orc_bf16_to_f32(GU[m * 2 * I + I + k]);"),
    # INT8 KV cache: another divisor than 255 for the scale
    "kv8_div256": ("        s = range / 255.0f;", "        s = range / 256.0f;"),
    # INT8 KV cache: zero point with the wrong sign
    "kv8_zero_sign": ("*z_out = rintf(-mn / s) + 0.0f;", "*z_out = rintf(mn / s) + 0.0f;"),
    # INT8 KV cache: ties away from zero
    "kv8_ties_away": ("    float q = rintf(t);", "    float q = roundf(t);"),
    # INT8 KV cache: truncation instead of rounding
    "kv8_trunc": ("    float q = rintf(t);", "    float q = truncf(t);"),
    # INT8 KV cache: groups along head_dim instead of the tokens
    "kv8_axis": ("float v = orc_bf16_to_f32(x[t * C]);", "float v = orc_bf16_to_f32(x[t]);"),
    # INT8 KV cache: a constant group with scale 1
    "kv8_const": ("        s = fabsf(mn);", "        s = 1.0f;"),
    # INT8 KV cache: dequantize adds the zero point
    "kv8_read_sign": ("const float d = (float)Q[i] - zero[gc];", "const float d = (float)Q[i] + zero[gc];"),
    # INT8 KV cache: the tail written over the history
    "kv8_tail_place": ("memcpy(out + Tq * C, resid,", "memcpy(out, resid,"),
    # INT8 KV cache: partial groups quantized
    "kv8_partial_group": ("return T < 128 ? 0 : 64 * ((T - 128) / 64);", "return T < 128 ? 0 : T - 128;"),
    # saturation missing (values above 448 become NaN)
    "no_satfinite": ("if (a >= 448.0) return (uint8_t)(sign | 0x7E);", "if (a >= 464.0) return (uint8_t)(sign | 0x7F);"),
}


@pytest.fixture(scope="module")
def src():
    with open(obuild.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, src, tmp_path):
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    c = tmp_path / f"mut_{name}.c"
    c.write_text(src.replace(old, new))
    so = tmp_path / f"libmut_{name}.so"
    subprocess.run(["gcc", *obuild.CFLAGS, str(c), "-o", str(so), "-lm"], check=True)
    mut = oracle.Oracle(str(so))
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(mut)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
