"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with what the format definition, a library
implementation of float8_e4m3fn, exact rational arithmetic or a closed form
fixes.  ``test_oracle_pins.py`` runs them on the oracle; ``test_oracle_mutants.py``
runs them on copies of the oracle with a planted mistake and expects a failure.
"""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FLT_MIN = np.float32(np.finfo(np.float32).tiny)


def lib_decode(codes):
    """float8_e4m3fn decode by ml_dtypes (a library implementation)."""
    return np.asarray(codes, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def lib_encode(values):
    """float8_e4m3fn encode by ml_dtypes: round to nearest even; it does not
    saturate, so only compare for |v| <= 464."""
    return np.asarray(values, np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def bf16_bits(x_f32):
    """Round fp32 values to bf16 with torch and return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ codec --

def pin_decode_table(o):
    codes = np.arange(256, dtype=np.uint8)
    d = o.e4m3_decode(codes)
    ref = lib_decode(codes)
    nan = np.isnan(d)
    assert np.array_equal(nan, np.isnan(ref)), "NaN codes differ from the library"
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}, "NaN must be S.1111.111 only"
    assert np.array_equal(d[~nan], ref[~nan]), "decoded values differ from the library"
    assert not np.isinf(d).any(), "e4m3fn has no infinities"
    assert np.nanmax(d) == 448.0 and np.nanmin(d) == -448.0
    assert d[0x01] == 2.0 ** -9 and d[0x08] == 2.0 ** -6 and d[0x38] == 1.0
    assert (~nan).sum() == 254


def pin_roundtrip(o):
    codes = np.arange(256, dtype=np.uint8)
    d = o.e4m3_decode(codes).astype(np.float32)
    back = o.e4m3_encode(d)
    finite = ~np.isnan(d)
    assert np.array_equal(back[finite], codes[finite]), "decode -> encode is not the identity"
    assert set(back[~finite].tolist()) <= {0x7F, 0xFF}


def read_rounding_cases():
    cases = []
    with open(os.path.join(GOLDEN, "e4m3_rounding_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            v, code = tok[0], int(tok[1], 16)
            if v.lstrip("-").startswith("0x"):
                val = float.fromhex(v)
            else:
                val = float(v)
            cases.append((np.float32(val), code, line))
    return cases


def pin_rounding_cases(o):
    cases = read_rounding_cases()
    vals = np.array([c[0] for c in cases], dtype=np.float32)
    got = o.e4m3_encode(vals)
    for (v, code, line), g in zip(cases, got):
        if np.isnan(v):
            assert (g & 0x7F) == 0x7F, line
        else:
            assert g == code, f"{line}: got 0x{g:02x}"


def pin_encode_vs_library(o, n=400_000, seed=11):
    rng = np.random.default_rng(seed)
    # magnitudes log-uniform over the whole e4m3 range and below it
    mag = np.exp2(rng.uniform(-14.0, math.log2(464.0), n)).astype(np.float32)
    v = np.where(rng.random(n) < 0.5, -mag, mag).astype(np.float32)
    # every midpoint between adjacent finite codes, and one fp32 ulp either side
    d = np.unique(lib_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((d[1:] + d[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(0))])
    v = np.concatenate([v, near, -near]).astype(np.float32)
    v = v[np.abs(v) <= 464.0]
    got = o.e4m3_encode(v)
    ref = lib_encode(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches vs library, first {v[bad[:4]]}"
    tv = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, tv), "mismatch vs torch float8_e4m3fn"


def pin_saturation(o):
    big = np.array([448.0, 448.5, 463.99, 464.0, 464.01, 500.0, 1e5, 3.0e38, np.inf],
                   dtype=np.float32)
    assert (o.e4m3_encode(big) == 0x7E).all()
    assert (o.e4m3_encode(-big) == 0xFE).all()
    assert (o.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F) == 0x7F


# ----------------------------------------------------------------- scales --

def _random_rows(rng, R, K, lo=-20, hi=20):
    x = rng.standard_normal((R, K)).astype(np.float32)
    x *= np.exp2(rng.uniform(lo, hi, (R, 1))).astype(np.float32)
    return bf16_bits(x)


def pin_scale_invariants(o, seed=5):
    rng = np.random.default_rng(seed)
    R, K = 64, 257
    xb = _random_rows(rng, R, K)
    x = bits_to_f32(xb).astype(np.float64)
    q, s = o.quantize_rows(xb)
    dq = o.e4m3_decode(q)
    # every code finite and within +-448
    assert not np.isnan(dq).any() and np.abs(dq).max() <= 448.0
    # a row's largest magnitude maps to +-448
    j = np.argmax(np.abs(x), axis=1)
    top = q[np.arange(R), j]
    assert np.all((top == 0x7E) | (top == 0xFE)), "absmax element must encode to +-448"
    # scale is the absmax over 448, up to one fp32 rounding
    amax = np.abs(x).max(axis=1)
    assert np.all(np.abs(s.astype(np.float64) * 448.0 - amax) <= amax * 2.0 ** -23)
    # reconstruction: half a 3-bit-mantissa step (2^-4 relative) in the
    # normal range, half the subnormal step (2^-10 * s) below it
    err = np.abs(dq * s[:, None] - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s[:, None].astype(np.float64))
    assert np.all(err <= bound * (1 + 2.0 ** -20)), "reconstruction error too large"
    # a scale depends on its own row only (data-free, no calibration set)
    perm = rng.permutation(R)
    q2, s2 = o.quantize_rows(xb[perm])
    assert np.array_equal(s2, s[perm]) and np.array_equal(q2, q[perm])
    # all-zero row: floor scale, all codes zero (sign kept)
    z = np.zeros((2, 32), np.uint16)
    z[1, :] = 0x8000  # -0.0
    qz, sz = o.quantize_rows(z)
    assert np.all(sz == FLT_MIN)
    assert np.all(qz[0] == 0x00) and np.all(qz[1] == 0x80)
    # tiny rows (bf16 subnormals) do not divide by zero and still reach 448
    t = np.zeros((1, 16), np.uint16)
    t[0, 3] = 0x0001  # smallest positive bf16 subnormal
    t[0, 5] = 0x8001
    qt, st = o.quantize_rows(t)
    assert st[0] == FLT_MIN
    assert qt[0, 3] != 0 and qt[0, 5] != 0 and np.all(np.delete(qt[0], [3, 5]) == 0)


def _ieee_scale(amax_f32):
    """fl32(amax / 448) by numpy's IEEE fp32 divide (correctly rounded),
    raised to FLT_MIN: the scale reading of the "MOSS-VL quantization README"
    FP8-Dynamic recipe (per-channel / per-token scale = absmax / 448)."""
    s = np.asarray(amax_f32, np.float32) / np.float32(448.0)
    # the same quotient through an fp64 divide rounded once to fp32 (an fp32
    # quotient rounded via fp64 is still correctly rounded: 53 >= 2*24 + 2)
    assert np.array_equal(s, (np.asarray(amax_f32, np.float64) / 448.0).astype(np.float32))
    return np.maximum(s, FLT_MIN).astype(np.float32)


def _ieee_codes(x_f32, s_f32):
    """e4m3(fl32(x / s)): numpy's fp32 divide, then the library encoder
    (ml_dtypes, round to nearest even) after saturating to +-448."""
    q = np.asarray(x_f32, np.float32) / np.asarray(s_f32, np.float32)
    return lib_encode(np.clip(q, np.float32(-448.0), np.float32(448.0)))


def _divide_sensitive_rows(rng, n_rows=48, K=24):
    """bf16 rows chosen so that a plausible rounding slip changes the bytes:
      - rows whose absmax a has fl32(a * fl32(1/448)) != fl32(a / 448), so a
        scale taken by reciprocal multiplication differs from the divide's;
      - rows holding values x with e4m3(fl32(x * fl32(1/s))) !=
        e4m3(fl32(x / s)), so codes taken by reciprocal multiplication differ.
    Both sets are found here by exhaustive numpy search over bf16 values."""
    pos = np.arange(1, 0x7F80, dtype=np.uint32)                  # positive finite bf16
    a_all = (pos << 16).view(np.float32)
    s_rec = (a_all * (np.float32(1.0) / np.float32(448.0))).astype(np.float32)
    scale_sensitive = pos[(a_all / np.float32(448.0)) != s_rec]
    rows = np.zeros((n_rows, K), np.uint16)
    r = 0
    # half the rows: a scale-sensitive absmax (normal range) and smaller values
    cand = scale_sensitive[(scale_sensitive > 0x0100) & (scale_sensitive < 0x7E00)]
    for ab in rng.choice(cand, n_rows // 2, replace=False):
        lo = rng.integers(0, ab, K - 1, dtype=np.uint32)
        rows[r, 0] = ab
        rows[r, 1:] = lo | (rng.integers(0, 2, K - 1, dtype=np.uint32) << 15)
        r += 1
    # the other half: values whose quotient sits where the reciprocal form
    # rounds to a different code
    for ab in rng.permutation(np.arange(0x3000, 0x5000, dtype=np.uint32)):
        if r == n_rows:
            break
        a = np.array([ab << 16], np.uint32).view(np.float32)[0]
        s = _ieee_scale(np.array([a], np.float32))[0]
        xb = np.arange(0, ab + 1, dtype=np.uint32)
        x = (xb << 16).view(np.float32)
        d = _ieee_codes(x, s) != lib_encode(np.clip(x * (np.float32(1.0) / s), -448, 448))
        hits = xb[d]
        if hits.size == 0:
            continue
        take = hits[:K - 1]
        rows[r, 0] = ab | 0x8000  # the absmax element, negative
        rows[r, 1:1 + take.size] = take | (rng.integers(0, 2, take.size, dtype=np.uint32) << 15).astype(np.uint32)
        r += 1
    assert r == n_rows, "not enough divide-sensitive values found"
    return rows


def pin_scale_and_quotient_rounding(o, seed=12):
    """Scales and codes equal, bit for bit, the IEEE fp32 divide forms
    s = fl32(max|x| / 448) (floored at FLT_MIN) and q = e4m3(fl32(x / s)),
    computed here by numpy and ml_dtypes alone, on random rows (every
    magnitude range, tiny rows included) and on rows where a reciprocal
    multiplication would round the scale or a code differently."""
    rng = np.random.default_rng(seed)
    xb = np.concatenate([_random_rows(rng, 32, 96, -140, 60), _divide_sensitive_rows(rng)[:, :24].repeat(4, 1)])
    x = bits_to_f32(xb)
    q, s = o.quantize_rows(xb)
    s_exp = _ieee_scale(np.abs(x).max(axis=1))
    assert np.array_equal(s.view(np.uint32), s_exp.view(np.uint32)), \
        f"scales differ from fl32(amax / 448) in {(s != s_exp).sum()} rows"
    q_exp = _ieee_codes(x, s_exp[:, None])
    bad = np.argwhere(q != q_exp)
    assert bad.size == 0, f"{bad.shape[0]} codes differ from e4m3(fl32(x / s)), first at {bad[0].tolist()}"


# ------------------------------------------------------------------- GEMM --

def pin_gemm_bruteforce(o, seed=3):
    """Exact rationals on tiny shapes: the library decodes the codes, Fraction
    sums them, and the oracle's fp64 result must be that value rounded once."""
    rng = np.random.default_rng(seed)
    for (M, N, K) in [(1, 1, 16), (3, 5, 32), (6, 4, 64), (2, 7, 48)]:
        x8, sa = o.quantize_rows(_random_rows(rng, M, K, -3, 3))
        w8, sw = o.quantize_rows(_random_rows(rng, N, K, -8, -4))
        y, sabs = o.linear_ref(x8, sa, w8, sw)
        xd, wd = lib_decode(x8), lib_decode(w8)
        for m in range(M):
            for n in range(N):
                dot = sum(Fraction(float(xd[m, k])) * Fraction(float(wd[n, k])) for k in range(K))
                dab = sum(abs(Fraction(float(xd[m, k])) * Fraction(float(wd[n, k]))) for k in range(K))
                sc = Fraction(float(sa[m])) * Fraction(float(sw[n]))
                exact, exact_abs = dot * sc, dab * sc
                assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 52), (M, N, K, m, n)
                assert abs(Fraction(sabs[m, n]) - exact_abs) <= exact_abs * Fraction(1, 2 ** 52)


def pin_gemm_int_vs_fp(o, seed=4):
    """The int64 and fp64 contractions agree exactly (the sum is exact)."""
    rng = np.random.default_rng(seed)
    M, N, K = 5, 9, 4096
    x8, sa = o.quantize_rows(_random_rows(rng, M, K, 0, 1))
    w8, sw = o.quantize_rows(_random_rows(rng, N, K, -6, -5))
    ones_a = np.ones(M, np.float32)
    ones_w = np.ones(N, np.float32)
    y, _ = o.linear_ref(x8, ones_a, w8, ones_w, want_abs=False)
    di = o.dot_int64(x8, w8)
    assert np.array_equal(y * 2.0 ** 18, di.astype(np.float64)), "fp64 sum is not exact"
    # all-448 worst case, K = 12288: the largest possible sum stays exact
    K2 = 12288
    a = np.full((1, K2), 0x7E, np.uint8)
    y2, _ = o.linear_ref(a, np.ones(1, np.float32), a, np.ones(1, np.float32), want_abs=False)
    assert y2[0, 0] == 448.0 * 448.0 * K2


def pin_onehot_closed_form(o, seed=6):
    """W rows with a single non-zero entry c_n at column j_n quantize to code
    +-448 there and 0 elsewhere, so y[m,n] = dec(X8[m,j_n]) * (+-448) * s_a[m] *
    s_w[n] exactly: checks the rescale and the (m, n) index mapping."""
    rng = np.random.default_rng(seed)
    M, N, K = 3, 7, 96
    x8, sa = o.quantize_rows(_random_rows(rng, M, K, -2, 2))
    j = rng.integers(0, K, N)
    c = (rng.standard_normal(N) * 3).astype(np.float32)
    w = np.zeros((N, K), np.float32)
    w[np.arange(N), j] = c
    wb = bf16_bits(w)
    w8, sw = o.quantize_rows(wb)
    cb = bits_to_f32(wb[np.arange(N), j])
    assert np.all(o.e4m3_decode(w8[np.arange(N), j]) == np.sign(cb) * 448.0)
    y, _ = o.linear_ref(x8, sa, w8, sw)
    xd = o.e4m3_decode(x8)
    for m in range(M):
        for n in range(N):
            expect = float(Fraction(float(xd[m, j[n]])) * Fraction(float(np.sign(cb[n]) * 448.0))
                           * Fraction(float(sa[m])) * Fraction(float(sw[n])))
            assert y[m, n] == expect, (m, n)


# ------------------------------------------------------------ KV cache --

def pin_bf16_rounding(o, seed=13):
    """fp32 -> bf16 against two library conversions (torch, ml_dtypes) on
    values over the whole range, exact ties both ways, and specials."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(6000) * np.exp2(rng.uniform(-130, 127, 6000))).astype(np.float32)
    base = rng.integers(0, 1 << 15, 2000, dtype=np.uint32) << 16
    ties = np.concatenate([base | 0x8000, base | 0x18000 & 0xFFFF8000, base | 0x7FFF, base | 0x8001]).astype(np.uint32)
    ties = ties[(ties & 0x7F800000) != 0x7F800000].view(np.float32)
    v = np.concatenate([v, ties, np.float32([0.0, -0.0, np.inf, -np.inf, 3.3895314e38])]).astype(np.float32)
    got = o.f32_to_bf16(v)
    ref_t = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ref_m = v.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(got, ref_t), f"{(got != ref_t).sum()} values differ from torch"
    assert np.array_equal(got, ref_m), f"{(got != ref_m).sum()} values differ from ml_dtypes"
    n = o.f32_to_bf16(np.float32([np.nan]))[0]
    assert (n & 0x7F80) == 0x7F80 and (n & 0x7F) != 0, "NaN must stay NaN"


def pin_kv_cache(o, seed=14):
    """KV-cache quantize is the activation rule on (token, head) rows;
    dequantize equals numpy's fp32 product rounded by ml_dtypes, and, with
    power-of-two scales, the exact product."""
    rng = np.random.default_rng(seed)
    T, H, D = 7, 8, 128
    kv = _random_rows(rng, T * H, D, -6, 6).reshape(T, H, D)
    q, s = o.kv_quantize(kv)
    q2, s2 = o.quantize_rows(kv.reshape(T * H, D))
    assert np.array_equal(q.reshape(T * H, D), q2) and np.array_equal(s.reshape(-1), s2)
    # heads are independent rows: permuting them permutes codes and scales
    perm = rng.permutation(H)
    qp, sp = o.kv_quantize(kv[:, perm, :])
    assert np.array_equal(qp, q[:, perm, :]) and np.array_equal(sp, s[:, perm])
    out = o.kv_dequantize(q, s)
    prod = (lib_decode(q).astype(np.float32) * s[:, :, None]).astype(np.float32)
    ref = prod.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(out, ref), f"{(out != ref).sum()} dequantized values differ"
    # power-of-two scales: the product is exact in bf16 (codes have 4 significant bits)
    s_pow2 = np.exp2(rng.integers(-20, 20, (T, H))).astype(np.float32)
    out2 = o.kv_dequantize(q, s_pow2)
    exact = lib_decode(q) * s_pow2[:, :, None].astype(np.float64)
    assert np.array_equal(bits_to_f32(out2).astype(np.float64), exact)


# ------------------------------------------------------- INT8 KV cache --

def _kv8_grid_case(rng, H=3, D=8):
    """128 tokens x H x D values on exact grids: in every column and group,
    token values (k - m) * 2^-e for a permutation k of 64 distinct codes that
    include 0 and 255, with m in [0, 255] and e per column and group.  Every
    value has at most 8 significant bits (bf16-exact), the range is 255 * 2^-e,
    so the fit is s = 2^-e, z = m, and the codes are k: no rounding anywhere."""
    G = 2
    k = np.empty((G * 64, H, D), np.int64)
    m = rng.integers(0, 256, (G, H, D))
    e = rng.integers(-20, 30, (G, H, D))
    for g in range(G):
        for h in range(H):
            for d in range(D):
                pick = np.concatenate([[0, 255], rng.choice(np.arange(1, 255), 62, replace=False)])
                k[g * 64:(g + 1) * 64, h, d] = rng.permutation(pick)
    mt = np.repeat(m, 64, axis=0)
    et = np.repeat(e, 64, axis=0)
    x = (k - mt) * np.exp2(-et.astype(np.float64))
    xb = bf16_bits(x.astype(np.float32))
    assert np.array_equal(bits_to_f32(xb).astype(np.float64), x), "grid values must be bf16-exact"
    return xb, k, np.exp2(-e.astype(np.float64)).astype(np.float32), m.astype(np.float32)


def pin_kv8_grid(o, seed=17):
    """Closed form of the min-max fit on grid-valued groups (a group is 64
    tokens of one column): scale 2^-e, zero m, codes k, and the read returns
    the inputs exactly.  A group formed along another axis, another divisor
    than 255, a flipped zero or a wrong dequantize formula all fail it."""
    rng = np.random.default_rng(seed)
    xb, k, s_ref, z_ref = _kv8_grid_case(rng)
    q, s, z = o.kv8_quantize(xb)
    assert np.array_equal(s, s_ref), "scale is not 2^-e"
    assert np.array_equal(z, z_ref), "zero is not m"
    assert np.array_equal(q.astype(np.int64), k), f"{(q != k).sum()} codes differ from the grid index"
    out = o.kv8_read(q, s, z, np.zeros((0,) + xb.shape[1:], np.uint16))
    assert np.array_equal(out, xb), "the read does not return grid values exactly"


def pin_kv8_ties(o, seed=18):
    """Half-way values round to the even code: groups of one column hold the
    minimum -m s, the maximum (255 - m) s and values (j + 1/2) s in between
    (s a power of two, |j + 1/2| < 128, so x / s + m is exact)."""
    rng = np.random.default_rng(seed)
    H, D = 2, 4
    x = np.empty((64, H, D), np.float64)
    want = np.empty((64, H, D), np.int64)
    for h in range(H):
        for d in range(D):
            m = int(rng.integers(64, 192))
            s = 2.0 ** int(rng.integers(-10, 10))
            lo, hi = max(-m, -127), min(255 - m - 1, 126)
            j = rng.integers(lo, hi + 1, 62)
            x[:, h, d] = np.concatenate([[-m * s, (255 - m) * s], (j + 0.5) * s])
            # x / s + m = j + m + 1/2 rounds to the even one of j + m and j + m + 1
            want[:, h, d] = np.concatenate([[0, 255], np.where((j + m) % 2 == 0, j + m, j + m + 1)])
    xb = bf16_bits(x.astype(np.float32))
    assert np.array_equal(bits_to_f32(xb).astype(np.float64), x), "tie values must be bf16-exact"
    q, _, _ = o.kv8_quantize(xb)
    assert np.array_equal(q.astype(np.int64), want), f"{(q != want).sum()} half-way codes not rounded to even"


def pin_kv8_invariants(o, seed=19):
    """Random groups: the minimum takes code 0 and the maximum 254 or 255 (the
    rounded zero point shifts the grid by at most half a step), codes are
    monotone in x within a group, the read is within half a step (s / 2) plus
    half a bf16 unit of x, permuting tokens inside a group permutes the codes
    and keeps the fit, a change to one value moves only its own group, and a
    constant group (0, small, negative, huge) is reproduced exactly."""
    rng = np.random.default_rng(seed)
    T, H, D = 192, 4, 16
    x = (rng.standard_normal((T, H, D)) * np.exp2(rng.uniform(-6, 6, (1, H, D)))
         + rng.uniform(-3, 3, (1, H, D))).astype(np.float32)
    xb = bf16_bits(x)
    xf = bits_to_f32(xb).astype(np.float64)
    q, s, z = o.kv8_quantize(xb)
    qi = q.astype(np.int64)
    for g in range(T // 64):
        blk, qb = xf[g * 64:(g + 1) * 64], qi[g * 64:(g + 1) * 64]
        amin, amax = blk.argmin(axis=0), blk.argmax(axis=0)
        assert np.all(np.take_along_axis(qb, amin[None], 0) == 0), "minimum is not code 0"
        top = np.take_along_axis(qb, amax[None], 0)
        assert np.all((top == 255) | (top == 254)), "maximum is not code 254 or 255"
        order = np.argsort(blk, axis=0, kind="stable")
        assert np.all(np.diff(np.take_along_axis(qb, order, 0), axis=0) >= 0), "codes not monotone in x"
    out = bits_to_f32(o.kv8_read(q, s, z, np.zeros((0, H, D), np.uint16))).astype(np.float64)
    srep = np.repeat(s, 64, axis=0).astype(np.float64)
    bound = 0.5 * srep * (1 + 2.0 ** -12) + np.abs(out) * 2.0 ** -8  # half a step + half a bf16 unit
    assert np.all(np.abs(out - xf) <= bound), "read farther than half a step from x"
    perm = np.concatenate([rng.permutation(64) + 64 * g for g in range(T // 64)])
    qp, sp, zp = o.kv8_quantize(xb[perm])
    assert np.array_equal(qp, q[perm]) and np.array_equal(sp, s) and np.array_equal(zp, z)
    xb2 = xb.copy()
    xb2[70, 1, 3] = bf16_bits(np.float32([1e4]))[0]
    q2, s2, z2 = o.kv8_quantize(xb2)
    changed = np.argwhere(s2 != s)
    assert changed.tolist() == [[1, 1, 3]], f"one value changed groups {changed.tolist()}"
    mask = np.ones_like(q, bool)
    mask[64:128, 1, 3] = False
    assert np.array_equal(q2[mask], q[mask])
    for c in (0.0, 1.5, -3.0e-30, -7.0, 2.0e30):
        cb = bf16_bits(np.full((64, 1, 2), c, np.float32))
        qc, sc, zc = o.kv8_quantize(cb)
        assert np.all(qc == qc.flat[0]), f"constant group {c}: codes differ"
        assert np.array_equal(o.kv8_read(qc, sc, zc, np.zeros((0, 1, 2), np.uint16)), cb), f"constant {c} not exact"


def pin_kv8_read_and_tail(o, seed=20):
    """The read is the dequantized history followed by the bf16 tail,
    bit for bit; the number of quantized positions keeps the latest 128
    positions in bf16 and quantizes older ones in whole groups of 64, no
    more than 191 positions staying bf16."""
    rng = np.random.default_rng(seed)
    H, D = 2, 8
    xb, k, s_ref, z_ref = _kv8_grid_case(rng, H, D)
    tail = bf16_bits(rng.standard_normal((37, H, D)).astype(np.float32))
    q, s, z = o.kv8_quantize(xb)
    out = o.kv8_read(q, s, z, tail)
    assert out.shape == (128 + 37, H, D)
    assert np.array_equal(out[:128], xb) and np.array_equal(out[128:], tail), "history or tail misplaced"
    for T in range(0, 1200):
        tq = o.kv8_history_tokens(T)
        assert tq % 64 == 0 and 0 <= tq <= T, (T, tq)
        assert T - tq >= min(T, 128), f"T={T}: fewer than the latest 128 positions in bf16"
        assert T - tq < 192, f"T={T}: a whole group older than the latest 128 is left in bf16"


# ------------------------------------------------------------ producers --

def pin_rmsnorm(o, seed=15):
    """RMSNorm against torch's rms_norm in float64 (a library routine), and
    the closed form of a constant row: c * g / sqrt(c^2 + eps)."""
    rng = np.random.default_rng(seed)
    M, K, eps = 6, 384, 1e-6
    xb = _random_rows(rng, M, K, -4, 4)
    gb = bf16_bits((1.0 + 0.3 * rng.standard_normal(K)).astype(np.float32))
    y = o.rmsnorm(xb, gb, eps)
    xt = torch.from_numpy(bits_to_f32(xb).astype(np.float64))
    gt = torch.from_numpy(bits_to_f32(gb).astype(np.float64))
    ref = torch.nn.functional.rms_norm(xt, (K,), gt, eps).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=0.0), "rmsnorm differs from torch"
    c = np.float32(-2.5)
    yc = o.rmsnorm(bf16_bits(np.full((1, 64), c, np.float32)), bf16_bits(np.ones(64, np.float32)), 0.25)
    cd = float(c)
    assert np.allclose(yc, cd / np.sqrt(cd * cd + 0.25), rtol=1e-15, atol=0.0)


def pin_silu_mul(o, seed=16):
    """SiLU(gate) * up against torch's silu in float64, on the packed
    [gate | up] layout (a transposed half would fail), and silu(0) = 0."""
    rng = np.random.default_rng(seed)
    M, I = 5, 200
    gu = _random_rows(rng, M, 2 * I, -3, 3)
    y = o.silu_mul(gu)
    v = torch.from_numpy(bits_to_f32(gu).astype(np.float64))
    ref = (torch.nn.functional.silu(v[:, :I]) * v[:, I:]).numpy()
    assert np.allclose(y, ref, rtol=1e-13, atol=0.0), "silu_mul differs from torch"
    z = np.zeros((1, 8), np.uint16)
    z[0, 4:] = bf16_bits(np.float32([1, 2, 3, 4]))
    assert np.all(o.silu_mul(z) == 0.0)


ALL_PINS = [pin_decode_table, pin_roundtrip, pin_rounding_cases, pin_encode_vs_library,
            pin_saturation, pin_scale_invariants, pin_scale_and_quotient_rounding, pin_gemm_bruteforce,
            pin_gemm_int_vs_fp, pin_onehot_closed_form, pin_bf16_rounding, pin_kv_cache,
            pin_rmsnorm, pin_silu_mul, pin_kv8_grid, pin_kv8_ties, pin_kv8_invariants, pin_kv8_read_and_tail]
