"""GPU quantize kernels against the CPU oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import bits16, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check_rows(x_bf16: torch.Tensor, which="act"):
    xb = bits16(x_bf16)
    if which == "act":
        q, s = mfp8.quantize_act(x_bf16)
    else:
        q, s = mfp8.quantize_weight(x_bf16)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_rows(xb)
    s_gpu = f32(s)
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    q_gpu = u8(q)
    bad = np.argwhere(q_gpu != q_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0]}: gpu {q_gpu[tuple(bad[0])]:#x} ref {q_ref[tuple(bad[0])]:#x}"


@pytest.mark.parametrize("M,K,kind", [
    (1, 16, "normal"), (3, 48, "normal"), (17, 4096, "normal"), (16, 4096, "normal"),
    (129, 12288, "rowscale"), (256, 4096, "rowscale"), (5, 2048 * 8 + 16, "normal"),  # loop kernel
    (2, 1040, "rowscale"), (7, 12304, "normal"),
])
def test_quantize_act_bitexact(M, K, kind):
    check_rows(W.make_x(M, K, seed=7, stream=M, kind=kind, device=DEV))


def test_quantize_act_full_size_rows():
    # the largest activation of the long-video workload: every code and scale
    x = W.make_x(16384, 4096, seed=3, kind="rowscale", device=DEV)
    check_rows(x)


def test_quantize_edge_rows():
    K = 64
    rows = []
    rows.append(torch.zeros(K))                        # all zero -> FLT_MIN scale
    rows.append(-torch.zeros(K))                       # negative zeros
    r = torch.zeros(K); r[5] = 1e-40; rows.append(r)   # bf16 subnormal only
    r = torch.zeros(K); r[0] = 3.0e38; r[1] = -1.0; rows.append(r)  # near bf16 max
    r = torch.full((K,), 448.0); rows.append(r)        # scale exactly 1
    # scale 1 with every e4m3 midpoint of [1, 2) and the tie cases of the golden file
    r = torch.tensor([448.0] + [1.0 + (2 * i + 1) / 16 for i in range(8)] + [1.0625, 1.1875, 2 ** -10, 3 * 2 ** -10]
                     + [0.0] * (K - 13))
    rows.append(r)
    r = torch.linspace(-7.0, 7.0, K); rows.append(r)
    r = torch.zeros(K); r[-1] = -2.5; rows.append(r)   # single negative entry
    x = torch.stack(rows).to(torch.bfloat16).to(DEV)
    check_rows(x)


@pytest.mark.parametrize("K", [64, 1040, 2048, 4096])
def test_quantize_edge_rows_warp_kernel(K):
    """Many rows (the warp-per-row kernel): the edge rows above spread among
    ordinary ones, with ragged K, plus rows whose scale is below 2^-64 (the
    quantizer's divide branch) and a row whose absmax is a bf16 subnormal."""
    g = torch.Generator().manual_seed(K)
    x = torch.randn(300, K, generator=g)
    x[3] = 0
    x[17] = -0.0
    x[40] = 0
    x[40, 5] = 1e-40
    x[41] *= 1e-30                      # scale about 1e-32: divide branch
    x[42] = 0
    x[42, K - 1] = -3e-25
    x[99] = 448.0
    x[100, : K // 2] = 3.0e38
    x[299] *= 1e4
    check_rows(x.to(torch.bfloat16).to(DEV))


@pytest.mark.parametrize("N,K", [(4096, 4096), (12288, 4096), (4096, 12288), (1024, 4096), (8, 16)])
def test_quantize_weight_bitexact(N, K):
    check_rows(W.make_w(N, K, seed=1, stream=N + K, device=DEV), which="weight")


def test_device_conversion_all_fp32_patterns():
    """Every fp32 bit pattern through the device's e4m3 conversion against
    the oracle encoder (NaN inputs: both must give a NaN code)."""
    chunk = 1 << 28
    for lo in range(0, 1 << 32, chunk):
        hi = lo + chunk
        bits = (torch.arange(chunk, dtype=torch.int64, device=DEV) + lo)
        bits = torch.where(bits >= (1 << 31), bits - (1 << 32), bits).to(torch.int32)
        vals = bits.view(torch.float32)
        got = u8(mfp8.e4m3_encode(vals))
        ref = oracle.e4m3_encode_bits_range(lo, hi)
        diff = got != ref
        if diff.any():
            idx = np.nonzero(diff)[0]
            b = (lo + idx).astype(np.uint64)
            exp_all_ones = ((b >> 23) & 0xFF) == 0xFF
            mant_nonzero = (b & 0x7FFFFF) != 0
            is_nan = exp_all_ones & mant_nonzero
            assert is_nan.all(), f"non-NaN mismatch at bits {int(b[~is_nan][0]):#010x}: gpu {got[idx[~is_nan][0]]:#x} ref {ref[idx[~is_nan][0]]:#x}"
            assert ((got[idx] & 0x7F) == 0x7F).all() and ((ref[idx] & 0x7F) == 0x7F).all()
        del bits, vals


def test_bounded_wait_reports_timeout_and_context_survives():
    assert mfp8.device_status() == mfp8.OK
    assert mfp8.mfp8_debug_bounded_wait(2000, torch.cuda.current_stream().cuda_stream) == mfp8.OK
    assert mfp8.device_status() == mfp8.ERR_TIMEOUT
    assert mfp8.device_status() == mfp8.OK  # read-and-clear
    x = torch.ones(4, 32, dtype=torch.bfloat16, device=DEV)
    q, s = mfp8.quantize_act(x)
    torch.cuda.synchronize()
    assert (u8(q) == 0x7E).all()


def _magnitude_sweep_rows(n_rows, seed):
    """Rows holding every finite bf16 magnitude up to the row's absmax, with
    random signs, under n_rows different absmax values spread over the whole
    bf16 range (including ones whose scale is raised to FLT_MIN)."""
    rng = np.random.default_rng(seed)
    mags = np.arange(0, 0x7F80, dtype=np.uint16)  # every finite non-negative bf16
    fixed = [0x7F7F, 0x43E0, 0x3F80, 0x0080, 0x0001, 0x0C00, 0x3C00, 0x4780]  # max, 448, 1, tiny, ...
    tops = np.array(fixed + list(rng.integers(0x0001, 0x7F80, n_rows - len(fixed))), dtype=np.uint16)
    K = 0x7F80 + 16
    rows = np.zeros((n_rows, K), dtype=np.uint16)
    for i, top in enumerate(tops):
        r = mags[mags <= top].copy()
        r = r | (rng.integers(0, 2, r.size, dtype=np.uint16) << 15)  # random signs
        rng.shuffle(r)
        rows[i, : r.size] = r
        rows[i, r.size] = top  # the row's absmax, positive
    return rows


def test_every_bf16_magnitude_under_many_scales():
    """The multiply-with-boundary-check quantizer against the oracle's
    division on every bf16 magnitude, under 256 row scales."""
    rows = _magnitude_sweep_rows(256, seed=21)
    x = torch.from_numpy(rows.view(np.int16)).view(torch.bfloat16).to(DEV)
    check_rows(x)


@pytest.mark.parametrize("path", [mfp8.PATH_SPLITK, mfp8.PATH_FUSED])
def test_decode_kernel_codes_every_bf16_magnitude(path):
    """The same sweep through the decode paths (the fused kernel quantizes on
    chip and can write its codes out), four tokens per call."""
    rows = _magnitude_sweep_rows(32, seed=22)
    K = rows.shape[1]
    W8, sw = mfp8.quantize_weight(W.make_w(128, K, seed=5, device=DEV))
    for i in range(0, rows.shape[0], 4):
        blk = rows[i:i + 4]
        x = torch.from_numpy(blk.view(np.int16)).view(torch.bfloat16).to(DEV)
        x8 = torch.empty((4, K), dtype=torch.uint8, device=DEV)
        xs = torch.empty((4,), dtype=torch.float32, device=DEV)
        mfp8.linear(x, W8, sw, path=path, x8_out=x8, xs_out=xs)
        torch.cuda.synchronize()
        q_ref, s_ref = oracle.quantize_rows(blk)
        assert np.array_equal(f32(xs).view(np.uint32), s_ref.view(np.uint32))
        assert np.array_equal(u8(x8), q_ref)


def test_divide_free_rounding_matches_ieee_divide_on_every_bf16_pair():
    """The quantizers round x / s with a multiply by the correctly rounded
    reciprocal and two fused multiply-adds.  On every absmax a (zero and each
    positive finite bf16, i.e. every scale a row can have) and every bf16 x
    with |x| <= a, both signs, the codes equal those of an IEEE divide."""
    out = torch.zeros(2, dtype=torch.int64, device=DEV)
    assert mfp8.mfp8_debug_quantize_check(out.data_ptr(), torch.cuda.current_stream().cuda_stream) == mfp8.OK
    torch.cuda.synchronize()
    bad, witness = (int(v) for v in out.cpu())
    assert bad == 0, f"{bad} codes differ; e.g. absmax bits {witness >> 16:#06x}, x bits {witness & 0xffff:#06x}"
