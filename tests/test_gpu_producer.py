"""The activation quantization fused into its producers (RMSNorm before
q/k/v and gate/up; SiLU(gate) * up on the packed gate_up output before down)
on the GPU against the CPU oracle.

The producers' bf16 output must be within one bf16 unit of the oracle's
exact fp64 value (the pages fix neither the norm's rounding nor the MLP
activation); the codes and scales must equal, bit for bit, the oracle's
quantization of the bf16 values the kernel wrote; and the codes, fed to the
FP8 GEMM, give Linear outputs within the acceptance tolerance."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import assert_linear_parity, bits16, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def within_one_bf16_unit(y_bits, y_ref):
    """Each bf16 value is within one unit in the last place of the exact
    value: 2^(e - 7) in y_ref's binade [2^e, 2^(e+1)), and no less than the
    spacing of bf16's subnormals, 2^-133."""
    y = (y_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    a = np.abs(y_ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.maximum(np.where(a > 0, np.exp2(e - 7), 0.0), 2.0 ** -133)
    return np.abs(y - y_ref) <= ulp


def gamma_for(K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (1.0 + 0.1 * torch.randn(K, generator=g)).to(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("M,K", [(1, 4096), (16, 4096), (2048, 4096), (37, 528), (5, 16384), (3, 12288), (4, 16)])
def test_rmsnorm_quantize(M, K):
    eps = 1e-6
    x = W.make_x(M, K, seed=M + K, kind="rowscale", device=DEV)
    g = gamma_for(K, K)
    y, codes, scales = mfp8.rmsnorm_quantize(x, g, eps)
    _, codes2, scales2 = mfp8.rmsnorm_quantize(x, g, eps, want_y=False)
    torch.cuda.synchronize()
    assert mfp8.device_status() == mfp8.OK
    y_ref = oracle.rmsnorm(bits16(x), bits16(g), eps)
    ok = within_one_bf16_unit(bits16(y), y_ref)
    assert ok.all(), f"{(~ok).sum()} normed values more than one bf16 unit from the exact value"
    q_ref, s_ref = oracle.quantize_rows(bits16(y))
    assert np.array_equal(u8(codes), q_ref), "codes differ from the oracle's quantization of y"
    assert np.array_equal(f32(scales).view(np.uint32), s_ref.view(np.uint32))
    assert torch.equal(codes, codes2) and torch.equal(scales.view(torch.int32), scales2.view(torch.int32))


@pytest.mark.parametrize("M,I", [(1, 12288), (8, 12288), (2048, 12288), (7, 528), (2, 16)])
def test_silu_mul_quantize(M, I):
    gu = W.make_x(M, 2 * I, seed=M + I, kind="rowscale", device=DEV)
    if M == 2:  # large negative gates, where e^-v overflows fp32, and large positive ones
        gu[0, :I] = torch.linspace(-120.0, 120.0, I, dtype=torch.float64).to(torch.bfloat16)
    y, codes, scales = mfp8.silu_mul_quantize(gu)
    _, codes2, _ = mfp8.silu_mul_quantize(gu, want_y=False)
    torch.cuda.synchronize()
    assert mfp8.device_status() == mfp8.OK
    y_ref = oracle.silu_mul(bits16(gu))
    ok = within_one_bf16_unit(bits16(y), y_ref)
    assert ok.all(), f"{(~ok).sum()} activation values more than one bf16 unit from the exact value"
    q_ref, s_ref = oracle.quantize_rows(bits16(y))
    assert np.array_equal(u8(codes), q_ref)
    assert np.array_equal(f32(scales).view(np.uint32), s_ref.view(np.uint32))
    assert torch.equal(codes, codes2)


def test_fused_producers_feed_the_linears():
    """One layer's prefill pipeline on codes from the fused producers: RMSNorm
    codes feed q_proj, SiLU(gate) * up codes of the packed gate_up output feed
    down_proj; outputs against the oracle on sampled rows."""
    M, H, I = 256, 4096, 12288
    x = W.make_x(M, H, seed=21, kind="rowscale", device=DEV)
    g = gamma_for(H, 21)
    _, xq, xs = mfp8.rmsnorm_quantize(x, g, 1e-6)
    Wq, swq = mfp8.quantize_weight(W.make_w(H, H, seed=22, device=DEV))
    yq = mfp8.gemm(xq, xs, Wq, swq)
    gu = W.make_x(M, 2 * I, seed=23, kind="rowscale", device=DEV)
    _, aq, asc = mfp8.silu_mul_quantize(gu)
    Wd, swd = mfp8.quantize_weight(W.make_w(H, I, seed=24, device=DEV))
    yd = mfp8.gemm(aq, asc, Wd, swd)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 77, 128, 255])
    assert_linear_parity(yq, u8(xq), f32(xs), u8(Wq), f32(swq), rows=rows, what="q_proj on fused RMSNorm codes")
    assert_linear_parity(yd, u8(aq), f32(asc), u8(Wd), f32(swd), rows=rows, what="down_proj on fused SiLU codes")
