"""The FP8 e4m3 KV cache ("MOSS-VL quantization README", SGLang paragraph:
--kv-cache-dtype fp8_e4m3) on the GPU against the CPU oracle.

Reading (the pages give only the flag): one scale per (token, head) row of a
[T, H, D] tensor by the activation rule; dequantize = bf16(fl32(dec * s)).
Codes, scales and dequantized values are compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import bits16, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make_kv(T, H, D, seed):
    """Keys/values [T, H, D]: N(0, 1) rows scaled per (token, head) by a
    log-uniform factor in [0.1, 10], with 0.1% outliers x50 (the activation
    recipe, one row per (token, head))."""
    return W.make_x(T * H, D, seed=seed, stream=D, kind="rowscale", device=DEV).view(T, H, D)


SHAPES = [(1, 8, 128), (4, 8, 128), (2048, 8, 128), (16384, 8, 128), (37, 3, 64), (5, 2, 16), (9, 4, 256),
          (3, 2, 512), (7, 1, 48)]


@pytest.mark.parametrize("T,H,D", SHAPES)
def test_kv_quantize_and_dequantize_bitexact(T, H, D):
    kv = make_kv(T, H, D, seed=T + D)
    codes, scales = mfp8.kv_quantize(kv)
    back = mfp8.kv_dequantize(codes, scales)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.kv_quantize(bits16(kv))
    assert np.array_equal(u8(codes), q_ref), "codes differ from the oracle"
    assert np.array_equal(f32(scales).view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    d_ref = oracle.kv_dequantize(q_ref, s_ref)
    assert np.array_equal(bits16(back), d_ref), "dequantized values differ from the oracle"
    # the same bytes as the activation quantizer on the [T*H, D] view
    x8, xs = mfp8.quantize_act(kv.view(T * H, D))
    assert torch.equal(x8.view(T, H, D), codes) and torch.equal(xs.view(T, H).view(torch.int32),
                                                                 scales.view(torch.int32))


def test_kv_edge_rows():
    """Zero, -0, subnormal and near-max rows; every bf16 magnitude class."""
    T, H, D = 4, 2, 128
    kv = torch.zeros((T, H, D), dtype=torch.bfloat16)
    kv[0, 1] = -0.0
    kv[1, 0, 3] = 1e-40          # a bf16 subnormal: scale floors at FLT_MIN
    kv[1, 1] = torch.linspace(-3e38, 3e38, D, dtype=torch.float64).to(torch.bfloat16)  # finite, up to near max
    kv[2, 0] = torch.tensor([(-1.0) ** i * 2.0 ** (i - 64) for i in range(D)]).to(torch.bfloat16)
    kv[3] = torch.randn(H, D).to(torch.bfloat16)
    kv = kv.to(DEV)
    codes, scales = mfp8.kv_quantize(kv)
    back = mfp8.kv_dequantize(codes, scales)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.kv_quantize(bits16(kv))
    assert np.array_equal(u8(codes), q_ref)
    assert np.array_equal(f32(scales).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(bits16(back), oracle.kv_dequantize(q_ref, s_ref))


def test_kv_writes_nothing_outside_its_buffers():
    T, H, D = 33, 8, 128
    kv = make_kv(T, H, D, seed=5)
    G = 4096
    raw_q = torch.full((T * H * D + 2 * G,), 0xA7, dtype=torch.uint8, device=DEV)
    raw_s = torch.full((T * H * 4 + 2 * G,), 0xA7, dtype=torch.uint8, device=DEV)
    raw_o = torch.full((T * H * D * 2 + 2 * G,), 0xA7, dtype=torch.uint8, device=DEV)
    h = torch.cuda.current_stream().cuda_stream
    q, s, o = raw_q[G:G + T * H * D], raw_s[G:G + T * H * 4], raw_o[G:G + T * H * D * 2]
    assert mfp8.mfp8_kv_quantize(kv.data_ptr(), T, H, D, q.data_ptr(), s.data_ptr(), h) == mfp8.OK
    assert mfp8.mfp8_kv_dequantize(q.data_ptr(), s.data_ptr(), T, H, D, o.data_ptr(), h) == mfp8.OK
    torch.cuda.synchronize()
    for raw, n in ((raw_q, T * H * D), (raw_s, T * H * 4), (raw_o, T * H * D * 2)):
        r = raw.cpu().numpy()
        assert (r[:G] == 0xA7).all() and (r[G + n:] == 0xA7).all(), "a write landed outside its buffer"
    q_ref, s_ref = oracle.kv_quantize(bits16(kv))
    assert np.array_equal(u8(q).reshape(T, H, D), q_ref)
    assert np.array_equal(bits16(o.view(torch.bfloat16)).reshape(T, H, D), oracle.kv_dequantize(q_ref, s_ref))
