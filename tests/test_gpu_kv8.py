"""The INT8 KV cache ("MOSS-VL quantization README", KV8 section: hqq
backend, nbits 8, q_group_size 64, axis 0, residual_length 128) on the GPU
against the CPU oracle.

Readings (the section gives settings, not HQQ's optimizer): a group is 64
consecutive tokens of one (head, channel) column; the asymmetric min-max fit
with an integer zero point in fp32; the read dequantizes the history and
appends the bf16 tail.  Codes, scales, zero points and read values are
compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import bits16, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check_quantize(kv):
    codes, scale, zero = mfp8.kv8_quantize(kv)
    torch.cuda.synchronize()
    q_ref, s_ref, z_ref = oracle.kv8_quantize(bits16(kv))
    assert np.array_equal(u8(codes), q_ref), f"{(u8(codes) != q_ref).sum()} codes differ from the oracle"
    assert np.array_equal(f32(scale).view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    assert np.array_equal(f32(zero).view(np.uint32), z_ref.view(np.uint32)), "zero points differ"
    return codes, scale, zero, q_ref, s_ref, z_ref


SHAPES = [(64, 8, 128), (192, 8, 128), (16384, 8, 128), (128, 3, 64), (64, 1, 16), (320, 4, 256), (64, 2, 48),
          (4096, 1, 512)]


@pytest.mark.parametrize("T,H,D", SHAPES)
def test_kv8_quantize_bitexact(T, H, D):
    check_quantize(W.make_kv(T, H, D, seed=T + D, device=DEV))


@pytest.mark.parametrize("Tq,Tr", [(0, 1), (64, 0), (64, 37), (256, 128), (1024, 191), (16256, 128), (0, 0)])
def test_kv8_read_bitexact(Tq, Tr):
    H, D = 8, 128
    kv = W.make_kv(Tq + Tr, H, D, seed=7, stream=Tq + Tr, device=DEV)
    codes, scale, zero = mfp8.kv8_quantize(kv[:Tq].contiguous())
    tail = kv[Tq:].contiguous()
    out = mfp8.kv8_read(codes, scale, zero, tail)
    torch.cuda.synchronize()
    q_ref, s_ref, z_ref = oracle.kv8_quantize(bits16(kv[:Tq]))
    ref = oracle.kv8_read(q_ref, s_ref, z_ref, bits16(tail))
    assert out.shape == (Tq + Tr, H, D)
    assert np.array_equal(bits16(out), ref), "read differs from the oracle"


def test_kv8_edge_groups():
    """Constant groups (0, -0, small, negative, huge), subnormal and tiny
    groups (scales below 2^-64 take the divide), near-max values of both
    signs, exact grid values and half-way values (ties to even)."""
    T, H, D = 64 * 3, 2, 64
    kv = torch.zeros((T, H, D), dtype=torch.float64)
    kv[:64, 0, 0] = 0.0
    kv[:64, 0, 1] = -0.0
    kv[:64, 0, 2] = 1.5
    kv[:64, 0, 3] = -7.0
    kv[:64, 0, 4] = 2.0e30
    kv[:64, 0, 5] = -3.0e-30
    kv[:32, 0, 6], kv[32:64, 0, 6] = 0.0, -0.0
    kv[:64, 0, 7] = torch.linspace(-1.5e38, 1.5e38, 64, dtype=torch.float64)
    kv[:64, 0, 8] = torch.tensor([(-1.0) ** i * 2.0 ** (-133 + (i % 7)) for i in range(64)])  # subnormal bf16
    kv[:64, 0, 9] = torch.tensor([(-1.0) ** i * 2.0 ** (-80 - (i % 5)) for i in range(64)])   # s < 2^-64
    kv[:64, 0, 10] = torch.tensor([2.0 ** (-70) * (1 + i / 64) for i in range(64)])
    gen = torch.Generator().manual_seed(3)
    for d in range(11, D):  # grids (k - m) 2^-e and half-way points (j + 1/2) 2^-e
        m = int(torch.randint(64, 192, (1,), generator=gen))
        e = int(torch.randint(-10, 10, (1,), generator=gen))
        k = torch.randperm(254, generator=gen)[:62] + 1
        vals = torch.cat([torch.tensor([0, 255]), k]).double() - m
        if d % 2:
            j = torch.randint(max(-m, -127), min(254 - m, 126) + 1, (62,), generator=gen).double()
            vals = torch.cat([torch.tensor([-m, 255 - m]).double(), j + 0.5])
        kv[:64, 0, d] = vals * 2.0 ** (-e)
    kv[64:, :, :] = torch.randn(T - 64, H, D, generator=gen, dtype=torch.float64) * 3 + 1
    kv[:64, 1, :] = torch.randn(64, D, generator=gen, dtype=torch.float64) * 1e-3 - 5
    kvb = kv.to(torch.bfloat16)
    assert torch.equal(kvb[:64, 0, 11:].double(), kv[:64, 0, 11:]), "grid and half-way values must be bf16-exact"
    kvb = kvb.to(DEV)
    codes, scale, zero, q_ref, s_ref, z_ref = check_quantize(kvb)
    out = mfp8.kv8_read(codes, scale, zero, kvb[:0])
    torch.cuda.synchronize()
    assert np.array_equal(bits16(out), oracle.kv8_read(q_ref, s_ref, z_ref, bits16(kvb[:0])))
    assert torch.equal(out[:64, 0, :6], kvb[:64, 0, :6]), "constant groups are not reproduced exactly"


def test_kv8_writes_nothing_outside_its_buffers():
    T, Tr, H, D = 192, 45, 4, 64
    kv = W.make_kv(T + Tr, H, D, seed=5, device=DEV)
    G, C = 4096, H * D
    sizes = {"q": T * C, "s": T // 64 * C * 4, "z": T // 64 * C * 4, "o": (T + Tr) * C * 2}
    raw = {k: torch.full((n + 2 * G,), 0xA7, dtype=torch.uint8, device=DEV) for k, n in sizes.items()}
    b = {k: raw[k][G:G + n] for k, n in sizes.items()}
    h = torch.cuda.current_stream().cuda_stream
    assert mfp8.mfp8_kv8_quantize(kv.data_ptr(), T, H, D, b["q"].data_ptr(), b["s"].data_ptr(), b["z"].data_ptr(),
                                  h) == mfp8.OK
    tail = kv[T:]
    assert mfp8.mfp8_kv8_read(b["q"].data_ptr(), b["s"].data_ptr(), b["z"].data_ptr(), T, tail.data_ptr(), Tr, H, D,
                              b["o"].data_ptr(), h) == mfp8.OK
    torch.cuda.synchronize()
    for k, n in sizes.items():
        r = raw[k].cpu().numpy()
        assert (r[:G] == 0xA7).all() and (r[G + n:] == 0xA7).all(), f"a write landed outside buffer {k}"
    q_ref, s_ref, z_ref = oracle.kv8_quantize(bits16(kv[:T]))
    assert np.array_equal(u8(b["q"]).reshape(T, H, D), q_ref)
    ref = oracle.kv8_read(q_ref, s_ref, z_ref, bits16(tail))
    assert np.array_equal(bits16(b["o"].view(torch.bfloat16)).reshape(T + Tr, H, D), ref)


def test_kv8_cache_streaming():
    """Positions appended in chunks of mixed sizes (single decode tokens and
    prefill chunks): after every append the history holds the oldest whole
    groups outside the latest 128 positions, and the read equals the oracle's
    read of the whole sequence quantized at once (groups are aligned to
    position 0, so the order of appends does not change them)."""
    H, D, cap = 4, 128, 1400
    seq = W.make_kv(cap, H, D, seed=9, device=DEV)
    cache = mfp8.Kv8Cache(cap, H, D, DEV)
    chunks = [1, 1, 63, 64, 200, 1, 1, 1, 130, 7, 300, 64, 1, 250, 2]
    T = 0
    for n in chunks:
        cache.append(seq[T:T + n])
        T += n
        tq = oracle.kv8_history_tokens(T)
        assert cache.T == T and cache.Tq == tq and cache.tail.shape[0] == T - tq
        out = cache.read()
        torch.cuda.synchronize()
        q_ref, s_ref, z_ref = oracle.kv8_quantize(bits16(seq[:tq]))
        ref = oracle.kv8_read(q_ref, s_ref, z_ref, bits16(seq[tq:T]))
        assert np.array_equal(bits16(out), ref), f"read after {T} positions differs from the oracle"


def test_kv8_divide_free_codes_match_the_divide():
    """The kernel's codes use a corrected quotient instead of x / s; on every
    finite bf16 x, over 2 x 65536 drawn scales and zero points, they equal the
    IEEE-divide codes."""
    out = torch.zeros(2, dtype=torch.int64, device=DEV)
    assert mfp8.mfp8_debug_kv8_code_check(out.data_ptr(), 65536, 7, torch.cuda.current_stream().cuda_stream) == mfp8.OK
    torch.cuda.synchronize()
    bad, witness = out.tolist()
    assert bad == 0, f"{bad} codes differ; scale bits {witness >> 32:08x}, x bits {witness & 0xffff:04x}"


def test_kv8_nonfinite_inputs_are_contained():
    """Non-finite values are outside the contract: the kernels must neither
    fault nor hang on them, and groups without them must still match the
    oracle bit for bit."""
    T, H, D = 128, 2, 64
    kv = W.make_kv(T, H, D, seed=11, device=DEV)
    kv[3, 0, 5] = float("inf")
    kv[70, 1, 9] = float("nan")
    kv[100, 0, 60] = float("-inf")
    codes, scale, zero = mfp8.kv8_quantize(kv)
    out = mfp8.kv8_read(codes, scale, zero, kv[:0])
    torch.cuda.synchronize()
    assert mfp8.device_status() == mfp8.OK
    q_ref, s_ref, z_ref = oracle.kv8_quantize(bits16(kv))
    bad = np.zeros((T // 64, H, D), bool)
    bad[0, 0, 5] = bad[1, 1, 9] = bad[1, 0, 60] = True
    ok = ~np.repeat(bad, 64, axis=0)
    assert np.array_equal(u8(codes)[ok], q_ref[ok])
    assert np.array_equal(f32(scale)[~bad].view(np.uint32), s_ref[~bad].view(np.uint32))
    assert np.array_equal(bits16(out)[ok], oracle.kv8_read(q_ref, s_ref, z_ref, bits16(kv[:0]))[ok])
