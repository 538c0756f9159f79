"""Out-of-bounds writes: every kernel path at ragged M and N, with each
buffer the library writes (Y, the caller's copies of the activation codes
and scales, the workspace) placed inside a larger allocation whose guard
bytes hold a known pattern.  After the call the guard bytes must be
untouched and the outputs must be right.  The epilogues of the decode and
split-K kernels store Y directly (no TMA clipping), so a wrong bound there
shows up as a changed guard byte."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import assert_linear_parity, bits16, f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096      # guard bytes on each side (a multiple of 16: the buffers stay aligned)
PATTERN = 0xA7


class Guarded:
    """`nbytes` usable bytes between two guard regions of PATTERN."""

    def __init__(self, nbytes):
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=DEV)
        self.body = self.raw[GUARD:GUARD + nbytes]

    def view(self, dtype, shape):
        return self.body.view(dtype).view(shape)

    def guards_intact(self):
        raw = self.raw.cpu().numpy()
        return bool((raw[:GUARD] == PATTERN).all() and (raw[GUARD + self.nbytes:] == PATTERN).all())


CASES = [  # (M, N, K): ragged in M and N, several tiles
    (1, 136, 272), (5, 264, 400), (13, 1032, 528), (16, 392, 1040),      # one-kernel decode path
    (17, 136, 272), (37, 264, 400), (100, 520, 528), (128, 1160, 400),   # cluster split-K
    (130, 264, 384), (201, 776, 528), (256, 1032, 400),                  # 1-CTA tiles, split-K
    (300, 520, 400), (513, 1032, 528),                                   # CTA pairs
    (3, 7, 272), (40, 101, 400), (200, 1001, 528), (600, 77, 400),       # N % 8 != 0: padded scratch + crop
]


def _paths(M):
    p = [mfp8.PATH_AUTO, mfp8.PATH_TILED, mfp8.PATH_PAIR]
    if M <= 256:
        p.append(mfp8.PATH_SPLITK)
    if M <= 16:
        p.append(mfp8.PATH_FUSED)
    return p


@pytest.mark.parametrize("M,N,K", CASES)
def test_linear_writes_nothing_outside_its_buffers(M, N, K):
    x = W.make_x(M, K, seed=M + N, kind="rowscale", device=DEV)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=M + N, device=DEV))
    x8_ref, xs_ref = oracle.quantize_rows(bits16(x))
    w8_h, sw_h = u8(W8), f32(sw)
    h = torch.cuda.current_stream().cuda_stream
    for path in _paths(M):
        for with_copies in (False, True):
            gy = Guarded(M * N * 2)
            ws_need = mfp8.mfp8_linear_workspace_bytes(M, N, K)
            gw = Guarded(ws_need)
            gx8, gxs = Guarded(M * K), Guarded(M * 4)
            x8p = gx8.body.data_ptr() if with_copies else None
            xsp = gxs.body.data_ptr() if with_copies else None
            st = mfp8.mfp8_linear_ex(x.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, gy.body.data_ptr(),
                                     gw.body.data_ptr(), ws_need, path, 0, x8p, xsp, h)
            assert st == mfp8.OK, (path, mfp8.mfp8_status_string(st))
            torch.cuda.synchronize()
            assert mfp8.device_status() == mfp8.OK
            what = f"M={M} N={N} K={K} path={path} copies={with_copies}"
            assert gy.guards_intact(), f"{what}: a write landed outside Y"
            assert gw.guards_intact(), f"{what}: a write landed outside the workspace"
            if with_copies:
                assert gx8.guards_intact() and gxs.guards_intact(), f"{what}: a write outside the code/scale copies"
                assert np.array_equal(u8(gx8.view(torch.uint8, (M, K))), x8_ref)
                assert np.array_equal(f32(gxs.view(torch.float32, (M,))).view(np.uint32), xs_ref.view(np.uint32))
            assert_linear_parity(gy.view(torch.bfloat16, (M, N)), x8_ref, xs_ref, w8_h, sw_h, what=what)


@pytest.mark.parametrize("M,N,K", [(5, 264, 400), (100, 520, 528), (300, 520, 400)])
def test_quantize_and_gemm_write_nothing_outside_their_buffers(M, N, K):
    x = W.make_x(M, K, seed=7, kind="rowscale", device=DEV)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=7, device=DEV))
    h = torch.cuda.current_stream().cuda_stream
    gx8, gxs = Guarded(M * K), Guarded(M * 4)
    assert mfp8.mfp8_quantize_act(x.data_ptr(), M, K, gx8.body.data_ptr(), gxs.body.data_ptr(), h) == mfp8.OK
    gw8, gsw = Guarded(N * K), Guarded(N * 4)
    w = W.make_w(N, K, seed=8, device=DEV)
    assert mfp8.mfp8_quantize_weight(w.data_ptr(), N, K, gw8.body.data_ptr(), gsw.body.data_ptr(), h) == mfp8.OK
    torch.cuda.synchronize()
    for g in (gx8, gxs, gw8, gsw):
        assert g.guards_intact()
    x8, xs = gx8.view(torch.uint8, (M, K)), gxs.view(torch.float32, (M,))
    for path in [mfp8.PATH_TILED, mfp8.PATH_PAIR] + ([mfp8.PATH_SPLITK] if M <= 256 else []):
        gy = Guarded(M * N * 2)
        st = mfp8.mfp8_gemm(x8.data_ptr(), xs.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N,
                            gy.body.data_ptr(), None, 0, path, h)
        assert st == mfp8.OK
        torch.cuda.synchronize()
        assert gy.guards_intact(), f"mfp8_gemm path={path}: a write landed outside Y"
        assert_linear_parity(gy.view(torch.bfloat16, (M, N)), u8(x8), f32(xs), u8(W8), f32(sw),
                             what=f"mfp8_gemm path={path}")
