"""The FP8_DYNAMIC Linear on the GPU against the CPU oracle.

Activation and weight codes/scales: bit-exact.  BF16 outputs: within
|y - y_ref| <= 2^-7 |y_ref| + 1e-5 * sum_k |a_k w_k| s_a s_w of the exact
rescaled product, element by element."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import assert_linear_parity, bits16, f32, rows_in_every_tile, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_case(M, N, K, path, seed=0, kind="normal", rows=None, check_codes=True, flags=0):
    x = W.make_x(M, K, seed=seed, stream=M, kind=kind, device=DEV)
    w = W.make_w(N, K, seed=seed, stream=N, device=DEV)
    W8, sw = mfp8.quantize_weight(w)
    x8 = torch.empty((M, K), dtype=torch.uint8, device=DEV)
    xs = torch.empty((M,), dtype=torch.float32, device=DEV)
    y = mfp8.linear(x, W8, sw, path=path, x8_out=x8, xs_out=xs, flags=flags)
    torch.cuda.synchronize()
    assert mfp8.device_status() == mfp8.OK
    w8_h, sw_h = u8(W8), f32(sw)
    x8_h, xs_h = u8(x8), f32(xs)
    if check_codes:
        w8_ref, sw_ref = oracle.quantize_rows(bits16(w))
        assert np.array_equal(w8_h, w8_ref) and np.array_equal(sw_h.view(np.uint32), sw_ref.view(np.uint32))
        x8_ref, xs_ref = oracle.quantize_rows(bits16(x))
        assert np.array_equal(x8_h, x8_ref), "activation codes differ from the oracle"
        assert np.array_equal(xs_h.view(np.uint32), xs_ref.view(np.uint32)), "activation scales differ"
    assert_linear_parity(y, x8_h, xs_h, w8_h, sw_h, rows=rows, what=f"M={M} N={N} K={K} path={path}")
    return x, W8, sw, y


SMALL = [  # (M, N, K): several tiles, ragged tails in M, N and K
    (1, 128, 128), (5, 256, 256), (16, 4096, 4096), (17, 384, 272), (64, 1024, 4096),
    (3, 136, 48), (2, 8, 16), (128, 512, 640), (33, 264, 400),
]
TILED_ONLY = [(130, 264, 384), (300, 520, 1040), (256, 1024, 4096), (1000, 2056, 528), (129, 4096, 128)]


@pytest.mark.parametrize("M,N,K", SMALL)
@pytest.mark.parametrize("path", [mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR, mfp8.PATH_FUSED,
                                  mfp8.PATH_AUTO])
def test_linear_small(M, N, K, path):
    if path == mfp8.PATH_FUSED and M > 16:
        pytest.skip("the fused decode kernel takes M <= 16")
    run_case(M, N, K, path, seed=M * 7 + N)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 12288, 4096), (16, 4096, 12288), (64, 1024, 4096),
                                   (33, 264, 400)])
@pytest.mark.parametrize("path", [mfp8.PATH_SPLITK, mfp8.PATH_FUSED])
def test_linear_static_weights_flag(M, N, K, path):
    if path == mfp8.PATH_FUSED and M > 16:
        pytest.skip("the fused decode kernel takes M <= 16")
    run_case(M, N, K, path, seed=M + 3, flags=mfp8.FLAG_STATIC_WEIGHTS)


ODD_N = [(4, 1, 64), (3, 7, 128), (16, 100, 528), (40, 13, 272), (100, 1001, 256), (200, 77, 640),
         (512, 1030, 1024), (2, 4099, 4096), (300, 4101, 128)]


@pytest.mark.parametrize("M,N,K", ODD_N)
@pytest.mark.parametrize("path", [mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR, mfp8.PATH_FUSED,
                                  mfp8.PATH_AUTO])
def test_linear_any_n(M, N, K, path):
    """N not a multiple of 8 (rows of Y not 16-byte aligned): the kernels run
    on N rounded up to 8 into a workspace scratch and the first N columns are
    copied out; codes bit-exact, outputs within the tolerance."""
    if path == mfp8.PATH_FUSED and M > 16:
        pytest.skip("the fused decode kernel takes M <= 16")
    if path == mfp8.PATH_SPLITK and M > 256:
        pytest.skip("the split-K kernel takes M <= 256")
    assert mfp8.mfp8_linear_workspace_bytes(M, N, K) > mfp8.mfp8_linear_workspace_bytes(M, (N + 7) // 8 * 8, K)
    run_case(M, N, K, path, seed=M + N, flags=mfp8.FLAG_STATIC_WEIGHTS if M <= 16 else 0)


@pytest.mark.parametrize("M,N,K", [(5, 13, 272), (64, 1001, 400), (700, 77, 528)])
def test_gemm_any_n(M, N, K):
    """mfp8_gemm on codes with N % 8 != 0 takes the scratch from its
    workspace (mfp8_gemm_workspace_bytes > 0 only then) and equals the
    Linear's output bit for bit."""
    assert mfp8.mfp8_gemm_workspace_bytes(M, N, K) > 0
    assert mfp8.mfp8_gemm_workspace_bytes(M, (N + 7) // 8 * 8, K) == 0
    x = W.make_x(M, K, seed=N, device=DEV)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=N, device=DEV))
    x8, xs = mfp8.quantize_act(x)
    for path in (mfp8.PATH_AUTO, mfp8.PATH_TILED, mfp8.PATH_PAIR):
        y = mfp8.gemm(x8, xs, W8, sw, path=path)
        y_lin = mfp8.linear(x, W8, sw, path=path)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_lin.view(torch.int16)), f"path {path}"
        assert_linear_parity(y, u8(x8), f32(xs), u8(W8), f32(sw), what=f"gemm M={M} N={N} K={K} path={path}")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    st = mfp8.mfp8_gemm(x8.data_ptr(), xs.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, out.data_ptr(), None, 0,
                        mfp8.PATH_AUTO, torch.cuda.current_stream().cuda_stream)
    assert st == mfp8.ERR_WORKSPACE


def test_linear_without_codes_out_matches_with():
    """The decode kernel writes the optional code copy only from its first
    cluster; the outputs must not depend on whether it is asked for."""
    for M in (1, 7, 64, 100):
        x = W.make_x(M, 4096, seed=9, device=DEV)
        W8, sw = mfp8.quantize_weight(W.make_w(1024, 4096, seed=9, device=DEV))
        y1 = mfp8.linear(x, W8, sw)
        x8 = torch.empty((M, 4096), dtype=torch.uint8, device=DEV)
        xs = torch.empty((M,), dtype=torch.float32, device=DEV)
        y2 = mfp8.linear(x, W8, sw, x8_out=x8, xs_out=xs)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# The one-kernel decode path: channel groups of 16..256 per CTA, one or
# several 32 KB code windows along K (8 or 16 code rows per K block), a
# ragged last K block, a partial last channel group (N % 16 == 8), grids
# above one CTA per SM, and every M from 1 to 16.
STREAM = [
    (1, 8, 16), (2, 24, 144), (7, 1032, 4112), (8, 1024, 12288), (9, 6144, 4096), (12, 264, 4992),
    (16, 24576, 4096), (4, 40960, 256), (13, 520, 1040), (16, 12296, 2064), (5, 4096, 8320),
]


@pytest.mark.parametrize("M,N,K", STREAM)
def test_fused_stream_geometry(M, N, K):
    run_case(M, N, K, mfp8.PATH_FUSED, seed=M * 5 + K, flags=mfp8.FLAG_STATIC_WEIGHTS if M % 2 else 0)


# The cluster split-K kernel on codes: token columns 16..256 (M rounded up
# to 16, with ragged M), cluster sizes 1..8, a ragged last K block, a K
# shorter than one block, a partial last channel tile (N % 128 != 0), grids
# of many tiles, and long K.
CLUSTER = [
    (17, 8, 16), (24, 136, 272), (48, 1032, 4112), (64, 6144, 4096), (80, 264, 4992), (96, 4096, 12288),
    (112, 520, 1040), (128, 12296, 2064), (33, 40960, 256), (127, 1024, 8320), (65, 24576, 4096),
    (129, 1032, 4112), (160, 264, 400), (192, 4096, 4096), (200, 12296, 2064), (255, 136, 272),
    (256, 1024, 8320), (176, 24576, 512), (240, 4096, 12288),
]


@pytest.mark.parametrize("M,N,K", CLUSTER)
def test_cluster_splitk_geometry(M, N, K):
    big = M * N * K > 1 << 30  # the oracle's exact contraction on sampled rows only
    run_case(M, N, K, mfp8.PATH_SPLITK, seed=M * 3 + K, kind="rowscale",
             rows=sampled_rows(M, 8, K) if big else None, flags=mfp8.FLAG_STATIC_WEIGHTS if M % 2 else 0)


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_fused_every_m(M):
    run_case(M, 4096, 4096, mfp8.PATH_FUSED, seed=100 + M, kind="rowscale" if M > 2 else "normal")


def test_fused_back_to_back_on_one_stream():
    """Consecutive decode kernels overlap on the GPU (the next one starts its
    weight stream while this one finishes); each reads its activations only
    after the previous kernel completed.  A chain where each Linear's input is
    the previous Linear's output must equal the same chain run one call at a
    time with a synchronisation in between."""
    M, H = 8, 4096
    Ws = [mfp8.quantize_weight(W.make_w(H, H, seed=60 + i, device=DEV)) for i in range(6)]
    x0 = W.make_x(M, H, seed=61, device=DEV)
    ws = torch.zeros((16,), dtype=torch.uint8, device=DEV)  # the path keeps nothing there
    torch.cuda.synchronize()

    def chain(sync):
        x = x0
        for W8, sw in Ws:
            x = mfp8.linear(x, W8, sw, workspace=ws, path=mfp8.PATH_FUSED, flags=mfp8.FLAG_STATIC_WEIGHTS)
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return x

    a, b = chain(False), chain(True)
    assert mfp8.device_status() == mfp8.OK
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.isfinite(a.float()).all()


@pytest.mark.parametrize("M,path", [(32, mfp8.PATH_SPLITK), (112, mfp8.PATH_SPLITK), (200, mfp8.PATH_SPLITK),
                                    (200, mfp8.PATH_TILED), (512, mfp8.PATH_PAIR)])
def test_dependent_chain_every_path(M, path):
    """Each call is a quantize pass that lets its GEMM start early and a GEMM
    that waits for the codes; consecutive calls overlap the same way.  A
    chain where each Linear's input is the previous Linear's output must
    equal the same chain run one call at a time with a synchronisation in
    between, bit for bit."""
    H = 2048
    Ws = [mfp8.quantize_weight(W.make_w(H, H, seed=70 + i, device=DEV)) for i in range(5)]
    x0 = W.make_x(M, H, seed=71, kind="rowscale", device=DEV)
    ws = torch.zeros((mfp8.mfp8_linear_workspace_bytes(M, H, H),), dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()

    def chain(sync):
        x = x0
        for W8, sw in Ws:
            x = mfp8.linear(x, W8, sw, workspace=ws, path=path, flags=mfp8.FLAG_STATIC_WEIGHTS)
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return x

    a, b = chain(False), chain(True)
    assert mfp8.device_status() == mfp8.OK
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.isfinite(a.float()).all()


@pytest.mark.parametrize("M,N,K", TILED_ONLY + [(513, 776, 1024), (2048, 1024, 4096)])
@pytest.mark.parametrize("path", [mfp8.PATH_TILED, mfp8.PATH_PAIR])
def test_linear_tiled_ragged(M, N, K, path):
    run_case(M, N, K, path, seed=11, kind="rowscale")


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (130, 264, 384), (64, 1024, 4096), (100, 512, 1024)])
@pytest.mark.parametrize("path", [mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR])
def test_gemm_entry_point(M, N, K, path):
    """mfp8_gemm on codes from mfp8_quantize_act: within tolerance of the
    oracle, and bit-identical to mfp8_linear through the same kernel."""
    if path == mfp8.PATH_SPLITK and M > 256:
        pytest.skip("split-K takes M <= 256")
    x = W.make_x(M, K, seed=5, device=DEV)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=5, device=DEV))
    x8, xs = mfp8.quantize_act(x)
    y2 = mfp8.gemm(x8, xs, W8, sw, path=path)
    torch.cuda.synchronize()
    assert_linear_parity(y2, u8(x8), f32(xs), u8(W8), f32(sw), what="mfp8_gemm")
    if True:
        y = mfp8.linear(x, W8, sw, path=path)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_deterministic():
    for path in (mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR, mfp8.PATH_FUSED):
        x = W.make_x(16, 4096, seed=0, device=DEV)
        W8, sw = mfp8.quantize_weight(W.make_w(4096, 4096, seed=0, device=DEV))
        ys = [mfp8.linear(x, W8, sw, path=path) for _ in range(3)]
        torch.cuda.synchronize()
        assert all(torch.equal(ys[0].view(torch.int16), t.view(torch.int16)) for t in ys[1:])


@pytest.mark.parametrize("M,paths", [(37, (mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR)),
                                     (11, (mfp8.PATH_FUSED, mfp8.PATH_SPLITK))])
def test_onehot_weights_exact_product(M, paths):
    """W rows with one non-zero at column j_n give y[m,n] = dec(x8[m,j_n]) *
    448 * s_a[m] * s_w[n]: a single product, so even the bf16 rounding is
    fixed.  Checks the (m, n) mapping and the rescale of each kernel."""
    N, K = 264, 384
    g = torch.Generator().manual_seed(3)
    j = torch.randint(0, K, (N,), generator=g)
    c = torch.randn(N, generator=g) * 3
    w = torch.zeros(N, K)
    w[torch.arange(N), j] = c
    w = w.to(torch.bfloat16).to(DEV)
    x = W.make_x(M, K, seed=3, device=DEV)
    W8, sw = mfp8.quantize_weight(w)
    x8, xs = mfp8.quantize_act(x)
    xd = oracle.e4m3_decode(u8(x8))
    wd = oracle.e4m3_decode(u8(W8))
    expect = (xd[:, j.numpy()] * wd[np.arange(N), j.numpy()][None, :]
              * f32(xs)[:, None].astype(np.float64) * f32(sw)[None, :].astype(np.float64))
    expect_bf16 = torch.from_numpy(expect).to(torch.bfloat16)
    for path in paths:
        y = mfp8.linear(x, W8, sw, path=path).cpu()
        # one product, rounded once: equal unless the kernel's fp32 rounding of
        # the product lands on the other side of a bf16 tie
        diff = (y.double() - expect_bf16.double()).abs()
        ulp = expect_bf16.double().abs() * 2.0 ** -7
        assert (diff <= ulp).all()
        assert (y.view(torch.int16) == expect_bf16.view(torch.int16)).float().mean() > 0.99


@pytest.mark.parametrize("M,paths", [(20, (mfp8.PATH_TILED, mfp8.PATH_SPLITK, mfp8.PATH_PAIR)),
                                     (16, (mfp8.PATH_FUSED,))])
def test_zero_activation_rows_give_zero_outputs(M, paths):
    N, K = 256, 512
    x = W.make_x(M, K, seed=4, device=DEV)
    x[3] = 0
    x[M - 1] = 0
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=4, device=DEV))
    for path in paths:
        y = mfp8.linear(x, W8, sw, path=path)
        torch.cuda.synchronize()
        assert (y[3] == 0).all() and (y[M - 1] == 0).all()


def test_empty_m_is_a_noop():
    W8, sw = mfp8.quantize_weight(W.make_w(64, 64, seed=0, device=DEV))
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    y = mfp8.linear(x, W8, sw)
    assert y.shape == (0, 64)


# ---------------------------------------------------- full-size workloads --

def sampled_rows(M, n=48, seed=0):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(M, size=min(n, M), replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(r))


def rows_per_tile(M, tile=256, seed=0):
    """One random row in every `tile`-row block of M (the 256-row tiles of
    the CTA-pair kernel, so every tile and every lap of its persistent
    schedule meets the oracle), plus the first and last rows."""
    return rows_in_every_tile(M, tile, seed)


@pytest.mark.parametrize("lin", W.LAYER_LINEARS, ids=lambda l: l.name)
@pytest.mark.parametrize("path", [mfp8.PATH_AUTO, mfp8.PATH_FUSED])
def test_decode_layer_full_size(lin, path):
    """Decode: the 7 Linears of one layer at M in {1, 4, 8}, every output."""
    for M in (1, 4, 8):
        run_case(M, lin.N, lin.K, path, seed=1, kind="normal", flags=mfp8.FLAG_STATIC_WEIGHTS)


@pytest.mark.parametrize("lin", W.LAYER_LINEARS, ids=lambda l: l.name)
def test_prefill_layer_full_size_sampled(lin):
    """Prefill M=2048: every code and scale, sampled output rows."""
    M = 2048
    run_case(M, lin.N, lin.K, mfp8.PATH_AUTO, seed=2, kind="rowscale",
             rows=np.union1d(sampled_rows(M, 16, lin.N), rows_per_tile(M, seed=lin.N)))


@pytest.mark.parametrize("lin", W.MLP_LINEARS, ids=lambda l: l.name)
def test_long_video_full_size_sampled(lin):
    """M = 16384: every code and scale, and one output row in each of the 64
    row tiles."""
    M = 16384
    run_case(M, lin.N, lin.K, mfp8.PATH_AUTO, seed=3, kind="rowscale", rows=rows_per_tile(M, seed=lin.K))


def test_workspace_reused_across_calls_and_shapes():
    """One workspace serves a sequence of calls of different sizes and
    paths, whatever earlier calls left in it: each is within tolerance."""
    cases = [(16, 12288, 4096, mfp8.PATH_AUTO), (1, 4096, 4096, mfp8.PATH_SPLITK), (8, 1024, 4096, mfp8.PATH_AUTO),
             (40, 2048, 1024, mfp8.PATH_SPLITK), (300, 512, 1024, mfp8.PATH_TILED), (3, 4096, 4096, mfp8.PATH_AUTO),
             (16, 12288, 4096, mfp8.PATH_SPLITK)]
    nbytes = max(mfp8.mfp8_linear_workspace_bytes(M, N, K) for M, N, K, _ in cases)
    big = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)  # not zero-filled: nothing needs it
    for i, (M, N, K, path) in enumerate(cases):
        x = W.make_x(M, K, seed=30 + i, device=DEV)
        W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=30 + i, device=DEV))
        y = mfp8.linear(x, W8, sw, workspace=big, path=path, flags=mfp8.FLAG_STATIC_WEIGHTS)
        torch.cuda.synchronize()
        x8_ref, xs_ref = oracle.quantize_rows(bits16(x))
        assert_linear_parity(y, x8_ref, xs_ref, u8(W8), f32(sw), what=f"reuse {i}")
    assert mfp8.device_status() == mfp8.OK


# ------------------------------------------------------ packed projections --

PACKS = {"qkv_proj": W.LAYER_LINEARS[0:3], "gate_up_proj": W.LAYER_LINEARS[4:6]}


@pytest.mark.parametrize("pack", sorted(PACKS))
@pytest.mark.parametrize("M", [1, 4, 8, 16, 64, 2048])
def test_packed_projection_equals_the_separate_ones(pack, M):
    """The README's packed modules (qkv_proj, gate_up_proj) are exact under
    per-channel weight scales: quantizing the stacked weight rows gives the
    stacked codes and scales, the activation codes and scales are those of
    the separate calls, and each block of the packed output is the separate
    projection's output.  Where the kernel sums K in the same order for
    both (the tile kernels at M = 2048) the blocks are equal bit for bit;
    the split-K kernels choose their K split from N, so there the blocks are
    each within tolerance of the oracle."""
    parts = PACKS[pack]
    K = parts[0].K
    ws = [W.make_w(p.N, K, seed=5, stream=i, device=DEV) for i, p in enumerate(parts)]
    q = [mfp8.quantize_weight(w) for w in ws]
    W8p, swp = mfp8.quantize_weight(torch.cat(ws, 0))
    torch.cuda.synchronize()
    assert torch.equal(W8p, torch.cat([a for a, _ in q], 0))
    assert torch.equal(swp.view(torch.int32), torch.cat([b for _, b in q], 0).view(torch.int32))
    x = W.make_x(M, K, seed=5, stream=M, kind="rowscale", device=DEV)
    paths = [mfp8.PATH_AUTO] + ([mfp8.PATH_PAIR, mfp8.PATH_TILED] if M >= 256 else [])
    rows = rows_per_tile(M, seed=M) if M > 64 else None
    x8_ref, xs_ref = oracle.quantize_rows(bits16(x))
    for path in paths:
        def run(W8, sw):
            x8 = torch.empty((M, K), dtype=torch.uint8, device=DEV)
            xs = torch.empty((M,), dtype=torch.float32, device=DEV)
            y = mfp8.linear(x, W8, sw, path=path, x8_out=x8, xs_out=xs, flags=mfp8.FLAG_STATIC_WEIGHTS)
            return y, x8, xs
        yp, x8p, xsp = run(W8p, swp)
        sep = [run(a, b) for a, b in q]
        torch.cuda.synchronize()
        assert mfp8.device_status() == mfp8.OK
        assert np.array_equal(u8(x8p), x8_ref) and np.array_equal(f32(xsp).view(np.uint32), xs_ref.view(np.uint32))
        off = 0
        for p, (a, b), (y, x8, xs) in zip(parts, q, sep):
            assert torch.equal(x8, x8p) and torch.equal(xs.view(torch.int32), xsp.view(torch.int32))
            blk = yp[:, off:off + p.N]
            if path in (mfp8.PATH_PAIR, mfp8.PATH_TILED):
                assert torch.equal(blk.contiguous().view(torch.int16), y.view(torch.int16)), \
                    f"{pack} M={M} path={path}: block {p.name} differs from the separate call"
            else:
                assert_linear_parity(blk.contiguous(), x8_ref, xs_ref, u8(a), f32(b), rows=rows,
                                     what=f"{pack} block {p.name} M={M}")
                assert_linear_parity(y, x8_ref, xs_ref, u8(a), f32(b), rows=rows, what=f"{p.name} M={M}")
            off += p.N
