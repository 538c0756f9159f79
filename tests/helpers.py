"""Shared test helpers: host copies of device tensors and the parity check."""
import numpy as np
import torch

import oracle


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint8)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().float().cpu().numpy()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_linear_parity(y_gpu: torch.Tensor, x8: np.ndarray, s_a: np.ndarray, w8: np.ndarray,
                         s_w: np.ndarray, rows=None, what=""):
    """Y from the GPU against the oracle's exact rescaled product on the
    given rows (all rows when None), under the acceptance rule
    |y - y_ref| <= 2^-7 |y_ref| + 1e-5 * s_abs."""
    if rows is not None:
        x8, s_a = x8[rows], s_a[rows]
        y = bf16_to_f64(y_gpu[torch.as_tensor(rows, device=y_gpu.device)])
    else:
        y = bf16_to_f64(y_gpu)
    y_ref, s_abs = oracle.linear_ref(x8, s_a, w8, s_w)
    ok = oracle.within_tolerance(y, y_ref, s_abs)
    if not ok.all():
        bad = np.argwhere(~ok)
        m, n = bad[0]
        raise AssertionError(
            f"{what}: {bad.shape[0]} of {ok.size} outputs outside tolerance; first at (row {m}, col {n}): "
            f"gpu {y[m, n]!r} ref {y_ref[m, n]!r} s_abs {s_abs[m, n]!r}")
    assert np.isfinite(y).all()


def rows_in_every_tile(M, tile=256, seed=0):
    """One random row in every `tile`-row block of M rows, plus rows 0 and
    M - 1, sorted."""
    rng = np.random.default_rng(seed)
    starts = np.arange(0, M, tile)
    picks = starts + rng.integers(0, tile, starts.size)
    picks = np.minimum(picks, M - 1)
    return np.union1d(picks, [0, M - 1])
