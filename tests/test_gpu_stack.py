"""The 252-Linear stack workload (36 self-attention layers x 7 projections,
per-layer weight std jittered by +-20%) swept at M in {1, 16, 128, 1024, 8192},
against the CPU oracle.

Weight and activation codes and scales are checked bit-exactly in full; the
BF16 outputs on sampled rows under the acceptance rule.  Three layers are
checked at every M (the first, a middle and the last self-attention layer),
so every projection shape meets every M with three different weight draws;
the oracle's exact contraction over all 252 Linears at M = 8192 would take
hours on the host."""
import numpy as np
import pytest
import torch

import oracle
from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W
from helpers import assert_linear_parity, bits16, f32, rows_in_every_tile, u8

pytestmark = pytest.mark.gpu
DEV = "cuda"
SEED = 4
STACK_MS = W.WORKLOADS[4]["Ms"]
JITTER = W.layer_std_jitter(SEED, len(W.SELF_LAYERS))
CHECKED_LAYERS = (0, len(W.SELF_LAYERS) // 2, len(W.SELF_LAYERS) - 1)  # indices into SELF_LAYERS


@pytest.mark.parametrize("M", STACK_MS)
def test_stack_layers_at_every_m(M):
    rng = np.random.default_rng(M)
    for li in CHECKED_LAYERS:
        for i, lin in enumerate(W.LAYER_LINEARS):
            x = W.make_x(M, lin.K, seed=SEED, stream=1000 * li + 10 * i + M, device=DEV)
            w = W.make_w(lin.N, lin.K, seed=SEED, stream=100 * li + i, std=0.02 * JITTER[li], device=DEV)
            W8, sw = mfp8.quantize_weight(w)
            x8 = torch.empty((M, lin.K), dtype=torch.uint8, device=DEV)
            xs = torch.empty((M,), dtype=torch.float32, device=DEV)
            y = mfp8.linear(x, W8, sw, x8_out=x8, xs_out=xs, flags=mfp8.FLAG_STATIC_WEIGHTS)
            torch.cuda.synchronize()
            assert mfp8.device_status() == mfp8.OK
            w8_ref, sw_ref = oracle.quantize_rows(bits16(w))
            assert np.array_equal(u8(W8), w8_ref)
            assert np.array_equal(f32(sw).view(np.uint32), sw_ref.view(np.uint32))
            x8_ref, xs_ref = oracle.quantize_rows(bits16(x))
            assert np.array_equal(u8(x8), x8_ref), f"layer {W.SELF_LAYERS[li]} {lin.name} M={M}: codes"
            assert np.array_equal(f32(xs).view(np.uint32), xs_ref.view(np.uint32))
            # every output row up to M = 128; above, one row in each row tile
            # of the kernel that runs (128 rows at M = 1024, the CTA-pair
            # kernel's 256 at M = 8192: every tile and persistent lap)
            rows = None if M <= 128 else rows_in_every_tile(M, 128 if M <= 1024 else 256,
                                                            seed=int(rng.integers(1 << 30)))
            assert_linear_parity(y, x8_ref, xs_ref, w8_ref, sw_ref, rows=rows,
                                 what=f"layer {W.SELF_LAYERS[li]} {lin.name} M={M}")
