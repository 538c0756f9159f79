"""mfp8_linear_noalloc: the Linear on the library's fixed scratch array,
through the C ABI, against mfp8_linear with a caller workspace.

Kept in a file collected last so that it runs both after every other GPU
test and, alone, in a fresh process (where its first call does the
per-device set-up)."""
import pytest
import torch

from fp8_w8a8_dynamic_b200 import mfp8
from fp8_w8a8_dynamic_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"

# decode sizes (the one-kernel path, no scratch), M = 64 (activation codes
# in the scratch, the cluster split-K kernel), a ragged mid-size M
# (128-row tiles), and a prefill-sized M (the CTA-pair kernel)
CASES = [(4, 1024, 4096), (16, 12288, 4096), (1, 4096, 12288), (64, 4096, 12288),
         (200, 4096, 4096), (1000, 4096, 4096)]


def _noalloc(x, W8, sw, y):
    M, K = x.shape
    N = W8.shape[0]
    return mfp8.mfp8_linear_noalloc(x.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)


def _with_workspace(x, W8, sw, y):
    M, K = x.shape
    N = W8.shape[0]
    nbytes = mfp8.mfp8_linear_workspace_bytes(M, N, K)
    ws = torch.zeros((nbytes,), dtype=torch.uint8, device=DEV)
    st = mfp8.mfp8_linear(x.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, y.data_ptr(), ws.data_ptr(),
                          nbytes, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def _same(y, y_ref):
    """Bit-equal: both calls take the same kernel for the same shape, and
    every kernel path is deterministic, so stale or misplaced scratch would
    show up as a changed bit."""
    return torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


@pytest.mark.parametrize("M,N,K", CASES)
def test_noalloc_matches_workspace_entry_point_twice(M, N, K):
    x = W.make_x(M, K, seed=31, stream=M, device=DEV)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=32, stream=N + K, device=DEV))
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    assert _with_workspace(x, W8, sw, y_ref) == mfp8.OK
    y1 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    assert _noalloc(x, W8, sw, y1) == mfp8.OK
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    assert _noalloc(x, W8, sw, y2) == mfp8.OK  # second call in a row, same scratch
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before  # nothing allocated
    assert mfp8.device_status() == mfp8.OK
    assert _same(y1, y_ref), "first no-alloc call differs from mfp8_linear"
    assert _same(y2, y_ref), "second no-alloc call differs from mfp8_linear"


def test_noalloc_back_to_back_different_shapes_on_one_stream():
    """Calls queued on one stream without a sync between them share the
    scratch in stream order."""
    shapes = [(8, 4096, 4096), (3, 12288, 4096), (8, 4096, 4096), (120, 1024, 4096)]
    runs = []
    for i, (M, N, K) in enumerate(shapes):
        x = W.make_x(M, K, seed=40 + i, device=DEV)
        W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=50 + i, device=DEV))
        runs.append((x, W8, sw, torch.empty((M, N), dtype=torch.bfloat16, device=DEV)))
    torch.cuda.synchronize()
    for x, W8, sw, y in runs:
        assert _noalloc(x, W8, sw, y) == mfp8.OK
    torch.cuda.synchronize()
    for x, W8, sw, y in runs:
        y_ref = torch.empty_like(y)
        assert _with_workspace(x, W8, sw, y_ref) == mfp8.OK
        assert _same(y, y_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    M, N, K = 2048, 1024, 12288  # codes alone: 24 MiB
    assert mfp8.mfp8_linear_workspace_bytes(M, N, K) > mfp8.STATIC_WORKSPACE_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    W8 = torch.zeros((N, K), dtype=torch.uint8, device=DEV)
    sw = torch.ones((N,), dtype=torch.float32, device=DEV)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device=DEV)
    assert _noalloc(x, W8, sw, y) == mfp8.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (y == 7.0).all()  # nothing ran
