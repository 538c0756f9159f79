"""The N > 1 path on CPU: two `gloo` ranks, as `bench.py` runs them under
torchrun with NCCL on GPUs.

The Linear partitions by tokens: the per-token scale is a function of the
token's own row, so a batch split into row blocks across ranks quantizes and
multiplies to the same bytes and values as the whole batch on one device.
The test checks that property with the oracle on each rank's block (gathered
on rank 0 and compared with the oracle on the whole batch), and the host
logic the bench wraps around its timed region: the barrier, the max over
ranks of a timing, whole-job throughput and per-rank input seeds."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2
M, N, K = 12, 48, 256  # 6 token rows per rank


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(WORLD))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    import oracle
    from fp8_w8a8_dynamic_b200 import workloads as W

    ctx = bench.DistCtx(torch, backend="gloo")
    assert (ctx.world, ctx.rank) == (WORLD, rank)
    dist = ctx.dist

    # max over ranks of a per-rank timing, as the bench reports it
    assert ctx.max(1.5 + rank) == 1.5 + WORLD - 1
    ctx.barrier()

    # every rank's batch is its own draw
    seeds = [None] * WORLD
    dist.all_gather_object(seeds, bench.rank_seed(1, rank))
    assert len(set(seeds)) == WORLD

    # data-parallel rows: this rank's block of the whole batch
    x = W.make_x(M, K, seed=7, stream=1, kind="rowscale")
    w = W.make_w(N, K, seed=7, stream=2)
    rows = slice(rank * M // WORLD, (rank + 1) * M // WORLD)
    xb = x[rows].contiguous().view(torch.int16).numpy().view(np.uint16)
    wb = w.contiguous().view(torch.int16).numpy().view(np.uint16)
    w8, s_w = oracle.quantize_rows(wb)
    x8, s_a = oracle.quantize_rows(xb)
    y, _ = oracle.linear_ref(x8, s_a, w8, s_w)
    parts = [None] * WORLD
    dist.gather_object((x8, s_a, y), parts if rank == 0 else None, dst=0)
    if rank == 0:
        np.savez(os.path.join(out_dir, "parts.npz"),
                 x8=np.concatenate([p[0] for p in parts]), s_a=np.concatenate([p[1] for p in parts]),
                 y=np.concatenate([p[2] for p in parts]))
    ctx.barrier()
    ctx.close()


def test_two_gloo_ranks_split_tokens_exactly(tmp_path):
    tmp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                        start_method="spawn")
    import oracle
    from fp8_w8a8_dynamic_b200 import workloads as W
    x = W.make_x(M, K, seed=7, stream=1, kind="rowscale")
    w = W.make_w(N, K, seed=7, stream=2)
    w8, s_w = oracle.quantize_rows(w.view(torch.int16).numpy().view(np.uint16))
    x8, s_a = oracle.quantize_rows(x.view(torch.int16).numpy().view(np.uint16))
    y, _ = oracle.linear_ref(x8, s_a, w8, s_w)
    got = np.load(tmp_path / "parts.npz")
    assert np.array_equal(got["x8"], x8)
    assert np.array_equal(got["s_a"].view(np.uint32), s_a.view(np.uint32))
    assert np.array_equal(got["y"], y)  # fp64 per element: the same value bit for bit


def test_job_throughput_counts_all_ranks_against_the_slowest():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 3 GB in 1.5 s (the slower rank) -> 4 GB/s
    assert bench.job_throughput(3e9, 2, 1500.0) == pytest.approx(4e9)
    assert bench.job_throughput(3e9, 1, 1500.0) == pytest.approx(2e9)
    assert bench.rank_seed(1, 0) != bench.rank_seed(1, 1)
