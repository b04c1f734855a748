"""The d'-sharded forward on two and three gloo ranks on the CPU: each rank
runs the oracle on its rows of W (the local compute is injected; on the GPU
it is the CUDA forward), the output columns are all-gathered, and the result
must equal the unsharded oracle forward bit for bit (every output row
depends on one row of W and on the full X only)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from test_weight_quantization_ttq_b200 import synth
from test_weight_quantization_ttq_b200.sharded import linear_forward_sharded, shard_rows


def test_shard_rows_cover_the_rows():
    for dp in (0, 1, 8, 200, 333, 4096, 4104):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_rows(dp, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == dp
            for (a, b), (c, _) in zip(spans, spans[1:]):
                assert b == c and a <= b
            # every shard that does not end the rows is a multiple of 8 rows
            assert all((b - a) % 8 == 0 for a, b in spans if b < dp)
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_local(X, W, A, B, p, lam, alpha, bits, group):
    import ttq_oracle
    out = ttq_oracle.get().forward(X.numpy().astype(np.float64), W.numpy(), p, lam, alpha, bits, group,
                                   A=None if A is None else A.numpy(), B=None if B is None else B.numpy())
    assert out["status"] == 0
    return torch.from_numpy(out["Y"])


def _rank_main(rank, world, port, spec, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        data = synth.generate(spec)
        a, b = shard_rows(spec.dp, world, rank)
        X = torch.from_numpy(data["X"])
        W = torch.from_numpy(np.ascontiguousarray(data["W"][a:b]))
        A = torch.from_numpy(data["A"]) if spec.r else None
        B = torch.from_numpy(np.ascontiguousarray(data["B"][a:b])) if spec.r else None
        Y = linear_forward_sharded(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                                   spec.dp, local_forward=_oracle_local)
        if rank == 0:
            result_q.put(Y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,spec", [
    (2, synth.LinearSpec("shard2", d=128, dp=200, T=9, bits=4, group=32, n_outliers=2, outlier_lo=20.0,
                         outlier_hi=50.0)),
    (3, synth.LinearSpec("shard3_lowrank", d=96, dp=70, T=5, bits=3, group=32, r=8, n_outliers=2,
                         outlier_lo=20.0, outlier_hi=50.0)),
])
def test_sharded_forward_equals_unsharded(world, spec):
    import ttq_oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, spec, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    Y = q.get(timeout=120)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    data = synth.generate(spec)
    ref = ttq_oracle.get().forward(data["X"].astype(np.float64), data["W"], spec.p, spec.lam, spec.alpha,
                                   spec.bits, spec.group, A=data.get("A"), B=data.get("B"))
    assert Y.shape == (spec.T, spec.dp)
    assert np.array_equal(Y, ref["Y"])


def _bench_rank_main(rank, world, port, result_q):
    import sys
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank timed a different number of milliseconds; the job's time
        # is the slowest rank's, on every rank
        ms = bench._max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        result_q.put((rank, ms, bench._job_throughput(world, 20, 2048, ms)))
    finally:
        dist.destroy_process_group()


def test_bench_times_the_job_by_its_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    assert [g[1] for g in got] == [15.0, 15.0]
    # two ranks x 20 steps x 2048 tokens in 15 ms
    assert all(abs(g[2] - 2 * 20 * 2048 / 0.015) < 1e-6 for g in got)
