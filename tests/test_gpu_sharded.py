"""The d'-sharded forward with the CUDA local compute, on the one GPU a
test run has: a one-rank NCCL group (the gather is then a copy), so the
sharded entry point must equal ttq_linear_forward bit for bit.  More ranks
are covered on the CPU with gloo (tests/test_sharded.py)."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist

import parity as P
from test_weight_quantization_ttq_b200 import synth, ttq
from test_weight_quantization_ttq_b200.sharded import linear_forward_sharded

pytestmark = pytest.mark.gpu


def test_one_rank_sharded_forward_equals_forward():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        spec = synth.LinearSpec("shard1", d=512, dp=264, T=40, bits=4, group=64, r=16, n_outliers=2,
                                outlier_lo=20.0, outlier_hi=50.0)
        data = P.inputs(spec)
        X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
        A, B = P.to_dev(data["A"], "bf16"), P.to_dev(data["B"], "bf16")
        Y = linear_forward_sharded(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                                   spec.dp, y_dtype=torch.float32)
        Y_ref = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                                       y_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y_ref)
    finally:
        dist.destroy_process_group()
