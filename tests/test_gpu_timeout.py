"""The bounded device waits run out, report TTQ_ERR_TIMEOUT and leave the
context usable.

Every pipeline wait in the kernels (the mbarrier phases of the product
kernels' TMA and tensor-core pipelines) gives up after a time limit instead
of spinning for ever.  A test hook makes one such wait that nothing can
complete (an mbarrier no one arrives on), with a limit of a few
milliseconds, through the kernels' own wait routine.  No GPU fault is
involved: the wait simply ends.
"""
import time

import numpy as np
import pytest
import torch

import parity as P
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000   # 2 ms


def test_wait_that_cannot_complete_times_out():
    spec = synth.C2.with_(dp=0)
    ws = ttq.new_workspace(spec.d, 0, spec.T, 0, 4, 32)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ttq.ttq_testing_wait_timeout(ttq.TTQ_TESTING_WAIT_MBARRIER, LIMIT_NS, 64, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 0.5, elapsed          # the wait ended on its own, near its limit
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_ERR_TIMEOUT and flags & ttq.TTQ_FLAG_TIMEOUT, (st, flags)
    # the context still works, and after ttq_workspace_init the same
    # workspace serves the statistic pass (whose merge tickets are the
    # counters that follow the status word) exactly like a fresh one
    ttq.ttq_workspace_init(ws)
    X = P.to_dev(synth.generate(spec, need_w=False)["X"], "bf16")
    D, Dr = ttq.ttq_act_norm(X, spec.p, spec.lam, spec.alpha, ws=ws)
    D0, Dr0 = ttq.ttq_act_norm(X, spec.p, spec.lam, spec.alpha)
    Ds, Drs, Xs = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha, ws=ws)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    assert torch.equal(D, D0) and torch.equal(Dr, Dr0)
    assert torch.equal(Ds, D0) and torch.equal(Drs, Dr0)
    assert not np.any(ws[:4096].view(torch.int32).cpu().numpy()[1:])   # counters back at zero


def test_wait_limit_bounds_are_checked():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for args in ((1, LIMIT_NS, 1), (0, 10, 1), (0, LIMIT_NS, 0), (0, LIMIT_NS, 149)):
        with pytest.raises(ttq.TTQError) as e:
            ttq.ttq_testing_wait_timeout(*args, ws)
        assert e.value.status == ttq.TTQ_ERR_INVALID_ARG, args
