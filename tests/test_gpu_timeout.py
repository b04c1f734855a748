"""The bounded device waits run out, report TTQ_ERR_TIMEOUT and leave the
context usable.

Every pipeline wait in the kernels (mbarrier phases, the statistic pass's
barrier among its blocks) gives up after a time limit instead of spinning
for ever.  A test hook makes one such wait that nothing can complete (an
mbarrier no one arrives on; a barrier told to expect one block more than
the grid has), with a limit of a few milliseconds, through the kernels' own
wait routines.  No GPU fault is involved: the wait simply ends.
"""
import time

import numpy as np
import pytest
import torch

import parity as P
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000   # 2 ms


@pytest.mark.parametrize("kind", [ttq.TTQ_TESTING_WAIT_MBARRIER, ttq.TTQ_TESTING_WAIT_GRID_BARRIER],
                         ids=["mbarrier", "grid_barrier"])
def test_wait_that_cannot_complete_times_out(kind):
    spec = synth.C2.with_(dp=0)
    ws = ttq.new_workspace(spec.d, 0, spec.T, 0, 4, 32)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ttq.ttq_testing_wait_timeout(kind, LIMIT_NS, 64, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 0.5, elapsed          # the wait ended on its own, near its limit
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_ERR_TIMEOUT and flags & ttq.TTQ_FLAG_TIMEOUT, (st, flags)
    header = ws[:4096].view(torch.int32).cpu().numpy()
    if kind == ttq.TTQ_TESTING_WAIT_GRID_BARRIER:
        # the barrier's counter is left off zero, as the header documents
        assert header[64] != 0

    # the context still works, and after ttq_workspace_init the same
    # workspace serves the fused statistic pass (which uses that counter)
    # exactly like a fresh one
    ttq.ttq_workspace_init(ws)
    X = P.to_dev(synth.generate(spec, need_w=False)["X"], "bf16")
    D, Dr, Xs = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha, ws=ws)
    D0, Dr0, Xs0 = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    assert torch.equal(D, D0) and torch.equal(Dr, Dr0)
    assert torch.equal(Xs.view(torch.int16), Xs0.view(torch.int16))
    assert not np.any(ws[:4096].view(torch.int32).cpu().numpy()[1:])   # counters back at zero


def test_wait_limit_bounds_are_checked():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for args in ((2, LIMIT_NS, 1), (0, 10, 1), (0, LIMIT_NS, 0), (1, LIMIT_NS, 149)):
        with pytest.raises(ttq.TTQError) as e:
            ttq.ttq_testing_wait_timeout(*args, ws)
        assert e.value.status == ttq.TTQ_ERR_INVALID_ARG, args
