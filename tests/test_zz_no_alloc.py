"""The allocation-free statistic entry point (ttq_act_norm_noalloc).

It exists for callers that cannot allocate device memory, such as a plug-in
living inside another framework's memory manager or a real-time loop that
must not allocate after start-up; it uses a fixed scratch array compiled
into the library instead of a caller workspace.  Its results must equal
those of ttq_act_norm, which uses a caller workspace, on consecutive calls
(the shared array keeps the previous call's contents, so a second call shows
that nothing stale leaks through).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import ttq_oracle
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu

D_RTOL = 1e-5  # the statistic's tolerance throughout the parity tests


def _check_oracle(got, ref):
    got = got.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)) and np.max(np.abs(got - ref) / np.abs(ref)) <= D_RTOL


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point(dtype):
    O = ttq_oracle.get()
    specs = [synth.LinearSpec("noalloc_a", d=4096, dp=0, T=2048, bits=4, group=128, dtype=dtype,
                              n_outliers=40, outlier_lo=20.0, outlier_hi=100.0, seed=3),
             synth.LinearSpec("noalloc_b", d=264, dp=0, T=45, bits=4, group=8, dtype=dtype, p=3.0,
                              n_outliers=3, seed=4)]
    for spec in specs:  # two calls in a row through the same scratch array
        x = synth.generate(spec, need_w=False)["X"]
        X = torch.from_numpy(x).cuda()
        X = X.to(torch.bfloat16) if dtype == "bf16" else X
        D0, Dr0 = ttq.ttq_act_norm(X, spec.p, spec.lam, spec.alpha)
        D1, Dr1 = ttq.ttq_act_norm_noalloc(X, spec.p, spec.lam, spec.alpha)
        torch.cuda.synchronize()
        # the same split plan, kernel and merge order as the workspace entry
        # point: the same bits
        assert torch.equal(D1, D0) and torch.equal(Dr1, Dr0)
        # and the oracle's D, D^(-1/2) within the statistic's tolerance
        pf, lf, af = (float(np.float32(v)) for v in (spec.p, spec.lam, spec.alpha))
        D_ref, Dr_ref, st = O.act_norm(x.astype(np.float64), pf, lf, af)
        assert st == 0
        _check_oracle(D1, D_ref)
        _check_oracle(Dr1, Dr_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    X = torch.zeros((4, 16392), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ttq.TTQError) as e:
        ttq.ttq_act_norm_noalloc(X, 2.0, 1e-3, 0.5)
    assert e.value.status == ttq.TTQ_ERR_UNSUPPORTED
