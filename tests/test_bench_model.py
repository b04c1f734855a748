"""The bench's floor model (CPU): the lower bound on one forward from the
method's algorithmic bytes and flops at given peaks, against the worked
values derived by hand from the cost model (statistic and quantiser at HBM
bandwidth, the product at the slower of its bytes and flops), and the
workload points the table mode covers."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from test_weight_quantization_ttq_b200 import synth  # noqa: E402

HBM = 6534.5e9     # bytes/s
TC = 1631.9e12     # flop/s


def _hand(d, dp, T, b, g, r=0, e=2):
    """The same floor written out term by term."""
    x_in, x_scaled, d_out = e * d * T, 2 * d * T, 8 * d
    w_in, codes_out, sz_out, d_in = e * dp * d, dp * d * b / 8, 4 * dp * d / g, 4 * d
    prod_bytes = dp * d * b / 8 + 4 * dp * d / g + 2 * d * T + e * T * dp
    if r:
        prod_bytes += 2 * r * (d + dp) + 2 * r * T
    flops = 2 * dp * d * T + 2 * r * (d + dp) * T
    first = (x_in + x_scaled + d_out + w_in + codes_out + sz_out + d_in) / HBM
    return 1e6 * (first + max(prod_bytes / HBM, flops / TC))


@pytest.mark.parametrize("spec,want_us", [
    (synth.C4.with_(T=1), 27.5),        # decode: the quantiser's pass over W dominates
    (synth.C5.with_(T=1), 95.1),
    (synth.C5.with_(T=4096), 1294.6),   # compute-bound product
    (synth.C3_GATE, 46.5),
])
def test_floor_matches_the_cost_model(spec, want_us):
    got, nbytes, flops = bench._floor_us(spec, HBM, TC)
    assert got == pytest.approx(_hand(spec.d, spec.dp, spec.T, spec.bits, spec.group, spec.r), rel=1e-12)
    assert got == pytest.approx(want_us, abs=0.1)
    assert flops == 2.0 * spec.dp * spec.d * spec.T + 2.0 * spec.r * (spec.d + spec.dp) * spec.T


def test_floor_grows_with_tokens_and_counts_float32_inputs():
    a = bench._floor_us(synth.C5.with_(T=16), HBM, TC)[0]
    b = bench._floor_us(synth.C5.with_(T=1024), HBM, TC)[0]
    assert b > a
    f32 = bench._floor_us(synth.C1, HBM, TC)[1]
    bf16 = bench._floor_us(synth.C1.with_(dtype="bf16"), HBM, TC)[1]
    # float32 X, W and Y move twice the bytes of their bf16 forms
    d, dp, T = synth.C1.d, synth.C1.dp, synth.C1.T
    assert f32 - bf16 == pytest.approx(2 * (d * T + dp * d + T * dp))
