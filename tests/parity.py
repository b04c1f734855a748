"""Helpers shared by the GPU parity tests: move seeded inputs to the device
and compare the CUDA path with the oracle."""
from __future__ import annotations

import numpy as np
import torch

from test_weight_quantization_ttq_b200 import synth

# Y tolerance of the layer: max |dY| <= 1e-2 * rms(Y_oracle) (bf16 operands,
# fp32 accumulation).  D tolerance: 1e-5 relative.
Y_TOL = 1e-2
D_RTOL = 1e-5


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def y_error(y_gpu: np.ndarray, y_ref: np.ndarray) -> float:
    """max |dY| / rms(Y_ref)."""
    rms = float(np.sqrt(np.mean(y_ref.astype(np.float64) ** 2)))
    if rms == 0.0:
        return float(np.abs(y_gpu).max()) if y_gpu.size else 0.0
    return float(np.abs(y_gpu.astype(np.float64) - y_ref).max()) / rms


def f32(v: float) -> float:
    """The binary32 value the C ABI receives for a float parameter (p,
    lambda, alpha); the oracle is given the same value."""
    return float(np.float32(v))


def params(spec: synth.LinearSpec) -> tuple[float, float, float]:
    return f32(spec.p), f32(spec.lam), f32(spec.alpha)


def inputs(spec: synth.LinearSpec, need_w: bool = True) -> dict:
    return synth.generate(spec, need_w=need_w)


_weights_cache: dict = {}


def inputs_shared_w(spec: synth.LinearSpec) -> dict:
    """synth.generate(spec), with W, A and B drawn once per weight recipe and
    reused across calls that differ only in T, p or alpha (those never
    change the weight's draw: it comes from its own seeded stream).  One
    recipe is kept at a time, so consecutive cases of one workload share it."""
    key = spec.with_(T=1, p=2.0, alpha=0.5, lam=1e-3)
    if key not in _weights_cache:
        _weights_cache.clear()
        full = synth.generate(spec.with_(T=1))
        _weights_cache[key] = {k: full[k] for k in ("W", "A", "B") if k in full}
    out = synth.generate(spec, need_w=False)
    out.update(_weights_cache[key])
    return out
