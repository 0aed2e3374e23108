"""Helpers for the GPU parity tests: moving seeded inputs to the device and
comparing CUDA outputs with the oracle under the stated tolerance.

Tolerance (benchmark spec, per output element):
    |y - y_exact| <= 2e-3 * sum_k |s_g(k) x_k|           (``bound`` below)
With BF16 output the final rounding of y itself can reach 2^-8 |y|, which for
inputs with |y| close to ``bound`` (all products of one sign) exceeds that
budget on its own; ``allow_output_rounding`` adds it for such cases.  The
random workloads are checked with the strict bound."""
from __future__ import annotations

import numpy as np
import pytest

REL_TOL = 2e-3


def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(cuda())


def x_to_dev(x_bits: np.ndarray):
    import torch
    return to_dev(x_bits.astype(np.int16), torch.bfloat16)


def y_to_f64(y) -> np.ndarray:
    import torch
    return y.detach().to(torch.float64).cpu().numpy()


def check_close(y, yref: np.ndarray, bound: np.ndarray, out_dtype: str = "bf16",
                strict: bool = True, what: str = "") -> float:
    """Assert the tolerance; returns max err / (2e-3 * bound)."""
    yv = y_to_f64(y) if not isinstance(y, np.ndarray) else y.astype(np.float64)
    assert yv.shape == yref.shape, (yv.shape, yref.shape)
    err = np.abs(yv - yref)
    allow = REL_TOL * bound
    if not strict:
        if out_dtype == "bf16":
            allow = allow + 2.0 ** -8 * (np.abs(yref) + REL_TOL * bound)
        else:
            allow = allow + 2.0 ** -23 * np.abs(yref)
    bad = ~(err <= allow)
    if bad.any():
        i = np.argwhere(bad)[0]
        pytest.fail(f"{what}: {bad.sum()} of {bad.size} outputs out of tolerance; first at {tuple(i)}: "
                    f"got {yv[tuple(i)]!r} want {yref[tuple(i)]!r} bound {bound[tuple(i)]!r}")
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / (REL_TOL * bound), np.where(err > 0, np.inf, 0.0))
    return float(ratio.max()) if ratio.size else 0.0
