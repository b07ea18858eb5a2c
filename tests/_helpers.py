"""Shared helpers for the parity tests: numpy <-> torch marshalling and tolerance checks.

Inputs come from `synth` (seeded); expected values come only from `oracle`.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

# Tolerances stated for the Lightning Attention forward: max|o - o_ref| relative to max|o_ref|.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(a: np.ndarray, device="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t) -> np.ndarray:
    import torch
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return synth.bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    got64 = as_f64(got)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got64).max())
    return float(np.abs(got64 - ref).max() / scale)


# Parity margins of the full-size workloads, printed in the session's terminal summary so
# that a passing run still records how far inside the tolerance each one landed.
MARGINS: list[tuple[str, str]] = []


def record_margin(name: str, **ratios: float) -> None:
    """Keep max|err|/max|ref| figures of one test for the end-of-run summary."""
    MARGINS.append((name, "  ".join(f"{k}={v:.3e}" for k, v in ratios.items())))


def assert_close(got, ref, dtype: str, what: str = "output"):
    e = rel_err(got, ref)
    assert np.all(np.isfinite(as_f64(got))), f"{what}: non-finite values"
    assert e <= TOL[dtype], f"{what}: max|err|/max|ref| = {e:.3e} > {TOL[dtype]:.0e}"
    return e


def mode_code(mode: str) -> int:
    return {"raw": oracle.MODE_RAW, "rmsnorm": oracle.MODE_RMSNORM, "rmsnorm_gate": oracle.MODE_RMSNORM_GATE}[mode]
