"""Shared helpers for the GPU tests: run the CUDA path through the binding, run the oracle on
the same seeded inputs, and compare with the tolerances of the method's statement."""
from __future__ import annotations

import numpy as np
import torch

# tolerances: |gpu - oracle| <= atol + rtol * |oracle|
LOGPROB_TOL = 2e-3
LOSS_TOL = 5e-3
GRAD_TOL = 5e-3  # norm-wise: |d| <= GRAD_TOL * (max|oracle| + |oracle|)


def assert_close(name, got, ref, atol, rtol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; worst rel "
                             f"{float(np.max(err / np.maximum(bound, 1e-300))):.3g}; first {i.tolist()} "
                             f"got {got.ravel()[i].tolist()} ref {ref.ravel()[i].tolist()}")


def assert_grad_close(name, got, ref, tol=GRAD_TOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = tol * (scale + np.abs(ref))
    bad = ~(err <= bound)
    if bad.any():
        i = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance (scale {scale:.3g}); "
                             f"first {i.tolist()} got {got.ravel()[i].tolist()} ref {ref.ravel()[i].tolist()}")


def to_dev(batch, device):
    b = batch.to(device)
    return b


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()
