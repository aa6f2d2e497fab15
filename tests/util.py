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


def diag_bounds(lp_gpu, lp_ref, logmu, mask) -> dict:
    """Absolute error bounds of the D3 mean and the k1 / k2 means of one call, propagated from the
    measured per-row log-probability errors through the arithmetic the kernels use.

    Per scored row the device forms delta = fl32(lp - log mu) (log mu is the same fp32 value on
    both sides), so |delta_gpu - delta| <= e_t + 2^-24 |delta|, e_t = |lp_gpu - lp_ref|.  Then
      * d3 = expm1f(delta) - delta: first order |expm1(delta)| |d delta|, plus expm1f's error
        (<= 2 ulp of expm1) and the rounding of the subtraction, <= 2^-21 (|expm1 delta| + |delta|);
        the cancellation in expm1(delta) - delta is why the bound is absolute, not relative;
      * k1 = -delta: |d delta|;
      * k2 = delta^2 / 2 (formed in fp64 from the fp32 delta): |delta| |d delta| + |d delta|^2 / 2.
    The means are summed in fp64 and rounded to fp32 once (2^-24 of the result).  The factor 2 in
    front of the first-order terms covers the second-order terms of the expansion."""
    m = np.asarray(mask, dtype=bool)
    e = np.abs(np.asarray(lp_gpu, np.float64)[m] - np.asarray(lp_ref, np.float64)[m])
    delta = np.asarray(lp_ref, np.float64)[m] - np.asarray(logmu, np.float64)[m]
    dd = e + 2.0 ** -24 * np.abs(delta)
    em1 = np.abs(np.expm1(delta))
    n = max(1, int(m.sum()))
    d3 = np.expm1(delta) - delta
    k2 = 0.5 * delta * delta
    return {
        "d3": 2.0 * float(np.sum(em1 * dd)) / n + 2.0 ** -21 * float(np.sum(em1 + np.abs(delta))) / n
              + 2.0 ** -24 * abs(float(np.mean(d3))) + 1e-30,
        "k1": 2.0 * float(np.sum(dd)) / n + 2.0 ** -24 * abs(float(np.mean(delta))) + 1e-30,
        "k2": 2.0 * float(np.sum(np.abs(delta) * dd + 0.5 * dd * dd)) / n + 2.0 ** -24 * float(np.mean(k2)) + 1e-30,
    }


def to_dev(batch, device):
    b = batch.to(device)
    return b


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()
