"""Plain fp64 CPU oracle for the batch-invariant dense layers: the bf16 GEMM and RMSNorm.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it and shares no code
with it.

Sources (page title, then section):

* [ZM-gap]  "Zero Mismatch, Simple Async RL" -- section "Only one probability
            gap comes from old weights": kernel selection by batch shape,
            reduction order and different prefill/decode arithmetic change
            logprobs although the parameters are the same.
* [ZM-val]  "Zero Mismatch, Simple Async RL" -- section "Large-model validation
            exposes concrete failure mechanisms": shape-selected library kernels
            are one of the sources of batch variance.
* [RZ-cn]   "REINFORCE Zero: 为什么内核对齐后..." -- the paragraph before Fig. 2:
            trainer-inference invariance removes the kernel-mismatch term with
            batch-invariant kernels and a matched forward computation.

The pages give no layer formulas; the readings (each listed in the design notes):

* GEMM: Y = X W^T with X [M, K] and W [N, K] (the linear-layer layout), bf16
  inputs, fp32 accumulation on the device, Y rounded to bf16.  The oracle is the
  exact product in fp64 of the inputs widened to fp64; the device's accumulation
  and output rounding enter the tests as a tolerance, not as oracle arithmetic.
* RMSNorm: y_t = x_t / sqrt(mean_j x_tj^2 + eps) * g (the normalisation of the
  Qwen and Llama families), computed per row on the device in fp32 and rounded
  to bf16; the oracle evaluates the same definition in fp64.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    """Widen a numpy / torch array to float64 (exact for bf16 and fp32)."""
    try:
        import torch  # local: the oracle works on plain numpy too
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def gemm(x, w) -> np.ndarray:
    """Y[m, n] = sum_k X[m, k] W[n, k] in float64."""
    return _f64(x) @ _f64(w).T


def gemm_abs(x, w) -> np.ndarray:
    """sum_k |X[m, k]| |W[n, k]|: the scale of each output's accumulation rounding error."""
    return np.abs(_f64(x)) @ np.abs(_f64(w)).T


def rmsnorm(x, g, eps: float) -> np.ndarray:
    """y_t = x_t / sqrt(mean_j x_tj^2 + eps) * g, row by row, in float64."""
    X = _f64(x)
    G = _f64(g)
    ms = np.mean(X * X, axis=1, keepdims=True)
    return X / np.sqrt(ms + float(eps)) * G[None, :]
