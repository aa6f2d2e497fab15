"""The batch-invariant dense layers (include/bi_model.h) against the fp64 oracle
(oracle/model_oracle.py), bit-for-bit invariance of every row across batch sizes and positions,
and the full-size linear layer of the 1.5B shape.

Tolerances, from the arithmetic:
* GEMM: the products of two bf16 values are exact in fp32; a sum of K of them in fp32, in any
  order, is within (K - 1) u sum_k |x_k w_k| of the exact sum (u = 2^-24), and rounding to bf16
  (8-bit significand) adds up to 2^-8 |y|.  The test allows K 2^-23 sum|x w| + 2^-7 |y|.
* RMSNorm: the fp32 sum of H squares is within H u of exact (relative), the rsqrt approximation
  within a few ulp, two fp32 products add 2u, the bf16 rounding up to 2^-8; the test allows
  (2^-7 + H 2^-24) |y|.
"""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import model_oracle as mo
from workloads import dense_inputs, norm_inputs

from .util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from async_rl_b200.build import build
    build()


def _f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def _check_gemm(x, w, y):
    ref = mo.gemm(x, w)
    K = x.shape[1]
    err = np.abs(_f64(y) - ref)
    bound = K * 2.0 ** -23 * mo.gemm_abs(x, w) + 2.0 ** -7 * np.abs(ref)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside; worst {float(np.max(err / np.maximum(bound, 1e-30))):.3g}; "
                           f"first {np.argwhere(bad)[:3].tolist()}")


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (7, 264, 136), (300, 520, 1536), (513, 8, 8),
                                   (256, 256, 4096), (1000, 1032, 200), (129, 776, 1544)])
def test_gemm_matches_oracle(M, N, K, cuda_device):
    """Ragged M, N and K: tiles that are part rows, part columns, part K chunk, and shapes smaller
    than one tile."""
    x, w = dense_inputs(M, K, N, seed=M * 7 + N + K)
    y, st = bi.gemm_bf16(x.to(cuda_device), w.to(cuda_device))
    torch.cuda.synchronize()
    bi.check_status(st)
    _check_gemm(x, w, y)


def test_gemm_closed_forms(cuda_device):
    """W = identity (Y = X exactly, every bf16 value representable) and a permutation of columns."""
    x, _ = dense_inputs(300, 512, 8, seed=11)
    eye = torch.eye(512, dtype=torch.bfloat16)
    y, st = bi.gemm_bf16(x.to(cuda_device), eye.to(cuda_device))
    torch.cuda.synchronize()
    bi.check_status(st)
    assert torch.equal(y.cpu(), x)
    perm = torch.randperm(512, generator=torch.Generator().manual_seed(3))[:264]
    p = torch.zeros(264, 512, dtype=torch.bfloat16)
    p[torch.arange(264), perm] = 1
    y, st = bi.gemm_bf16(x.to(cuda_device), p.to(cuda_device))
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), x[:, perm])


def test_gemm_empty_batch(cuda_device):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda_device)
    w = torch.ones(16, 64, dtype=torch.bfloat16, device=cuda_device)
    y, st = bi.gemm_bf16(x, w)
    torch.cuda.synchronize()
    assert y.shape == (0, 16) and int(st.item()) == 0


def test_gemm_rows_bitwise_invariant(cuda_device):
    """Each probe row's output has the same bits alone (M = 1, decode) and packed into batches of
    every size at random positions (both halves of a 256-row tile, tail tiles)."""
    K, N = 1536, 1032
    probes, w = dense_inputs(48, K, N, seed=5)
    w = w.to(cuda_device)
    probes = probes.to(cuda_device)
    alone = torch.cat([bi.gemm_bf16(probes[i:i + 1], w)[0] for i in range(probes.shape[0])])
    gen = torch.Generator().manual_seed(9)
    for M in (7, 256, 257, 1000, 4096):
        filler, _ = dense_inputs(M, K, 8, seed=M)
        x = filler.to(cuda_device)
        k = min(M, 48)
        pos = torch.randperm(M, generator=gen)[:k].to(cuda_device)
        x[pos] = probes[:k]
        y, st = bi.gemm_bf16(x, w)
        torch.cuda.synchronize()
        bi.check_status(st)
        assert torch.equal(y[pos], alone[:k]), f"a probe row changed bits at M = {M}"


def test_gemm_full_size_linear_layer(cuda_device):
    """The gate/up projection of the 1.5B shape: M = 76,239 rows, K = 1536, N = 8960, in the launch
    configuration the benchmark times; sampled rows against the oracle."""
    M, K, N = 76239, 1536, 8960
    x, w = dense_inputs(M, K, N, seed=1234)
    y, st = bi.gemm_bf16(x.to(cuda_device), w.to(cuda_device))
    torch.cuda.synchronize()
    bi.check_status(st)
    rows = np.unique(np.concatenate([np.random.default_rng(0).choice(M, 40, replace=False), [0, 255, 256, M - 1]]))
    _check_gemm(x[rows], w, y[torch.tensor(rows, device=cuda_device)])


def _check_norm(x, g, eps, y):
    ref = mo.rmsnorm(x, g, eps)
    H = x.shape[1]
    assert_close("rmsnorm", _f64(y), ref, 0.0, 2.0 ** -7 + H * 2.0 ** -24)


@pytest.mark.parametrize("M,H,eps", [(1, 1536, 1e-6), (7, 2048, 1e-5), (300, 2560, 1e-6), (1000, 8, 0.0),
                                     (33, 4104, 1e-2)])
def test_rmsnorm_matches_oracle(M, H, eps, cuda_device):
    x, g = norm_inputs(M, H, seed=M + H)
    y, st = bi.rmsnorm(x.to(cuda_device), g.to(cuda_device), eps)
    torch.cuda.synchronize()
    bi.check_status(st)
    _check_norm(x, g, eps, y)


def test_rmsnorm_zero_and_constant_rows(cuda_device):
    """A zero row with eps > 0 gives zeros; a constant row c gives c / sqrt(c^2 + eps) g."""
    H = 512
    x = torch.zeros(3, H, dtype=torch.bfloat16)
    x[1] = 2.0
    x[2] = -0.5
    g = torch.linspace(-2, 2, H).to(torch.bfloat16)
    y, st = bi.rmsnorm(x.to(cuda_device), g.to(cuda_device), 0.25)
    torch.cuda.synchronize()
    bi.check_status(st)
    assert torch.all(y[0] == 0)
    _check_norm(x, g, 0.25, y)


def test_rmsnorm_rows_bitwise_invariant(cuda_device):
    H = 1536
    probes, g = norm_inputs(40, H, seed=77)
    probes, g = probes.to(cuda_device), g.to(cuda_device)
    alone = torch.cat([bi.rmsnorm(probes[i:i + 1], g, 1e-6)[0] for i in range(40)])
    gen = torch.Generator().manual_seed(4)
    for M in (5, 64, 513, 20000):
        x, _ = norm_inputs(M, H, seed=M)
        x = x.to(cuda_device)
        k = min(M, 40)
        pos = torch.randperm(M, generator=gen)[:k].to(cuda_device)
        x[pos] = probes[:k]
        y, st = bi.rmsnorm(x, g, 1e-6)
        torch.cuda.synchronize()
        bi.check_status(st)
        assert torch.equal(y[pos], alone[:k]), f"a probe row changed bits at M = {M}"
