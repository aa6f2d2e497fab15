"""Pins of the dense-layer oracle (oracle/model_oracle.py) against closed forms, brute force and
invariants, so that a plausible slip (a transposed operand, a sum for a mean, eps outside the
square root, a dropped gain) fails a test.  CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle import model_oracle as mo


def _bf16(a):
    return torch.tensor(np.asarray(a), dtype=torch.float32).to(torch.bfloat16)


def test_gemm_identity_returns_input_exactly():
    rng = np.random.default_rng(0)
    x = _bf16(rng.standard_normal((5, 16)))
    y = mo.gemm(x, torch.eye(16, dtype=torch.bfloat16))
    assert np.array_equal(y, x.double().numpy())


def test_gemm_permutation_selects_columns():
    """W = rows of a permutation matrix: Y[:, n] = X[:, perm[n]] (catches a transposed operand)."""
    rng = np.random.default_rng(1)
    K, N = 12, 7
    x = _bf16(rng.standard_normal((4, K)))
    perm = rng.permutation(K)[:N]
    w = torch.zeros(N, K, dtype=torch.bfloat16)
    w[torch.arange(N), torch.tensor(perm)] = 1
    y = mo.gemm(x, w)
    assert np.array_equal(y, x.double().numpy()[:, perm])


def test_gemm_constant_operands_closed_form():
    """X = a everywhere, W = b everywhere: every output is K a b."""
    M, N, K, a, b = 3, 5, 96, 0.75, -1.5
    y = mo.gemm(torch.full((M, K), a, dtype=torch.bfloat16), torch.full((N, K), b, dtype=torch.bfloat16))
    assert np.all(y == K * a * b)


def test_gemm_brute_force_triple_loop():
    rng = np.random.default_rng(2)
    M, N, K = 3, 4, 5
    x = rng.integers(-4, 5, size=(M, K)).astype(np.float64)
    w = rng.integers(-4, 5, size=(N, K)).astype(np.float64)
    ref = [[sum(x[m][k] * w[n][k] for k in range(K)) for n in range(N)] for m in range(M)]
    assert np.array_equal(mo.gemm(x, w), np.array(ref))


def test_gemm_abs_bounds_the_product():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 40))
    w = rng.standard_normal((9, 40))
    assert np.all(np.abs(mo.gemm(x, w)) <= mo.gemm_abs(x, w) + 1e-12)
    assert np.array_equal(mo.gemm_abs(np.abs(x), np.abs(w)), mo.gemm(np.abs(x), np.abs(w)))


@pytest.mark.parametrize("c,eps", [(3.0, 0.0), (-0.5, 1e-6), (2.0, 0.25)])
def test_rmsnorm_constant_row_closed_form(c, eps):
    """x = c everywhere: mean(x^2) = c^2, so y_j = c / sqrt(c^2 + eps) g_j (a sum for the mean or
    eps outside the root breaks this for H > 1)."""
    H = 64
    g = np.linspace(-2.0, 2.0, H)
    y = mo.rmsnorm(np.full((1, H), c), g, eps)
    assert np.allclose(y[0], c / math.sqrt(c * c + eps) * g, rtol=1e-15, atol=0)


def test_rmsnorm_unit_gain_has_unit_mean_square():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((8, 300)) * rng.uniform(0.1, 10.0, size=(8, 1))
    y = mo.rmsnorm(x, np.ones(300), 0.0)
    assert np.allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-13)


def test_rmsnorm_scale_invariance_without_eps():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 128))
    g = rng.standard_normal(128)
    assert np.allclose(mo.rmsnorm(37.0 * x, g, 0.0), mo.rmsnorm(x, g, 0.0), rtol=1e-13, atol=0)


def test_rmsnorm_brute_force_loops():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, 5))
    g = rng.standard_normal(5)
    eps = 1e-3
    ref = []
    for row in x:
        r = math.sqrt(sum(v * v for v in row) / len(row) + eps)
        ref.append([row[j] / r * g[j] for j in range(len(row))])
    assert np.allclose(mo.rmsnorm(x, g, eps), np.array(ref), rtol=1e-14, atol=0)


def test_rmsnorm_zero_row_and_row_independence():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 32))
    x[2] = 0.0
    g = rng.standard_normal(32)
    y = mo.rmsnorm(x, g, 1e-6)
    assert np.all(y[2] == 0.0)
    for r in range(5):
        assert np.array_equal(mo.rmsnorm(x[r:r + 1], g, 1e-6)[0], y[r])


def test_dense_input_generators_are_seeded_and_follow_the_recipe():
    """The seeded generators behind the dense-layer tests and the dense bench: deterministic, bf16,
    and the stated distributions (x ~ N(0, 1), W ~ N(0, 0.02); RMSNorm rows N(0, s^2) with
    s ~ U[0.05, 20], gains 1 + N(0, 0.1))."""
    from workloads import dense_inputs, norm_inputs
    x1, w1 = dense_inputs(2000, 512, 300, seed=7)
    x2, w2 = dense_inputs(2000, 512, 300, seed=7)
    assert torch.equal(x1, x2) and torch.equal(w1, w2)
    assert x1.dtype == torch.bfloat16 and w1.shape == (300, 512)
    assert abs(float(x1.float().std()) - 1.0) < 0.01 and abs(float(w1.float().std()) - 0.02) < 0.001
    x, g = norm_inputs(4000, 256, seed=8)
    assert torch.equal(x, norm_inputs(4000, 256, seed=8)[0]) and g.shape == (256,)
    # a row's RMS is s times the RMS of 256 standard normals (within a few percent of 1)
    s = x.float().pow(2).mean(dim=1).sqrt()
    assert float(s.min()) > 0.05 * 0.8 and float(s.max()) < 20.0 * 1.25 and float(s.median()) > 5.0
    assert abs(float(g.float().mean()) - 1.0) < 0.03 and 0.07 < float(g.float().std()) < 0.13
