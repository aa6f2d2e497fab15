"""Parity at the full size of the throughput workload (H = 1536, V = 151936, 8 x 8 responses of
U[256, 2048] rows, T = 76,239), in the launch configuration bench.py times.

The fp64 oracle cannot score 76K rows against a 152K vocabulary in a test's time, so it checks
outputs it can compute one by one (log pi and dH of sampled rows, with the batch's exact
coefficients), and the rest is checked through properties that hold at any size (dW columns sum
to zero because every row of dZ does; diff-0).  The rollout log-probabilities are drawn by the
test itself, so no oracle input comes from the CUDA path."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for

from .util import GRAD_TOL, LOGPROB_TOL, assert_close, assert_grad_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def full(cuda_device):
    from async_rl_b200.build import build
    build()
    b = make_batch(spec_for("qwen1.5b"), with_w_roll=False)
    gen = torch.Generator().manual_seed(4242)
    mu = (torch.randn(b.n_rows, generator=gen) * 0.3 - 12.0).to(torch.float32)
    d = b.to(cuda_device)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, mu.to(cuda_device), d.rewards, d.resp_offsets,
                             d.group_offsets)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    return {"b": b, "mu": mu, "d": d, "out": out}


def _sample_rows(n_rows, k, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(n_rows, size=k, replace=False)
    return np.sort(np.concatenate([rows, [0, n_rows - 1]]))


def test_fullsize_sampled_logprob_and_dh(full):
    b, mu, out = full["b"], full["mu"], full["out"]
    rows = _sample_rows(b.n_rows, 40, seed=7)
    lp_ref, _ = orc.token_logprob(b.hidden, b.w, b.targets, rows=rows)
    assert_close("logprob", f64(out.logprob)[rows], lp_ref, LOGPROB_TOL, LOGPROB_TOL)
    # the oracle's coefficients of the sampled rows: g_t = -c_i w_t with the batch's exact c_i
    A = orc.advantages(b.rewards, b.group_offsets)
    _, c = orc.response_coefficients(A, b.resp_offsets, None)
    off = b.resp_offsets.numpy()
    resp = np.searchsorted(off, rows, side="right") - 1
    w_ref = np.exp(lp_ref - mu.double().numpy()[rows])
    assert_close("is_weight", f64(out.is_weight)[rows], w_ref, LOGPROB_TOL, LOGPROB_TOL)
    g = -c[resp] * w_ref
    dh_ref = orc.grad_rows(b.hidden, b.w, b.targets, g, rows)
    assert_grad_close("grad_hidden", f64(out.grad_hidden)[rows], dh_ref, GRAD_TOL)


def test_fullsize_dw_columns_sum_to_zero(full):
    """sum_v dW[v, :] = sum_t (sum_v dZ_tv) h_t = 0: each column sum is small against the column's
    absolute mass (what is left is the rounding of bf16 dZ)."""
    gw = full["out"].grad_w
    col = gw.double().sum(dim=0)
    mass = gw.double().abs().sum(dim=0)
    assert torch.all(col.abs() <= 2e-3 * mass + 1e-12), float((col.abs() / mass).max())
    assert torch.isfinite(gw).all()


def test_fullsize_diff_zero(full, cuda_device):
    """Rollout logprobs from the library's own forward on the same packed batch: w == 1 and D3 == 0
    exactly for all 76K rows (the logprob-only path and the loss path share their bits)."""
    d = full["d"]
    lp, _, st = bi.logprob_fwd(d.hidden, d.w, d.targets)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, lp, d.rewards, d.resp_offsets, d.group_offsets)
    torch.cuda.synchronize()
    bi.check_status(st)
    bi.check_status(out.status)
    assert torch.equal(out.logprob, lp)
    assert torch.all(out.is_weight == 1.0)
    d3 = out.d3()
    assert d3["mean"] == 0.0 and d3["max"] == 0.0 and d3["k1"] == 0.0 and d3["count"] == d.n_rows
