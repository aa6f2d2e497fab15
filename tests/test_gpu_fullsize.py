"""Parity at the full sizes of the three loss workloads, in the launch configuration bench.py times
(the default path; the 1.5B shape also on the opt-in P store):

* 1.5B shape: H = 1536, V = 151936, 8 x 8 responses of U[256, 2048] rows (T = 76,239);
* 8K reasoning budget: H = 1536, 4 x 8 responses of U[1024, 8192] rows (about 147K rows);
* 4B shape, long context: H = 2560, 2 x 8 responses of 16,384 rows whose first 12,288 are prompt
  (262,144 rows, 65,536 scored).

The fp64 oracle cannot score 10^5 rows against a 152K vocabulary in a test's time, so it checks
outputs it can compute one by one (log pi, w and dH of sampled rows, with the batch's exact
coefficients), and the rest is checked through properties that hold at any size (dW columns sum
to zero because every row of dZ does; diff-0 over every row).  The rollout log-probabilities are
drawn by the test itself, so no oracle input comes from the CUDA path."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for

from .util import GRAD_TOL, LOGPROB_TOL, assert_close, assert_grad_close, f64

pytestmark = pytest.mark.gpu

# every workload on the default path (nothing of size T x V in memory; dW recomputes the logits),
# and the 1.5B shape once more on the opt-in P store
FULL_CASES = [("qwen1.5b", False), ("reason8k", False), ("qwen4b_lag64", False), ("qwen1.5b", True)]


@pytest.fixture(scope="module", params=FULL_CASES, ids=lambda c: c[0] + ("-pstore" if c[1] else ""))
def full(request, cuda_device):
    from async_rl_b200.build import build
    build()
    name, pstore = request.param
    b = make_batch(spec_for(name), with_w_roll=False)
    gen = torch.Generator().manual_seed(4242)
    mu = (torch.randn(b.n_rows, generator=gen) * 0.3 - 12.0).to(torch.float32)
    d = b.to(cuda_device)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, mu.to(cuda_device), d.rewards, d.resp_offsets,
                             d.group_offsets, d.prompt_lens, pstore=pstore)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    state = {"name": name, "pstore": pstore, "b": b, "mu": mu, "d": d, "out": out}
    yield state
    state.clear()
    del d, out
    torch.cuda.empty_cache()


def _scored_mask(b) -> np.ndarray:
    return orc.scored_rows(b.resp_offsets, b.prompt_lens, b.n_rows)


def _sample_rows(b, k, seed):
    """k scored rows at random plus the first and last scored rows; with prompts, 8 prompt rows too."""
    rng = np.random.default_rng(seed)
    scored = np.flatnonzero(_scored_mask(b))
    rows = [rng.choice(scored, size=k, replace=False), scored[[0, -1]]]
    if b.prompt_lens is not None:
        rows.append(rng.choice(np.flatnonzero(~_scored_mask(b)), size=8, replace=False))
    return np.unique(np.concatenate(rows))


def test_fullsize_sampled_logprob_and_dh(full):
    b, mu, out = full["b"], full["mu"], full["out"]
    rows = _sample_rows(b, 40, seed=7)
    sc = _scored_mask(b)[rows]
    hs, ys = b.hidden[rows], b.targets[rows]          # only the sampled rows are widened to fp64
    lp_ref, _ = orc.token_logprob(hs, b.w, ys)
    lp_ref = np.where(sc, lp_ref, 0.0)
    assert_close("logprob", f64(out.logprob)[rows], lp_ref, LOGPROB_TOL, LOGPROB_TOL)
    # the oracle's coefficients of the sampled rows: g_t = -c_i w_t with the batch's exact c_i
    A = orc.advantages(b.rewards, b.group_offsets)
    _, c = orc.response_coefficients(A, b.resp_offsets, b.prompt_lens)
    resp = np.searchsorted(b.resp_offsets.numpy(), rows, side="right") - 1
    w_ref = np.where(sc, np.exp(lp_ref - mu.double().numpy()[rows]), 0.0)
    assert_close("is_weight", f64(out.is_weight)[rows], w_ref, LOGPROB_TOL, LOGPROB_TOL)
    g = -c[resp] * w_ref
    dh_ref = orc.grad_rows(hs, b.w, ys, g, np.arange(rows.shape[0]))
    assert_grad_close("grad_hidden", f64(out.grad_hidden)[rows], dh_ref, GRAD_TOL)
    if not sc.all():
        assert torch.all(out.grad_hidden[torch.tensor(rows[~sc], device=out.grad_hidden.device)] == 0)


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
    exactly on every scored row (the logprob-only path and the loss path share their bits)."""
    b, d = full["b"], full["d"]
    lp, _, st = bi.logprob_fwd(d.hidden, d.w, d.targets)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, lp, d.rewards, d.resp_offsets, d.group_offsets,
                             d.prompt_lens, pstore=full["pstore"])
    torch.cuda.synchronize()
    bi.check_status(st)
    bi.check_status(out.status)
    sc = torch.tensor(_scored_mask(b), device=cuda_device)
    assert torch.equal(out.logprob[sc], lp[sc])
    assert torch.all(out.is_weight[sc] == 1.0)
    assert torch.all(out.logprob[~sc] == 0.0) and torch.all(out.is_weight[~sc] == 0.0)
    d3 = out.d3()
    assert d3["mean"] == 0.0 and d3["max"] == 0.0 and d3["k1"] == 0.0 and d3["count"] == int(sc.sum())
