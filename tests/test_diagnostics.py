"""Host-side update tracker against the oracle's order statistics (CPU), and a simulated run
through the CUDA path where injected logprob mismatch spikes the D3 peak/median (GPU)."""
import math

import numpy as np
import pytest
import torch

from async_rl_b200.diagnostics import UpdateTracker
from oracle import isloss_oracle as orc


def _fake(d3, k1, k2, rej=0, n=100):
    return {"mean": d3, "k1": k1, "k2": k2, "n_rejected": rej, "count": n}


def test_tracker_matches_oracle_statistics():
    rng = np.random.default_rng(4)
    d3 = rng.gamma(2.0, 1e-4, size=41)
    d3[17] = 0.5  # one excursion
    k1 = rng.normal(1e-4, 2e-5, size=41)
    tr = UpdateTracker()
    for a, b in zip(d3, k1):
        tr.add(_fake(a, b, b * b))
    ref = orc.d3_peak_median(d3)
    assert math.isclose(tr.d3_peak_over_median(), ref["ratio"], rel_tol=1e-15)
    assert math.isclose(tr.kl_drift(10), orc.kl_drift(d3, 10), rel_tol=1e-15)
    assert math.isclose(tr.kl_drift(7, "k1"), orc.kl_drift(k1, 7), rel_tol=1e-15)
    with pytest.raises(ValueError):
        tr.kl_drift(42)


def test_tracker_rejection_rate():
    tr = UpdateTracker()
    for rej in (0, 1, 3, 2):
        tr.add(_fake(1.0, 0.0, 0.0, rej))
    assert tr.rejection_rate([10, 10, 10, 10], 2) == 5 / 20


@pytest.mark.gpu
def test_simulated_updates_aligned_vs_mismatched(cuda_device):
    """Twelve updates of a small step.  Aligned: the rollout logprobs come from the library's own
    forward under lagged weights, so D3 moves smoothly.  Mismatched: the same, with an execution
    mismatch injected (noise on the rollout logprobs) on two updates.  The tracker's peak/median
    separates the two runs, and each update's D3 equals the oracle's D3 of that update."""
    import async_rl_b200 as bi
    from workloads import make_batch, spec_for

    spec = spec_for("tiny", H=256, V=3001, groups=2, per_group=4, len_lo=16, len_hi=48)
    runs = {}
    for name, spikes in (("aligned", ()), ("mismatched", (5, 9))):
        tr = UpdateTracker()
        for u in range(12):
            b = make_batch(spec, seed=500 + u).to(cuda_device)
            mu, _, st = bi.logprob_fwd(b.hidden, b.w_roll, b.targets)
            bi.check_status(st)
            if u in spikes:
                g = torch.Generator(device="cpu").manual_seed(u)
                mu = mu + (torch.randn(mu.shape[0], generator=g) * 0.5).to(cuda_device)
            out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
            bi.check_status(out.status)
            d3 = out.d3()
            tr.add(d3)
            ref = orc.d3_stats(out.logprob.double().cpu().numpy(), mu.double().cpu().numpy())
            assert math.isclose(d3["mean"], ref["mean"], rel_tol=1e-3, abs_tol=1e-9)
        runs[name] = tr
    assert runs["aligned"].d3_peak_over_median() < 5.0
    assert runs["mismatched"].d3_peak_over_median() > 100.0
