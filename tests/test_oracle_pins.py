"""Pins for the fp64 oracle: closed forms, invariants, library special cases,
brute force on tiny inputs and finite differences.  No GPU.

Each test names the passage it follows (page title, section); the quantities
are defined in the oracle module's header.
"""
import math

import numpy as np
import pytest
import torch

from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for
from workloads.synth import random_inputs

LN2, LN3 = math.log(2.0), math.log(3.0)


# --- log-softmax / token logprob ---------------------------------------------

def test_uniform_logits_give_minus_log_v():
    """W = 0 (or h = 0): every logit is 0, so log pi = -log V exactly."""
    for V in (2, 7, 512, 151936 // 64):
        h = np.random.default_rng(V).normal(size=(3, 16))
        w = np.zeros((V, 16))
        lp, lse = orc.token_logprob(h, w, np.array([0, V - 1, V // 2]))
        assert np.all(lp == orc.minus_log_v(V)) or np.allclose(lp, -math.log(V), rtol=0, atol=1e-15)
        assert np.allclose(lse, math.log(V), rtol=0, atol=1e-15)
        lp0, _ = orc.token_logprob(np.zeros((2, 16)), np.random.default_rng(1).normal(size=(V, 16)),
                                   np.array([1, 0]))
        assert np.allclose(lp0, -math.log(V), rtol=0, atol=1e-15)


def test_two_token_vocab_closed_form():
    """V = 2: log pi_y = -log(1 + exp(z_other - z_y)) (logistic)."""
    rng = np.random.default_rng(7)
    h = rng.normal(size=(50, 8))
    w = rng.normal(size=(2, 8))
    y = rng.integers(0, 2, size=50)
    lp, _ = orc.token_logprob(h, w, y)
    z = h @ w.T
    zo = z[np.arange(50), 1 - y]
    zy = z[np.arange(50), y]
    assert np.allclose(lp, -np.log1p(np.exp(zo - zy)), rtol=0, atol=1e-13)


def test_hand_worked_probabilities():
    """z = (ln 3, 0, 0, 0): p = (1/2, 1/6, 1/6, 1/6), lse = ln 6."""
    w = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0], [0.0, 0.0]])
    h = np.array([[LN3, 0.0]] * 4)
    lp, lse = orc.token_logprob(h, w, np.array([0, 1, 2, 3]))
    assert np.allclose(lp, [math.log(0.5)] + [math.log(1 / 6)] * 3, rtol=0, atol=1e-15)
    assert np.allclose(lse, math.log(6.0), rtol=0, atol=1e-15)


def test_matches_torch_log_softmax_fp64():
    """Library special case: torch.log_softmax in float64 on the tiny workload."""
    b = make_batch(spec_for("tiny"))
    lp, _ = orc.token_logprob(b.hidden, b.w, b.targets)
    z = b.hidden.double() @ b.w.double().T
    ref = torch.log_softmax(z, dim=1).gather(1, b.targets.long()[:, None])[:, 0].numpy()
    assert np.allclose(lp, ref, rtol=0, atol=1e-12)


def test_brute_force_direct_exp_ratio():
    """Brute force on a tiny case with no max shift: log(exp(z_y) / sum exp(z))."""
    rng = np.random.default_rng(3)
    h = rng.normal(size=(5, 3))
    w = rng.normal(size=(7, 3)) * 0.5
    y = np.array([0, 6, 3, 3, 1])
    lp, _ = orc.token_logprob(h, w, y)
    for t in range(5):
        zs = [sum(h[t, k] * w[v, k] for k in range(3)) for v in range(7)]
        ref = math.log(math.exp(zs[y[t]]) / sum(math.exp(s) for s in zs))
        assert abs(lp[t] - ref) < 1e-13


def test_probabilities_sum_to_one():
    rng = np.random.default_rng(5)
    z = rng.normal(size=(9, 1000)) * 3
    logp, _ = orc.log_softmax_rows(z)
    assert np.allclose(np.exp(logp).sum(1), 1.0, rtol=0, atol=1e-13)


def test_large_logits_stay_finite():
    """Shift invariance: adding 1000 to every logit leaves log p unchanged."""
    rng = np.random.default_rng(6)
    z = rng.normal(size=(4, 50))
    a, _ = orc.log_softmax_rows(z)
    b, _ = orc.log_softmax_rows(z + 1000.0)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


# --- IS weight, decomposition, D3 ----------------------------------------------

def test_decomposition_identity_and_weight_factorisation():
    """'Zero Mismatch' -- 'Only one probability gap comes from old weights':
    log pi_k - log mu_v = (log pi_k - log pi_v) + (log pi_v - log mu_v), so the IS
    weight factors into a lag part and a kernel-mismatch part."""
    b = make_batch(spec_for("tiny"))
    lp_k, _ = orc.token_logprob(b.hidden, b.w, b.targets)          # learner at theta_k
    lp_v, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)     # learner at theta_v
    logmu = lp_v + np.random.default_rng(0).normal(size=lp_v.shape) * 1e-3  # rollout with mismatch
    w, delta = orc.is_weight(lp_k, logmu)
    w_lag, _ = orc.is_weight(lp_k, lp_v)
    w_mis, _ = orc.is_weight(lp_v, logmu)
    assert np.allclose(delta, (lp_k - lp_v) + (lp_v - logmu), rtol=0, atol=1e-14)
    assert np.allclose(w, w_lag * w_mis, rtol=1e-14, atol=0)


def test_diff_zero_gives_unit_weight_and_zero_d3():
    """'diff 0': rollout logprobs equal to the learner's give w == 1 and D3 == 0 exactly."""
    b = make_batch(spec_for("tiny"))
    lp, _ = orc.token_logprob(b.hidden, b.w, b.targets)
    w, delta = orc.is_weight(lp, lp)
    assert np.all(w == 1.0) and np.all(delta == 0.0)
    st = orc.d3_stats(lp, lp)
    assert st["mean"] == 0.0 and st["max"] == 0.0 and st["n_nonfinite"] == 0


def test_d3_nonnegative_and_series():
    """w - 1 - log w >= 0 (exp(x) >= 1 + x); for small delta it is delta^2/2 + delta^3/6 + ..."""
    d = np.concatenate([np.linspace(-30, 30, 2001), np.logspace(-12, -1, 200),
                        -np.logspace(-12, -1, 200)])
    t = orc.d3_terms(d)
    assert np.all(t >= 0)
    small = np.abs(d) < 1e-3
    series = d**2 / 2 + d**3 / 6 + d**4 / 24 + d**5 / 120
    # expm1(d) - d cancels: its absolute error is a few ulp of |d|
    err = np.abs(t[small] - series[small])
    assert np.all(err <= 4 * np.finfo(float).eps * np.abs(d[small]) + 1e-9 * series[small])
    big = np.abs(d) > 1
    assert np.allclose(t[big], np.exp(d[big]) - 1 - d[big], rtol=1e-12, atol=0)


def test_weights_are_not_clipped():
    """Unclipped token-level IS ('REINFORCE-Zero' -- 'Core insight'): w = e^delta for any delta."""
    lp = np.array([0.0, -1.0, -2.0, -20.0])
    mu = np.array([-5.0, -1.0, 3.0, -40.0])
    w, _ = orc.is_weight(lp, mu)
    assert np.allclose(w, np.exp([5.0, 0.0, -5.0, 20.0]), rtol=1e-15, atol=0)


def test_nonfinite_rollout_logprob_propagates():
    st = orc.d3_stats(np.array([-1.0, -2.0]), np.array([-np.inf, -2.0]))
    assert st["n_nonfinite"] == 1 and not np.isfinite(st["mean"])


# --- advantages, coefficients, loss ---------------------------------------------

def test_group_mean_advantages():
    """Reward minus group mean ('Alignment permits a simpler learning path')."""
    A = orc.advantages(np.array([1.0, 0.0, 0.0, 1.0, 1.0, 1.0, 1.0]), np.array([0, 4, 5, 7]))
    assert np.array_equal(A, [0.5, -0.5, -0.5, 0.5, 0.0, 0.0, 0.0])
    rng = np.random.default_rng(1)
    r = (rng.random(64) < 0.4).astype(float)
    A = orc.advantages(r, np.arange(0, 65, 8))
    for g in range(8):
        assert np.sum(A[8 * g:8 * g + 8]) == 0.0          # dyadic means: exact


def test_on_policy_loss_is_zero():
    """w == 1 everywhere: L = -(1/R) sum_i A_i = 0 for group-mean advantages."""
    b = make_batch(spec_for("tiny"))
    lp, _ = orc.token_logprob(b.hidden, b.w, b.targets)
    out = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, lp, b.rewards, b.resp_offsets,
                              b.group_offsets, want_grads=False)
    assert out["loss"] == 0.0 or abs(out["loss"]) < 1e-15
    assert np.all(out["is_weight"] == 1.0)


def _worked_example():
    """Two one-token responses in one group.  W rows e1, e2, 0, 0 (V=4, H=2).
    Row 0: h = (ln3, 0), y = 0 -> p = (1/2, 1/6, 1/6, 1/6), log pi = -ln2; log mu = -ln4 -> w = 2.
    Row 1: h = (0, ln3), y = 1 -> p = (1/6, 1/2, 1/6, 1/6), log pi = -ln2; log mu = -ln2 -> w = 1.
    Rewards (1, 0) -> A = (1/2, -1/2); n = (1, 1); R = 2 -> c = (1/4, -1/4).
    L = -(c0 w0 + c1 w1) = -(1/2 - 1/4) = -1/4.  g = -c w = (-1/2, 1/4).
    dZ0 = -1/2 (e0 - p0) = (-1/4, 1/12, 1/12, 1/12);  dZ1 = 1/4 (e1 - p1) = (-1/24, 1/8, -1/24, -1/24).
    dH0 = dZ0 W = (-1/4, 1/12);  dH1 = (-1/24, 1/8).
    dW_v = dZ0_v h0 + dZ1_v h1.
    """
    w = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0], [0.0, 0.0]])
    h = np.array([[LN3, 0.0], [0.0, LN3]])
    return dict(hidden=h, w=w, targets=np.array([0, 1]),
                rollout_logprob=np.array([-math.log(4.0), -LN2]),
                rewards=np.array([1.0, 0.0]), resp_offsets=np.array([0, 1, 2]),
                group_offsets=np.array([0, 2]))


def test_worked_example_closed_form():
    out = orc.is_loss_fwd_bwd(**_worked_example())
    assert abs(out["loss"] - (-0.25)) < 1e-15
    assert np.allclose(out["is_weight"], [2.0, 1.0], rtol=1e-15)
    assert np.allclose(out["token_loss"], [-0.5, 0.25], rtol=1e-15)
    assert abs(out["d3"]["mean"] - (1 - LN2) / 2) < 1e-15
    assert np.allclose(out["grad_hidden"], [[-1 / 4, 1 / 12], [-1 / 24, 1 / 8]], rtol=0, atol=1e-15)
    dz0 = np.array([-1 / 4, 1 / 12, 1 / 12, 1 / 12])
    dz1 = np.array([-1 / 24, 1 / 8, -1 / 24, -1 / 24])
    dW = np.outer(dz0, [LN3, 0.0]) + np.outer(dz1, [0.0, LN3])
    assert np.allclose(out["grad_w"], dW, rtol=0, atol=1e-15)


def test_resp_normalizer_and_prompt_mask():
    """Prompt rows are not scored; n_i counts scored rows; R* overrides R."""
    ex = _worked_example()
    ex2 = dict(ex)
    # prepend one prompt row to response 0 (same data shifted); it must not change anything
    ex2["hidden"] = np.vstack([[5.0, -5.0], ex["hidden"]])
    ex2["targets"] = np.array([2, 0, 1])
    ex2["rollout_logprob"] = np.array([-123.0, -math.log(4.0), -LN2])
    ex2["resp_offsets"] = np.array([0, 2, 3])
    out = orc.is_loss_fwd_bwd(**ex2, prompt_lens=np.array([1, 0]))
    assert abs(out["loss"] - (-0.25)) < 1e-15
    assert out["token_loss"][0] == 0.0 and np.all(out["grad_hidden"][0] == 0.0)
    out4 = orc.is_loss_fwd_bwd(**ex, resp_normalizer=4.0)
    assert abs(out4["loss"] - (-0.125)) < 1e-15


# --- gradients -----------------------------------------------------------------

def test_finite_difference_gradients():
    """Central differences of the fp64 oracle loss on random entries of H and W."""
    rng = np.random.default_rng(11)
    T, H, V = 12, 6, 9
    h = rng.normal(size=(T, H))
    w = rng.normal(size=(V, H)) * 0.7
    y = rng.integers(0, V, size=T)
    off = np.array([0, 3, 7, 12])
    goff = np.array([0, 2, 3])
    r = np.array([1.0, 0.0, 1.0])
    mu = orc.token_logprob(h, w + rng.normal(size=w.shape) * 0.05, y)[0]
    pl = np.array([1, 0, 2])
    args = dict(targets=y, rollout_logprob=mu, rewards=r, resp_offsets=off,
                group_offsets=goff, prompt_lens=pl, resp_normalizer=5.0)
    out = orc.is_loss_fwd_bwd(h, w, **args)
    eps = 1e-6
    for _ in range(32):
        i, k = rng.integers(0, T), rng.integers(0, H)
        hp, hm = h.copy(), h.copy()
        hp[i, k] += eps
        hm[i, k] -= eps
        fd = (orc.loss_only(hp, w, **args) - orc.loss_only(hm, w, **args)) / (2 * eps)
        assert abs(fd - out["grad_hidden"][i, k]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-10
    for _ in range(32):
        v, k = rng.integers(0, V), rng.integers(0, H)
        wp, wm = w.copy(), w.copy()
        wp[v, k] += eps
        wm[v, k] -= eps
        fd = (orc.loss_only(h, wp, **args) - orc.loss_only(h, wm, **args)) / (2 * eps)
        assert abs(fd - out["grad_w"][v, k]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-10


def test_gradient_invariants():
    """sum_v dZ_tv = 0, so the column sums of dW vanish; equal W rows give dH = 0."""
    b = make_batch(spec_for("tiny"))
    lp, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
    out = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, lp, b.rewards, b.resp_offsets, b.group_offsets)
    assert np.allclose(out["grad_w"].sum(0), 0.0, rtol=0, atol=1e-13)
    w_eq = np.tile(np.random.default_rng(2).normal(size=(1, 128)), (512, 1))
    out2 = orc.is_loss_fwd_bwd(b.hidden, w_eq, b.targets, lp, b.rewards, b.resp_offsets, b.group_offsets)
    assert np.allclose(out2["grad_hidden"], 0.0, rtol=0, atol=1e-14)


def test_grad_rows_matches_full():
    b = make_batch(spec_for("tiny"))
    lp, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
    out = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, lp, b.rewards, b.resp_offsets, b.group_offsets)
    rows = np.array([0, 5, 17, b.n_rows - 1])
    g = out["token_loss"][rows]
    dh = orc.grad_rows(b.hidden, b.w, b.targets, g, rows)
    assert np.allclose(dh, out["grad_hidden"][rows], rtol=0, atol=1e-15)


def test_kl_estimators_small_delta():
    """k3 equals the D3 term; for small delta k1 ~ -mean(delta), k2 ~ k3 ~ delta^2/2."""
    rng = np.random.default_rng(4)
    lp = rng.normal(size=1000)
    mu = lp + rng.normal(size=1000) * 1e-3
    k = orc.kl_estimators(lp, mu)
    assert abs(k["k3"] - orc.d3_stats(lp, mu)["mean"]) < 1e-18
    assert abs(k["k2"] - k["k3"]) < 1e-3 * k["k2"]


def test_synthetic_generator_is_seeded():
    a = make_batch(spec_for("tiny"))
    b = make_batch(spec_for("tiny"))
    assert torch.equal(a.hidden, b.hidden) and torch.equal(a.targets, b.targets)
    assert torch.equal(a.w_roll, b.w_roll) and torch.equal(a.resp_offsets, b.resp_offsets)
    assert a.n_rows == int(a.resp_offsets[-1]) and 8 * 8 <= a.n_rows <= 8 * 32
    assert a.hidden.dtype == torch.bfloat16 and a.targets.dtype == torch.int32
    h, w, y = random_inputs(5, 64, 100, seed=1)
    assert h.shape == (5, 64) and w.shape == (100, 64) and int(y.max()) < 100
