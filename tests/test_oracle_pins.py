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
    assert st["n_nonfinite"] == 1 and not np.isfinite(st["mean"]) and np.isnan(st["max"])


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


def test_grad_w_rows_matches_full_and_worked_example():
    """dW rows of selected vocabulary ids (any T): the hand-worked two-row example's closed-form
    rows, and the full gradient's rows on a prompt-masked batch with a tail id and a target id."""
    ex = _worked_example()
    out = orc.is_loss_fwd_bwd(**ex)
    dz0 = np.array([-1 / 4, 1 / 12, 1 / 12, 1 / 12])
    dz1 = np.array([-1 / 24, 1 / 8, -1 / 24, -1 / 24])
    rows = orc.grad_w_rows(ex["hidden"], ex["w"], ex["targets"], out["token_loss"], out["lse"], [3, 0, 1])
    ref = np.outer(dz0, [LN3, 0.0]) + np.outer(dz1, [0.0, LN3])
    assert np.allclose(rows, ref[[3, 0, 1]], rtol=0, atol=1e-15)
    b = make_batch(spec_for("tiny", prompt_len=3))
    lp, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
    full = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, lp, b.rewards, b.resp_offsets, b.group_offsets,
                               b.prompt_lens)
    ids = np.array([0, int(b.targets[7]), 200, 511])
    got = orc.grad_w_rows(b.hidden, b.w, b.targets, full["token_loss"], full["lse"], ids)
    assert np.allclose(got, full["grad_w"][ids], rtol=1e-12, atol=1e-17)


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


# ---------------------------------------------------------------------------
# Comparison variants and diagnostics (the pages' baselines and stability statistics)
# ---------------------------------------------------------------------------

def _variant_case(seed=21, lag=0.35):
    """Tiny step whose rollout log-probabilities carry enough noise that some weights leave
    [0.8, 1.2] (clipping) and some responses have a large mean log-ratio (gating)."""
    rng = np.random.default_rng(seed)
    T, H, V = 14, 6, 9
    h = rng.normal(size=(T, H))
    w = rng.normal(size=(V, H)) * 0.7
    y = rng.integers(0, V, size=T)
    off = np.array([0, 3, 7, 10, 14])
    goff = np.array([0, 2, 4])
    r = np.array([1.0, 0.0, 0.0, 1.0])
    mu = orc.token_logprob(h, w, y)[0] + rng.normal(size=T) * lag
    pl = np.array([1, 0, 0, 1])
    args = dict(targets=y, rollout_logprob=mu, rewards=r, resp_offsets=off, group_offsets=goff,
                prompt_lens=pl, resp_normalizer=4.0)
    return h, w, args


def test_ppo_clip_hand_example():
    """Two responses of two tokens, R* = 2, clip range [0.8, 1.2].  A = +1: w = 1.5 is clipped
    (l = -1.2/4, g = 0), w = 0.9 is not (l = g = -0.9/4).  A = -1: w = 0.5 is clipped at 0.8
    (l = +0.8/4, g = 0), w = 1.5 is not (min picks -1.5: l = g = +1.5/4).  L = 0.05."""
    w = np.array([1.5, 0.9, 0.5, 1.5])
    A_row = np.array([1.0, 1.0, -1.0, -1.0])
    n_row = np.full(4, 2.0)
    resp = np.array([0, 0, 1, 1])
    mask = np.ones(4, dtype=bool)
    c_row = A_row / (2.0 * n_row)
    t = orc.token_terms("ppo_clip", w, np.log(w), A_row, n_row, 2.0, resp, mask, c_row, 0.2, 0.2)
    assert np.allclose(t["token_loss"], [-0.3, -0.225, 0.2, 0.375], rtol=0, atol=1e-15)
    assert np.allclose(t["g"], [0.0, -0.225, 0.0, 0.375], rtol=0, atol=1e-15)
    assert t["n_clipped"] == 2
    assert abs(float(np.sum(t["token_loss"])) - 0.05) < 1e-15


def test_ppo_clip_wide_range_is_unclipped():
    h, w, args = _variant_case()
    ref = orc.is_loss_fwd_bwd(h, w, **args)
    wide = orc.is_loss_fwd_bwd(h, w, variant="ppo_clip", eps_low=1.0, eps_high=1e9, **args)
    assert abs(wide["loss"] - ref["loss"]) <= 1e-15 * max(1.0, abs(ref["loss"]))
    assert np.allclose(wide["grad_hidden"], ref["grad_hidden"], rtol=1e-14, atol=1e-18)
    assert np.allclose(wide["grad_w"], ref["grad_w"], rtol=1e-14, atol=1e-18)
    assert wide["n_clipped"] == 0


def test_ppo_clip_finite_differences():
    """The clipped loss is piecewise smooth in log pi; away from the kinks its gradient is the
    oracle's dH/dW (a wrong clip side or a gradient through the constant bound fails here)."""
    h, w, args = _variant_case()
    v = dict(variant="ppo_clip", eps_low=0.2, eps_high=0.2)
    out = orc.is_loss_fwd_bwd(h, w, **args, **v)
    wts = out["is_weight"][out["mask"]]
    assert np.min(np.abs(np.concatenate([wts - 0.8, wts - 1.2]))) > 1e-3  # no token at a kink
    assert 0 < out["n_clipped"] < int(out["mask"].sum())                    # both branches occur
    rng = np.random.default_rng(5)
    eps = 1e-6
    for _ in range(24):
        i, k = rng.integers(0, h.shape[0]), rng.integers(0, h.shape[1])
        hp, hm = h.copy(), h.copy()
        hp[i, k] += eps
        hm[i, k] -= eps
        fd = (orc.loss_only(hp, w, **args, **v) - orc.loss_only(hm, w, **args, **v)) / (2 * eps)
        assert abs(fd - out["grad_hidden"][i, k]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-10
    for _ in range(24):
        a, k = rng.integers(0, w.shape[0]), rng.integers(0, w.shape[1])
        wp, wm = w.copy(), w.copy()
        wp[a, k] += eps
        wm[a, k] -= eps
        fd = (orc.loss_only(h, wp, **args, **v) - orc.loss_only(h, wm, **args, **v)) / (2 * eps)
        assert abs(fd - out["grad_w"][a, k]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-10


def test_seq_gate_hand_example_and_limits():
    """rho = mean delta of a response: (0.1 + 0.5) / 2 = 0.3 is rejected at gate 0.2 and kept at
    0.4; an infinite gate is the unclipped loss; a zero gate rejects every response whose rho is
    not exactly 0."""
    w = np.exp(np.array([0.1, 0.5, -0.05, 0.05]))
    A_row = np.array([1.0, 1.0, -1.0, -1.0])
    n_row = np.full(4, 2.0)
    resp = np.array([0, 0, 1, 1])
    mask = np.ones(4, dtype=bool)
    c_row = A_row / (2.0 * n_row)
    lo = orc.token_terms("seq_gate", w, np.log(w), A_row, n_row, 2.0, resp, mask, c_row, gate=0.2)
    hi = orc.token_terms("seq_gate", w, np.log(w), A_row, n_row, 2.0, resp, mask, c_row, gate=0.4)
    assert lo["n_rejected"] == 1 and list(lo["rejected"]) == [True, False]
    assert np.all(lo["token_loss"][:2] == 0.0) and np.all(lo["g"][:2] == 0.0)
    assert np.allclose(lo["token_loss"][2:], -c_row[2:] * w[2:], rtol=0, atol=0)
    assert hi["n_rejected"] == 0 and np.allclose(hi["token_loss"], -c_row * w, rtol=0, atol=0)
    h, wm, args = _variant_case()
    ref = orc.is_loss_fwd_bwd(h, wm, **args)
    inf = orc.is_loss_fwd_bwd(h, wm, variant="seq_gate", gate=math.inf, **args)
    assert inf["loss"] == ref["loss"] and inf["n_rejected"] == 0
    assert np.array_equal(inf["grad_hidden"], ref["grad_hidden"])
    zero = orc.is_loss_fwd_bwd(h, wm, variant="seq_gate", gate=0.0, **args)
    assert zero["loss"] == 0.0 and zero["n_rejected"] == 4
    assert not np.any(zero["grad_hidden"]) and not np.any(zero["grad_w"])


def test_seq_gate_drops_exactly_the_rejected_responses():
    """Rows of rejected responses get dH = 0; the rows of kept responses are unchanged from the
    unclipped step (the gate removes terms, it does not rescale the others)."""
    h, w, args = _variant_case()
    ref = orc.is_loss_fwd_bwd(h, w, **args)
    gated = orc.is_loss_fwd_bwd(h, w, variant="seq_gate", gate=0.15, **args)
    rho = gated["rho"]
    assert 0 < gated["n_rejected"] < 4
    off = args["resp_offsets"]
    for i in range(4):
        rows = slice(off[i], off[i + 1])
        if gated["rejected"][i]:
            assert abs(rho[i]) > 0.15 and not np.any(gated["grad_hidden"][rows])
        else:
            assert np.array_equal(gated["grad_hidden"][rows], ref["grad_hidden"][rows])


def test_kl_estimators_unbiased_on_exact_expectation():
    """With tokens drawn from mu in exact proportions (counts 1..7 of 28), the plain means of k1
    and k3 equal KL(mu || pi) = sum mu log(mu / pi); k2 equals it to second order only."""
    rng = np.random.default_rng(3)
    counts = np.arange(1, 8)
    mu = counts / counts.sum()
    pi = rng.dirichlet(np.ones(7))
    kl = float(np.sum(mu * np.log(mu / pi)))
    logmu = np.repeat(np.log(mu), counts)
    logpi = np.repeat(np.log(pi), counts)
    est = orc.kl_estimators(logpi, logmu)
    assert abs(est["k1"] - kl) < 1e-14 and abs(est["k3"] - kl) < 1e-14
    near = np.exp(np.log(mu) + 1e-3 * rng.normal(size=7))
    near /= near.sum()
    kl_near = float(np.sum(mu * np.log(mu / near)))
    est_near = orc.kl_estimators(np.repeat(np.log(near), counts), logmu)
    assert abs(est_near["k2"] - kl_near) < 1e-3 * kl_near
    const = orc.kl_estimators(np.full(5, 0.3), np.zeros(5))
    assert abs(const["k1"] + 0.3) < 1e-15 and abs(const["k2"] - 0.045) < 1e-15
    assert abs(const["k3"] - (math.expm1(0.3) - 0.3)) < 1e-15


def test_d3_peak_median_and_kl_drift():
    s = orc.d3_peak_median([1.0, 2.0, 3.0, 100.0])
    assert s["peak"] == 100.0 and s["median"] == 2.5 and s["ratio"] == 40.0
    assert orc.kl_drift([1.0, 1.0, 2.0, 2.0, 10.0, 30.0], 2) == 20.0
    with pytest.raises(ValueError):
        orc.kl_drift([1.0], 2)
