"""Parity of the CUDA path against the fp64 oracle on the same seeded inputs.

Sizes span several tiles and ragged tails (rows not a multiple of 128, vocabularies not a
multiple of 256 or 32) and include the full H = 1536, V = 151936 head."""
import math

import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for
from workloads.synth import random_inputs

from .util import GRAD_TOL, LOGPROB_TOL, LOSS_TOL, assert_close, assert_grad_close, diag_bounds, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from async_rl_b200.build import build
    build()


def _logprob_case(T, H, V, seed, cuda_device, w_std=0.02):
    h, w, y = random_inputs(T, H, V, seed, w_std=w_std)
    lp_ref, lse_ref = orc.token_logprob(h, w, y)
    lp, lse, st = bi.logprob_fwd(h.to(cuda_device), w.to(cuda_device), y.to(cuda_device), want_lse=True)
    torch.cuda.synchronize()
    bi.check_status(st)
    assert_close("logprob", f64(lp), lp_ref, LOGPROB_TOL, LOGPROB_TOL)
    assert_close("lse", f64(lse), lse_ref, LOGPROB_TOL, LOGPROB_TOL)
    return lp


@pytest.mark.parametrize("T,H,V", [(1, 128, 512), (7, 128, 549), (160, 128, 512), (300, 256, 1000),
                                   (129, 192, 4133), (257, 1536, 151936)])
def test_logprob_matches_oracle(T, H, V, cuda_device):
    _logprob_case(T, H, V, seed=T * 7 + H + V, cuda_device=cuda_device)


def test_logprob_peaky_logits(cuda_device):
    """Large logits (W ~ N(0, 0.5)): the running max moves across chunks; no overflow."""
    _logprob_case(200, 256, 3001, seed=5, cuda_device=cuda_device, w_std=0.5)


def test_logprob_empty_batch(cuda_device):
    h = torch.empty(0, 128, dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros(512, 128, dtype=torch.bfloat16, device=cuda_device)
    y = torch.empty(0, dtype=torch.int32, device=cuda_device)
    lp, _, st = bi.logprob_fwd(h, w, y)
    torch.cuda.synchronize()
    bi.check_status(st)
    assert lp.numel() == 0


def test_logprob_uniform_closed_form(cuda_device):
    """W = 0: every logit is 0 and log pi = -log V for every row."""
    T, H, V = 130, 128, 1000
    h = torch.randn(T, H).to(torch.bfloat16).to(cuda_device)
    w = torch.zeros(V, H, dtype=torch.bfloat16, device=cuda_device)
    y = torch.randint(0, V, (T,), dtype=torch.int32).to(cuda_device)
    lp, _, st = bi.logprob_fwd(h, w, y)
    torch.cuda.synchronize()
    bi.check_status(st)
    assert np.allclose(f64(lp), -np.log(V), rtol=0, atol=2e-6)


def test_bad_target_sets_status(cuda_device):
    h, w, y = random_inputs(10, 128, 512, seed=1)
    y[3] = 512
    lp, _, st = bi.logprob_fwd(h.to(cuda_device), w.to(cuda_device), y.to(cuda_device))
    torch.cuda.synchronize()
    assert int(st.item()) == 6
    assert np.isnan(f64(lp)[3]) and np.isfinite(np.delete(f64(lp), 3)).all()


def _loss_case(batch, cuda_device, rollout_lp=None, resp_normalizer=0.0, check_dw=True, tight=1e-4,
               pstore=False, variant_kw=None):
    b = batch
    if rollout_lp is None:
        rollout_lp, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
        rollout_lp = rollout_lp + b.logmu_noise.double().numpy()
    mu = torch.tensor(rollout_lp, dtype=torch.float32)
    mu64 = mu.double().numpy()   # the oracle sees exactly the fp32 values the GPU sees
    vkw = dict(variant_kw or {})
    ref = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu64, b.rewards, b.resp_offsets, b.group_offsets,
                              b.prompt_lens, resp_normalizer, want_grad_w=check_dw, **vkw)
    d = b.to(cuda_device)
    ws = bi.make_workspace(d.n_rows, d.hidden.shape[1], d.w.shape[0], d.R, cuda_device, pstore=pstore)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, mu.to(cuda_device), d.rewards, d.resp_offsets,
                             d.group_offsets, d.prompt_lens, resp_normalizer, ws=ws, pstore=pstore, **vkw)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    assert_close("loss", f64(out.loss), [ref["loss"]], LOSS_TOL, LOSS_TOL)
    # tighter: the loss error is small against the sum of |token losses| (each token loss carries
    # the relative error of its IS weight, i.e. the absolute error of its log-probability)
    scale = float(np.sum(np.abs(ref["token_loss"])))
    assert abs(float(out.loss.item()) - ref["loss"]) <= tight * scale + 1e-9
    assert_close("logprob", f64(out.logprob), ref["logprob"], LOGPROB_TOL, LOGPROB_TOL)
    assert_close("is_weight", f64(out.is_weight), ref["is_weight"], LOGPROB_TOL, LOGPROB_TOL)
    assert_close("token_loss", f64(out.token_loss), ref["token_loss"], LOSS_TOL * np.max(np.abs(ref["token_loss"])),
                 LOSS_TOL)
    d3 = out.d3()
    assert d3["count"] == ref["d3"]["count"] and d3["n_nonfinite"] == 0
    # D3 and the KL estimators: bounds propagated from this call's measured logprob errors
    bnd = diag_bounds(f64(out.logprob), ref["logprob"], mu64, ref["mask"])
    assert_close("d3.mean", [d3["mean"]], [ref["d3"]["mean"]], bnd["d3"], 0.0)
    assert_close("kl.k1", [d3["k1"]], [ref["kl"]["k1"]], bnd["k1"], 0.0)
    assert_close("kl.k2", [d3["k2"]], [ref["kl"]["k2"]], bnd["k2"], 0.0)
    assert d3["n_clipped"] == ref["n_clipped"] and d3["n_rejected"] == ref["n_rejected"]
    assert_grad_close("grad_hidden", f64(out.grad_hidden), ref["grad_hidden"])
    if check_dw:
        assert_grad_close("grad_w", f64(out.grad_w), ref["grad_w"])
    return out, ref


def test_loss_tiny(cuda_device):
    _loss_case(make_batch(spec_for("tiny")), cuda_device)


def test_loss_tiny_prompt_masked_and_normaliser(cuda_device):
    spec = spec_for("tiny", prompt_len=5)
    _loss_case(make_batch(spec), cuda_device, resp_normalizer=13.0)


def test_loss_odd_shapes(cuda_device):
    """V not a multiple of 32, rows not a multiple of 128, groups of unequal size, an empty response."""
    spec = spec_for("tiny", V=549, H=192, groups=3, per_group=3, len_lo=1, len_hi=70)
    b = make_batch(spec, lengths=[37, 0, 64, 129, 5, 1, 70, 33, 2])
    b.group_offsets = torch.tensor([0, 2, 3, 9], dtype=torch.int32)
    _loss_case(b, cuda_device)


@pytest.mark.parametrize("case", ["all_prompt", "no_rows"])
def test_loss_without_scored_rows(case, cuda_device):
    """No scored token at all (every row a prompt row, or no rows): the loss and both gradients are
    exactly zero, D3 counts nothing, the status is clean ("Zero Mismatch, Simple Async RL", section
    "Alignment permits a simpler learning path": a response contributes its token mean, an empty
    one nothing)."""
    lengths = [5, 7, 3, 9, 2, 4, 6, 8] if case == "all_prompt" else [0] * 8
    spec = spec_for("tiny", groups=2, per_group=4, len_lo=0, len_hi=9, prompt_len=16 if case == "all_prompt" else 0)
    b = make_batch(spec, lengths=lengths).to(cuda_device)
    mu = torch.full((b.n_rows,), -6.0, dtype=torch.float32, device=cuda_device)
    out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets,
                             b.prompt_lens, 0.0)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    assert float(out.loss.item()) == 0.0
    assert not bool(out.grad_w.any()) and not bool(out.grad_hidden.any())
    assert out.d3()["count"] == 0


def test_loss_cluster_split_h2048(cuda_device):
    """H = 2048: eight CTAs share each tile (256 columns each)."""
    spec = spec_for("tiny", H=2048, V=3000, groups=2, per_group=2, len_lo=40, len_hi=150)
    _loss_case(make_batch(spec), cuda_device)


def test_loss_cluster_split_h2560(cuda_device):
    """H = 2560: 320 columns per CTA, two MMA column chunks of 192 and 128."""
    spec = spec_for("tiny", H=2560, V=2000, groups=2, per_group=2, len_lo=40, len_hi=150, prompt_len=16)
    _loss_case(make_batch(spec), cuda_device)


@pytest.mark.parametrize("name,kw", [("tiny", dict(prompt_len=3)), ("h2560", dict(H=2560, V=2000, len_lo=40, len_hi=150)),
                                     ("odd", dict(V=549, H=192, len_lo=1, len_hi=70))])
def test_loss_default_and_pstore_paths(name, kw, cuda_device):
    """The default path (dW recomputes the logits; nothing of size T x V in memory) and the opt-in
    P store (dW from the stored probability tiles), each against the oracle, and against each
    other: identical bits except grad_w."""
    b = make_batch(spec_for("tiny", **kw))
    lo, ref = _loss_case(b, cuda_device, pstore=False)
    hi, _ = _loss_case(b, cuda_device, pstore=True)
    for f in ("loss", "logprob", "is_weight", "token_loss", "grad_hidden", "d3_raw"):
        assert torch.equal(getattr(lo, f), getattr(hi, f)), f
    assert not torch.equal(lo.grad_w, hi.grad_w) or b.n_rows == 0  # two different dW kernels ran


def test_pstore_needs_its_workspace(cuda_device):
    """BI_LOSS_STORE_P with the default-size workspace is refused on the host (nothing launched)."""
    b = make_batch(spec_for("tiny")).to(cuda_device)
    mu = torch.full((b.n_rows,), -6.0, dtype=torch.float32, device=cuda_device)
    ws = bi.make_workspace(b.n_rows, 128, 512, b.R, cuda_device)
    assert ws.numel() < bi.workspace_bytes(b.n_rows, 128, 512, b.R, pstore=True)
    with pytest.raises(bi.BiError) as e:
        bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets, ws=ws,
                           pstore=True)
    assert e.value.code == 3  # BI_ERR_WORKSPACE


def _variant_batch(H=256, V=3001, noise=0.35):
    """A batch whose rollout log-probabilities carry N(0, noise) on top of the lagged head, so that
    weights leave the clip range and responses differ in their mean log-ratio."""
    b = make_batch(spec_for("tiny", H=H, V=V, groups=3, per_group=4, len_lo=8, len_hi=40, prompt_len=2))
    mu, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
    mu = mu + np.random.default_rng(99).normal(size=mu.shape[0]) * noise
    return b, mu


def _away_from(values, x, margin):
    return bool(np.all(np.abs(np.asarray(values, dtype=np.float64) - x) > margin))


@pytest.mark.parametrize("pstore", [False, True])
def test_loss_ppo_clip(pstore, cuda_device):
    """The clipped-surrogate baseline: token losses, the gradient only where w itself is the
    selected term, and the count of clipped tokens (no weight within 1e-3 of the clip bounds, so
    the fp32 and fp64 decisions agree)."""
    b, mu = _variant_batch()
    mu32 = torch.tensor(mu, dtype=torch.float32).double().numpy()
    w_ref = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu32, b.rewards, b.resp_offsets, b.group_offsets,
                                b.prompt_lens, want_grads=False)["is_weight"]
    eps = 0.2
    while not (_away_from(w_ref[w_ref != 0], 1 - eps, 1e-3) and _away_from(w_ref[w_ref != 0], 1 + eps, 1e-3)):
        eps += 0.0037
    out, ref = _loss_case(b, cuda_device, rollout_lp=mu, pstore=pstore,
                          variant_kw=dict(variant="ppo_clip", eps_low=eps, eps_high=eps))
    assert 0 < ref["n_clipped"] < int(ref["mask"].sum())


@pytest.mark.parametrize("pstore", [False, True])
def test_loss_sequence_gate(pstore, cuda_device):
    """The rejection-gate baseline with the threshold half-way between two responses' |rho|:
    rejected responses have zero token losses and zero dH rows; the rejection count matches."""
    b, mu = _variant_batch()
    mu32 = torch.tensor(mu, dtype=torch.float32).double().numpy()
    probe = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu32, b.rewards, b.resp_offsets, b.group_offsets,
                                b.prompt_lens, want_grads=False, variant="seq_gate", gate=math.inf)
    a = np.sort(np.abs(probe["rho"]))
    gate = float(0.5 * (a[len(a) // 2 - 1] + a[len(a) // 2]))
    assert _away_from(np.abs(probe["rho"]), gate, 1e-4)
    out, ref = _loss_case(b, cuda_device, rollout_lp=mu, pstore=pstore,
                          variant_kw=dict(variant="seq_gate", gate=gate))
    assert 0 < ref["n_rejected"] < b.R
    off = b.resp_offsets.numpy()
    dh = f64(out.grad_hidden)
    for i in np.nonzero(ref["rejected"])[0]:
        assert not np.any(dh[off[i]:off[i + 1]])


@pytest.mark.parametrize("H,V", [(256, 3001), (1536, 8000)])
def test_loss_reference_moves_mid_sweep(H, V, cuda_device):
    """Logit scale growing along the vocabulary (W_v scaled by 1 + 60 (v/V)^2): the per-row
    reference is raised on many tiles after the first, so the accumulated O is rescaled between
    slice updates, on one CTA (H = 256) and across a cluster (H = 1536)."""
    b = make_batch(spec_for("tiny", H=H, V=V))
    ramp = (1.0 + 60.0 * (torch.arange(V, dtype=torch.float32) / V) ** 2)[:, None]
    b.w = (b.w.float() * ramp).to(torch.bfloat16)
    b.w_roll = (b.w_roll.float() * ramp).to(torch.bfloat16)
    # logits reach |z| ~ 200 here; fp32 accumulation over H products leaves ~1e-4 of absolute error
    # in one logit, hence in log pi and in the relative error of each IS weight
    _loss_case(b, cuda_device, tight=1e-3)


def test_loss_confident_targets(cuda_device):
    """Targets with p_y ~ 0.999: dH = g sum_{v != y} p_v (W_y - W_v) is ~1e-3 of |g W_y|; a form
    that subtracts two O(|W_y|) terms rounded to bf16 would lose it."""
    spec = spec_for("tiny", H=256, V=3001)
    b = make_batch(spec)
    T = b.n_rows
    gen = torch.Generator().manual_seed(77)
    b.targets = torch.randperm(spec.V, generator=gen)[:T].to(torch.int32)
    h = b.hidden.float()
    rows = (15.0 * h / (h * h).sum(dim=1, keepdim=True)).to(torch.bfloat16)
    b.w[b.targets.long()] = rows
    b.w_roll[b.targets.long()] = rows
    out, ref = _loss_case(b, cuda_device)
    assert float(np.min(ref["logprob"])) > -5e-3  # the case is what it claims to be


@pytest.mark.slow
def test_loss_full_head_1536(cuda_device):
    """Full H = 1536, V = 151936 LM head with a few hundred rows over several tiles."""
    spec = spec_for("qwen1.5b", groups=2, per_group=2, len_lo=60, len_hi=130)
    _loss_case(make_batch(spec), cuda_device)
