"""Seeded synthetic workloads with the shapes of the REINFORCE Zero learner step.

The pages ("Zero Mismatch, Simple Async RL", sections "Alignment permits a
simpler learning path" and "Keep throughput, lag and quality conditions
separate") describe grouped responses scored by a learner whose weights are a
few versions ahead of the rollout's.  Nothing of the pages' data or weights is
available, so every tensor here is random with the shapes of the named models:

* hidden states h ~ N(0, 1), LM-head W ~ N(0, 0.02), both rounded to bf16;
* rollout weights W_roll = bf16(fp32(W) + N(0, sigma_lag)) stand in for policy lag;
* target ids uniform in [0, V); response lengths uniform in [lo, hi] inclusive;
* rewards Bernoulli(p) (or U[0, 1]); groups of equal size.

"N(0, s)" means standard deviation s.  Random numbers are drawn from a
``torch.Generator`` seeded with ``1234 + config index``.  The rollout
log-probabilities themselves are NOT produced here: each side (the CUDA path
when it plays the rollout engine, the oracle in the tests) computes them from
``w_roll``; this module only supplies the optional per-row additive noise that
the 8K-budget workload puts on 1% of the rows.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class ConfigSpec:
    name: str
    index: int
    H: int
    V: int
    groups: int
    per_group: int
    len_lo: int
    len_hi: int
    sigma_lag: float
    reward: str            # "bernoulli:<p>" or "uniform"
    prompt_len: int = 0    # leading rows of each response that are not scored
    noisy_frac: float = 0.0
    noisy_sigma: float = 0.0


CONFIGS = {
    "tiny": ConfigSpec("tiny", 0, H=128, V=512, groups=2, per_group=4,
                       len_lo=8, len_hi=32, sigma_lag=1e-3, reward="bernoulli:0.5"),
    "qwen1.5b": ConfigSpec("qwen1.5b", 1, H=1536, V=151936, groups=8, per_group=8,
                           len_lo=256, len_hi=2048, sigma_lag=1e-4, reward="bernoulli:0.4"),
    "reason8k": ConfigSpec("reason8k", 2, H=1536, V=151936, groups=4, per_group=8,
                           len_lo=1024, len_hi=8192, sigma_lag=4e-4, reward="bernoulli:0.4",
                           noisy_frac=0.01, noisy_sigma=0.05),
    "qwen4b_lag64": ConfigSpec("qwen4b_lag64", 3, H=2560, V=151936, groups=2, per_group=8,
                               len_lo=16384, len_hi=16384, sigma_lag=2e-3, reward="uniform",
                               prompt_len=12288),
    "invariance": ConfigSpec("invariance", 4, H=2048, V=151936, groups=64, per_group=1,
                             len_lo=512, len_hi=512, sigma_lag=1e-4, reward="bernoulli:0.5"),
}


def spec_for(name: str, **overrides) -> ConfigSpec:
    """The named spec, optionally with fields replaced (e.g. fewer groups)."""
    return dataclasses.replace(CONFIGS[name], **overrides)


@dataclasses.dataclass
class Batch:
    spec: ConfigSpec
    hidden: torch.Tensor          # [n_rows, H] bf16
    w: torch.Tensor               # [V, H] bf16, learner LM head
    w_roll: torch.Tensor          # [V, H] bf16, rollout LM head (lagged)
    targets: torch.Tensor         # [n_rows] int32
    rewards: torch.Tensor         # [R] float32
    resp_offsets: torch.Tensor    # [R+1] int64, row offsets of responses
    group_offsets: torch.Tensor   # [G+1] int32, response offsets of groups
    prompt_lens: Optional[torch.Tensor]  # [R] int32 or None
    logmu_noise: torch.Tensor     # [n_rows] float32, additive noise on log mu (zeros mostly)

    @property
    def n_rows(self) -> int:
        return int(self.hidden.shape[0])

    @property
    def R(self) -> int:
        return int(self.rewards.shape[0])

    @property
    def G(self) -> int:
        return int(self.group_offsets.shape[0]) - 1

    def to(self, device) -> "Batch":
        mv = lambda t: None if t is None else t.to(device)
        return Batch(self.spec, mv(self.hidden), mv(self.w), mv(self.w_roll), mv(self.targets),
                     mv(self.rewards), mv(self.resp_offsets), mv(self.group_offsets),
                     mv(self.prompt_lens), mv(self.logmu_noise))


def _randn_bf16(gen, shape, std, device):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    step = max(1, (1 << 24) // max(1, shape[1]))   # bounded fp32 temporaries
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        tmp = torch.randn((r1 - r0, shape[1]), generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        out[r0:r1] = tmp.to(torch.bfloat16)
    return out


def _perturb_bf16(gen, base, std, device):
    out = torch.empty_like(base)
    rows, cols = base.shape
    step = max(1, (1 << 24) // max(1, cols))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        tmp = torch.randn((r1 - r0, cols), generator=gen, device=device, dtype=torch.float32)
        tmp.mul_(std).add_(base[r0:r1].to(torch.float32))
        out[r0:r1] = tmp.to(torch.bfloat16)
    return out


def make_batch(spec: ConfigSpec, seed: Optional[int] = None, device="cpu",
               lengths: Optional[list] = None, with_w_roll: bool = True) -> Batch:
    """Draw one seeded batch for ``spec`` (seed defaults to 1234 + spec.index).

    ``lengths`` overrides the per-response row counts (used by tests that need
    an exact shape).  ``with_w_roll=False`` skips the lagged rollout head.
    """
    seed = 1234 + spec.index if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    R = spec.groups * spec.per_group
    if lengths is None:
        lens = torch.randint(spec.len_lo, spec.len_hi + 1, (R,), generator=gen, device=device)
        lens = lens.cpu().to(torch.int64)
    else:
        assert len(lengths) == R
        lens = torch.tensor(lengths, dtype=torch.int64)
    resp_offsets = torch.zeros(R + 1, dtype=torch.int64)
    resp_offsets[1:] = torch.cumsum(lens, 0)
    n_rows = int(resp_offsets[-1])
    group_offsets = torch.arange(0, R + 1, spec.per_group, dtype=torch.int32)
    prompt_lens = None
    if spec.prompt_len > 0:
        prompt_lens = torch.clamp(lens, max=spec.prompt_len).to(torch.int32)

    hidden = _randn_bf16(gen, (n_rows, spec.H), 1.0, device)
    w = _randn_bf16(gen, (spec.V, spec.H), 0.02, device)
    w_roll = _perturb_bf16(gen, w, spec.sigma_lag, device) if with_w_roll else w
    targets = torch.randint(0, spec.V, (n_rows,), generator=gen, device=device, dtype=torch.int64)
    targets = targets.to(torch.int32)
    if spec.reward.startswith("bernoulli:"):
        p = float(spec.reward.split(":")[1])
        rewards = (torch.rand((R,), generator=gen, device=device) < p).to(torch.float32)
    elif spec.reward == "uniform":
        rewards = torch.rand((R,), generator=gen, device=device, dtype=torch.float32)
    else:
        raise ValueError(spec.reward)
    noise = torch.zeros(n_rows, dtype=torch.float32, device=device)
    if spec.noisy_frac > 0:
        k = max(1, int(round(spec.noisy_frac * n_rows)))
        rows = torch.randperm(n_rows, generator=gen, device=device)[:k]
        noise[rows] = torch.randn((k,), generator=gen, device=device) * spec.noisy_sigma
    return Batch(spec, hidden, w, w_roll, targets, rewards.to(torch.float32),
                 resp_offsets.to(device), group_offsets.to(device),
                 None if prompt_lens is None else prompt_lens.to(device), noise)


def make_global_batch(spec: ConfigSpec, world: int, seed: Optional[int] = None, device="cpu") -> Batch:
    """The batch of a data-parallel step on ``world`` ranks: ``world`` sub-batches of ``spec``
    (sub-batch k drawn by ``make_batch`` with seed + 1000 k) packed one after another, sharing the
    LM heads of sub-batch 0.  With world = 1 it is ``make_batch(spec, seed)`` itself, so the
    per-GPU workload stays the same as the number of ranks grows."""
    seed = 1234 + spec.index if seed is None else seed
    subs = []
    for k in range(world):
        b = make_batch(spec, seed=seed + 1000 * k, device=device, with_w_roll=(k == 0))
        subs.append(b if k == 0 else dataclasses.replace(b, w=None, w_roll=None))
    if world == 1:
        return subs[0]
    row_base, resp_base = 0, 0
    offs, goffs, plens = [torch.zeros(1, dtype=torch.int64, device=device)], [torch.zeros(1, dtype=torch.int32, device=device)], []
    for b in subs:
        offs.append(b.resp_offsets[1:] + row_base)
        goffs.append(b.group_offsets[1:] + resp_base)
        if b.prompt_lens is not None:
            plens.append(b.prompt_lens)
        row_base += b.n_rows
        resp_base += b.R
    cat = lambda name: torch.cat([getattr(b, name) for b in subs])
    return Batch(spec, cat("hidden"), subs[0].w, subs[0].w_roll, cat("targets"), cat("rewards"),
                 torch.cat(offs), torch.cat(goffs), torch.cat(plens) if plens else None, cat("logmu_noise"))


def random_inputs(T: int, H: int, V: int, seed: int, w_std: float = 0.02, device="cpu"):
    """Plain (hidden, W, targets) triple for shape sweeps: h ~ N(0,1), W ~ N(0,w_std)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    hidden = _randn_bf16(gen, (T, H), 1.0, device)
    w = _randn_bf16(gen, (V, H), w_std, device)
    targets = torch.randint(0, V, (T,), generator=gen, device=device, dtype=torch.int64).to(torch.int32)
    return hidden, w, targets


def dense_inputs(M: int, K: int, N: int, seed: int, w_std: float = 0.02, device="cpu"):
    """(x [M, K], w [N, K]) for the linear-layer GEMM: x ~ N(0, 1), W ~ N(0, w_std), both bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return _randn_bf16(gen, (M, K), 1.0, device), _randn_bf16(gen, (N, K), w_std, device)


def norm_inputs(M: int, H: int, seed: int, device="cpu"):
    """(x [M, H], g [H]) for RMSNorm: rows x ~ N(0, s_m^2) with a per-row scale s_m ~ U[0.05, 20]
    (hidden states of very different magnitudes), gains g ~ 1 + N(0, 0.1), both bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn((M, H), generator=gen, device=device)
    x.mul_(torch.rand((M, 1), generator=gen, device=device) * 19.95 + 0.05)
    g = 1.0 + 0.1 * torch.randn((H,), generator=gen, device=device)
    return x.to(torch.bfloat16), g.to(torch.bfloat16)


def logprob_pair_inputs(T: int, seed: int, device="cpu"):
    """(learner log-probs, rollout log-probs, mask) for the D3 statistics: learner log pi ~
    N(-8, 2^2), rollout log mu = log pi + N(0, 0.05^2) with 1% of the tokens moved by a further
    N(0, 1) (mismatch spikes), and a mask that scores 80% of the tokens; fp32, fp32, u8."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    lp = torch.randn(T, generator=gen, device=device) * 2.0 - 8.0
    mu = lp + torch.randn(T, generator=gen, device=device) * 0.05
    spikes = torch.randperm(T, generator=gen, device=device)[: max(1, T // 100)]
    mu[spikes] += torch.randn(spikes.shape[0], generator=gen, device=device)
    mask = (torch.rand(T, generator=gen, device=device) < 0.8).to(torch.uint8)
    return lp.float(), mu.float(), mask
