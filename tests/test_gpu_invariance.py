"""Bitwise batch invariance of the CUDA path ("Zero Mismatch, Simple Async RL", sections
"Alignment permits a simpler learning path" and "Large-model validation exposes concrete failure
mechanisms": bit-identical logprobs for the same weights and tokens whatever the batch shape and
whether a row is scored alone (decode) or packed (prefill)), the diff-0 condition, and the
device-side error paths (bounded-wait timeout, non-finite weights)."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from workloads.synth import random_inputs

pytestmark = pytest.mark.gpu

H, V = 2048, 151936          # the batch-invariance workload's head
N_PROBE = 128
R0 = 64.0                    # fixed response normaliser


@pytest.fixture(scope="module")
def probe(cuda_device):
    from async_rl_b200.build import build
    build()
    gen = torch.Generator().manual_seed(1238)
    h, w, y = random_inputs(N_PROBE, H, V, seed=1238)
    mu = (torch.randn(N_PROBE, generator=gen) * 0.5 - 12.0).to(torch.float32)
    d = cuda_device
    return {"h": h.to(d), "w": w.to(d), "y": y.to(d), "mu": mu.to(d)}


def _pack(probe, M, pos_rows, n_probe_in, gen, device):
    """A batch of M rows: probes [pos_rows] at the given positions, N(0,1) filler elsewhere.
    Each probe row is a one-row response in a group with two empty responses (rewards 1, 0, 0);
    each filler row is a one-row response in a group of its own."""
    hid = torch.randn(M, H, generator=gen).to(torch.bfloat16).to(device)
    tg = torch.randint(0, V, (M,), generator=gen, dtype=torch.int32).to(device)
    mu = (torch.randn(M, generator=gen) * 0.5 - 12.0).to(torch.float32).to(device)
    for k, r in enumerate(pos_rows):
        hid[r] = probe["h"][n_probe_in[k]]
        tg[r] = probe["y"][n_probe_in[k]]
        mu[r] = probe["mu"][n_probe_in[k]]
    is_probe = set(int(r) for r in pos_rows)
    offs, gos, rew = [0], [0], []
    for r in range(M):
        if r in is_probe:
            offs += [r + 1, r + 1, r + 1]
            rew += [1.0, 0.0, 0.0]
            gos.append(gos[-1] + 3)
        else:
            offs.append(r + 1)
            rew.append(float(r % 2))
            gos.append(gos[-1] + 1)
    t = lambda x, dt: torch.tensor(x, dtype=dt, device=device)
    return hid, tg, mu, t(rew, torch.float32), t(offs, torch.int64), t(gos, torch.int32)


def _decode_reference(probe, device):
    """Each probe row scored alone (T = 1 per call)."""
    ref = {"lp": [], "w": [], "tl": [], "dh": [], "lp_fwd": []}
    for i in range(N_PROBE):
        hid = probe["h"][i:i + 1].contiguous()
        tg = probe["y"][i:i + 1].contiguous()
        mu = probe["mu"][i:i + 1].contiguous()
        rew = torch.tensor([1.0, 0.0, 0.0], device=device)
        offs = torch.tensor([0, 1, 1, 1], dtype=torch.int64, device=device)
        gos = torch.tensor([0, 3], dtype=torch.int32, device=device)
        out = bi.is_loss_fwd_bwd(hid, probe["w"], tg, mu, rew, offs, gos, None, R0)
        lp, _, st = bi.logprob_fwd(hid, probe["w"], tg)
        torch.cuda.synchronize()
        bi.check_status(out.status)
        bi.check_status(st)
        ref["lp"].append(out.logprob.clone())
        ref["w"].append(out.is_weight.clone())
        ref["tl"].append(out.token_loss.clone())
        ref["dh"].append(out.grad_hidden.clone())
        ref["lp_fwd"].append(lp.clone())
    return {k: torch.cat(v) for k, v in ref.items()}


def test_decode_equals_logprob_fwd(probe, cuda_device):
    ref = _decode_reference(probe, cuda_device)
    assert torch.equal(ref["lp"], ref["lp_fwd"])
    lp, _, st = bi.logprob_fwd(probe["h"], probe["w"], probe["y"])
    torch.cuda.synchronize()
    assert torch.equal(lp, ref["lp"])


@pytest.mark.parametrize("M,per_batch", [(7, 3), (64, 16), (513, 64), (4096, 128), (32768, 128)])
def test_bitwise_across_batch_shapes(probe, cuda_device, M, per_batch):
    ref = _decode_reference(probe, cuda_device) if not hasattr(test_bitwise_across_batch_shapes, "_ref") else \
        test_bitwise_across_batch_shapes._ref
    test_bitwise_across_batch_shapes._ref = ref
    gen = torch.Generator().manual_seed(M)
    order = torch.randperm(N_PROBE, generator=gen).tolist()
    for b0 in range(0, N_PROBE, per_batch):
        ids = order[b0:b0 + per_batch]
        pos = torch.randperm(M, generator=gen)[:len(ids)].tolist()
        hid, tg, mu, rew, offs, gos = _pack(probe, M, pos, ids, gen, cuda_device)
        out = bi.is_loss_fwd_bwd(hid, probe["w"], tg, mu, rew, offs, gos, None, R0)
        lp, _, st = bi.logprob_fwd(hid, probe["w"], tg)
        torch.cuda.synchronize()
        bi.check_status(out.status)
        bi.check_status(st)
        p = torch.tensor(pos, device=cuda_device)
        q = torch.tensor(ids, device=cuda_device)
        assert torch.equal(lp[p], ref["lp"][q]), f"logprob_fwd differs at M={M}"
        assert torch.equal(out.logprob[p], ref["lp"][q]), f"logprob differs at M={M}"
        assert torch.equal(out.is_weight[p], ref["w"][q]), f"is_weight differs at M={M}"
        assert torch.equal(out.token_loss[p], ref["tl"][q]), f"token_loss differs at M={M}"
        assert torch.equal(out.grad_hidden[p], ref["dh"][q]), f"grad_hidden differs at M={M}"


def test_diff_zero(cuda_device):
    """Rollout logprobs taken from the library's own decode-mode calls: w == 1 and D3 == 0 exactly."""
    from workloads import make_batch, spec_for
    b = make_batch(spec_for("tiny")).to(cuda_device)
    mu = torch.empty(b.n_rows, dtype=torch.float32, device=cuda_device)
    for t in range(b.n_rows):
        lp, _, st = bi.logprob_fwd(b.hidden[t:t + 1].contiguous(), b.w, b.targets[t:t + 1].contiguous())
        mu[t:t + 1] = lp
    out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    assert torch.all(out.is_weight == 1.0)
    d3 = out.d3()
    assert d3["mean"] == 0.0 and d3["max"] == 0.0 and d3["count"] == b.n_rows
    scale = float(out.token_loss.abs().sum())
    assert abs(float(out.loss.item())) <= 1e-6 * scale
    raw, st = bi.d3_stats(out.logprob, mu)
    torch.cuda.synchronize()
    assert bi.decode_d3(raw)["mean"] == 0.0


def test_dw_is_deterministic(cuda_device):
    from workloads import make_batch, spec_for
    b = make_batch(spec_for("tiny", H=1536, V=20000, groups=2, per_group=4, len_lo=100, len_hi=300)).to(cuda_device)
    mu = torch.full((b.n_rows,), -9.0, device=cuda_device)
    o1 = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
    g1 = o1.grad_w.clone()
    o2 = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
    torch.cuda.synchronize()
    assert torch.equal(g1, o2.grad_w) and torch.equal(o1.grad_hidden, o2.grad_hidden)
    assert torch.equal(o1.loss, o2.loss)


def test_nonfinite_rollout_logprob_is_reported(cuda_device):
    from workloads import make_batch, spec_for
    b = make_batch(spec_for("tiny")).to(cuda_device)
    mu = torch.full((b.n_rows,), -6.0, device=cuda_device)
    mu[4] = float("-inf")
    out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
    torch.cuda.synchronize()
    assert int(out.status.item()) == 7
    d3 = out.d3()
    assert d3["n_nonfinite"] == 1
    assert not np.isfinite(d3["mean"]) and not np.isfinite(d3["max"])  # the NaN term is kept in both
    assert torch.isinf(out.is_weight[4])


def test_bounded_wait_timeout_returns_status(cuda_device):
    """A wait that nothing satisfies runs out after its limit: BI_ERR_TIMEOUT, no hang, and the
    context stays usable."""
    h, w, y = random_inputs(300, 256, 4000, seed=9)
    h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
    bi.debug_force_timeout_once(20_000_000)  # 20 ms
    lp, _, st = bi.logprob_fwd(h, w, y)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    lp2, _, st2 = bi.logprob_fwd(h, w, y)
    lp3, _, st3 = bi.logprob_fwd(h, w, y)
    torch.cuda.synchronize()
    bi.check_status(st2)
    assert torch.equal(lp2, lp3) and torch.isfinite(lp2).all()
