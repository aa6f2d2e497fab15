"""bi_d3_stats (D3 and the sampled KL estimators of two logprob arrays; "Zero Mismatch, Simple
Async RL", section "Only one probability gap comes from old weights") against the fp64 oracle:
many 256-row blocks with a ragged tail, a mask, spike rows, a non-finite row, empty inputs.

Tolerance: each term is formed in fp32 from the fp32 inputs, delta = lp - mu carries an absolute
rounding of about 2^-24 |lp| (|lp| <= 30 here), d3 = expm1(delta) - delta then moves by about
|delta| times that, and the device sums the terms in fp64; the test allows 1e-4 relative on the
means of d3 and delta^2 / 2 and on the max, and 1e-5 absolute on the mean of -delta.  The count is
an integer: exact."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from async_rl_b200.build import build
    build()


def _inputs(T, seed):
    g = torch.Generator().manual_seed(seed)
    lp = torch.randn(T, generator=g) * 2.0 - 8.0
    mu = lp + torch.randn(T, generator=g) * 0.05
    spikes = torch.randperm(T, generator=g)[: max(1, T // 100)]
    mu[spikes] += torch.randn(spikes.shape[0], generator=g)
    mask = (torch.rand(T, generator=g) < 0.8).to(torch.uint8)
    return lp.float(), mu.float(), mask


def _run(lp, mu, mask, dev):
    raw, st = bi.d3_stats(lp.to(dev), mu.to(dev), None if mask is None else mask.to(dev))
    torch.cuda.synchronize()
    return bi.decode_d3(raw), int(st.item())


@pytest.mark.parametrize("masked", [False, True])
def test_d3_stats_match_oracle(masked, cuda_device):
    T = 100003
    lp, mu, mask = _inputs(T, seed=21)
    m = mask if masked else None
    got, st = _run(lp, mu, m, cuda_device)
    assert st == 0
    sel = None if m is None else m.numpy()
    ref = orc.d3_stats(lp.double().numpy(), mu.double().numpy(), sel)
    kl = orc.kl_estimators(lp.double().numpy(), mu.double().numpy(), sel)
    assert got["count"] == ref["count"] and got["n_nonfinite"] == 0
    assert abs(got["mean"] - ref["mean"]) <= 1e-4 * abs(ref["mean"])
    assert abs(got["max"] - ref["max"]) <= 1e-4 * abs(ref["max"])
    assert abs(got["k1"] - kl["k1"]) <= 1e-5
    assert abs(got["k2"] - kl["k2"]) <= 1e-4 * abs(kl["k2"])
    assert got["n_clipped"] == 0 and got["n_rejected"] == 0


def test_d3_stats_nonfinite_row_is_counted(cuda_device):
    """log mu = -inf gives w = +inf and d3 = inf - inf = NaN: counted, mean non-finite, status set."""
    lp, mu, _ = _inputs(1000, seed=3)
    mu[417] = -float("inf")
    got, st = _run(lp, mu, None, cuda_device)
    ref = orc.d3_stats(lp.double().numpy(), mu.double().numpy())
    assert got["count"] == 1000 and got["n_nonfinite"] == ref["n_nonfinite"] == 1
    assert not np.isfinite(got["mean"]) and not np.isfinite(got["max"])  # a NaN term is not dropped
    assert np.isnan(ref["max"])
    assert st == 7  # BI_ERR_NONFINITE


def test_d3_stats_empty_and_fully_masked(cuda_device):
    empty = torch.empty(0, dtype=torch.float32)
    got, st = _run(empty, empty, None, cuda_device)
    assert st == 0 and got["count"] == 0 and got["mean"] == 0.0
    lp, mu, _ = _inputs(300, seed=4)
    got, st = _run(lp, mu, torch.zeros(300, dtype=torch.uint8), cuda_device)
    assert st == 0 and got["count"] == 0 and got["mean"] == 0.0 and got["max"] == 0.0


def test_d3_stats_unaligned_arrays_give_the_same_sums(cuda_device):
    """Arrays starting 4 bytes (and the mask 1 byte) past an alignment boundary take the kernel's
    element loads instead of its 16-byte loads; the sums, formed in the same order, are the same
    bits, and both agree with the oracle."""
    T = 70001
    lp, mu, mask = _inputs(T + 1, seed=33)
    lpd, mud, md = lp.to(cuda_device), mu.to(cuda_device), mask.to(cuda_device)
    # the same T values, once 16-byte aligned (fresh copies) and once at an offset of one element
    a_lp, a_mu, a_m = lpd[1:].clone(), mud[1:].clone(), md[1:].clone()
    u_lp, u_mu, u_m = lpd[1:], mud[1:], md[1:]
    assert u_lp.data_ptr() % 16 != 0 and u_m.data_ptr() % 4 != 0
    ga, sa = _run(a_lp, a_mu, a_m, cuda_device)
    gu, su = _run(u_lp, u_mu, u_m, cuda_device)
    assert sa == su == 0
    assert ga == gu
    ref = orc.d3_stats(lp[1:].double().numpy(), mu[1:].double().numpy(), mask[1:].numpy())
    assert gu["count"] == ref["count"]
    assert abs(gu["mean"] - ref["mean"]) <= 1e-4 * abs(ref["mean"])
