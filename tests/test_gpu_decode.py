"""Decode-style scoring (bi_logprob_fwd with T <= 128 rows, computed on every SM in one cooperative
pass over W that keeps only sub-tile maxima, references and 32-column partial sums) gives the same bits
as the cluster kernel that scores packed batches ("Zero Mismatch, Simple Async RL", section
"Alignment permits a simpler learning path": rollout and learner logprobs bit-identical whether a
row is scored alone or packed), for the tilings of several hidden sizes, and matches the oracle."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc
from workloads.synth import random_inputs

from .util import LOGPROB_TOL, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from async_rl_b200.build import build
    build()


def _lp(h, w, y, dev, ws_rows=None):
    T = h.shape[0]
    ws = bi.make_workspace(ws_rows if ws_rows is not None else T, h.shape[1], w.shape[0], 0, dev)
    lp, lse, st = bi.logprob_fwd(h, w, y, want_lse=True, ws=ws)
    torch.cuda.synchronize()
    bi.check_status(st)
    return lp, lse


# (H, V): tilings C = 1 (H = 128, 192), C = 6 (1536, NZ = 256), C = 8 with NZ = 192 (2560); V ragged
@pytest.mark.parametrize("H,V", [(128, 549), (192, 4099), (1536, 32771), (2560, 20011)])
def test_few_rows_bitwise_equal_to_packed_batch(H, V, cuda_device):
    h, w, y = random_inputs(300, H, V, seed=H + V)
    h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
    packed_lp, packed_lse = _lp(h, w, y, cuda_device)          # 300 rows: the cluster kernel
    # 1, 3, 9, 12 and 20 rows keep their hidden rows resident (one, two or four 8-row atoms); 33,
    # 40, 100 and 128 rows stream them with every stage, in a box of the rows rounded up to 8.
    # Past 8 rows the sub-tile maxima are stored sub-tile-major.
    for rows in ([0], [5, 17, 299], list(range(128)), list(range(172, 300)), list(range(40, 52)), list(range(7, 27)),
                 list(range(60, 69)), list(range(200, 233)), list(range(3, 43)), list(range(150, 250))):
        r = torch.tensor(rows, device=cuda_device)
        lp, lse = _lp(h[r].contiguous(), w, y[r].contiguous(), cuda_device)   # <= 128 rows: every SM
        assert torch.equal(lp, packed_lp[r]), f"logprob bits differ (H={H}, V={V}, {len(rows)} rows)"
        assert torch.equal(lse, packed_lse[r]), f"lse bits differ (H={H}, V={V}, {len(rows)} rows)"
    # and the few-row path against the fp64 oracle
    lp, _ = _lp(h[:7].contiguous(), w, y[:7].contiguous(), cuda_device)
    ref, _ = orc.token_logprob(h[:7].cpu(), w.cpu(), y[:7].cpu())
    assert_close("logprob", lp.double().cpu().numpy(), ref, LOGPROB_TOL, LOGPROB_TOL)


def test_few_rows_with_moving_reference_bitwise_equal_to_packed_batch(cuda_device):
    """Logits growing along the vocabulary (W_v scaled by 1 + 60 (v/V)^2): each row's reference
    is raised on many tiles, so the chain, the per-class rescales and the class combine of the
    single-pass path all take their rarely used branches."""
    H, V = 1536, 40000
    h, w, y = random_inputs(300, H, V, seed=77)
    ramp = (1.0 + 60.0 * (torch.arange(V, dtype=torch.float32) / V) ** 2)[:, None]
    w = (w.float() * ramp).to(torch.bfloat16)
    h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
    packed_lp, packed_lse = _lp(h, w, y, cuda_device)
    for rows in ([3], list(range(10, 30)), list(range(40, 72)), list(range(100, 228))):
        r = torch.tensor(rows, device=cuda_device)
        lp, lse = _lp(h[r].contiguous(), w, y[r].contiguous(), cuda_device)
        assert torch.equal(lp, packed_lp[r]) and torch.equal(lse, packed_lse[r])


@pytest.mark.parametrize("T", [5, 100])
def test_few_rows_with_minimum_workspace_take_the_cluster_kernel(T, cuda_device):
    """A workspace without room for the all-SM path's partial sums is accepted (the cluster
    kernel scores the rows, loading a hidden-row box of the rows rounded up to 8); the bits are
    the same."""
    h, w, y = random_inputs(T, 1536, 8192, seed=3)
    h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
    fast, _ = _lp(h, w, y, cuda_device)
    small = torch.empty(bi.workspace_bytes(T, 1536, 8192, 0, minimal=True), dtype=torch.uint8, device=cuda_device)
    assert small.numel() < bi.workspace_bytes(T, 1536, 8192, 0)
    lp, _, st = bi.logprob_fwd(h, w, y, ws=small)
    torch.cuda.synchronize()
    bi.check_status(st)
    assert torch.equal(lp, fast)


def test_few_rows_bad_target_sets_status(cuda_device):
    h, w, y = random_inputs(3, 128, 512, seed=9)
    y[1] = 512
    lp, _, st = bi.logprob_fwd(h.to(cuda_device), w.to(cuda_device), y.to(cuda_device))
    torch.cuda.synchronize()
    assert int(st.item()) == 6
    assert torch.isnan(lp[1]).item() and torch.isfinite(lp[0]).item() and torch.isfinite(lp[2]).item()
