"""Data parallelism by whole groups on one GPU: the 1.5B-shape batch (8 groups of 8 responses,
T = 76,239) scored whole, then as 2 and as 4 whole-group shards (dp.shard_by_groups, the sharding
bench.py uses) called one after another with the global R* -- what N ranks would each do.

Every per-row output (log pi, w, token loss, dH row) of a shard must have the bits of the same row
in the whole-batch call: each is row-local, and the kernels' arithmetic for a row does not depend
on the batch it sits in.  The sum over shards of dW and of the loss (in rank order) must equal the
whole batch's within the gradient and loss tolerances: those are sums over rows, so their rounding
depends on how the rows are split.  ("Zero Mismatch, Simple Async RL", section "Alignment permits
a simpler learning path": group-mean advantages keep a group on one rank.)"""
import pytest
import torch

import async_rl_b200 as bi
from async_rl_b200.dp import shard_of
from workloads import make_batch, spec_for

from .util import GRAD_TOL, LOSS_TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def whole(cuda_device):
    from async_rl_b200.build import build
    build()
    b = make_batch(spec_for("qwen1.5b"), with_w_roll=False).to(cuda_device)
    gen = torch.Generator().manual_seed(99)
    mu = (torch.randn(b.n_rows, generator=gen) * 0.3 - 12.0).to(torch.float32).to(cuda_device)
    out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    return b, mu, out


@pytest.mark.parametrize("world", [2, 4])
def test_group_shards_match_the_whole_batch(whole, world, cuda_device):
    b, mu, full = whole
    dw_sum = torch.zeros_like(full.grad_w)
    loss_sum = 0.0
    covered = 0
    for rank in range(world):
        row0, row1, r0, r1, loff, lgoff = shard_of(b.resp_offsets.cpu(), b.group_offsets.cpu(), None, world, rank)
        assert row0 == covered
        covered = row1
        sl = slice(row0, row1)
        out = bi.is_loss_fwd_bwd(b.hidden[sl].contiguous(), b.w, b.targets[sl].contiguous(), mu[sl].contiguous(),
                                 b.rewards[r0:r1].contiguous(), torch.as_tensor(loff, device=cuda_device),
                                 torch.as_tensor(lgoff, device=cuda_device), None, float(b.R))
        torch.cuda.synchronize()
        bi.check_status(out.status)
        for f in ("logprob", "is_weight", "token_loss", "grad_hidden"):
            assert torch.equal(getattr(out, f), getattr(full, f)[sl]), (f, world, rank)
        dw_sum += out.grad_w
        loss_sum += float(out.loss.item())
        del out
    assert covered == b.n_rows
    ref = full.grad_w.double()
    err = (dw_sum.double() - ref).abs()
    assert bool((err <= GRAD_TOL * (ref.abs().max() + ref.abs())).all())
    ref_loss = float(full.loss.item())
    scale = float(full.token_loss.double().abs().sum().item())
    assert abs(loss_sum - ref_loss) <= LOSS_TOL * (1.0 + abs(ref_loss))
    assert abs(loss_sum - ref_loss) <= 1e-4 * scale + 1e-9
