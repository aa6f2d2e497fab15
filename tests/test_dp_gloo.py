"""Data-parallel host logic on CPU: world size 2, gloo.

Each rank evaluates the fp64 oracle on its shard of whole groups with the global normaliser R*,
the ranks sum dW and the loss, and the result must equal the single-process full batch.  Per-row
outputs of each shard must equal the full batch's rows (they are row-local)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from async_rl_b200.dp import allreduce_step, local_slices, shard_by_groups
from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for


def _batch():
    b = make_batch(spec_for("tiny", groups=4, per_group=3, len_lo=3, len_hi=20, V=97, H=64, prompt_len=2))
    mu, _ = orc.token_logprob(b.hidden, b.w_roll, b.targets)
    return b, mu


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b, mu = _batch()
        shards = shard_by_groups(b.resp_offsets, b.group_offsets, b.prompt_lens, world)
        g0, g1 = shards[rank]
        row0, row1, r0, r1, loff, lgoff = local_slices(b.resp_offsets, b.group_offsets, g0, g1)
        out = orc.is_loss_fwd_bwd(b.hidden[row0:row1], b.w, b.targets[row0:row1], mu[row0:row1],
                                  b.rewards[r0:r1], loff, lgoff, b.prompt_lens[r0:r1],
                                  resp_normalizer=float(b.R))
        gw = torch.tensor(out["grad_w"])
        loss = torch.tensor([out["loss"]], dtype=torch.float64)
        allreduce_step(dist, gw, loss)
        q.put((rank, row0, row1, loss.item(), gw.numpy(), out["logprob"], out["grad_hidden"]))
    finally:
        dist.destroy_process_group()


def test_shard_covers_all_groups_contiguously():
    b, _ = _batch()
    for world in (1, 2, 3, 4, 6, 8):   # more ranks than groups leaves some ranks empty
        sh = shard_by_groups(b.resp_offsets, b.group_offsets, b.prompt_lens, world)
        assert len(sh) == world and sh[0][0] == 0 and sh[-1][1] == b.G
        assert all(sh[k][1] == sh[k + 1][0] for k in range(world - 1))
        assert all(g0 <= g1 for g0, g1 in sh)


def test_dp_two_ranks_matches_single_process():
    b, mu = _batch()
    full = orc.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets,
                               b.prompt_lens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, row0, row1, loss, gw, lp, dh in res:
        assert abs(loss - full["loss"]) <= 1e-12 * max(1.0, abs(full["loss"]))
        assert np.allclose(gw, full["grad_w"], rtol=1e-10, atol=1e-15)
        assert np.array_equal(lp, full["logprob"][row0:row1])
        assert np.allclose(dh, full["grad_hidden"][row0:row1], rtol=0, atol=1e-15)
