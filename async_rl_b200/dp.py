"""Data-parallel plumbing for the fused IS loss.

The learner step shards by whole groups ("Zero Mismatch, Simple Async RL", section "Alignment
permits a simpler learning path": the advantage is a response's reward minus its group mean, so a
group must stay on one rank).  Every per-row output is row-local and batch-invariant, hence
identical to the single-GPU result; the only exchange is the sum over ranks of dW and of the loss.
Each rank passes the global number of responses as the normaliser R*.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def shard_by_groups(resp_offsets: Sequence[int], group_offsets: Sequence[int], prompt_lens=None,
                    world: int = 1) -> List[Tuple[int, int]]:
    """Contiguous group ranges [g0, g1) per rank, balancing the scored rows.

    Greedy: rank k takes groups until its cumulative scored rows reach (k+1)/world of the total.
    Deterministic for given offsets.
    """
    off = np.asarray(resp_offsets, dtype=np.int64)
    goff = np.asarray(group_offsets, dtype=np.int64)
    lens = off[1:] - off[:-1]
    if prompt_lens is not None:
        lens = lens - np.asarray(prompt_lens, dtype=np.int64)
    G = goff.shape[0] - 1
    per_group = np.array([lens[goff[g]:goff[g + 1]].sum() for g in range(G)], dtype=np.int64)
    cum = np.concatenate([[0], np.cumsum(per_group)])
    total = int(cum[-1])
    bounds = [0]
    for k in range(1, world):
        target = total * k / world
        g = int(np.searchsorted(cum, target, side="left"))
        g = max(bounds[-1], min(G, g))
        bounds.append(g)
    bounds.append(G)
    return [(bounds[k], bounds[k + 1]) for k in range(world)]


def local_slices(resp_offsets, group_offsets, g0: int, g1: int):
    """Row range, response range and rebased offsets of groups [g0, g1).

    Returns (row0, row1, r0, r1, local_resp_offsets, local_group_offsets).
    """
    off = np.asarray(resp_offsets, dtype=np.int64)
    goff = np.asarray(group_offsets, dtype=np.int64)
    r0, r1 = int(goff[g0]), int(goff[g1])
    row0, row1 = int(off[r0]), int(off[r1])
    loff = off[r0:r1 + 1] - row0
    lgoff = (goff[g0:g1 + 1] - r0).astype(np.int32)
    return row0, row1, r0, r1, loff, lgoff


def shard_of(resp_offsets, group_offsets, prompt_lens, world: int, rank: int):
    """This rank's whole-group shard of a global batch: (row0, row1, r0, r1, local_resp_offsets,
    local_group_offsets), from ``shard_by_groups`` then ``local_slices``."""
    g0, g1 = shard_by_groups(resp_offsets, group_offsets, prompt_lens, world)[rank]
    return local_slices(resp_offsets, group_offsets, g0, g1)


def pin_collectives(env=None) -> dict:
    """Fix NCCL's all-reduce algorithm and protocol (unless the caller already chose them), so that
    the dW sum over ranks takes the same reduction order on every step and every run.  Must run
    before the first NCCL communicator is created.  Returns the settings in force."""
    import os
    env = os.environ if env is None else env
    env.setdefault("NCCL_ALGO", "Ring")
    env.setdefault("NCCL_PROTO", "Simple")
    return {"NCCL_ALGO": env["NCCL_ALGO"], "NCCL_PROTO": env["NCCL_PROTO"]}


def allreduce_step(dist, grad_w, loss, group=None) -> None:
    """Sum dW and the loss over the ranks (the one exchange step of data parallelism)."""
    dist.all_reduce(grad_w, group=group)
    dist.all_reduce(loss, group=group)
