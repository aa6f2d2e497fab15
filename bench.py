#!/usr/bin/env python
"""Throughput of the fused token-logprob + unclipped IS-loss forward+backward on B200.

One step = one call of bi_is_loss_fwd_bwd over one synthetic batch with the shapes of the
1.5B-parameter workload (H = 1536, V = 151936, 8 groups x 8 responses of U[256, 2048] tokens):
forward logits + log-softmax + target gather, IS weight, D3, advantages, loss, dH and dW.
Inputs (hidden 0.2 GB, W 0.47 GB) are larger than the 126 MB L2, so no flush is needed between
steps.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload loss|dense|decode|d3]

The default line runs the path that never writes anything of size T x V to device memory: the
fused forward + dH kernel, then the dW kernel that recomputes the logits tile by tile.  The opt-in
P store (every exponentiated logit tile kept in a 23 GB workspace, dW as one GEMM over it) is
timed beside it as the extra key "pstore_opt_in" at N = 1.

N > 1 runs one process per GPU (bench.py re-launches itself under torchrun when WORLD_SIZE is not
set).  One global batch of N sub-batches of the workload is drawn on every rank; each rank scores
its whole-group shard (dp.shard_by_groups) with R* = the global number of responses (weak scaling:
about one sub-batch per rank), and the ranks sum dW and the loss with NCCL (algorithm and protocol
pinned), the one exchange step of data parallelism.

--dry-run checks that plumbing on CPU (gloo ranks, the tiny workload, no kernels).

--workload dense times the batch-invariant dense layers instead (not the default line): one step is
RMSNorm of the 1.5B-shape hidden states [76239, 1536] followed by the gate/up projection
Y = X W^T with W [8960, 1536] (bi_rmsnorm + bi_gemm_bf16); ranks are independent replicas.

--workload decode times decode-style scoring (not the default line): one bi_logprob_fwd call per
step on one row of the 1.5B head (the all-SM path: one pass over W on every SM, then the
per-row combine), with the cluster kernel's latency beside it.

--workload d3 times bi_d3_stats (not the default line): the D3 statistic and the KL estimators of
2^24 tokens' learner and rollout log-probabilities with a mask, an HBM-bound reduction, in GB/s.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused logprob+IS-loss fwd+bwd tokens/s at H1536 V151936; % bf16 tensor peak"
UNIT = "tokens/s"
CONFIG = "qwen1.5b"
CPU_SAMPLE_ROWS = 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--small", action="store_true",
                    help="profiling case: same head, 4 responses of 1408 rows (T=5632: two full rounds of "
                         "22 clusters); not a bench line")
    ap.add_argument("--workload", choices=["loss", "dense", "decode", "d3"], default="loss",
                    help="loss: the fused LM-head step (default line); dense: RMSNorm + linear layer; "
                         "decode: one-row logprob scoring latency; d3: bi_d3_stats over 2^24 tokens")
    ap.add_argument("--dry-run", action="store_true",
                    help="CPU check of the multi-rank plumbing (gloo, tiny workload, no GPU kernels)")
    ap.add_argument("--no-pstore", action="store_true", help="skip the opt-in P-store comparison key")
    return ap.parse_args()


def relaunch_if_needed(args):
    """--gpus N > 1 without a torchrun environment: run this script again as N ranks (torchrun on
    127.0.0.1, bounded by `timeout`).  Under torchrun, refuse a world size other than --gpus."""
    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1:
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                   f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
                   os.path.abspath(__file__)] + sys.argv[1:]
            os.execvp(cmd[0], cmd)
        return
    world = int(os.environ["WORLD_SIZE"])
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}, "fallback"


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "k_lm_fwd_dh_k_lm_dw_T5632.md")
CSRC_HASHED = ("sm100.cuh", "kernels_lm.cuh")  # the forward + dH kernel's sources


def sources_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in CSRC_HASHED:
        with open(os.path.join(ROOT, "async_rl_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, T: int, H: int):
    """DRAM bytes per launch of `kernel` at T rows, scaled from the committed small-case ncu record
    (`traffic <kernel> <bytes per launch> <T_small> <sha256 of the CUDA sources>`), or None when the
    sources changed since that capture.  The forward + dH kernel reads W once per round of
    clusters and the hidden rows once, and writes dH once: the bytes beyond 4 T H (hidden in, dH
    out) are scaled by T (the number of 128-row units, hence of rounds), the 4 T H part is exact."""
    if not os.path.exists(TRAFFIC_RECORD) or kernel != "k_lm_fwd_dh":
        return None
    digest = sources_hash()
    with open(TRAFFIC_RECORD) as fh:
        for ln in fh:
            parts = ln.split()
            if len(parts) == 5 and parts[0] == "traffic" and parts[1] == kernel and parts[4] == digest:
                small, t_small = int(parts[2]), int(parts[3])
                per_row_fixed = 4.0 * H
                return int((small - per_row_fixed * t_small) * T / t_small + per_row_fixed * T)
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def sub_batch(b, nrows):
    """The first `nrows` packed rows with the responses and groups that cover them (host tensors)."""
    off = b.resp_offsets.cpu().numpy()
    goff = b.group_offsets.cpu().numpy()
    keep = int(np.searchsorted(off, nrows, side="left"))  # responses starting before nrows
    new_off = np.minimum(off[:keep + 1], nrows)
    if new_off[-1] < nrows:
        new_off = np.append(new_off, nrows)
    R = len(new_off) - 1
    new_goff = [0]
    for g in range(len(goff) - 1):
        hi = min(goff[g + 1], R)
        if hi > new_goff[-1]:
            new_goff.append(hi)
        if hi >= R:
            break
    return new_off, np.array(new_goff), b.rewards.cpu().numpy()[:R]


def cpu_oracle_sample(b, logmu_host, nrows):
    """Time the fp64 oracle (test infrastructure) on a bounded slice of the same workload."""
    from oracle import isloss_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    off, goff, rew = sub_batch(b, nrows)
    h = b.hidden[:nrows].cpu()
    w = b.w.cpu()
    y = b.targets[:nrows].cpu()
    t0 = time.perf_counter()
    orc.is_loss_fwd_bwd(h, w, y, logmu_host[:nrows].astype(np.float64), rew, off, goff)
    dt = time.perf_counter() - t0
    return {"value": nrows / dt, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"first {nrows} rows of the {CONFIG} batch (fwd + loss + dH + dW in fp64 NumPy), {dt:.1f} s"}


def loss_workload(spec, T):
    """The loss step's workload name, the same in both arms' `config`."""
    return (f"{CONFIG}: H={spec.H} V={spec.V}, {spec.groups}x{spec.per_group} responses "
            f"U[{spec.len_lo},{spec.len_hi}] rows, T={T} scored rows per rank")


def run_reference(args):
    """--impl reference: the fp64 CPU oracle on the machine's host cores, a bounded slice per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from workloads import make_batch, spec_for
    from oracle import isloss_oracle as orc
    b = make_batch(spec_for(CONFIG))
    nrows = 256
    lp_roll, _ = orc.token_logprob(b.hidden[:nrows], b.w_roll, b.targets[:nrows])
    logmu = lp_roll + b.logmu_noise[:nrows].double().numpy()
    times = []
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(b, logmu, nrows)
        if i >= args.warmup:
            times.append(nrows / r["value"])
    ms = 1e3 * statistics.mean(times)
    val = nrows / (ms * 1e-3)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": loss_workload(b.spec, b.n_rows), "global_batch_tokens": int(b.n_rows),
                       "parallelism": "dp1"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                             "sample": f"first {nrows} rows of that batch per step (fwd + loss + dH + dW in "
                                       f"fp64 NumPy), throughput scaled to tokens/s"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def local_shard(gb, world, rank):
    """This rank's whole-group shard of the global batch (a Batch of its own rows and responses)
    and the global number of responses R*."""
    from async_rl_b200.dp import shard_of
    from workloads import Batch
    pl = None if gb.prompt_lens is None else gb.prompt_lens.cpu()
    row0, row1, r0, r1, loff, lgoff = shard_of(gb.resp_offsets.cpu(), gb.group_offsets.cpu(), pl, world, rank)
    dev = gb.hidden.device
    b = Batch(gb.spec, gb.hidden[row0:row1].contiguous(), gb.w, gb.w_roll, gb.targets[row0:row1].contiguous(),
              gb.rewards[r0:r1].contiguous(), torch.as_tensor(loff, device=dev), torch.as_tensor(lgoff, device=dev),
              None if gb.prompt_lens is None else gb.prompt_lens[r0:r1].contiguous(),
              gb.logmu_noise[row0:row1].contiguous())
    return b, gb.R, (row0, row1)


def run_dry(args):
    """--dry-run: the multi-rank plumbing on CPU with gloo: the global tiny batch, each rank's
    whole-group shard, R*, the pinned collective settings and one all-reduce; no GPU kernels."""
    import datetime
    import torch.distributed as dist
    from async_rl_b200.dp import pin_collectives
    from workloads import make_global_batch, spec_for
    rank, world, _ = dist_env()
    pinned = pin_collectives()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    gb = make_global_batch(spec_for("tiny"), world)
    b, rstar, rows = local_shard(gb, world, rank)
    tok = torch.tensor([float(b.n_rows)], dtype=torch.float64)
    shards = [rows]
    if world > 1:
        dist.all_reduce(tok)
        shards = [None] * world
        dist.all_gather_object(shards, rows)
    if rank == 0:
        print(json.dumps({"dry_run": True, "metric": METRIC, "n_gpus": world, "global_rows": gb.n_rows,
                          "rows_all_ranks": int(tok.item()), "resp_normalizer": rstar, "shards": shards,
                          "collectives": pinned}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_ours(args):
    rank, world, local = dist_env()
    import async_rl_b200 as bi
    from async_rl_b200.build import build
    from async_rl_b200.dp import allreduce_step, pin_collectives
    from workloads import make_global_batch, spec_for

    if rank == 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    pinned = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        pinned = pin_collectives()
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        dist.barrier()
        pg = dist
    spec = spec_for(CONFIG)
    if args.small:
        spec = spec_for(CONFIG, groups=1, per_group=4, len_lo=1408, len_hi=1408)
    gb = make_global_batch(spec, world, device=dev)
    b, rstar, _ = local_shard(gb, world, rank)
    del gb
    T, H, V, R = b.n_rows, spec.H, spec.V, b.R
    # rollout log-probabilities from the lagged head (the rollout engine's role), plus noise rows
    logmu, _, st = bi.logprob_fwd(b.hidden, b.w_roll, b.targets)
    logmu += b.logmu_noise
    bi.check_status(st)
    b.w_roll = None
    ws = bi.make_workspace(T, H, V, R, dev)
    out = bi.LossOutputs.allocate(T, H, V, dev)
    rnorm = float(rstar)

    def step():
        bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, logmu, b.rewards, b.resp_offsets, b.group_offsets,
                           None, rnorm, ws=ws, out=out)
        if pg is not None:
            allreduce_step(pg, out.grad_w, out.loss)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    bi.check_status(out.status)

    clocks = ClockSampler(local)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    bi.profile_reset()
    bi.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    bi.profile_enable(False)
    if pg is not None:
        pg.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    prof = bi.profile_read()
    bi.check_status(out.status)

    tok = torch.tensor([float(T), ms], dtype=torch.float64, device=dev)
    if pg is not None:
        tot = tok[:1].clone()
        pg.all_reduce(tot)
        mx = tok[1:].clone()
        pg.all_reduce(mx, op=pg.ReduceOp.MAX)
        total_tokens, ms_max = float(tot.item()), float(mx.item())
    else:
        total_tokens, ms_max = float(T), ms
    value = total_tokens / (ms_max * 1e-3)

    # end to end through the public API with host buffers (pinned): every step copies its inputs
    # host -> device and reads its loss and diagnostics back.  The copy of step i+1's inputs runs on
    # a second stream while step i computes (two device buffer sets), as a prefetching data loader
    # would; every copy and read of the K steps lies inside the timed region.
    e2e = None
    if not args.no_e2e:
        host = {k: getattr(b, k).cpu().pin_memory() for k in ("hidden", "targets", "rewards", "resp_offsets",
                                                              "group_offsets")}
        host["logmu"] = logmu.cpu().pin_memory()
        dbufs = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
        loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
        d3_h = torch.empty(out.d3_raw.numel(), dtype=torch.uint8).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = loss_h.numel() * 4 + d3_h.numel()
        main_s = torch.cuda.current_stream(dev)
        copy_s = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(i, after=None):
            bufs = dbufs[i % 2]
            with torch.cuda.stream(copy_s):
                if after is not None:
                    copy_s.wait_event(after)
                copy_s.wait_event(used[i % 2])  # the step that last read these buffers
                for k in host:
                    bufs[k].copy_(host[k], non_blocking=True)
                copied[i % 2].record(copy_s)

        def e2e_run(nsteps, start_event=None):
            issue_copy(0, start_event)
            for i in range(nsteps):
                if i + 1 < nsteps:
                    issue_copy(i + 1)
                main_s.wait_event(copied[i % 2])
                d = dbufs[i % 2]
                bi.is_loss_fwd_bwd(d["hidden"], b.w, d["targets"], d["logmu"], d["rewards"], d["resp_offsets"],
                                   d["group_offsets"], None, rnorm, ws=ws, out=out)
                used[i % 2].record(main_s)
                if pg is not None:
                    allreduce_step(pg, out.grad_w, out.loss)
                loss_h.copy_(out.loss, non_blocking=True)
                d3_h.copy_(out.d3_raw, non_blocking=True)

        e2e_run(2)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(main_s)
        e2e_run(args.steps, start_event=f0)
        f1.record(main_s)
        torch.cuda.synchronize()
        ems = torch.tensor([f0.elapsed_time(f1) / args.steps], dtype=torch.float64, device=dev)
        if pg is not None:
            pg.all_reduce(ems, op=pg.ReduceOp.MAX)
        e2e = {"value": total_tokens / (float(ems.item()) * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "h2d": "pinned host buffers, prefetched one step ahead on a copy stream"}

    # the opt-in P store beside it (N = 1 only): same batch, its own 23 GB workspace
    pstore = None
    if world == 1 and not args.no_pstore:
        ws_p = bi.make_workspace(T, H, V, R, dev, pstore=True)
        out_p = bi.LossOutputs.allocate(T, H, V, dev)

        def pstep():
            bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, logmu, b.rewards, b.resp_offsets, b.group_offsets,
                               None, rnorm, ws=ws_p, out=out_p, pstore=True)

        for _ in range(args.warmup):
            pstep()
        torch.cuda.synchronize()
        n_p = min(args.steps, 5)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(n_p):
            pstep()
        p1.record()
        torch.cuda.synchronize()
        bi.check_status(out_p.status)
        pms = p0.elapsed_time(p1) / n_p
        pstore = {"ms_per_step": pms, "tokens_per_s": T / (pms * 1e-3), "steps": n_p,
                  "workspace_gb": ws_p.numel() / 1e9,
                  "note": "opt-in BI_LOSS_STORE_P: every exponentiated logit tile kept in device memory "
                          "(materialises T x V), dW as one GEMM over it; not the headline"}
        del ws_p, out_p
        torch.cuda.empty_cache()

    peaks, peak_src = measured_peaks()
    peak_tf = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    flops_tvh = 2.0 * T * V * H  # one LM-head contraction over the batch
    # algorithmic: logits + dH in the fused forward, dW in the second kernel; executed adds the
    # logit recompute of the dW kernel
    alg = {"k_lm_fwd": flops_tvh, "k_lm_fwd_dh": 2 * flops_tvh, "k_lm_dw": flops_tvh, "k_dw_stream": flops_tvh}
    executed = {"k_lm_fwd": flops_tvh, "k_lm_fwd_dh": 2 * flops_tvh, "k_lm_dw": 2 * flops_tvh,
                "k_dw_stream": flops_tvh}
    dom = max(alg, key=lambda k: prof.get(k, (0.0, 1))[0])
    dms, dn = prof.get(dom, (float("nan"), 1))
    davg = dms / max(dn, 1)
    achieved = alg[dom] / (davg * 1e-3) / 1e12
    step_tflops = 6.0 * T * V * H / (ms * 1e-3) / 1e12
    kernels = {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches": v[1]} for k, v in prof.items()}
    launches = int(sum(v[1] for v in prof.values()))

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": loss_workload(spec, T),
                       "global_batch_tokens": int(total_tokens), "parallelism": f"dp{world}",
                       "path": "default: no T x V array in device memory (dW recomputes the logits)",
                       "workspace_gb": ws.numel() / 1e9,
                       "sharding": "whole groups of one global batch (shard_by_groups), R* = global responses",
                       "collectives": pinned,
                       "l2": "inputs larger than L2 (hidden 0.23 GB, W 0.47 GB); no flush"},
            "pct_bf16_peak": 100.0 * step_tflops / peak_tf,
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": achieved / peak_tf,
                         "traffic": recorded_traffic(dom, T, H) if (CONFIG == "qwen1.5b" and not args.small) else None,
                         "traffic_source": "ncu small case (T=5632) scaled to this launch by T; null when the "
                                           "CUDA sources changed since the capture",
                         "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "algorithmic_flops_per_launch": alg[dom],
                         "executed_frac": executed[dom] / (davg * 1e-3) / 1e12 / peak_tf},
            "step_roofline": {"achieved": step_tflops, "frac": step_tflops / peak_tf,
                              "algorithmic_flops": 6.0 * T * V * H, "unit": "TFLOP/s"},
            "kernels": kernels, "gpu_launches": launches, "clocks": clk, "e2e": e2e}
    if pstore is not None:
        pstore["pct_bf16_peak"] = 100.0 * 6.0 * T * V * H / (pstore["ms_per_step"] * 1e-3) / 1e12 / peak_tf
        line["pstore_opt_in"] = pstore
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(b, logmu.cpu().double().numpy(), CPU_SAMPLE_ROWS)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


DENSE_M, DENSE_K, DENSE_N = 76239, 1536, 8960  # 1.5B shape: tokens, hidden size, MLP width
DENSE_METRIC = "batch-invariant RMSNorm + bf16 GEMM (gate/up) TFLOP/s at M76239 K1536 N8960"
DENSE_CPU_ROWS = 32768


def dense_workload():
    """The dense step's workload name, the same in both arms' `config`."""
    return (f"dense: RMSNorm [{DENSE_M}, {DENSE_K}] then Y = X W^T, W [{DENSE_N}, {DENSE_K}] "
            f"(1.5B shape gate/up)")


def run_dense_reference(args):
    """--impl reference --workload dense: the fp64 oracle on the machine's host cores, a bounded slice
    of rows per step (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from workloads import dense_inputs, norm_inputs
    M, K, N = DENSE_M, DENSE_K, DENSE_N
    rows = 4096
    x, g = norm_inputs(rows, K, seed=1234)
    _, w = dense_inputs(8, K, N, seed=4321)
    times, cores = [], 1
    for i in range(args.warmup + args.steps):
        dt, cores = dense_cpu_sample(x, g, w, rows)
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * statistics.mean(times)
    val = 2.0 * rows * N * K / (ms * 1e-3) / 1e12
    print(json.dumps({"impl": "reference", "metric": DENSE_METRIC, "value": val, "unit": "TFLOP/s",
                      "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic",
                      "config": {"workload": dense_workload()},
                      "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                       "sample": f"{rows} rows of [{M}, {K}] per step (fp64 RMSNorm + GEMM)"},
                      "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def dense_cpu_sample(x, g, w, rows):
    """The fp64 oracle (test infrastructure) on the first `rows` rows of the dense step."""
    from oracle import model_oracle as mo
    try:
        from threadpoolctl import threadpool_info
        cores = max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    xs, gs, ws = x[:rows].cpu(), g.cpu(), w.cpu()
    t0 = time.perf_counter()
    for r0 in range(0, rows, 8192):  # row chunks keep the fp64 output small
        h = mo.rmsnorm(xs[r0:r0 + 8192], gs, 1e-6)
        mo.gemm(torch.tensor(h, dtype=torch.float32).to(torch.bfloat16), ws)
    dt = time.perf_counter() - t0
    return dt, int(cores)


def run_dense(args):
    """--workload dense: RMSNorm then the gate/up GEMM on one synthetic batch per step."""
    rank, world, local = dist_env()
    import async_rl_b200 as bi
    from async_rl_b200.build import build
    from workloads import dense_inputs, norm_inputs

    if rank == 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        dist.barrier()
        pg = dist
    M, K, N = DENSE_M, DENSE_K, DENSE_N
    x, g = norm_inputs(M, K, seed=1234 + 1000 * rank)
    _, w = dense_inputs(8, K, N, seed=4321)
    xd, gd, wd = x.to(dev), g.to(dev), w.to(dev)
    h = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    st = torch.empty(1, dtype=torch.int32, device=dev)

    def step(src):
        bi.rmsnorm(src, gd, 1e-6, out=h, status=st)
        bi.gemm_bf16(h, wd, out=y, status=st)

    for _ in range(args.warmup):
        step(xd)
    torch.cuda.synchronize()
    bi.check_status(st)
    clocks = ClockSampler(local)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    bi.profile_reset()
    bi.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step(xd)
    e1.record()
    torch.cuda.synchronize()
    bi.profile_enable(False)
    clk = clocks.stop()
    ms = torch.tensor([e0.elapsed_time(e1) / args.steps], dtype=torch.float64, device=dev)
    if pg is not None:
        pg.all_reduce(ms, op=pg.ReduceOp.MAX)
    ms = float(ms.item())
    prof = bi.profile_read()
    flops = 2.0 * M * N * K
    value = world * flops / (ms * 1e-3) / 1e12

    # end to end: x copied in from pinned host memory and all of y read back, every step
    xh = x.pin_memory()
    yh = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    xin = torch.empty_like(xd)

    def e2e_step():
        xin.copy_(xh, non_blocking=True)
        step(xin)
        yh.copy_(y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    ems = torch.tensor([f0.elapsed_time(f1) / args.steps], dtype=torch.float64, device=dev)
    if pg is not None:
        pg.all_reduce(ems, op=pg.ReduceOp.MAX)
    e2e = {"value": world * flops / (float(ems.item()) * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(y.numel() * 2),
           "h2d": "pinned host buffers, copies in series with the step (x in, all of y out)"}

    peaks, peak_src = measured_peaks()
    peak_tf = float(peaks.get("bf16_tflops"))
    peak_gb = float(peaks.get("hbm_gbs"))
    gms, gn = prof.get("k_gemm_pair", (float("nan"), 1))
    nms, nn = prof.get("k_rmsnorm", (float("nan"), 1))
    g_tf = flops / (gms / max(gn, 1) * 1e-3) / 1e12
    n_gb = 2.0 * 2 * M * K / (nms / max(nn, 1) * 1e-3) / 1e9
    line = {"metric": DENSE_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": dense_workload(),
                       "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (x 0.23 GB, y 1.37 GB); no flush"},
            "roofline": {"bound": "tensor", "kernel": "k_gemm_pair", "achieved": g_tf, "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": g_tf / peak_tf, "traffic": None,
                         "peak_source": f"{peak_src} bf16_tflops (burst: short kernel timed alone)",
                         "algorithmic_flops_per_launch": flops},
            "rmsnorm_roofline": {"bound": "hbm", "kernel": "k_rmsnorm", "achieved": n_gb, "peak": peak_gb,
                                 "unit": "GB/s", "frac": n_gb / peak_gb,
                                 "algorithmic_bytes_per_launch": 2.0 * 2 * M * K},
            "kernels": {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches": v[1]} for k, v in prof.items()},
            "gpu_launches": int(sum(v[1] for v in prof.values())), "clocks": clk, "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = DENSE_CPU_ROWS
        dt, cores = dense_cpu_sample(x, g, w, rows)
        line["cpu_baseline"] = {"value": 2.0 * rows * N * K / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"first {rows} rows of the dense step (fp64 NumPy RMSNorm + GEMM), {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


DECODE_METRIC = "decode-style logprob scoring latency, one row per call, at H1536 V151936"


def decode_workload(H, V):
    """The decode line's workload name, the same in both arms' `config`."""
    return f"decode: 1 row per bi_logprob_fwd call, H={H} V={V}"


def run_decode_reference(args):
    """--impl reference --workload decode: the fp64 oracle scoring one row per step on the host cores."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from oracle import isloss_oracle as orc
    from workloads.synth import random_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    h, w, y = random_inputs(1, 1536, 151936, seed=1234)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        orc.token_logprob(h, w, y)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    print(json.dumps({"impl": "reference", "metric": DECODE_METRIC, "value": ms, "unit": "ms per call",
                      "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                      "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic",
                      "config": {"workload": decode_workload(1536, 151936)},
                      "cpu_baseline": {"value": ms, "unit": "ms per call", "cores": int(cores), "kind": "oracle",
                                       "sample": "one row per step"},
                      "e2e": {"value": ms, "unit": "ms per call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def run_decode(args):
    """--workload decode: one-row bi_logprob_fwd calls (all-SM path), ms per call."""
    rank, world, local = dist_env()
    import async_rl_b200 as bi
    from async_rl_b200.build import build
    from workloads.synth import random_inputs

    if rank == 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    H, V = 1536, 151936
    h, w, y = random_inputs(128, H, V, seed=1234 + rank)
    h, w, y = h.to(dev), w.to(dev), y.to(dev)
    h1, y1 = h[:1].contiguous(), y[:1].contiguous()
    out = torch.empty(1, dtype=torch.float32, device=dev)
    st = torch.empty(1, dtype=torch.int32, device=dev)
    ws_fast = bi.make_workspace(1, H, V, 0, dev)
    ws_min = torch.empty(bi.workspace_bytes(1, H, V, 0, minimal=True), dtype=torch.uint8, device=dev)

    def timed(ws, n, T=1, profiled=False):
        hh, yy = h[:T].contiguous(), y[:T].contiguous()
        o = torch.empty(T, dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            bi.logprob_fwd(hh, w, yy, ws=ws, out=o, status=st)
        torch.cuda.synchronize()
        if profiled:  # only the timed calls are recorded
            bi.profile_reset()
            bi.profile_enable(True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            bi.logprob_fwd(hh, w, yy, ws=ws, out=o, status=st)
        e1.record()
        torch.cuda.synchronize()
        if profiled:
            bi.profile_enable(False)
        bi.check_status(st)
        return e0.elapsed_time(e1) / n

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = timed(ws_fast, args.steps)
    # per-kernel times from a second pass (the event pairs around each launch would otherwise sit
    # between the pass and its dependent combine kernel)
    timed(ws_fast, args.steps, profiled=True)
    clk = clocks.stop()
    prof = bi.profile_read()
    ms_128 = timed(bi.make_workspace(128, H, V, 0, dev), args.steps, T=128)
    ms_cluster = timed(ws_min, args.steps)
    # end to end: the row copied in from pinned memory and its logprob read back, every call
    hh = h1.cpu().pin_memory()
    yh = y1.cpu().pin_memory()
    oh = torch.empty(1, dtype=torch.float32).pin_memory()
    hd, yd = torch.empty_like(h1), torch.empty_like(y1)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        hd.copy_(hh, non_blocking=True)
        yd.copy_(yh, non_blocking=True)
        bi.logprob_fwd(hd, w, yd, ws=ws_fast, out=out, status=st)
        oh.copy_(out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    ems = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = measured_peaks()
    w_bytes = 2.0 * V * H
    # the kernel that streams W (the cluster kernel's launches when the device has no cooperative launch)
    wk = "k_lm_decode1" if "k_lm_decode1" in prof else "k_lm_fwd"
    zt = prof.get(wk, (float("nan"), 1))
    zt_ms = zt[0] / max(zt[1], 1)
    line = {"metric": DECODE_METRIC, "value": ms, "unit": "ms per call", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": decode_workload(H, V),
                       "parallelism": f"replicas{world}", "l2": "W 0.47 GB exceeds L2; no flush"},
            "rows_128_ms": ms_128, "cluster_kernel_ms": ms_cluster,
            "roofline": {"bound": "hbm", "kernel": wk, "achieved": w_bytes / (zt_ms * 1e-3) / 1e9,
                         "peak": float(peaks.get("hbm_gbs")), "unit": "GB/s",
                         "frac": w_bytes / (zt_ms * 1e-3) / 1e9 / float(peaks.get("hbm_gbs")), "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": w_bytes},
            "kernels": {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches": v[1]} for k, v in prof.items()},
            "gpu_launches": int(sum(v[1] for v in prof.values())), "clocks": clk,
            "e2e": {"value": ems, "unit": "ms per call", "h2d_bytes_per_step": int(H * 2 + 4),
                    "d2h_bytes_per_step": 4, "h2d": "pinned host row and target in, logprob out, every call"}}
    if rank == 0:
        print(json.dumps(line), flush=True)


D3_T = 1 << 24
D3_METRIC = "bi_d3_stats (D3 and the KL estimators) GB/s over 16,777,216 tokens"
D3_BYTES_PER_TOKEN = 9  # fp32 learner and rollout log-probabilities, u8 mask


def d3_workload():
    """The D3 line's workload name, the same in both arms' `config`."""
    return f"d3: bi_d3_stats over {D3_T} tokens (fp32 log pi and log mu, u8 mask scoring 80%)"


def d3_cpu_sample(lp, mu, mask, rows):
    """The fp64 oracle's D3 statistics over the first `rows` tokens: (seconds, cores)."""
    from oracle import isloss_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    t0 = time.perf_counter()
    orc.d3_stats(lp[:rows], mu[:rows], mask[:rows])
    return time.perf_counter() - t0, int(cores)


def run_d3_reference(args):
    """--impl reference --workload d3: the fp64 oracle on the host cores, a 2^21-token slice per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from workloads import logprob_pair_inputs
    rows = 1 << 21
    lp, mu, mask = logprob_pair_inputs(rows, seed=1234)
    times, cores = [], 1
    for i in range(args.warmup + args.steps):
        dt, cores = d3_cpu_sample(lp, mu, mask, rows)
        if i >= args.warmup:
            times.append(dt)
    sec = statistics.mean(times)
    val = D3_BYTES_PER_TOKEN * rows / sec / 1e9
    print(json.dumps({"impl": "reference", "metric": D3_METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "config": {"workload": d3_workload()},
                      "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                       "sample": f"the first {rows} tokens per step (fp64 NumPy)"},
                      "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def run_d3(args):
    """--workload d3: bi_d3_stats over 2^24 tokens, HBM-bound; GB/s of algorithmic bytes."""
    rank, world, local = dist_env()
    import async_rl_b200 as bi
    from async_rl_b200.build import build
    from workloads import logprob_pair_inputs

    if rank == 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T = D3_T
    lp, mu, mask = logprob_pair_inputs(T, seed=1234 + rank, device=dev)
    ws = bi.make_workspace(T, 64, 1, 0, dev)
    nbytes = D3_BYTES_PER_TOKEN * T

    def call(a, b, m):
        return bi.d3_stats(a, b, m, ws=ws)

    for _ in range(args.warmup):
        call(lp, mu, mask)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        raw, st = call(lp, mu, mask)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    bi.profile_reset()
    bi.profile_enable(True)
    for _ in range(args.steps):
        raw, st = call(lp, mu, mask)
    torch.cuda.synchronize()
    bi.profile_enable(False)
    clk = clocks.stop()
    prof = bi.profile_read()
    bi.check_status(st)
    # end to end: the three arrays copied in from pinned memory and the 40-byte result read back
    lph, muh, mh = lp.cpu().pin_memory(), mu.cpu().pin_memory(), mask.cpu().pin_memory()
    rawh = torch.empty(40, dtype=torch.uint8).pin_memory()
    lpd, mud, md = torch.empty_like(lp), torch.empty_like(mu), torch.empty_like(mask)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        lpd.copy_(lph, non_blocking=True)
        mud.copy_(muh, non_blocking=True)
        md.copy_(mh, non_blocking=True)
        raw, st = call(lpd, mud, md)
        rawh.copy_(raw, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    ems = f0.elapsed_time(f1) / args.steps
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        rows = 1 << 21
        sec, cores = d3_cpu_sample(lph, muh, mh, rows)
        cpu = {"value": D3_BYTES_PER_TOKEN * rows / sec / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"the first {rows} tokens (fp64 NumPy), {sec:.2f} s"}
    peaks, peak_src = measured_peaks()
    kp = prof.get("k_d3_partial", (float("nan"), 1))
    kp_ms = kp[0] / max(kp[1], 1)
    achieved = nbytes / (kp_ms * 1e-3) / 1e9
    line = {"metric": D3_METRIC, "value": nbytes / (ms * 1e-3) / 1e9 * world, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": d3_workload(), "parallelism": f"replicas{world}",
                       "l2": "inputs 151 MB, larger than L2; no flush"},
            "roofline": {"bound": "hbm", "kernel": "k_d3_partial", "achieved": achieved,
                         "peak": float(peaks.get("hbm_gbs")), "unit": "GB/s",
                         "frac": achieved / float(peaks.get("hbm_gbs")), "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": nbytes},
            "kernels": {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches": v[1]} for k, v in prof.items()},
            "gpu_launches": int(sum(v[1] for v in prof.values())), "clocks": clk,
            "e2e": {"value": nbytes / (ems * 1e-3) / 1e9 * world, "unit": "GB/s", "h2d_bytes_per_step": nbytes,
                    "d2h_bytes_per_step": 40,
                    "h2d": "pinned host arrays in, the 40-byte result out, every call"}}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    relaunch_if_needed(args)
    if args.dry_run:
        run_dry(args)
        return
    if args.workload == "decode":
        if args.impl == "reference":
            run_decode_reference(args)
        else:
            run_decode(args)
    elif args.workload == "dense":
        if args.impl == "reference":
            run_dense_reference(args)
        else:
            run_dense(args)
    elif args.workload == "d3":
        if args.impl == "reference":
            run_d3_reference(args)
        else:
            run_d3(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
