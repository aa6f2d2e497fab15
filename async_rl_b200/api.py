"""Python binding of the batch-invariant logprob + unclipped IS-loss library.

Argument marshalling only: every step of the computation runs in the CUDA kernels behind the C
ABI (include/bi_isloss.h).  PyTorch provides device memory and the current stream.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import _lib

D3_DTYPE_BYTES = 40  # bi_d3: f32 mean, f32 max, i64 count, i64 n_nonfinite, f32 k1, f32 k2, i32 n_clipped, i32 n_rejected


class BiError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {_lib.STATUS_NAMES.get(self.code, 'BI_UNKNOWN')} ({self.code})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_cuda(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device):
    # the library dereferences every pointer on the GPU: host memory must never reach it
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor, got {t.device}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_buffers(dev: torch.device, **named):
    """Caller-supplied outputs, workspace and status words: CUDA tensors on `dev`, contiguous."""
    for name, t in named.items():
        if t is None:
            continue
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError(f"{name} must be a CUDA tensor on {dev}, got {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def workspace_bytes(T: int, H: int, V: int, R: int = 0, minimal: bool = False, pstore: bool = False) -> int:
    """Workspace of the default path (nothing of size T x V), the smallest accepted one
    (minimal=True), or the one of the opt-in P store (pstore=True, loss calls only), which keeps
    every exponentiated logit tile of the forward in device memory."""
    lib = _lib.load()
    if pstore:
        return int(lib.bi_workspace_bytes_pstore(T, H, V, R))
    fn = lib.bi_workspace_bytes_min if minimal else lib.bi_workspace_bytes
    return int(fn(T, H, V, R))


def make_workspace(T: int, H: int, V: int, R: int = 0, device="cuda", minimal: bool = False,
                   pstore: bool = False) -> torch.Tensor:
    n = workspace_bytes(T, H, V, R, minimal, pstore)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def check_status(status: torch.Tensor, where: str = "bi") -> None:
    code = int(status.item())
    if code != 0:
        raise BiError(code, where)


def _raise_host(code: int, where: str):
    if code != 0:
        raise BiError(code, where)


def logprob_fwd(hidden: torch.Tensor, w: torch.Tensor, targets: torch.Tensor, want_lse: bool = False,
                ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None):
    """log pi(y_t | h_t) for each row.  Returns (logprob[T] f32, lse[T] f32 or None, status[1] i32)."""
    dev = hidden.device
    T, H = hidden.shape
    V = w.shape[0]
    _check_cuda(hidden, "hidden", torch.bfloat16, dev)
    _check_cuda(w, "w", torch.bfloat16, dev)
    _check_cuda(targets, "targets", torch.int32, dev)
    lib = _lib.load()
    if ws is None:
        ws = make_workspace(T, H, V, 0, dev)
    _check_buffers(dev, ws=ws, out=out, status=status)
    if out is not None and (out.dtype != torch.float32 or out.numel() < T):
        raise ValueError("out must be float32 with at least T elements")
    logprob = out if out is not None else torch.empty(T, dtype=torch.float32, device=dev)
    lse = torch.empty(T, dtype=torch.float32, device=dev) if want_lse else None
    st = status if status is not None else torch.empty(1, dtype=torch.int32, device=dev)
    code = lib.bi_logprob_fwd(_ptr(hidden), _ptr(w), _ptr(targets), T, H, V, _ptr(logprob), _ptr(lse),
                              _ptr(st), _ptr(ws), ws.numel(), _stream(dev))
    _raise_host(code, "bi_logprob_fwd")
    return logprob, lse, st


@dataclasses.dataclass
class LossOutputs:
    loss: torch.Tensor         # [1] f32
    logprob: torch.Tensor      # [T] f32
    is_weight: torch.Tensor    # [T] f32
    token_loss: torch.Tensor   # [T] f32
    d3_raw: torch.Tensor       # [40] u8 (bi_d3)
    grad_hidden: torch.Tensor  # [T, H] bf16
    grad_w: torch.Tensor       # [V, H] f32
    status: torch.Tensor       # [1] i32

    def d3(self) -> dict:
        return decode_d3(self.d3_raw)

    @staticmethod
    def allocate(T: int, H: int, V: int, device) -> "LossOutputs":
        z = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=device)
        return LossOutputs(z(1), z(T), z(T), z(T), z(D3_DTYPE_BYTES, dt=torch.uint8), z(T, H, dt=torch.bfloat16),
                           z(V, H), z(1, dt=torch.int32))


def is_loss_fwd_bwd(hidden, w, targets, rollout_logprob, rewards, resp_offsets, group_offsets,
                    prompt_lens=None, resp_normalizer: float = 0.0, ws: Optional[torch.Tensor] = None,
                    out: Optional[LossOutputs] = None, variant: str = "unclipped", eps_low: float = 0.2,
                    eps_high: float = 0.2, gate: float = float("inf"), pstore: bool = False) -> LossOutputs:
    """Fused forward + backward of the token-level IS REINFORCE loss (see the C header).

    ``variant`` is "unclipped" (the method), or one of the comparison baselines "ppo_clip"
    (clip range [1 - eps_low, 1 + eps_high]) and "seq_gate" (rejects responses whose mean token
    log-ratio exceeds ``gate`` in absolute value).  ``pstore`` opts in to the P store (dW as a
    GEMM over the stored exponentiated logit tiles; needs a ``workspace_bytes(..., pstore=True)``
    workspace); by default nothing of size T x V is written to device memory."""
    dev = hidden.device
    T, H = hidden.shape
    V = w.shape[0]
    R = rewards.shape[0]
    G = group_offsets.shape[0] - 1
    _check_cuda(hidden, "hidden", torch.bfloat16, dev)
    _check_cuda(w, "w", torch.bfloat16, dev)
    _check_cuda(targets, "targets", torch.int32, dev)
    _check_cuda(rollout_logprob, "rollout_logprob", torch.float32, dev)
    _check_cuda(rewards, "rewards", torch.float32, dev)
    _check_cuda(resp_offsets, "resp_offsets", torch.int64, dev)
    _check_cuda(group_offsets, "group_offsets", torch.int32, dev)
    if prompt_lens is not None:
        _check_cuda(prompt_lens, "prompt_lens", torch.int32, dev)
    lib = _lib.load()
    if ws is None:
        ws = make_workspace(T, H, V, R, dev, pstore=pstore)
    o = out if out is not None else LossOutputs.allocate(T, H, V, dev)
    _check_buffers(dev, ws=ws, loss=o.loss, logprob=o.logprob, is_weight=o.is_weight, token_loss=o.token_loss,
                   d3_raw=o.d3_raw, grad_hidden=o.grad_hidden, grad_w=o.grad_w, status=o.status)
    if variant not in _lib.LOSS_VARIANTS:
        raise ValueError(f"unknown loss variant {variant!r}")
    cfg = _lib.LossCfg(_lib.LOSS_VARIANTS[variant], float(eps_low), float(eps_high), float(gate),
                       _lib.LOSS_STORE_P if pstore else 0)
    import ctypes
    code = lib.bi_is_loss_fwd_bwd(_ptr(hidden), _ptr(w), _ptr(targets), _ptr(rollout_logprob), _ptr(rewards),
                                  _ptr(resp_offsets), _ptr(group_offsets), _ptr(prompt_lens), R, G,
                                  float(resp_normalizer), ctypes.addressof(cfg), T, H, V, _ptr(o.loss), _ptr(o.logprob),
                                  _ptr(o.is_weight), _ptr(o.token_loss), _ptr(o.d3_raw), _ptr(o.grad_hidden),
                                  _ptr(o.grad_w), _ptr(o.status), _ptr(ws), ws.numel(), _stream(dev))
    _raise_host(code, "bi_is_loss_fwd_bwd")
    return o


def d3_stats(learner_logprob, rollout_logprob, mask=None, ws=None):
    """D3 and KL statistics of two logprob arrays.  Returns (bi_d3 bytes [40] u8, status)."""
    dev = learner_logprob.device
    T = learner_logprob.shape[0]
    _check_cuda(learner_logprob, "learner_logprob", torch.float32, dev)
    _check_cuda(rollout_logprob, "rollout_logprob", torch.float32, dev)
    if mask is not None:
        _check_cuda(mask, "mask", torch.uint8, dev)
    lib = _lib.load()
    if ws is None:
        ws = make_workspace(T, 64, 1, 0, dev)  # the R = 0 layout covers the block partials
    _check_buffers(dev, ws=ws)
    raw = torch.empty(D3_DTYPE_BYTES, dtype=torch.uint8, device=dev)
    st = torch.empty(1, dtype=torch.int32, device=dev)
    code = lib.bi_d3_stats(_ptr(learner_logprob), _ptr(rollout_logprob), _ptr(mask), T, _ptr(raw), _ptr(st),
                           _ptr(ws), ws.numel(), _stream(dev))
    _raise_host(code, "bi_d3_stats")
    return raw, st


def decode_d3(raw: torch.Tensor) -> dict:
    """bi_d3 bytes -> {mean, max, count, n_nonfinite, k1, k2, n_clipped, n_rejected}."""
    raw = raw.cpu()
    f = raw[:8].view(torch.float32)
    i = raw[8:24].view(torch.int64)
    k = raw[24:32].view(torch.float32)
    c = raw[32:40].view(torch.int32)
    return {"mean": float(f[0]), "max": float(f[1]), "count": int(i[0]), "n_nonfinite": int(i[1]),
            "k1": float(k[0]), "k2": float(k[1]), "n_clipped": int(c[0]), "n_rejected": int(c[1])}


def gemm_bf16(x: torch.Tensor, w: torch.Tensor, out: Optional[torch.Tensor] = None,
              status: Optional[torch.Tensor] = None):
    """Y = X W^T (include/bi_model.h).  Returns (y [M, N] bf16, status [1] i32)."""
    dev = w.device
    M, K = x.shape
    N = w.shape[0]
    _check_cuda(x, "x", torch.bfloat16, dev)
    _check_cuda(w, "w", torch.bfloat16, dev)
    if w.shape[1] != K:
        raise ValueError(f"x has K = {K} columns, w has {w.shape[1]}")
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    _check_cuda(y, "out", torch.bfloat16, dev)
    if tuple(y.shape) != (M, N):
        raise ValueError(f"out must be [{M}, {N}]")
    _check_buffers(dev, status=status)
    st = status if status is not None else torch.empty(1, dtype=torch.int32, device=dev)
    code = _lib.load().bi_gemm_bf16(_ptr(x), _ptr(w), _ptr(y), M, N, K, _ptr(st), _stream(dev))
    _raise_host(code, "bi_gemm_bf16")
    return y, st


def rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float, out: Optional[torch.Tensor] = None,
            status: Optional[torch.Tensor] = None):
    """y = x / sqrt(mean(x^2) + eps) * g per row (include/bi_model.h).  Returns (y, status)."""
    dev = x.device
    M, H = x.shape
    _check_cuda(x, "x", torch.bfloat16, dev)
    _check_cuda(g, "g", torch.bfloat16, dev)
    if g.shape != (H,):
        raise ValueError(f"g must be [{H}]")
    y = out if out is not None else torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    _check_cuda(y, "out", torch.bfloat16, dev)
    _check_buffers(dev, status=status)
    if y.shape != x.shape:
        raise ValueError(f"out must be [{M}, {H}]")
    st = status if status is not None else torch.empty(1, dtype=torch.int32, device=dev)
    code = _lib.load().bi_rmsnorm(_ptr(x), _ptr(g), float(eps), _ptr(y), M, H, _ptr(st), _stream(dev))
    _raise_host(code, "bi_rmsnorm")
    return y, st


def debug_force_timeout_once(limit_ns: int) -> None:
    """Test hook: the next logprob_fwd on this thread exercises the bounded-wait timeout path."""
    _lib.load().bi_debug_force_timeout_once(int(limit_ns))


def profile_enable(on: bool = True) -> None:
    """Record CUDA events around each kernel launch of later calls on this thread."""
    _lib.load().bi_profile_enable(1 if on else 0)


def profile_reset() -> None:
    _lib.load().bi_profile_reset()


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} accumulated since the last reset (synchronises)."""
    import ctypes
    lib = _lib.load()
    n = 32
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    m = lib.bi_profile_read(names, ms, cnt, n)
    if m < 0:
        raise RuntimeError("bi_profile_read: CUDA event failure")
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(m) if cnt[i] > 0}
