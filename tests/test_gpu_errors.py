"""Device-detected argument errors and optional outputs of bi_is_loss_fwd_bwd (include/bi_isloss.h):
inconsistent offsets set BI_ERR_BAD_OFFSETS without a hang and leave the context usable; the
optional outputs (is_weight, token_loss, d3) may be NULL and the other outputs keep their bits."""
import ctypes

import pytest
import torch

import async_rl_b200 as bi
from async_rl_b200 import _lib
from workloads import make_batch, spec_for

pytestmark = pytest.mark.gpu

BAD_OFFSETS = 8


@pytest.fixture(scope="module")
def tiny(cuda_device):
    from async_rl_b200.build import build
    build()
    b = make_batch(spec_for("tiny", prompt_len=3)).to(cuda_device)
    mu = torch.full((b.n_rows,), -6.0, device=cuda_device)
    return b, mu


def _status(b, mu, resp_offsets, group_offsets, prompt_lens):
    out = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, resp_offsets, group_offsets, prompt_lens)
    torch.cuda.synchronize()
    return int(out.status.item())


def test_bad_offsets_set_status_and_context_survives(tiny):
    b, mu = tiny
    assert _status(b, mu, b.resp_offsets, b.group_offsets, b.prompt_lens) == 0
    off = b.resp_offsets.clone()
    off[-1] -= 1                                   # the responses do not cover the rows
    assert _status(b, mu, off, b.group_offsets, b.prompt_lens) == BAD_OFFSETS
    off = b.resp_offsets.clone()
    off[2], off[3] = off[3].item(), off[2].item()  # not monotone
    assert _status(b, mu, off, b.group_offsets, b.prompt_lens) == BAD_OFFSETS
    goff = b.group_offsets.clone()
    goff[-1] -= 1                                  # the groups do not cover the responses
    assert _status(b, mu, b.resp_offsets, goff, b.prompt_lens) == BAD_OFFSETS
    plen = b.prompt_lens.clone()
    plen[0] = int((b.resp_offsets[1] - b.resp_offsets[0]).item()) + 1   # prompt longer than the response
    assert _status(b, mu, b.resp_offsets, b.group_offsets, plen) == BAD_OFFSETS
    assert _status(b, mu, b.resp_offsets, b.group_offsets, b.prompt_lens) == 0


def test_optional_outputs_may_be_null(tiny, cuda_device):
    b, mu = tiny
    T, H = b.hidden.shape
    V = b.w.shape[0]
    full = bi.is_loss_fwd_bwd(b.hidden, b.w, b.targets, mu, b.rewards, b.resp_offsets, b.group_offsets,
                              b.prompt_lens)
    o = bi.LossOutputs.allocate(T, H, V, cuda_device)
    ws = bi.make_workspace(T, H, V, b.R, cuda_device)
    cfg = _lib.LossCfg(0, 0.2, 0.2, float("inf"))
    p = lambda t: t.data_ptr()
    code = _lib.load().bi_is_loss_fwd_bwd(
        p(b.hidden), p(b.w), p(b.targets), p(mu), p(b.rewards), p(b.resp_offsets), p(b.group_offsets),
        p(b.prompt_lens), b.R, b.G, 0.0, ctypes.addressof(cfg), T, H, V, p(o.loss), p(o.logprob),
        None, None, None, p(o.grad_hidden), p(o.grad_w), p(o.status), p(ws), ws.numel(),
        torch.cuda.current_stream(cuda_device).cuda_stream)
    torch.cuda.synchronize()
    assert code == 0 and int(o.status.item()) == 0 and int(full.status.item()) == 0
    for name in ("loss", "logprob", "grad_hidden", "grad_w"):
        assert torch.equal(getattr(o, name), getattr(full, name)), name
