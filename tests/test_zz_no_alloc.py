"""bi_logprob_fwd_noalloc: the entry point for callers that cannot allocate device memory (code
inside a host framework that owns every device allocation, so it cannot pass a workspace).  It
must give the bits of bi_logprob_fwd, call after call, from its fixed scratch array, whose size
does not depend on T.  This file is collected last on purpose."""
import pytest
import torch

from async_rl_b200 import _lib
from async_rl_b200.build import build
from workloads.synth import random_inputs


pytestmark = pytest.mark.gpu


def _call_noalloc(lib, h, w, y, want_lse=True):
    T, H = h.shape
    V = w.shape[0]
    lp = torch.empty(T, dtype=torch.float32, device=h.device)
    lse = torch.empty(T, dtype=torch.float32, device=h.device) if want_lse else None
    st = torch.empty(1, dtype=torch.int32, device=h.device)
    code = lib.bi_logprob_fwd_noalloc(h.data_ptr(), w.data_ptr(), y.data_ptr(), T, H, V, lp.data_ptr(),
                                      None if lse is None else lse.data_ptr(), st.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    return code, lp, lse, st


def _call_with_workspace(lib, h, w, y):
    T, H = h.shape
    V = w.shape[0]
    ws_bytes = lib.bi_workspace_bytes(T, H, V, 0)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=h.device)
    lp = torch.empty(T, dtype=torch.float32, device=h.device)
    lse = torch.empty(T, dtype=torch.float32, device=h.device)
    st = torch.empty(1, dtype=torch.int32, device=h.device)
    code = lib.bi_logprob_fwd(h.data_ptr(), w.data_ptr(), y.data_ptr(), T, H, V, lp.data_ptr(), lse.data_ptr(),
                              st.data_ptr(), ws.data_ptr(), ws_bytes, torch.cuda.current_stream().cuda_stream)
    return code, lp, lse, st


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_device):
    build()
    lib = _lib.load()
    # calls in a row, the second smaller, so stale scratch from the first would show up; the third
    # has more rows than any fixed per-row scratch of a few MB could hold
    for (T, H, V, seed) in [(3000, 1536, 151936, 31), (701, 1536, 151936, 32), (20000, 1536, 151936, 33)]:
        h, w, y = random_inputs(T, H, V, seed)
        h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
        code, lp, lse, st = _call_noalloc(lib, h, w, y)
        assert code == 0, _lib.STATUS_NAMES.get(code, code)
        rcode, rlp, rlse, rst = _call_with_workspace(lib, h, w, y)
        assert rcode == 0
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(rst.item()) == 0
        assert torch.equal(lp, rlp) and torch.equal(lse, rlse)
        assert torch.isfinite(lp).all()


def test_noalloc_matches_decode_sized_calls_and_null_lse(cuda_device):
    """Decode-sized calls (T = 1 and T = 128): bi_logprob_fwd with its default workspace scores them
    on every SM in one pass, the no-allocation entry point on the cluster kernel; the header
    promises the same bits.  Then a call with lse = NULL must give the same logprob bits."""
    lib = _lib.load()
    for (T, seed) in [(1, 41), (128, 42)]:
        h, w, y = random_inputs(T, 1536, 151936, seed)
        h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
        code, lp, lse, st = _call_noalloc(lib, h, w, y)
        assert code == 0, _lib.STATUS_NAMES.get(code, code)
        rcode, rlp, rlse, rst = _call_with_workspace(lib, h, w, y)
        assert rcode == 0
        code2, lp2, lse2, st2 = _call_noalloc(lib, h, w, y, want_lse=False)
        assert code2 == 0 and lse2 is None
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(rst.item()) == 0 and int(st2.item()) == 0
        assert torch.equal(lp, rlp) and torch.equal(lse, rlse)
        assert torch.equal(lp2, lp)


def test_noalloc_refuses_unsupported_shape_without_launching(cuda_device):
    lib = _lib.load()
    T, H = 16, 704  # no column split of H = 704 over <= 8 CTAs has 64-multiple slices
    h = torch.zeros(T, H, dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros(512, H, dtype=torch.bfloat16, device=cuda_device)
    y = torch.zeros(T, dtype=torch.int32, device=cuda_device)
    code, _, _, _ = _call_noalloc(lib, h, w, y, want_lse=False)
    assert code == 2  # BI_ERR_UNSUPPORTED_SHAPE: nothing launched
