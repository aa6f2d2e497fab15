"""bi_logprob_fwd_noalloc: the entry point for callers that cannot allocate device memory (code
inside a host framework that owns every device allocation, so it cannot pass a workspace).  It
must give the results of bi_logprob_fwd, call after call, from its fixed scratch array, and refuse
sizes beyond that array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from async_rl_b200 import _lib
from async_rl_b200.build import build
from workloads.synth import random_inputs

from .util import LOGPROB_TOL

pytestmark = pytest.mark.gpu

NOALLOC_MAX_ROWS = 8192


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


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.all(np.abs(a - b) <= LOGPROB_TOL + LOGPROB_TOL * np.abs(b))


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_device):
    build()
    lib = _lib.load()
    # two calls in a row, the second smaller, so stale scratch from the first would show up
    for (T, H, V, seed) in [(3000, 1536, 151936, 31), (701, 1536, 151936, 32)]:
        h, w, y = random_inputs(T, H, V, seed)
        h, w, y = h.to(cuda_device), w.to(cuda_device), y.to(cuda_device)
        code, lp, lse, st = _call_noalloc(lib, h, w, y)
        assert code == 0, _lib.STATUS_NAMES.get(code, code)
        rcode, rlp, rlse, rst = _call_with_workspace(lib, h, w, y)
        assert rcode == 0
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(rst.item()) == 0
        assert _close(lp, rlp) and _close(lse, rlse)


def test_noalloc_refuses_more_rows_than_its_scratch(cuda_device):
    lib = _lib.load()
    T = NOALLOC_MAX_ROWS + 1
    h = torch.zeros(T, 128, dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros(512, 128, dtype=torch.bfloat16, device=cuda_device)
    y = torch.zeros(T, dtype=torch.int32, device=cuda_device)
    code, _, _, _ = _call_noalloc(lib, h, w, y, want_lse=False)
    assert code == 3  # BI_ERR_WORKSPACE: nothing launched
