"""The C-ABI library loads and exports every symbol the header declares; host-side argument
checks return their error codes before any CUDA call.  No GPU needed."""
import ctypes
import os
import re

import pytest

from async_rl_b200 import _lib
from async_rl_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("bi_logprob_fwd", "bi_is_loss_fwd_bwd", "bi_d3_stats", "bi_workspace_bytes", "bi_status_string",
                 "bi_gemm_bf16", "bi_rmsnorm"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTED) <= set(declared_functions())


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.bi_status_string(code).decode() == name
    assert lib.bi_status_string(99).decode() == "BI_UNKNOWN"
    assert lib.bi_version() >= 100


def test_workspace_bytes(lib):
    # the logprob-only workspace holds per-CTA partials: its size does not grow with T until the
    # block partials of bi_d3_stats (32 bytes per 256 rows) need more
    a = lib.bi_workspace_bytes(1000, 1536, 151936, 0)
    b = lib.bi_workspace_bytes(2000, 1536, 151936, 0)
    assert 0 < a == b
    big = 1 << 30
    assert lib.bi_workspace_bytes(big, 1536, 151936, 0) >= (big // 256) * 32
    c = lib.bi_workspace_bytes(1000, 1536, 151936, 64)
    d = lib.bi_workspace_bytes(2000, 1536, 151936, 64)
    assert b < c < d
    assert lib.bi_workspace_bytes(-1, 128, 512, 0) == 0
    # the compact copy of the hidden states is part of the loss workspace
    assert d - c >= 1000 * 1536 * 2
    # the default loss workspace is O(T H + R): nothing of size T x V; it is also the minimum
    lo = lib.bi_workspace_bytes_min(2000, 1536, 151936, 64)
    assert lo == d and d < 2000 * 1536 * 2 * 4 + (64 << 20)
    # the opt-in P store holds the bf16 probability tiles (T x (V + 256) rounded to 128 rows)
    ps = lib.bi_workspace_bytes_pstore(2000, 1536, 151936, 64)
    assert ps - d >= 2048 * 151936 * 2
    assert lib.bi_workspace_bytes_pstore(2000, 1536, 151936, 0) == 0
    assert lib.bi_workspace_bytes_min(2000, 1536, 151936, 0) == b
    # up to 128 rows the logprob workspace also holds the all-SM path's per-tile maxima, references
    # and 32-column partial sums: about 1/32 of the rows' logits, never the logits themselves
    dec = lib.bi_workspace_bytes(128, 1536, 151936, 0)
    assert b < dec < b + 128 * 151936 * 4 // 16
    assert lib.bi_workspace_bytes_min(128, 1536, 151936, 0) == b


FAKE = 1 << 20  # aligned non-null address; never dereferenced on the paths below


def test_logprob_argument_checks(lib):
    st = FAKE
    ws_bytes = lib.bi_workspace_bytes(10, 128, 512, 0)
    # NULL hidden
    assert lib.bi_logprob_fwd(None, FAKE, FAKE, 10, 128, 512, FAKE, None, st, FAKE, ws_bytes, None) == 1
    # misaligned hidden
    assert lib.bi_logprob_fwd(FAKE + 2, FAKE, FAKE, 10, 128, 512, FAKE, None, st, FAKE, ws_bytes, None) == 1
    # unsupported H
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 100, 512, FAKE, None, st, FAKE, ws_bytes, None) == 2
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 704, 512, FAKE, None, st, FAKE, ws_bytes, None) == 2
    # workspace too small (below the minimum; between the minimum and bi_workspace_bytes the call
    # runs on the cluster kernel instead of every SM) / missing / misaligned
    ws_min = lib.bi_workspace_bytes_min(10, 128, 512, 0)
    assert ws_min < ws_bytes
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 128, 512, FAKE, None, st, FAKE, ws_min - 1, None) == 3
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 128, 512, FAKE, None, st, None, ws_bytes, None) == 3
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 128, 512, FAKE, None, st, FAKE + 16, ws_bytes, None) == 3
    # negative sizes
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, -1, 128, 512, FAKE, None, st, FAKE, ws_bytes, None) == 1
    assert lib.bi_logprob_fwd(FAKE, FAKE, FAKE, 10, 128, 0, FAKE, None, st, FAKE, ws_bytes, None) == 1


def test_is_loss_argument_checks(lib):
    T, H, V, R = 40, 128, 512, 4
    ws_bytes = lib.bi_workspace_bytes(T, H, V, R)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, R, 2, 0.0, None, T, H, V,
            FAKE, FAKE, None, None, None, FAKE, FAKE, FAKE, FAKE, ws_bytes, None]

    def call(**kw):
        a = list(args)
        idx = {"hidden": 0, "R": 8, "G": 9, "rnorm": 10, "cfg": 11, "H": 13, "grad_w": 21, "ws_bytes": 24,
               "loss": 15}
        for k, v in kw.items():
            a[idx[k]] = v
        return lib.bi_is_loss_fwd_bwd(*a)

    assert call(hidden=None) == 1
    assert call(R=0) == 1
    assert call(G=5) == 1          # more groups than responses
    assert call(rnorm=-1.0) == 1
    assert call(loss=None) == 1
    assert call(grad_w=FAKE + 4) == 1  # misaligned
    assert call(H=704) == 2            # 11 * 64: no split into <= 384-column multiples of 64 with C <= 8
    bad_variant = _lib.LossCfg(7, 0.2, 0.2, 1.0)
    assert call(cfg=ctypes.addressof(bad_variant)) == 1
    bad_eps = _lib.LossCfg(1, -0.1, 0.2, 1.0)
    assert call(cfg=ctypes.addressof(bad_eps)) == 1
    bad_gate = _lib.LossCfg(2, 0.2, 0.2, float("nan"))
    assert call(cfg=ctypes.addressof(bad_gate)) == 1
    ws_min = lib.bi_workspace_bytes_min(T, H, V, R)
    assert 0 < ws_min == ws_bytes
    assert call(ws_bytes=ws_min - 1) == 3
    # the opt-in P store with a default-size workspace, and unknown flag bits
    store = _lib.LossCfg(0, 0.0, 0.0, 0.0, _lib.LOSS_STORE_P)
    assert call(cfg=ctypes.addressof(store)) == 3
    assert lib.bi_workspace_bytes_pstore(T, H, V, R) > ws_bytes
    bad_flags = _lib.LossCfg(0, 0.0, 0.0, 0.0, 4)
    assert call(cfg=ctypes.addressof(bad_flags)) == 1


def test_d3_argument_checks(lib):
    assert lib.bi_d3_stats(None, FAKE, None, 10, FAKE, FAKE, FAKE, 256, None) == 1
    assert lib.bi_d3_stats(FAKE, FAKE, None, 10, None, FAKE, FAKE, 256, None) == 1
    assert lib.bi_d3_stats(FAKE, FAKE, None, 1000, FAKE, FAKE, FAKE, 16, None) == 3


def test_gemm_argument_checks(lib):
    """Host checks of bi_gemm_bf16 (include/bi_model.h) return before any CUDA call."""
    p = ctypes.c_void_p(4096)      # 16-byte aligned stand-in pointers, never dereferenced
    odd = ctypes.c_void_p(4104)
    st = ctypes.c_void_p(8192)
    f = lib.bi_gemm_bf16
    assert f(p, p, p, 16, 256, 64, None, None) == 1            # no status pointer
    assert f(None, p, p, 16, 256, 64, st, None) == 1           # no input
    assert f(p, odd, p, 16, 256, 64, st, None) == 1            # misaligned weight
    assert f(p, p, p, -1, 256, 64, st, None) == 1              # negative M
    assert f(p, p, p, 16, 250, 64, st, None) == 2              # N not a multiple of 8
    assert f(p, p, p, 16, 256, 60, st, None) == 2              # K not a multiple of 8
    assert f(p, p, p, 16, 0, 64, st, None) == 2
    assert f(p, p, p, 16, 256, 0, st, None) == 2


def test_rmsnorm_argument_checks(lib):
    p = ctypes.c_void_p(4096)
    q = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p(4100)
    st = ctypes.c_void_p(8192)
    f = lib.bi_rmsnorm
    assert f(p, p, 1e-6, q, 4, 64, None, None) == 1            # no status pointer
    assert f(p, None, 1e-6, q, 4, 64, st, None) == 1           # no gain
    assert f(odd, p, 1e-6, q, 4, 64, st, None) == 1            # misaligned input
    assert f(p, p, -1.0, q, 4, 64, st, None) == 1              # negative eps
    assert f(p, p, float("nan"), q, 4, 64, st, None) == 1
    assert f(p, p, 1e-6, p, 4, 64, st, None) == 1              # output aliases input
    assert f(p, p, 1e-6, q, 4, 60, st, None) == 2              # H not a multiple of 8
