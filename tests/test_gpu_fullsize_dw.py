"""Element-wise parity at the full 1536 x 151936 LM head with 4431 rows over 8 responses, on
both dW paths (the default one, whose dW kernel recomputes the logits, and the opt-in P store).

dW is compared element by element on 80 vocabulary rows spread over the tiles, the ragged tail
tile and the targets of a few rows, against the fp64 oracle evaluated over every row of the batch
(``grad_w_rows`` needs the logits of the selected ids only, plus every row's lse).  log pi and w are
compared on every row, dH on sampled rows, the loss against the oracle's.  The second case scales
W_v by 1 + 60 (v / V)^2, so that each row's reference is raised on many tiles late in the sweep:
the dW kernel's per-column lse, the P store's per-step reference fix-up and the online rescale of
the forward all take their rarely used branches at the full vocabulary.  The rollout
log-probabilities are the oracle's own plus seeded noise; nothing here comes from the CUDA path.

Definitions: "Zero Mismatch, Simple Async RL", sections "Only one probability gap comes from old
weights" and "Alignment permits a simpler learning path"."""
import numpy as np
import pytest
import torch

import async_rl_b200 as bi
from oracle import isloss_oracle as orc
from workloads import make_batch, spec_for

from .util import GRAD_TOL, LOGPROB_TOL, LOSS_TOL, assert_close, assert_grad_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["plain", "ramp"])
def case(request):
    from async_rl_b200.build import build
    build()
    b = make_batch(spec_for("qwen1.5b", groups=2, per_group=4, len_lo=480, len_hi=640), with_w_roll=False)  # T = 4431
    V = b.w.shape[0]
    if request.param == "ramp":
        ramp = (1.0 + 60.0 * (torch.arange(V, dtype=torch.float32) / V) ** 2)[:, None]
        b.w = (b.w.float() * ramp).to(torch.bfloat16)
    lp, lse = orc.token_logprob(b.hidden, b.w, b.targets)          # every row, fp64
    rng = np.random.default_rng(2024)
    mu32 = torch.tensor(lp + rng.normal(size=lp.shape[0]) * 0.05, dtype=torch.float32)
    mu = mu32.double().numpy()
    A = orc.advantages(b.rewards, b.group_offsets)
    _, c = orc.response_coefficients(A, b.resp_offsets, None)
    resp = np.repeat(np.arange(b.R), np.diff(b.resp_offsets.numpy()))
    w_ref = np.exp(lp - mu)
    g = -c[resp] * w_ref
    ids = np.unique(np.concatenate([rng.choice(V, size=64, replace=False), [0, 1, 255, 256, V - 129, V - 2, V - 1],
                                    b.targets.numpy()[rng.choice(b.n_rows, size=8, replace=False)]]))
    rows = np.unique(np.concatenate([rng.choice(b.n_rows, size=32, replace=False), [0, b.n_rows - 1]]))
    ref = {"lp": lp, "w": w_ref, "loss": float(np.sum(g)), "abs_loss": float(np.sum(np.abs(g))), "ids": ids,
           "rows": rows, "dw": orc.grad_w_rows(b.hidden, b.w, b.targets, g, lse, ids),
           "dh": orc.grad_rows(b.hidden[rows], b.w, b.targets[rows], g[rows], np.arange(rows.shape[0]))}
    yield {"name": request.param, "b": b, "mu32": mu32, "ref": ref}


@pytest.mark.parametrize("pstore", [False, True])
def test_fullhead_elementwise_dw_dh_logprob(case, pstore, cuda_device):
    b, ref = case["b"], case["ref"]
    d = b.to(cuda_device)
    out = bi.is_loss_fwd_bwd(d.hidden, d.w, d.targets, case["mu32"].to(cuda_device), d.rewards, d.resp_offsets,
                             d.group_offsets, pstore=pstore)
    torch.cuda.synchronize()
    bi.check_status(out.status)
    assert_close("logprob", f64(out.logprob), ref["lp"], LOGPROB_TOL, LOGPROB_TOL)
    assert_close("is_weight", f64(out.is_weight), ref["w"], LOGPROB_TOL, LOGPROB_TOL)
    assert_close("loss", f64(out.loss), [ref["loss"]], LOSS_TOL, LOSS_TOL)
    # the loss error against the sum of |token losses|: each token loss carries the relative error of
    # its weight, i.e. the absolute error of its logprob (~1e-4 where the ramp drives |z| to ~200)
    tight = 1e-3 if case["name"] == "ramp" else 1e-4
    assert abs(float(out.loss.item()) - ref["loss"]) <= tight * ref["abs_loss"] + 1e-9
    assert_grad_close("grad_hidden", f64(out.grad_hidden[torch.as_tensor(ref["rows"], device=cuda_device)]),
                      ref["dh"], GRAD_TOL)
    got = f64(out.grad_w[torch.as_tensor(ref["ids"], device=cuda_device)])
    assert_grad_close("grad_w", got, ref["dw"], GRAD_TOL)
    # the sampled rows carry real mass: the check is not passed by zeros
    assert np.max(np.abs(ref["dw"])) > 0 and np.max(np.abs(got)) > 0
