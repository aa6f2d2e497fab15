"""Plain fp64 CPU oracle for the batch-invariant token logprob + unclipped IS REINFORCE loss.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it and shares no code
with it.

Every quantity follows the plain definition, evaluated in float64 on the bf16
inputs widened exactly to float64.  Sources (page title, then section):

* [ZM-gap]   "Zero Mismatch, Simple Async RL" -- section "Only one probability
             gap comes from old weights": the learner/rollout log-ratio and its
             decomposition, and the D3 diagnostic (per-update token mean of
             w - 1 - log w).
* [ZM-path]  "Zero Mismatch, Simple Async RL" -- section "Alignment permits a
             simpler learning path": token-level IS weight (learner probability
             over rollout probability, no clipping, no rejection gate); the
             advantage is the response reward minus its group mean; tokens are
             averaged within each response.
* [RZ-core]  "REINFORCE-Zero: kernel alignment + unclipped IS enables 20K-step
             stable async RL" -- "Core insight": unclipped token-level IS.
* [RZ-cn]    "REINFORCE Zero: 为什么内核对齐后..." -- the paragraph around Fig. 2:
             the IS coefficient is the exponential of a log-probability
             difference; D3 is a batch mean.

Readings where the pages are silent (each one is listed in the design notes):

* loss value form: L = -(1/R*) sum_i (1/n_i) sum_{t in i} w_t A_i (ratio form).
  Its gradient equals the REINFORCE form's, since dw/dlogpi = w.
* advantage: A_i = r_i - mean_{j in group(i)} r_j, no std division.
* aggregation over responses: a plain mean over the R* responses of the call
  (R* = R unless the caller passes a normaliser); a response with no scored
  token contributes 0 and still counts in R*.
* rows that are not scored (prompt rows) get logprob = w = token loss = 0 and a
  zero gradient row.
* D3 statistics are over every scored token of the call: mean, max, count, and
  the number of non-finite terms (mean and max are non-finite when any term is).
* rollout-to-learner KL (the pages plot a "sampled estimate" without a formula):
  the plain sampled estimators of KL(mu || pi) from tokens drawn from mu, with
  delta = log pi - log mu: k1 = -delta, k2 = delta^2 / 2, k3 = e^delta - 1 - delta
  (the D3 term); means over the scored tokens.  E_mu[k1] = E_mu[k3] = KL(mu||pi).
* comparison variants (the baselines the pages argue against; no formula given):
  - "ppo_clip": the clipped surrogate per token,
      l_t = -min(r A_i, clip(r, 1 - eps_low, 1 + eps_high) A_i) / (R* n_i),
    r = w_t, differentiated through r only (the clip bound is a constant);
  - "seq_gate": response i is rejected when its mean token log-ratio
    rho_i = (1/n_i) sum_t delta_t has |rho_i| > gate (or is not finite); a
    rejected response contributes no loss and no gradient and still counts in
    R*.  The rejection rate is n_rejected / (responses with a scored token).
* D3 peak/median across updates: max over the per-update D3 means divided by
  their median; KL drift: median over the last window of updates divided by
  the median over the first window.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

_ROW_CHUNK = 64


def _f64(a) -> np.ndarray:
    """Widen a numpy / torch array to float64 (exact for bf16 and fp32)."""
    try:
        import torch  # local: the oracle works on plain numpy too
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").to(torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.int64)


# ---------------------------------------------------------------------------
# Token log-probability  [ZM-gap], [ZM-path], [RZ-cn]
# ---------------------------------------------------------------------------

def logits(hidden_rows, w) -> np.ndarray:
    """z[t, v] = <W_v, h_t>: the LM-head logits of the given rows (float64)."""
    return _f64(hidden_rows) @ _f64(w).T


def log_softmax_rows(z: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(log p, lse) per row: lse = m + log sum_v exp(z_v - m), m = max_v z_v."""
    m = np.max(z, axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.sum(np.exp(z - m), axis=1))
    return z - lse[:, None], lse


def token_logprob(hidden, w, targets, rows: Optional[np.ndarray] = None):
    """log pi(y_t | h_t) = z_{t,y_t} - lse_t for each row (or each row in ``rows``).

    Returns (logprob, lse) as float64 arrays.
    """
    H = _f64(hidden) if not isinstance(hidden, np.ndarray) or hidden.dtype != np.float64 else hidden
    W = _f64(w) if not isinstance(w, np.ndarray) or w.dtype != np.float64 else w
    y = _i64(targets)
    idx = np.arange(H.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    lp = np.empty(idx.shape[0])
    lse = np.empty(idx.shape[0])
    for s in range(0, idx.shape[0], _ROW_CHUNK):
        r = idx[s:s + _ROW_CHUNK]
        z = H[r] @ W.T
        _, l = log_softmax_rows(z)
        lse[s:s + _ROW_CHUNK] = l
        lp[s:s + _ROW_CHUNK] = z[np.arange(r.shape[0]), y[r]] - l
    return lp, lse


# ---------------------------------------------------------------------------
# IS weight and D3  [ZM-gap], [ZM-path], [RZ-core]
# ---------------------------------------------------------------------------

def is_weight(logpi, logmu) -> tuple[np.ndarray, np.ndarray]:
    """delta = log pi - log mu and the unclipped weight w = exp(delta)."""
    delta = _f64(logpi) - _f64(logmu)
    with np.errstate(over="ignore", invalid="ignore"):
        return np.exp(delta), delta


def d3_terms(delta) -> np.ndarray:
    """w - 1 - log w with w = exp(delta), written as expm1(delta) - delta."""
    d = _f64(delta)
    with np.errstate(over="ignore", invalid="ignore"):
        return np.expm1(d) - d


def d3_stats(learner_logprob, rollout_logprob, mask=None) -> dict:
    """Per-call D3 statistics over the rows selected by ``mask`` (all when None)."""
    _, delta = is_weight(learner_logprob, rollout_logprob)
    if mask is not None:
        delta = delta[np.asarray(mask).astype(bool)]
    d = d3_terms(delta)
    n = int(d.shape[0])
    nonfinite = int(np.sum(~np.isfinite(d)))
    if n == 0:
        return {"mean": 0.0, "max": 0.0, "count": 0, "n_nonfinite": 0}
    with np.errstate(invalid="ignore"):
        return {"mean": float(np.sum(d) / n), "max": float(np.max(d)),
                "count": n, "n_nonfinite": nonfinite}


# ---------------------------------------------------------------------------
# Advantages and per-response coefficients  [ZM-path]
# ---------------------------------------------------------------------------

def advantages(rewards, group_offsets) -> np.ndarray:
    """A_i = r_i - mean of r over the group holding response i."""
    r = _f64(rewards)
    g = _i64(group_offsets)
    A = np.zeros_like(r)
    for k in range(g.shape[0] - 1):
        a, b = int(g[k]), int(g[k + 1])
        if b > a:
            A[a:b] = r[a:b] - np.mean(r[a:b])
    return A


def scored_rows(resp_offsets, prompt_lens, n_rows: int) -> np.ndarray:
    """Boolean mask of the scored rows: response rows after their prompt prefix."""
    off = _i64(resp_offsets)
    pl = None if prompt_lens is None else _i64(prompt_lens)
    mask = np.zeros(n_rows, dtype=bool)
    for i in range(off.shape[0] - 1):
        a, b = int(off[i]), int(off[i + 1])
        p = 0 if pl is None else int(pl[i])
        mask[a + p:b] = True
    return mask


def response_coefficients(A, resp_offsets, prompt_lens, resp_normalizer: float = 0.0):
    """n_i (scored tokens of response i) and c_i = A_i / (R* n_i) (0 when n_i = 0)."""
    off = _i64(resp_offsets)
    R = off.shape[0] - 1
    lens = off[1:] - off[:-1]
    n = lens - (0 if prompt_lens is None else _i64(prompt_lens))
    n = np.maximum(n, 0)
    Rstar = float(R) if resp_normalizer == 0 else float(resp_normalizer)
    c = np.zeros(R)
    nz = n > 0
    c[nz] = _f64(A)[nz] / (Rstar * n[nz])
    return n, c


# ---------------------------------------------------------------------------
# Full step: loss, per-token terms, D3 and gradients
# ---------------------------------------------------------------------------

def token_terms(variant: str, w, delta, A_row, n_row, rstar: float, resp_of_row, mask, c_row,
                eps_low: float = 0.2, eps_high: float = 0.2, gate: float = math.inf) -> dict:
    """Per-token loss l_t and gradient coefficient g_t = dL/dlog pi_t of each loss variant.

    unclipped: l_t = -w A / (R* n),  g_t = l_t                         ([ZM-path], [RZ-core])
    ppo_clip:  l_t = -min(w A, clip(w) A) / (R* n); g_t = -w A / (R* n) where the first
               argument is the minimum (ties included), else 0
    seq_gate:  the unclipped terms, zeroed on every row of a rejected response
    """
    T = w.shape[0]
    with np.errstate(invalid="ignore", over="ignore", divide="ignore"):
        denom = rstar * n_row
        if variant == "unclipped":
            l = np.where(mask, -c_row * w, 0.0)
            return {"token_loss": l, "g": l.copy(), "n_clipped": 0, "n_rejected": 0,
                    "rejected": np.zeros(0, dtype=bool)}
        if variant == "ppo_clip":
            first = w * A_row
            second = np.clip(w, 1.0 - eps_low, 1.0 + eps_high) * A_row
            sur = np.minimum(first, second)
            active = first <= second
            l = np.where(mask, -sur / np.where(mask, denom, 1.0), 0.0)
            g = np.where(mask & active, -first / np.where(mask, denom, 1.0), 0.0)
            n_clipped = int(np.sum(mask & ~active & (A_row != 0)))
            return {"token_loss": l, "g": g, "n_clipped": n_clipped, "n_rejected": 0,
                    "rejected": np.zeros(0, dtype=bool)}
        if variant == "seq_gate":
            R = int(np.max(resp_of_row)) + 1 if T else 0
            R = max(R, 0)
            sums = np.zeros(R)
            cnt = np.zeros(R)
            for t in range(T):
                if mask[t]:
                    sums[resp_of_row[t]] += delta[t]
                    cnt[resp_of_row[t]] += 1
            rho = np.where(cnt > 0, sums / np.maximum(cnt, 1), 0.0)
            rejected = (cnt > 0) & ~(np.abs(rho) <= gate)
            keep_row = mask & ~rejected[resp_of_row] if T else mask
            l = np.where(keep_row, -c_row * w, 0.0)
            return {"token_loss": l, "g": l.copy(), "n_clipped": 0, "n_rejected": int(np.sum(rejected)),
                    "rejected": rejected, "rho": rho}
    raise ValueError(f"unknown loss variant {variant!r}")


def is_loss_fwd_bwd(hidden, w, targets, rollout_logprob, rewards, resp_offsets, group_offsets,
                    prompt_lens=None, resp_normalizer: float = 0.0, want_grads: bool = True,
                    want_grad_w: bool = True, variant: str = "unclipped", eps_low: float = 0.2,
                    eps_high: float = 0.2, gate: float = math.inf) -> dict:
    """Everything the fused learner step returns, in float64.

    L   = sum_t l_t over the scored tokens (l_t of the variant, see ``token_terms``;
          unclipped: l_t = -c_i w_t, c_i = A_i / (R* n_i))
    g_t = dL/dlog pi_t  (0 on unscored rows)
    dZ  = g_t (onehot(y_t) - p_t),  p_t = softmax(z_t)
    dH  = dZ W,   dW = dZ^T H
    """
    Hm = _f64(hidden)
    Wm = _f64(w)
    y = _i64(targets)
    off = _i64(resp_offsets)
    T = Hm.shape[0]
    assert int(off[-1]) == T and int(off[0]) == 0
    logmu = _f64(rollout_logprob)

    A = advantages(rewards, group_offsets)
    n, c = response_coefficients(A, off, prompt_lens, resp_normalizer)
    mask = scored_rows(off, prompt_lens, T)
    resp_of_row = np.repeat(np.arange(off.shape[0] - 1), off[1:] - off[:-1])
    c_row = c[resp_of_row]

    lp_all, lse_all = token_logprob(Hm, Wm, y, rows=np.nonzero(mask)[0])
    logprob = np.zeros(T)
    lse = np.zeros(T)
    logprob[mask] = lp_all
    lse[mask] = lse_all
    wgt = np.zeros(T)
    delta = np.zeros(T)
    w_s, d_s = is_weight(lp_all, logmu[mask])
    wgt[mask] = w_s
    delta[mask] = d_s
    rstar = float(resp_normalizer) if resp_normalizer > 0 else float(off.shape[0] - 1)
    terms = token_terms(variant, wgt, delta, A[resp_of_row], n[resp_of_row].astype(np.float64), rstar,
                        resp_of_row, mask, c_row, eps_low, eps_high, gate)
    token_loss = terms["token_loss"]
    with np.errstate(invalid="ignore", over="ignore"):
        loss = float(np.sum(token_loss))
    d3 = d3_stats(lp_all, logmu[mask])
    kl = kl_estimators(lp_all, logmu[mask])

    out = {"loss": loss, "logprob": logprob, "lse": lse, "is_weight": wgt, "delta": delta,
           "token_loss": token_loss, "d3": d3, "kl": kl, "advantages": A, "n_scored": n, "coef": c,
           "mask": mask, "n_clipped": terms["n_clipped"], "n_rejected": terms["n_rejected"],
           "rejected": terms["rejected"]}
    if "rho" in terms:
        out["rho"] = terms["rho"]
    if not want_grads:
        return out
    g = terms["g"]
    dH = np.zeros_like(Hm)
    dW = np.zeros_like(Wm) if want_grad_w else None
    rows = np.nonzero(mask)[0]
    for s in range(0, rows.shape[0], _ROW_CHUNK):
        r = rows[s:s + _ROW_CHUNK]
        z = Hm[r] @ Wm.T
        logp, _ = log_softmax_rows(z)
        dZ = -np.exp(logp)
        dZ[np.arange(r.shape[0]), y[r]] += 1.0
        dZ *= g[r][:, None]
        dH[r] = dZ @ Wm
        if want_grad_w:
            dW += dZ.T @ Hm[r]
    out["grad_hidden"] = dH
    out["grad_w"] = dW
    return out


def grad_rows(hidden, w, targets, g_rows, rows) -> np.ndarray:
    """dH rows for the given rows and per-row coefficients g (row-local, any size)."""
    Hm = _f64(hidden)
    Wm = _f64(w)
    y = _i64(targets)
    r = np.asarray(rows, dtype=np.int64)
    out = np.empty((r.shape[0], Wm.shape[1]))
    for s in range(0, r.shape[0], _ROW_CHUNK):
        rr = r[s:s + _ROW_CHUNK]
        z = Hm[rr] @ Wm.T
        logp, _ = log_softmax_rows(z)
        dZ = -np.exp(logp)
        dZ[np.arange(rr.shape[0]), y[rr]] += 1.0
        dZ *= np.asarray(g_rows[s:s + _ROW_CHUNK], dtype=np.float64)[:, None]
        out[s:s + _ROW_CHUNK] = dZ @ Wm
    return out


def grad_w_rows(hidden, w, targets, g_rows, lse_rows, vocab_ids) -> np.ndarray:
    """dW rows for the given vocabulary ids: dW_v = sum_t dZ_tv h_t over every row t, with
    dZ_tv = g_t (1[v = y_t] - exp(z_tv - lse_t)) (g_t = 0 on unscored rows).  Needs only the
    logits of the selected ids, so any T fits; ``lse_rows`` comes from ``token_logprob``."""
    Hm = _f64(hidden)
    Wm = _f64(w)
    y = _i64(targets)
    v = np.asarray(vocab_ids, dtype=np.int64)
    g = np.asarray(g_rows, dtype=np.float64)
    lse = np.asarray(lse_rows, dtype=np.float64)
    out = np.zeros((v.shape[0], Wm.shape[1]))
    for s in range(0, Hm.shape[0], 4096):
        z = Hm[s:s + 4096] @ Wm[v].T
        dZ = -np.exp(z - lse[s:s + 4096, None])
        dZ += (y[s:s + 4096, None] == v[None, :])
        dZ *= g[s:s + 4096, None]
        out += dZ.T @ Hm[s:s + 4096]
    return out


def kl_estimators(learner_logprob, rollout_logprob, mask=None) -> dict:
    """Sampled estimators of KL(mu || pi) from rollout samples, r = w = pi/mu:
    k1 = -log r, k2 = (log r)^2 / 2, k3 = r - 1 - log r (the D3 term); means over tokens."""
    _, delta = is_weight(learner_logprob, rollout_logprob)
    if mask is not None:
        delta = delta[np.asarray(mask).astype(bool)]
    if delta.shape[0] == 0:
        return {"k1": 0.0, "k2": 0.0, "k3": 0.0}
    return {"k1": float(np.mean(-delta)), "k2": float(np.mean(0.5 * delta * delta)),
            "k3": float(np.mean(d3_terms(delta)))}


def d3_peak_median(d3_means) -> dict:
    """Peak over median of per-update D3 means ([ZM-gap]: 1.50x aligned, 442.54x standard)."""
    d = np.asarray(d3_means, dtype=np.float64)
    if d.shape[0] == 0:
        return {"peak": 0.0, "median": 0.0, "ratio": float("nan")}
    med = float(np.median(d))
    peak = float(np.max(d))
    return {"peak": peak, "median": med, "ratio": peak / med if med != 0 else float("inf")}


def kl_drift(values, window: int) -> float:
    """Median over the last ``window`` updates divided by the median over the first ``window``
    ([ZM-path] Fig. 1: median rollout-to-learner KL rises 83.33x with standard kernels)."""
    v = np.asarray(values, dtype=np.float64)
    if v.shape[0] < window or window <= 0:
        raise ValueError("need at least one full window of updates")
    return float(np.median(v[-window:]) / np.median(v[:window]))


def loss_only(hidden, w, targets, rollout_logprob, rewards, resp_offsets, group_offsets,
              prompt_lens=None, resp_normalizer: float = 0.0, **variant) -> float:
    """The scalar loss (no gradients); used by finite-difference pins."""
    return is_loss_fwd_bwd(hidden, w, targets, rollout_logprob, rewards, resp_offsets,
                           group_offsets, prompt_lens, resp_normalizer, want_grads=False, **variant)["loss"]


def minus_log_v(V: int) -> float:
    """-log V: the log-probability of any token under a uniform softmax."""
    return -math.log(V)
