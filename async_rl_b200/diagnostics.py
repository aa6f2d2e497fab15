"""Stability diagnostics across updates, host side.

"Zero Mismatch, Simple Async RL" reads two statistics over a run:
* section "Only one probability gap comes from old weights": the per-update D3 (token mean of
  w - 1 - log w) and the ratio of its peak to its median over the run (1.50x with aligned kernels,
  442.54x with standard kernels);
* section "Alignment permits a simpler learning path", Fig. 1: the median rollout-to-learner KL
  over the first and the last thousand updates (it rises 83.33x with standard kernels), and the
  fraction of sequences a rejection gate discards.

Each update's numbers come from the device-written ``bi_d3`` of ``bi_is_loss_fwd_bwd`` (decoded
by ``LossOutputs.d3()``); this module only keeps the series and takes order statistics.
"""
from __future__ import annotations

import statistics
from typing import Dict, List


class UpdateTracker:
    """Series of per-update diagnostics: D3 (= the k3 KL estimator), k1, k2, rejections."""

    def __init__(self) -> None:
        self.d3: List[float] = []
        self.k1: List[float] = []
        self.k2: List[float] = []
        self.n_rejected: List[int] = []
        self.n_tokens: List[int] = []

    def add(self, d3: Dict) -> None:
        """Record one update's decoded ``bi_d3`` dictionary."""
        self.d3.append(float(d3["mean"]))
        self.k1.append(float(d3["k1"]))
        self.k2.append(float(d3["k2"]))
        self.n_rejected.append(int(d3.get("n_rejected", 0)))
        self.n_tokens.append(int(d3["count"]))

    def __len__(self) -> int:
        return len(self.d3)

    def d3_peak_over_median(self) -> float:
        """Largest per-update D3 over the median per-update D3 (inf when the median is 0)."""
        if not self.d3:
            raise ValueError("no updates recorded")
        med = statistics.median(self.d3)
        peak = max(self.d3)
        return peak / med if med != 0 else float("inf")

    def kl_drift(self, window: int, estimator: str = "k3") -> float:
        """Median of the chosen KL estimator over the last ``window`` updates divided by its median
        over the first ``window`` updates."""
        series = {"k1": self.k1, "k2": self.k2, "k3": self.d3}[estimator]
        if window <= 0 or len(series) < window:
            raise ValueError("need at least one full window of updates")
        return statistics.median(series[-window:]) / statistics.median(series[:window])

    def rejection_rate(self, n_responses: List[int], window: int) -> float:
        """Rejected responses over the responses of the last ``window`` updates."""
        if window <= 0 or len(self.n_rejected) < window or len(n_responses) != len(self.n_rejected):
            raise ValueError("need one response count per update and a full window")
        return sum(self.n_rejected[-window:]) / max(1, sum(n_responses[-window:]))
