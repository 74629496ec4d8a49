"""Acceptance telemetry of a run of verify steps (host-side bookkeeping, no GPU).

Gemma 4 MTP serving guide, section 6 "observability": the guide watches the overall
acceptance rate, the mean accepted length per step (MAL) and the per-position decay of
acceptance.  With a_s accepted drafts in step s (0 <= a_s <= k):

  position rate r_i   = P(a >= i), i = 1..k        (cumulative: the draft at position i
                                                    was accepted, so were all before it)
  conditional rate    = P(a >= i | a >= i-1)
  MAL                 = 1 + sum_i r_i = E[a + 1]    (tokens emitted per step)
  overall acceptance  = sum_i r_i / k = E[a] / k

Section 2 of the same guide prints r = (0.47, 0.24) and MAL 1.71 at k = 2, consistent
with the cumulative reading (1 + 0.47 + 0.24 = 1.71).
"""
from __future__ import annotations

import numpy as np


def acceptance_telemetry(n_accepted, k: int) -> dict:
    a = np.asarray(n_accepted, np.int64).ravel()
    if a.size == 0:
        raise ValueError("no steps")
    if k < 0 or a.min() < 0 or a.max() > k:
        raise ValueError("accepted counts must lie in [0, k]")
    rates = [float((a >= i).mean()) for i in range(1, k + 1)]
    cond = []
    prev = 1.0
    for r in rates:
        cond.append(r / prev if prev > 0 else 0.0)
        prev = r
    return dict(k=k, steps=int(a.size), position_rates=rates, conditional_rates=cond,
                mal=1.0 + float(sum(rates)),
                overall_acceptance=float(sum(rates) / k) if k else 0.0)
