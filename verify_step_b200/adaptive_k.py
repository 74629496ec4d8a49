"""Choosing the number of drafts k from acceptance telemetry (host side, no GPU).

Gemma 4 MTP serving guide (butteryoon.github.io), section 2 "measured benchmark" and
section 6 "observability", and its closing checklist:
  * raise k step by step and fix it where the mean acceptance length per step (MAL) stops
    improving; the guide's own workload settles at k = 2 (MAL 1.00, 1.45, 1.71 at k = 0, 1, 2,
    k >= 3 dropped because the extra verification ate the gain);
  * if position 0 accepts normally but position 1 accepts below 15 %, cut k to 1;
  * overall acceptance below 25 % for a sustained period signals domain drift (realign the
    drafter); section 5 adds that below 20 % speculation costs verification without a speedup.

Readings taken where the guide gives no number:
  * "stops improving": the relative MAL gain of k over k - 1 is below ``plateau_gain``.  MAL alone
    cannot see the verification cost; 0.10 makes the policy settle at k = 2 on the guide's own
    telemetry (gain 1 -> 2 is 17.9 %, gain 2 -> 3 with the guide's decay is about 7 %).
  * "position 0 accepts normally": P(a >= 1) within 25 % of the guide's reference 0.47 (>= 0.35).
  * "sustained": the whole observation window.
Position rates are cumulative, r_i = P(a >= i) (``telemetry.acceptance_telemetry``).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .telemetry import acceptance_telemetry


@dataclass
class Decision:
    k: int                      # drafts to use for the next window
    phase: str                  # "explore" (still raising k) or "hold"
    reasons: list = field(default_factory=list)
    alerts: list = field(default_factory=list)
    telemetry: dict | None = None


class AdaptiveK:
    """Windowed controller: feed it the accepted counts of every verify step
    (``observe``); after ``window`` steps at the current k it returns a ``Decision``."""

    def __init__(self, k_init: int = 1, k_min: int = 1, k_max: int = 6, window: int = 2000,
                 plateau_gain: float = 0.10, pos1_floor: float = 0.15, pos0_normal: float = 0.35,
                 drift_floor: float = 0.25, no_gain_floor: float = 0.20):
        if not (1 <= k_min <= k_init <= k_max):
            raise ValueError("need 1 <= k_min <= k_init <= k_max")
        if window < 1:
            raise ValueError("window must be positive")
        self.k_min, self.k_max, self.window = k_min, k_max, window
        self.plateau_gain, self.pos1_floor, self.pos0_normal = plateau_gain, pos1_floor, pos0_normal
        self.drift_floor, self.no_gain_floor = drift_floor, no_gain_floor
        self.k = k_init
        self.phase = "explore"
        self.mal = {}              # k -> MAL measured over a full window at that k
        self._buf = []

    def observe(self, n_accepted) -> Decision | None:
        """Adds one verify step's accepted counts (one per sequence); returns a decision when a
        window is complete, else None."""
        a = np.asarray(n_accepted, np.int64).ravel()
        if a.size and (a.min() < 0 or a.max() > self.k):
            raise ValueError(f"accepted counts must lie in [0, {self.k}]")
        self._buf.append(a)
        if sum(x.size for x in self._buf) < self.window:
            return None
        counts = np.concatenate(self._buf)
        self._buf = []
        return self._decide(counts)

    def _decide(self, counts) -> Decision:
        t = acceptance_telemetry(counts, self.k)
        d = Decision(k=self.k, phase=self.phase, telemetry=t)
        rates = t["position_rates"]
        if t["overall_acceptance"] < self.no_gain_floor:
            d.alerts.append(f"overall acceptance {t['overall_acceptance']:.3f} < "
                            f"{self.no_gain_floor}: verification without speedup")
        elif t["overall_acceptance"] < self.drift_floor:
            d.alerts.append(f"overall acceptance {t['overall_acceptance']:.3f} < "
                            f"{self.drift_floor}: drafter drift, realign it")
        # position-1 collapse: cut to one draft (both phases)
        if self.k >= 2 and rates[0] >= self.pos0_normal and rates[1] < self.pos1_floor:
            d.reasons.append(f"pos0 {rates[0]:.3f} normal but pos1 {rates[1]:.3f} < "
                             f"{self.pos1_floor}: k -> 1")
            self.k, self.phase = max(1, self.k_min), "hold"
            d.k, d.phase = self.k, self.phase
            return d
        self.mal[self.k] = t["mal"]
        if self.phase == "explore":
            prev = self.mal.get(self.k - 1)
            if prev is not None and t["mal"] < prev * (1.0 + self.plateau_gain):
                d.reasons.append(f"MAL {t['mal']:.3f} at k={self.k} gains < "
                                 f"{self.plateau_gain:.0%} over {prev:.3f}: hold k={self.k - 1}")
                self.k, self.phase = self.k - 1, "hold"
            elif self.k < self.k_max:
                d.reasons.append(f"MAL {t['mal']:.3f} at k={self.k}: try k={self.k + 1}")
                self.k += 1
            else:
                d.reasons.append(f"k_max={self.k_max} reached: hold")
                self.phase = "hold"
        d.k, d.phase = self.k, self.phase
        return d
