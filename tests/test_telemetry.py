"""Telemetry definitions pinned to the serving guide's printed numbers."""
import json
import os

import numpy as np
import pytest

from verify_step_b200.telemetry import acceptance_telemetry

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mal_telemetry.json")


def test_printed_numbers_are_consistent_with_cumulative_reading():
    g = json.load(open(GOLDEN))
    r1, r2 = g["per_position_acceptance_cumulative"]
    # 100 steps with exactly these cumulative rates: 24 x a=2, 23 x a=1, 53 x a=0
    a = np.array([2] * round(100 * r2) + [1] * round(100 * (r1 - r2)) + [0] * round(100 * (1 - r1)))
    t = acceptance_telemetry(a, g["k"])
    assert t["position_rates"] == pytest.approx([r1, r2])
    assert t["mal"] == pytest.approx(g["mal_printed"], abs=1e-12)
    lo, hi = g["overall_acceptance_range_printed"]
    assert lo <= t["overall_acceptance"] <= hi
    # the conditional reading of "pos1 ~24%" would not reproduce the printed MAL
    assert abs((1 + r1 + r1 * r2) - g["mal_printed"]) > 0.1


def test_k1_row():
    g = json.load(open(GOLDEN))
    a = np.array([1] * 45 + [0] * 55)
    assert acceptance_telemetry(a, 1)["mal"] == pytest.approx(g["mal_k1_printed"])


def test_invalid_counts_rejected():
    with pytest.raises(ValueError):
        acceptance_telemetry([3], 2)
    with pytest.raises(ValueError):
        acceptance_telemetry([], 2)
