"""CPU checks of the host-side summary that the bench reports for the
staleness sweep: errors grouped by the factor's age (steps since its
refresh), and the falsifier's flag (the stalest factor's error in whitened
coordinates reaching the Euclidean one)."""
import numpy as np
import pytest

from geometry_aware_fp8_b200 import staleness


def _fake(T, K):
    age = np.arange(T) % K
    white = (0.02 + 0.01 * age).tolist()
    frob = (0.03 + 0.001 * age).tolist()
    return {"euclid": {"frob": [0.026] * T, "white": [0.05] * T}, K: {"frob": frob, "white": white}}


def test_summary_groups_errors_by_age():
    T, K = 12, 4
    s = staleness.summary(_fake(T, K), [K])
    v = s[f"K={K}"]
    assert v["white_fresh"] == pytest.approx(0.02)
    assert v["white_stalest"] == pytest.approx(0.05)  # age K - 1 = 3
    assert v["frob_stalest"] == pytest.approx(0.033)
    assert v["white_mean"] == pytest.approx(np.mean(0.02 + 0.01 * (np.arange(T) % K)))
    assert v["stalest_reaches_euclid_white"]  # 0.05 >= 0.05
    assert s["euclid"]["white"] == pytest.approx(0.05)


def test_summary_when_the_sweep_is_shorter_than_the_interval():
    # T < K: the stalest age seen is T - 1
    s = staleness.summary(_fake(3, 10), [10])
    assert s["K=10"]["white_stalest"] == pytest.approx(0.04)
    assert not s["K=10"]["stalest_reaches_euclid_white"]
