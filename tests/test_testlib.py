"""The comparison helper of the parity tests, on the CPU: absolute figures
are always recorded, and a magnitude-relative bound is refused for tensors
that are not sums over windows or tokens."""
import numpy as np
import pytest

from tests import rib_testlib as T


def test_absolute_figures_are_recorded_even_when_normalised():
    ref = np.full(10, 40.0)
    got = ref + 0.05
    n = len(T.RECORDS)
    msg = T.check_close(got, ref, "dQp", normalize=True)
    assert msg == ""                    # 0.05 / 40 = 1.25e-3, within 2e-2 / 2e-3
    r = T.RECORDS[n]
    assert r["what"] == "dQp" and r["max_abs"] == pytest.approx(0.05)
    assert r["abs_within"] is False and r["within"] is True
    assert r["normalised_by"] == 40.0


def test_normalised_bound_refused_for_outputs():
    with pytest.raises(AssertionError, match="not allowed"):
        T.check_close(np.zeros(3), np.ones(3), "out", normalize=True)
    assert T.check_close(np.ones(3), np.ones(3), "out", normalize=True, grown_inputs=True) == ""


def test_plain_bound():
    assert T.check_close(np.zeros(4), np.full(4, 1e-3), "dqkv") == ""
    assert "beyond" in T.check_close(np.zeros(4), np.full(4, 3e-2), "dqkv")
