"""The seeded input helpers shared by the CUDA path's tests and the oracle's
callers (no arithmetic of the method lives there)."""
import pytest

from reduction_epilogue_b200 import synth


@pytest.mark.parametrize("M,n", [(16, 64), (128, 128), (1024, 1024), (2048, 64), (5, 3), (1, 64), (300, 1),
                                 (32768, 128)])
def test_sample_rows_gives_exactly_the_rows_asked_for(M, n):
    rows = synth.sample_rows(M, n, seed=1)
    assert len(rows) == min(M, n) == len(set(rows))
    assert rows == sorted(rows) and all(0 <= r < M for r in rows)
    if min(M, n) >= 2:
        assert rows[0] == 0 and rows[-1] == M - 1  # both tile edges
    assert rows == synth.sample_rows(M, n, seed=1)  # seeded


def test_linear_inputs_follow_the_stated_distribution():
    x, W, b = synth.linear_inputs(64, 256, 96, seed=3)
    bound = 1.0 / 16.0
    assert x.shape == (64, 256) and W.shape == (96, 256) and b.shape == (96,)
    assert W.abs().max() <= bound and b.abs().max() <= bound
    assert abs(float(x.mean())) < 0.05 and abs(float(x.std()) - 1.0) < 0.05
