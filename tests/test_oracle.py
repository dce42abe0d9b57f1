"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test below checks the oracle against something other than itself: the
pages' worked values (tests/golden/), closed forms, exact integer arithmetic,
exact rational brute force, or numpy's float64 matmul.  The cases are chosen so
that a plausible slip in the oracle (a dropped bias, a transposed weight, an
off-by-one in the k loop, scale and clamp swapped, tanh-GELU for erf-GELU, a
max taken before the GELU, sum instead of mean in the pool, a wrong window
count) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

SQRT2 = math.sqrt(2.0)


@pytest.fixture(scope="module")
def normal_values(golden_dir):
    with open(os.path.join(golden_dir, "normal_values.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# The contraction y = x W^T + b
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N", [(1, 1, 1), (3, 5, 7), (7, 3, 5), (5, 7, 3), (16, 33, 9), (2, 64, 130)])
def test_linear_matches_numpy_float64(M, K, N):
    x, W, b = synth.linear_inputs(M, K, N, seed=M * 100 + K * 10 + N)
    x, W, b = x.numpy(), W.numpy(), b.numpy()
    y = oracle.linear_rows(x, W, b)
    ref = x.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    assert y.shape == (M, N)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_linear_exact_integers_brute_force():
    # Small integers: every product and partial sum is exact in fp64, so the
    # oracle must equal Python's exact integer dot products.
    M, K, N = 4, 11, 6
    x, W, b = synth.integer_inputs(M, K, N, seed=3)
    x, W, b = x.numpy(), W.numpy(), b.numpy()
    y = oracle.linear_rows(x, W, b)
    for m in range(M):
        for n in range(N):
            exact = int(b[n]) + sum(int(x[m, k]) * int(W[n, k]) for k in range(K))
            assert y[m, n] == exact


def test_linear_exact_rational_brute_force():
    # Exact rational arithmetic on the fp32 values: the oracle's fp64 result
    # must be within a few fp64 ulps of the exact sum.
    M, K, N = 3, 9, 4
    x, W, b = synth.linear_inputs(M, K, N, seed=11)
    x, W, b = x.numpy(), W.numpy(), b.numpy()
    y = oracle.linear_rows(x, W, b)
    for m in range(M):
        for n in range(N):
            exact = Fraction(float(b[n])) + sum(Fraction(float(x[m, k])) * Fraction(float(W[n, k])) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(1, 2**45) * (1 + abs(exact))


def test_linear_uses_W_rows_not_columns_and_the_last_k():
    # W[n] is row n of a [N,K] matrix; a transposed read or a k loop that stops
    # one short both change these values.
    x = np.array([[1.0, 10.0, 100.0]], dtype=np.float32)
    W = np.array([[1.0, 0.0, 0.0], [0.0, 0.0, 1.0]], dtype=np.float32)
    b = np.array([0.5, -0.5], dtype=np.float32)
    y = oracle.linear_rows(x, W, b)
    assert y.tolist() == [[1.5, 99.5]]
    assert oracle.linear_rows(x, W, None).tolist() == [[1.0, 100.0]]


def test_row_subset_equals_full():
    M, K, N = 9, 17, 5
    x, W, b = synth.linear_inputs(M, K, N, seed=5)
    full = oracle.forward_rows(x.numpy(), W.numpy(), b.numpy(), **oracle.PROBLEMS["scale_hardtanh_gelu"])
    rows = [8, 0, 4]
    sub = oracle.forward_rows(x.numpy(), W.numpy(), b.numpy(), rows=rows, **oracle.PROBLEMS["scale_hardtanh_gelu"])
    np.testing.assert_array_equal(sub, full[rows])


# --------------------------------------------------------------------------
# GELU, the normal CDF and the pages' printed values
# --------------------------------------------------------------------------

def test_gelu_against_normal_table(normal_values):
    for e in normal_values["textbook_values"]:
        v = float(e["quantity"][4:-1])  # "Phi(x)"
        # GELU(v)/v = Phi(v) for v != 0
        assert abs(oracle.gelu(v) / v - e["value"]) <= e["abs_tol"] + 1e-16, e


def test_gelu_against_page_values(normal_values):
    pv = {e["quantity"]: e for e in normal_values["page_values"]}
    e = pv["erf(2/sqrt(2))"]
    # GELU(2) = 2 * (1 + erf(2/sqrt2)) / 2
    assert abs((oracle.gelu(2.0) - 1.0) - e["value"]) <= e["abs_tol"]
    e = pv["Phi(-1)"]
    assert abs(oracle.gelu(-1.0) / -1.0 - e["value"]) <= e["abs_tol"]
    # derivative by central differences: GELU'(x) = Phi(x) + x phi(x)
    h = 1e-5
    d = (oracle.gelu(-1.0 + h) - oracle.gelu(-1.0 - h)) / (2 * h)
    e = pv["gelu_derivative(-1)"]
    assert abs(d - e["value"]) <= e["abs_tol"]
    # and phi(-1) = GELU'(-1) - Phi(-1), divided by x = -1
    phi_m1 = (d - oracle.gelu(-1.0) / -1.0) / -1.0
    e = pv["phi(-1)"]
    assert abs(phi_m1 - e["value"]) <= e["abs_tol"]


def test_gelu_closed_forms():
    assert oracle.gelu(0.0) == 0.0
    for v in [0.1, 0.75, 1.0, 1.7, 2.0, 3.3]:
        # Phi(-v) = 1 - Phi(v)  =>  GELU(v) - GELU(-v) = v
        assert abs((oracle.gelu(v) - oracle.gelu(-v)) - v) < 1e-15
    assert oracle.gelu(40.0) == 40.0
    assert oracle.gelu(-40.0) == 0.0 or abs(oracle.gelu(-40.0)) < 1e-300
    # global minimum near x = -0.7518 at about -0.16997
    xs = np.linspace(-3, 0, 30001)
    g = np.array([oracle.gelu(v) for v in xs])
    assert abs(xs[g.argmin()] - (-0.7518)) < 2e-4
    assert abs(g.min() - (-0.16997)) < 1e-5


def test_gelu_is_erf_form_not_tanh_form():
    # The tanh approximation differs from the erf form by up to ~4.7e-4;
    # at x = -2.699 the gap is at its largest.
    v = -2.699
    tanh_form = 0.5 * v * (1 + math.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3)))
    erf_form = v * 0.5 * math.erfc(-v / SQRT2)
    assert abs(oracle.gelu(v) - erf_form) < 1e-15
    assert abs(oracle.gelu(v) - tanh_form) > 4e-4


# --------------------------------------------------------------------------
# Epilogue (a): scale -> hardtanh -> GELU
# --------------------------------------------------------------------------

def test_gelu_tanh_form_closed_forms():
    # The tanh form (page l2_p53's first fused kernel): v/2 (1 + tanh(c (v +
    # 0.044715 v^3))), c = sqrt(2/pi).  tanh is odd, so the same identity as
    # the erf form holds: G(v) - G(-v) = v; G(0) = 0; G(v) -> v and -> 0.
    assert oracle.gelu_tanh(0.0) == 0.0
    for v in [0.1, 0.75, 1.0, 1.7, 2.0, 3.3]:
        assert abs((oracle.gelu_tanh(v) - oracle.gelu_tanh(-v)) - v) < 1e-15
    assert abs(oracle.gelu_tanh(30.0) - 30.0) < 1e-12
    assert abs(oracle.gelu_tanh(-30.0)) < 1e-12
    # curvature at 0: G(h) + G(-h) = h tanh(c (h + 0.044715 h^3)) ~ c h^2,
    # which pins c = sqrt(2/pi) = 0.7978845608...
    h = 1e-4
    assert abs((oracle.gelu_tanh(h) + oracle.gelu_tanh(-h)) / h**2 - 0.7978845608) < 1e-6


def test_gelu_tanh_form_distance_from_erf_form():
    # Against the (independently pinned) erf form: the approximation is off
    # by at most 4.73e-4, at |v| ~ 2.70, and by 9.80e-5 at v = 2 (the page's
    # printed figure for that gap is garbled; these are the values of the two
    # closed forms).  A wrong constant or a dropped factor moves both (e.g.
    # 0.04715 for 0.044715 gives a 1.5e-3 gap).
    xs = np.linspace(-8, 8, 16001)
    d = np.array([oracle.gelu_tanh(v) - oracle.gelu(v) for v in xs])
    i = int(np.abs(d).argmax())
    assert 4.6e-4 < abs(d[i]) < 4.8e-4
    assert 2.6 < abs(xs[i]) < 2.8
    assert abs((oracle.gelu_tanh(2.0) - oracle.gelu(2.0)) - 9.80e-5) < 1e-6
    # the gap is even in v (both forms satisfy G(v) - G(-v) = v)
    assert np.allclose(d, d[::-1], rtol=0, atol=1e-13)


def test_forward_with_tanh_form():
    # gelu_tanh switches the GELU of epilogues (a) and (c), nothing else
    x = np.array([[1.0, -2.0, 0.5, 3.0]], dtype=np.float32)
    W = np.array([[0.5, 0.25, -1.0, 0.125], [1.0, 1.0, 1.0, 1.0]], dtype=np.float32)
    b = np.array([0.25, -0.5], dtype=np.float32)
    y = oracle.linear_rows(x, W, b)[0]
    a = oracle.forward_rows(x, W, b, gelu_tanh=True, **oracle.PROBLEMS["scale_hardtanh_gelu"])[0]
    for n in range(2):
        t = min(max(0.5 * y[n], -2.0), 2.0)
        assert a[n] == np.float32(oracle.gelu_tanh(t))
    sw = oracle.forward_rows(x, W, b, gelu_tanh=True, **oracle.PROBLEMS["swish_scale"])
    assert (sw == oracle.forward_rows(x, W, b, **oracle.PROBLEMS["swish_scale"])).all()
    Wp = np.tile(W, (8, 1))  # N = 16: one pool window
    bp = np.tile(b, 8)
    c = oracle.forward_rows(x, Wp, bp, gelu_tanh=True, **oracle.PROBLEMS["avgpool_gelu_scale_rowmax"])[0]
    p = oracle.linear_rows(x, Wp, bp)[0].mean()
    assert c == np.float32(2.0 * oracle.gelu_tanh(p))


def test_epilogue_a_saturation_and_order(normal_values):
    tb = {e["quantity"]: e["value"] for e in normal_values["textbook_values"]}
    f = oracle.scale_hardtanh_gelu
    assert f(0.0) == 0.0
    # 0.5*y >= 2 saturates at 2*Phi(2); <= -2 at -2*Phi(-2)
    for y in [4.0, 4.5, 10.0, 1e6]:
        assert abs(f(y) - 2 * tb["Phi(2)"]) < 1e-15
    for y in [-4.0, -7.0, -1e6]:
        assert abs(f(y) - (-2 * tb["Phi(-2)"])) < 1e-16
    # scale first: y = 3 gives GELU(1.5); clamping first would give GELU(1)
    assert abs(f(3.0) - 1.5 * tb["Phi(1.5)"]) < 1e-15
    assert abs(f(2.0) - tb["Phi(1)"]) < 1e-15
    # asymmetric clamp: a swapped lo/hi changes the result
    assert abs(f(10.0, 0.5, -1.0, 0.5) - 0.5 * tb["Phi(0.5)"]) < 1e-15
    assert abs(f(-10.0, 0.5, -1.0, 0.5) - (-1.0 * (1 - tb["Phi(1)"]))) < 1e-15


# --------------------------------------------------------------------------
# Epilogue (b): swish -> scale
# --------------------------------------------------------------------------

def test_epilogue_b_closed_forms():
    f = oracle.swish_scale
    assert f(0.0) == 0.0
    # sigmoid(0) = 1/2, sigmoid(1) = e/(1+e)
    assert abs(f(1.0, 2.0) - 2.0 * math.e / (1 + math.e)) < 1e-15
    # sigmoid(-y) = 1 - sigmoid(y)  =>  swish(y) - swish(-y) = y
    for y in [0.3, 1.0, 2.5, 7.0]:
        assert abs((f(y, 1.0) - f(-y, 1.0)) - y) < 1e-14
        assert abs((f(y, 2.0) - f(-y, 2.0)) - 2 * y) < 1e-14
    assert f(100.0, 2.0) == 200.0
    v = f(-1000.0, 2.0)
    assert v == 0.0 and not math.isnan(v)
    assert f(-5.0, 2.0) < 0


# --------------------------------------------------------------------------
# Epilogue (c): AvgPool1d(k) -> GELU -> scale -> row max
# --------------------------------------------------------------------------

def test_pool_fold_toy_from_page(golden_dir):
    with open(os.path.join(golden_dir, "pool_fold_toy.json")) as f:
        g = json.load(f)
    x = np.array(g["x"], dtype=np.float32)
    W = np.array(g["W"], dtype=np.float32)
    b = np.array(g["b"], dtype=np.float32)
    y = oracle.linear_rows(x, W, b)
    assert y[0].tolist() == g["linear_out"]
    k = g["pool_k"]
    # Route 1: the oracle's pooled max equals 2*GELU of the larger window mean
    out = oracle.forward_rows(x, W, b, kind=oracle.EPI_AVGPOOL_GELU_SCALE_ROWMAX, scale=2.0, pool_k=k)
    assert out.shape == (1,)
    assert out[0] == np.float32(2.0 * oracle.gelu(g["pooled"][1]))
    # Route 2: the pooled weights through the oracle's Linear give the same means
    y2 = oracle.linear_rows(x, np.array(g["pooled_W"], dtype=np.float32), np.zeros(2, np.float32))
    assert y2[0].tolist() == g["pooled"]
    # and the row max of the pooled row equals the oracle's max
    assert oracle.pool_gelu_scale_max(y[0], k=k, s=2.0) == 2.0 * oracle.gelu(max(g["pooled"]))


def test_pool_window_count_from_page(golden_dir):
    with open(os.path.join(golden_dir, "problem_shapes.json")) as f:
        probs = json.load(f)["problems"]
    p = [q for q in probs if q["epilogue"] == "avgpool_gelu_scale_rowmax"][0]
    assert oracle.pool_windows(p["N"], p["pool_k"]) == p["pooled_len"]
    assert oracle.pool_windows(40, 16) == 2
    assert oracle.pool_windows(16, 16) == 1
    assert oracle.pool_windows(15, 16) == 0
    assert oracle.pool_windows(10, 4, 3) == 3  # floor((10-4)/3)+1


def test_pool_max_is_taken_after_gelu():
    # GELU is not monotone: window means -3 and -0.75.  max of GELU is
    # GELU(-3) ~ -0.00405, while GELU(max mean) = GELU(-0.75) ~ -0.170.
    y = np.array([-3.0] * 16 + [-0.75] * 16)
    out = oracle.pool_gelu_scale_max(y, k=16, s=2.0)
    assert abs(out - 2 * oracle.gelu(-3.0)) < 1e-15
    assert abs(out - 2 * oracle.gelu(-0.75)) > 0.3


def test_pool_uses_mean_and_ignores_tail():
    y = np.zeros(40)
    y[0:16] = np.arange(16)            # mean 7.5
    y[16:32] = 0.25                    # mean 0.25
    y[32:40] = 1e6                     # trailing columns: no full window
    out = oracle.pool_gelu_scale_max(y, k=16, s=2.0)
    assert abs(out - 2 * oracle.gelu(7.5)) < 1e-12
    # the window starts move by the stride: a stride-8 pool of width 16 over
    # the same row sees the window [8, 24) with mean (sum(8..15) + 8*0.25)/16
    out8 = oracle.pool_gelu_scale_max(y, k=16, stride=8, s=1.0)
    # windows: [0,16) 7.5, [8,24) (92+2)/16, [16,32) .25, [24,40) (2 + 8e6)/16
    assert abs(out8 - oracle.gelu((2 + 8e6) / 16)) < 1e-6


def test_pool_rowmax_invariants_random():
    M, K, N = 6, 40, 96
    x, W, b = synth.linear_inputs(M, K, N, seed=21)
    x, W, b = x.numpy(), W.numpy(), b.numpy()
    y = oracle.linear_rows(x, W, b)
    out = oracle.forward_rows(x, W, b, **oracle.PROBLEMS["avgpool_gelu_scale_rowmax"])
    for m in range(M):
        # each window mean recomputed from the 16 dot products
        g = [2.0 * oracle.gelu(sum(y[m, 16 * j + t] for t in range(16)) / 16) for j in range(N // 16)]
        assert all(out[m] >= np.float32(v) for v in g)
        assert any(out[m] == np.float32(v) for v in g)
        assert out[m] >= 2 * -0.16998


def test_forward_rounds_once_to_float32():
    M, K, N = 3, 12, 8
    x, W, b = synth.linear_inputs(M, K, N, seed=2)
    x, W, b = x.numpy(), W.numpy(), b.numpy()
    y = oracle.linear_rows(x, W, b)
    out = oracle.forward_rows(x, W, b, **oracle.PROBLEMS["swish_scale"])
    assert out.dtype == np.float32
    for m in range(M):
        for n in range(N):
            assert out[m, n] == np.float32(oracle.swish_scale(y[m, n], 2.0))
    none = oracle.forward_rows(x, W, b, kind=oracle.EPI_NONE)
    np.testing.assert_array_equal(none, y.astype(np.float32))


def test_oracle_rejects_bad_arguments():
    x = np.zeros((2, 4), np.float32)
    W = np.zeros((8, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.forward_rows(x, W, None, kind=oracle.EPI_AVGPOOL_GELU_SCALE_ROWMAX, pool_k=16)
    with pytest.raises(ValueError):
        oracle.forward_rows(x, W, None, kind=7)
    with pytest.raises(ValueError):
        oracle.forward_rows(x, W, None, kind=0, rows=[2])
