"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on the same seeded inputs.

Tolerances (elementwise, ref = oracle):
  3xTF32   |got - ref| <= 1e-4 + 1e-4 |ref|
  TF32     |got - ref| <= 5e-3 + 5e-3 |ref|
Small shapes (several tiles plus ragged tails, both the direct and the
swapped operand order) are compared in full; the full-size workloads on a
seeded sample of at least 64 whole rows (every row where M <= 128, and the
whole [M] output of the pool epilogue), in the same launch plan the
benchmark times.

Inputs of large magnitude (x ~ N(0, 50^2)) make TF32's operand rounding,
not the accumulation, the dominant error.  There the single-pass TF32 result
is checked twice: against the oracle run on the same operands truncated to
TF32 (what the tensor core multiplies; checked on the device by
test_tf32_input_conversion_truncates), at the single-pass tolerance, which
is the tight check; and against the oracle on the exact operands, at that
tolerance plus the largest change operand truncation can cause, derived per
element below (a worst case: it holds for every input, so it is loose).
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = {"3xtf32": (1e-4, 1e-4), "tf32": (5e-3, 5e-3)}


@pytest.fixture(scope="module")
def fle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import reduction_epilogue_b200 as m
    from reduction_epilogue_b200 import build
    build.build()
    m.load()
    return m


def _oracle(x, W, b, problem, rows=None):
    return oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), None if b is None else b.cpu().numpy(),
                               rows=rows, **oracle.PROBLEMS[problem])


def _assert_close(got, ref, precision, what=""):
    atol, rtol = TOL[precision]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), what + ": non-finite output"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        pytest.fail(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                    f"got {got[i]!r} ref {ref[i]!r} err {err[i]:.3e} bound {bound[i]:.3e}")


def _tf32(a):
    """fp32 values with the low 13 mantissa bits cleared: the TF32 operand
    the tensor core reads for an fp32 input."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return (a.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


# Largest slope of the exact-form GELU on [-2, 2]: GELU'(t) = Phi(t) + t phi(t)
# peaks at t = sqrt(2), where it is Phi(sqrt 2) + sqrt(2) phi(sqrt 2) = 1.1289.
GELU_SLOPE_2 = 1.13


def _truncation_bound(x, W, scale):
    """Per-element bound on how far epilogue (a) can move when both operands
    are truncated to TF32: each truncation changes a value by less than 2^-10
    of itself, so a product by less than 2^-9 of |x||W| (to first order),
    and y by less than 2^-9 sum_k |x_mk| |W_nk|; the clamp is 1-Lipschitz and
    GELU on [-2, 2] at most 1.13-Lipschitz, after the scale."""
    ax = np.abs(np.asarray(x.cpu().numpy(), dtype=np.float64))
    aw = np.abs(np.asarray(W.cpu().numpy(), dtype=np.float64))
    return GELU_SLOPE_2 * abs(scale) * 2.0 ** -9 * (ax @ aw.T)


def _assert_tf32_large_magnitude(got, x, W, b, what):
    """The two single-pass TF32 checks of large-magnitude inputs (module
    docstring), for epilogue (a) with the pages' constants."""
    atol, rtol = TOL["tf32"]
    got = np.asarray(got, dtype=np.float64)
    xt, Wt = _tf32(x.cpu().numpy()), _tf32(W.cpu().numpy())
    ref_t = oracle.forward_rows(xt, Wt, None if b is None else b.cpu().numpy(),
                                **oracle.PROBLEMS["scale_hardtanh_gelu"])
    _assert_close(got, ref_t, "tf32", what + " (TF32 operands)")
    ref = _oracle(x, W, b, "scale_hardtanh_gelu").astype(np.float64)
    bound = atol + rtol * np.abs(ref) + _truncation_bound(x, W, 0.5)
    err = np.abs(got - ref)
    assert (err <= bound).all(), f"{what}: max err {err.max():.3e} outside the derived bound"


def _run(fle, x, W, b, problem, precision):
    out = fle.linear_epilogue(x, W, b, problem, precision)
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    return out


SMALL = [(1, 4, 1), (7, 36, 33), (16, 64, 130), (33, 100, 257), (128, 1024, 1024),
         (130, 68, 300), (257, 260, 520), (300, 132, 1000), (200, 64, 301)]
PROBLEMS = ["scale_hardtanh_gelu", "swish_scale", "avgpool_gelu_scale_rowmax", "none"]


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("problem", PROBLEMS)
@pytest.mark.parametrize("M,K,N", SMALL)
def test_small_full_compare(fle, M, K, N, problem, precision):
    if problem == "avgpool_gelu_scale_rowmax" and N < 16:
        pytest.skip("pool needs N >= 16")
    x, W, b = synth.linear_inputs(M, K, N, seed=M + 7 * K + 13 * N, device="cuda")
    out = _run(fle, x, W, b, problem, precision)
    _assert_close(out.cpu().numpy(), _oracle(x, W, b, problem), precision, f"{problem} {M}x{K}x{N}")


# Full-size workloads: (M, K, N, problem, sampled rows); at least 64 rows,
# all rows where M <= 128 and the whole [M] output of the pool epilogue
FULL = [
    (2048, 8192, 8192, "scale_hardtanh_gelu", 64),
    (1024, 8192, 8192, "avgpool_gelu_scale_rowmax", 1024),
    (128, 32768, 32768, "swish_scale", 128),
    (128, 1024, 1024, "scale_hardtanh_gelu", 128),
] + [(m, 8192, 8192, "scale_hardtanh_gelu", 64) for m in (16, 64, 256, 1024, 4096)]


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M,K,N,problem,nrows", FULL)
def test_full_size_sampled_rows(fle, M, K, N, problem, nrows, precision):
    x, W, b = synth.linear_inputs(M, K, N, seed=0, device="cuda")
    out = _run(fle, x, W, b, problem, precision)
    rows = synth.sample_rows(M, nrows, seed=1)
    assert len(rows) == min(M, nrows) and len(rows) >= min(M, 64)
    got = out.cpu().numpy()[rows]
    ref = _oracle(x, W, b, problem, rows=rows)
    _assert_close(got, ref, precision, f"{problem} {M}x{K}x{N} rows={len(rows)}")
    del x, W, b, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M,K,N", [(300, 1024, 520), (100, 1024, 300), (5, 2048, 77)])
def test_integer_inputs_are_exact(fle, M, K, N, precision):
    # Integers in [-4, 4] are exact in TF32; every partial sum stays below 2^24,
    # so the contraction is exact in any order: bit-exact against the oracle.
    x, W, b = synth.integer_inputs(M, K, N, seed=4, device="cuda")
    out = _run(fle, x, W, b, "none", precision)
    ref = _oracle(x, W, b, "none")
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M", [64, 512])
def test_hardtanh_saturation(fle, M, precision):
    # x ~ N(0, 50^2) drives most of 0.5*y past +-2: both clamp branches fire.
    # Single-pass TF32 is checked as the module docstring says; 3xTF32 keeps
    # its own bound unchanged.
    K, N = 256, 384
    x, W, b = synth.linear_inputs(M, K, N, seed=9, device="cuda", x_std=50.0)
    out = _run(fle, x, W, b, "scale_hardtanh_gelu", precision)
    ref = _oracle(x, W, b, "scale_hardtanh_gelu")
    assert (ref > 1.95).mean() > 0.1 and (ref < -0.045).mean() > 0.1
    if precision == "tf32":
        _assert_tf32_large_magnitude(out.cpu().numpy(), x, W, b, "saturation")
    else:
        _assert_close(out.cpu().numpy(), ref, precision, "saturation")


def test_gelu_is_the_erf_form(fle):
    # y = W[:, 0] exactly (x = e0, no bias).  Where tanh-GELU and erf-GELU
    # differ by more than 2e-4 inside the clamp range, the 3xTF32 result must
    # follow erf-GELU to 1e-4 + 1e-4|ref|.
    ts = np.linspace(-2.0, 2.0, 4001)
    tanh_g = 0.5 * ts * (1 + np.tanh(math.sqrt(2 / math.pi) * (ts + 0.044715 * ts ** 3)))
    erf_g = np.array([oracle.gelu(t) for t in ts])
    pick = ts[np.abs(tanh_g - erf_g) > 2e-4]
    assert pick.size > 0
    N = int(pick.size)
    W = torch.zeros(N, 4, dtype=torch.float32)
    W[:, 0] = torch.from_numpy(2.0 * pick).float()  # y = 2t so that 0.5*y = t
    x = torch.zeros(3, 4, dtype=torch.float32)
    x[:, 0] = 1.0
    x, W = x.cuda(), W.cuda()
    out = _run(fle, x, W, None, "scale_hardtanh_gelu", "3xtf32")
    ref = _oracle(x, W, None, "scale_hardtanh_gelu")
    _assert_close(out.cpu().numpy(), ref, "3xtf32", "erf-GELU")
    tanh_ref = 0.5 * 2 * pick * 0.5 * (1 + np.tanh(math.sqrt(2 / math.pi) * (pick + 0.044715 * pick ** 3)))
    assert np.abs(out.cpu().numpy()[0] - tanh_ref).max() > 1.5e-4


def test_pool_max_after_gelu(fle):
    # Two windows with means -3 and -0.75: the row max of GELU*2 is
    # 2*GELU(-3) ~ -0.0081, not 2*GELU(-0.75) ~ -0.34.
    N, K = 32, 4
    W = torch.zeros(N, K)
    W[:16, 0] = -3.0
    W[16:, 0] = -0.75
    x = torch.zeros(2, K)
    x[:, 0] = 1.0
    out = _run(fle, x.cuda(), W.cuda(), None, "avgpool_gelu_scale_rowmax", "3xtf32")
    ref = _oracle(x, W, None, "avgpool_gelu_scale_rowmax")
    _assert_close(out.cpu().numpy(), ref, "3xtf32", "pool order")
    assert abs(float(out[0]) - 2 * oracle.gelu(-3.0)) < 1e-5


@pytest.mark.parametrize("problem", PROBLEMS)
def test_k_zero_gives_epilogue_of_bias(fle, problem):
    M, N = 5, 48
    _, _, b = synth.linear_inputs(M, 4, N, seed=3, device="cuda")
    b = b * 10
    x = torch.empty(M, 0, device="cuda")
    W = torch.empty(N, 0, device="cuda")
    out = _run(fle, x, W, b, problem, "tf32")
    ref = _oracle(x, W, b, problem)
    _assert_close(out.cpu().numpy(), ref, "3xtf32", "K=0")


def test_no_bias(fle):
    x, W, _ = synth.linear_inputs(200, 96, 260, seed=12, device="cuda")
    out = _run(fle, x, W, None, "swish_scale", "3xtf32")
    _assert_close(out.cpu().numpy(), _oracle(x, W, None, "swish_scale"), "3xtf32", "no bias")


def test_empty_m_is_a_no_op(fle):
    x = torch.empty(0, 64, device="cuda")
    W = torch.randn(32, 64, device="cuda")
    out = fle.linear_epilogue(x, W, None, "scale_hardtanh_gelu")
    assert out.shape == (0, 32)


def test_misaligned_operand_is_rejected(fle):
    base = torch.zeros(4 * 64 + 1, device="cuda")
    x = base[1:].view(4, 64)  # 4-byte offset: not 16-byte aligned
    W = torch.zeros(8, 64, device="cuda")
    with pytest.raises(fle.FleError) as e:
        fle.linear_epilogue(x, W, None, "none")
    assert e.value.status == 3


def test_repeat_calls_are_deterministic(fle):
    x, W, b = synth.linear_inputs(512, 1024, 2048, seed=5, device="cuda")
    a = _run(fle, x, W, b, "avgpool_gelu_scale_rowmax", "tf32")
    c = _run(fle, x, W, b, "avgpool_gelu_scale_rowmax", "tf32")
    assert torch.equal(a, c)
    a = _run(fle, x, W, b, "scale_hardtanh_gelu", "3xtf32")
    c = _run(fle, x, W, b, "scale_hardtanh_gelu", "3xtf32")
    assert torch.equal(a, c)


def test_bounded_wait_expires_cleanly(fle):
    # A barrier nothing arrives on: the wait gives up after 2 ms, records
    # FLE_ERR_TIMEOUT and the kernel returns; the context stays usable.
    lib = fle.load()
    assert lib.fle_test_bounded_wait(2000, None) == 0
    assert fle.device_status() == 8
    assert fle.device_status() == 0
    x, W, b = synth.linear_inputs(64, 64, 64, seed=1, device="cuda")
    out = _run(fle, x, W, b, "none", "3xtf32")
    _assert_close(out.cpu().numpy(), _oracle(x, W, b, "none"), "3xtf32", "after timeout")


def test_plan_choices(fle):
    d = fle.desc_for("swish_scale", "tf32")
    assert "swap=1" in fle.plan_string(128, 32768, 32768, d)
    d = fle.desc_for("scale_hardtanh_gelu", "tf32")
    assert "swap=0" in fle.plan_string(2048, 8192, 8192, d)


def test_tf32_input_conversion_truncates(fle, capsys):
    # The 3xTF32 split writes only the low part lo = x - trunc13(x) and lets
    # the tensor core read the raw fp32 x as the high part, which is exact
    # only if kind::tf32 drops the low 13 mantissa bits of an fp32 operand
    # (rather than rounding).  Checked here on values whose dropped bits
    # would round up.
    v = 1.0 + 2.0 ** -11 + 2.0 ** -12
    x = torch.full((1, 4), v, device="cuda")
    W = torch.ones(1, 4, device="cuda")
    out = _run(fle, x, W, None, "none", "tf32")
    got = float(out[0, 0])
    trunc, rn = 4.0, 4.0 * (1.0 + 2.0 ** -10)
    with capsys.disabled():
        print(f"\n[tf32 operand conversion: {'truncate' if got == trunc else 'round-to-nearest' if got == rn else got}]")
    assert got == trunc, got


def test_tensor_core_accumulation_rounding_probe(fle, capsys):
    # One tile, 15 k-blocks (too few to be split across CTAs): x = 1, W[0,0] = 1
    # and every other W = 1.5 * 2^-27, so each 8-deep MMA after the first adds
    # 0.75 ulp(1) to an accumulator of 1.0.  Truncating accumulation keeps 1.0;
    # round-to-nearest climbs by one ulp per instruction; the exact sum is about
    # 1 + 45 ulp.  Informational: the 3xTF32 path sums 128-deep slices in
    # registers, which bounds the error whichever way the hardware rounds.
    K = 15 * 32
    x = torch.ones(1, K, device="cuda")
    W = torch.full((1, K), 1.5 * 2.0 ** -27, device="cuda")
    W[0, 0] = 1.0
    out = _run(fle, x, W, None, "none", "tf32")
    ulps = (float(out[0, 0]) - 1.0) / 2.0 ** -23
    assert -0.5 <= ulps <= 61, ulps
    mode = "truncating (round toward zero)" if ulps < 0.5 else f"{ulps:.0f} ulp above 1 (rounding)"
    with capsys.disabled():
        print(f"\n[tensor-core fp32 accumulation: {mode}]")


@pytest.mark.parametrize("precision", ["3xtf32"])
def test_long_k_accuracy_3xtf32(fle, precision):
    # The accumulation chain grows with K; 3xTF32 must keep the fp32-faithful
    # bound at K = 32768 on unit-scale data (direct and swapped order).
    for M, N in ((128, 640), (300, 260)):
        x, W, b = synth.linear_inputs(M, 32768, N, seed=M, device="cuda")
        out = _run(fle, x, W, b, "none", precision)
        rows = synth.sample_rows(M, 32, seed=2)
        _assert_close(out.cpu().numpy()[rows], _oracle(x, W, b, "none", rows=rows), precision, f"K=32768 {M}x{N}")


@pytest.mark.parametrize("which", [0, 1, 2, 3, 4])
def test_epilogue_math_against_fp64_and_cuda(fle, which):
    # The epilogue evaluates erf by Abramowitz & Stegun 7.1.26 (|error| <=
    # 1.5e-7) and the sigmoid with a fast exponential and divide; bound both
    # against fp64 and against CUDA's erff / expf on a dense grid and at
    # saturating magnitudes.
    from scipy.special import erf as erf64
    lib = fle.load()
    lib.fle_test_epilogue_math.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_void_p]
    # a dense grid plus magnitudes where exp over- or underflows in fp32
    extremes = torch.tensor([-1e4, -500.0, -100.0, -88.0, -50.0, 50.0, 88.0, 100.0, 500.0, 1e4])
    xs = torch.cat([torch.linspace(-9.0, 9.0, 360001), extremes]).cuda()
    got = torch.empty_like(xs)
    cuda_ref = torch.empty_like(xs)
    assert lib.fle_test_epilogue_math(xs.data_ptr(), got.data_ptr(), xs.numel(), which, 0, None) == 0
    assert lib.fle_test_epilogue_math(xs.data_ptr(), cuda_ref.data_ptr(), xs.numel(), which, 1, None) == 0
    torch.cuda.synchronize()
    x = xs.cpu().numpy().astype(np.float64)
    g = got.cpu().numpy().astype(np.float64)
    c = cuda_ref.cpu().numpy().astype(np.float64)
    if which == 0:
        exact = erf64(x)
        bound = 6e-7 * np.ones_like(x)  # A&S bound 1.5e-7 plus fast exp and reciprocal rounding
    elif which == 1:
        exact = x * 0.5 * (1 + erf64(x / np.sqrt(2)))
        bound = 2.5e-7 * np.maximum(1.0, np.abs(x))
    elif which == 2:
        with np.errstate(over="ignore"):
            exact = x / (1 + np.exp(-x))
        bound = 4e-6 * np.maximum(1.0, np.abs(x))
    elif which == 3:
        exact = 0.5 * x * (1 + np.tanh(np.sqrt(2 / np.pi) * (x + 0.044715 * x ** 3)))
        bound = 5e-7 * np.maximum(1.0, np.abs(x))
    else:
        # the polynomial GELU is only used on [-2, 2] (epilogue (a) clamps there)
        keep = np.abs(x) <= 2.0
        x, g, c = x[keep], g[keep], c[keep]
        exact = x * 0.5 * (1 + erf64(x / np.sqrt(2)))
        bound = 2.5e-7 * np.maximum(1.0, np.abs(x))
    assert np.isfinite(g).all()
    assert np.abs(g - exact).max() <= bound.max() and (np.abs(g - exact) <= bound).all()
    assert (np.abs(g - c) <= 2 * bound).all()


_STAGE_VARIANT_SCRIPT = r"""
import sys, numpy as np, torch
import oracle
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import synth
fle.load()
bad = []
for (M, K, N, problem) in [(16, 2080, 300, "scale_hardtanh_gelu"), (100, 1056, 520, "swish_scale"),
                           (300, 1056, 600, "scale_hardtanh_gelu"), (520, 2080, 1100, "avgpool_gelu_scale_rowmax"),
                           (33, 20000, 3000, "none")]:
    x, W, b = synth.linear_inputs(M, K, N, seed=7, device="cuda")
    out = fle.linear_epilogue(x, W, b, problem, "tf32")
    torch.cuda.synchronize()
    rows = synth.sample_rows(M, 24, seed=3)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows,
                              **oracle.PROBLEMS[problem]).astype(np.float64)
    got = out.cpu().numpy()[rows].astype(np.float64)
    err = np.abs(got - ref) - (5e-3 + 5e-3 * np.abs(ref))
    if fle.device_status() != 0 or not np.isfinite(got).all() or (err > 0).any():
        bad.append((M, K, N, problem, float(err.max())))
print("PLAN", fle.plan_string(300, 1056, 600, fle.desc_for("scale_hardtanh_gelu", "tf32")))
print("BAD", bad)
sys.exit(1 if bad else 0)
"""


@pytest.mark.parametrize("kps", ["1", "2"])
def test_one_and_two_kblocks_per_stage(fle, kps):
    # Ring stages hold one or two 32-wide k-blocks (the planner picks per
    # plan; FLE_KPS forces one).  Both forms, in both kernels and with odd
    # k-block counts per unit (K = 1056, 2080 and 20000 are 33, 65 and 625
    # k-blocks), against the oracle, in a fresh process.
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, FLE_KPS=kps, PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", _STAGE_VARIANT_SCRIPT], cwd=root, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert f"kps={kps}" in r.stdout


@pytest.mark.parametrize("problem", ["scale_hardtanh_gelu", "swish_scale"])
@pytest.mark.parametrize("M", [1, 45, 100, 128])
def test_swapped_pair_tiles(fle, M, problem):
    # Skinny M with at least one 256-row weight tile per CTA pair runs the
    # swapped pair kernel (each CTA of a pair: 128 weight rows, half of the
    # activation rows).  Ragged M (BN = 32, 64, 128), ragged N (75 tiles, the
    # last one 93 rows short) and a ragged K tail.
    M, K, N = M, 520, 75 * 256 - 93
    d = fle.desc_for(problem, "tf32")
    plan = fle.plan_string(M, K, N, d)
    assert "pair=1 swap=1" in plan, plan
    x, W, b = synth.linear_inputs(M, K, N, seed=11, device="cuda")
    out = _run(fle, x, W, b, problem, "tf32")
    _assert_close(out.cpu().numpy(), _oracle(x, W, b, problem), "tf32", f"{M}x{K}x{N} {plan}")


_PAIR_3X_SCRIPT = r"""
import sys, numpy as np, torch
import oracle
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import synth
lib = fle.load()
bad = []
for (M, K, N, problem) in [(128, 520, 75 * 256 - 93, "scale_hardtanh_gelu"), (45, 2080, 40 * 256, "swish_scale"),
                           (100, 4096, 2000, "none"), (1, 1056, 19107, "swish_scale"),
                           (64, 4096, 29100, "scale_hardtanh_gelu")]:
    d = fle.desc_for(problem, "3xtf32")
    plan = fle.plan_string(M, K, N, d)
    if "pair=1 swap=1" not in plan:
        bad.append(("not the swapped pair kernel", plan))
        continue
    x, W, b = synth.linear_inputs(M, K, N, seed=M + K, device="cuda")
    outs = []
    for mode in (1, 2, 0):  # FLE_FINISH_OWN, FLE_FINISH_LAST, FLE_FINISH_AUTO
        lib.fle_test_set_finisher(mode)
        out = fle.linear_epilogue(x, W, b, problem, "3xtf32")
        torch.cuda.synchronize()
        if fle.device_status() != 0:
            bad.append(("status", M, K, N, mode, plan))
        outs.append(out.cpu().numpy())
    lib.fle_test_set_finisher(0)
    if not all(np.array_equal(outs[0], o) for o in outs[1:]):
        bad.append(("finisher branches differ", M, K, N, plan))
    cols = np.arange(N) if N <= 20000 else np.unique(np.r_[0:256, N - 256:N, np.arange(0, N, 97)])
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy()[cols], b.cpu().numpy()[cols],
                              **oracle.PROBLEMS[problem]).astype(np.float64)
    got = outs[0][:, cols].astype(np.float64)
    err = np.abs(got - ref)
    if not np.isfinite(got).all() or (err > 1e-4 + 1e-4 * np.abs(ref)).any():
        bad.append(("oracle", M, K, N, problem, float(err.max()), plan))
    print("PLAN", plan)
print("BAD", bad)
sys.exit(1 if bad else 0)
"""


def test_swapped_pair_tiles_3xtf32():
    # The swapped pair kernel in 3xTF32 (FLE_PAIR=1 forces it for skinny M):
    # ragged M, N and K, whole tiles, tiles split k-aligned over pairs and an
    # uneven last wave spread over all pairs (64 x 4096 x 29100), both
    # finisher branches bitwise equal, against the oracle at the 3xTF32
    # tolerance (on a spread of output columns for the widest weight).
    import os
    import subprocess
    import sys
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, FLE_PAIR="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", _PAIR_3X_SCRIPT], cwd=root, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
    assert r.stdout.count("PLAN tile=256x") == 5, r.stdout


OPTION_SHAPES = [(7, 36, 33), (100, 1056, 520), (200, 64, 301), (300, 132, 1000), (128, 520, 19107)]


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("problem", ["scale_hardtanh_gelu", "avgpool_gelu_scale_rowmax"])
@pytest.mark.parametrize("M,K,N", OPTION_SHAPES)
def test_gelu_tanh_option(fle, M, K, N, problem, precision):
    # FLE_FLAG_GELU_TANH: the tanh form of GELU in (a) and (c), against the
    # oracle's tanh form (the swapped, direct and swapped-pair kernels).
    if problem == "avgpool_gelu_scale_rowmax" and N < 16:
        pytest.skip("pool needs N >= 16")
    x, W, b = synth.linear_inputs(M, K, N, seed=3 * M + K + N, device="cuda")
    out = fle.linear_epilogue(x, W, b, problem, precision, gelu="tanh")
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), gelu_tanh=True,
                              **oracle.PROBLEMS[problem])
    _assert_close(out.cpu().numpy(), ref, precision, f"tanh GELU {problem} {M}x{K}x{N}")
    # and it is not the erf form: the two differ by up to 4.7e-4 per element
    if problem == "scale_hardtanh_gelu":
        erf_ref = _oracle(x, W, b, problem)
        assert np.abs(ref.astype(np.float64) - erf_ref).max() > 1e-6


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M,K,N", OPTION_SHAPES)
def test_fold_scale_option(fle, M, K, N, precision):
    # FLE_FLAG_FOLD_SCALE: (a) as s*acc + s*b in one FMA; the same function,
    # so the same oracle and tolerance; and the saturated region too.
    x, W, b = synth.linear_inputs(M, K, N, seed=5 * M + K + N, device="cuda")
    x50 = x * 50.0
    for xin in (x, x50):
        out = fle.linear_epilogue(xin, W, b, "scale_hardtanh_gelu", precision, fold_scale=True)
        torch.cuda.synchronize()
        assert fle.device_status() == 0
        if xin is x50 and precision == "tf32":
            # operand truncation dominates: the checks of the module docstring
            _assert_tf32_large_magnitude(out.cpu().numpy(), xin, W, b, f"fold scale x50 {M}x{K}x{N}")
        else:
            ref = _oracle(xin, W, b, "scale_hardtanh_gelu")
            _assert_close(out.cpu().numpy(), ref, precision, f"fold scale {M}x{K}x{N}")


def test_concurrent_calls_on_two_streams(fle):
    # Two calls in flight at once on two streams, each with its own
    # workspace (split-K plans): no CTA waits for another CTA, so the grids
    # may share the GPU in any proportion; both results match the oracle.
    shapes = [(16, 8192, 4096, "scale_hardtanh_gelu"), (300, 4096, 1100, "avgpool_gelu_scale_rowmax")]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    runs = []
    for (M, K, N, problem), s in zip(shapes, streams):
        x, W, b = synth.linear_inputs(M, K, N, seed=M + N, device="cuda")
        d = fle.desc_for(problem, "tf32")
        out = torch.empty((M,) if problem.startswith("avgpool") else (M, N), device="cuda")
        wsb = fle.workspace_size(M, K, N, d)
        assert wsb > 0  # both plans split K
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        runs.append((x, W, b, problem, out, d, ws, wsb, s))
    torch.cuda.synchronize()
    for _ in range(3):
        for x, W, b, problem, out, d, ws, wsb, s in runs:
            fle.forward(x, W, b, out, d, workspace=ws, workspace_bytes=wsb, stream=s)
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    for x, W, b, problem, out, d, ws, wsb, s in runs:
        rows = synth.sample_rows(x.shape[0], 16, seed=5)
        _assert_close(out.cpu().numpy()[rows], _oracle(x, W, b, problem, rows=rows), "tf32",
                      f"concurrent {problem}")
