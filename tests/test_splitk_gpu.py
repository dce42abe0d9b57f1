"""GPU checks of tiles whose k-blocks are split over several CTAs.

Such a tile is finished without any CTA waiting for another: the CTA holding
the tile's k-block 0 adds the parked fp32 partials of the other contributors
to its own accumulator when it finds them all parked ("own"), and otherwise
parks its partial too, and the last contributor to arrive sums every partial
from zero ("last").  Timing picks the branch; the test hooks of
include/fle_testing.h pin one branch (FLE_FINISH_OWN / FLE_FINISH_LAST) and
count which branch finished each tile.  Both branches add the partials in
contributor order, so their outputs are bitwise equal, and both match the
oracle.  Every kernel that splits tiles is covered: the one-CTA swapped
kernel, the CTA-pair kernel in direct and swapped operand order, in both
precisions.
"""
import contextlib
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOL = {"3xtf32": (1e-4, 1e-4), "tf32": (5e-3, 5e-3)}
FINISH_AUTO, FINISH_OWN, FINISH_LAST = 0, 1, 2


@pytest.fixture(scope="module")
def fle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import reduction_epilogue_b200 as m
    from reduction_epilogue_b200 import build
    build.build()
    m.load()
    return m


@contextlib.contextmanager
def finisher(fle, mode):
    lib = fle.load()
    prev = lib.fle_test_set_finisher(mode)
    assert prev in (FINISH_AUTO, FINISH_OWN, FINISH_LAST)
    try:
        yield
    finally:
        torch.cuda.synchronize()
        lib.fle_test_set_finisher(prev)


def finish_counts(fle, reset=True):
    counts = (ctypes.c_uint32 * 2)()
    assert fle.load().fle_test_finisher_counts(counts, 1 if reset else 0, None) == 0
    return int(counts[0]), int(counts[1])


def split_tiles(plan):
    """Tiles the plan splits over CTAs, counted per CTA of a pair."""
    sk = int(re.search(r"sk_tiles=(\d+)", plan).group(1))
    return sk * (2 if "pair=1" in plan else 1)


def assert_close(got, ref, precision, what):
    atol, rtol = TOL[precision]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert (err <= atol + rtol * np.abs(ref)).all(), f"{what}: max err {err.max():.3e}"


# (M, K, N, problem, precision, plan fragment naming the kernel)
CASES = [
    (16, 8192, 4096, "scale_hardtanh_gelu", "tf32", "pair=0 swap=1"),
    (16, 8192, 4096, "scale_hardtanh_gelu", "3xtf32", "pair=0 swap=1"),
    (100, 4096, 2000, "swish_scale", "3xtf32", "pair=0 swap=1"),
    (512, 2048, 2560, "avgpool_gelu_scale_rowmax", "tf32", "pair=1 swap=0"),
    (512, 2048, 2560, "avgpool_gelu_scale_rowmax", "3xtf32", "pair=1 swap=0"),
    (300, 2048, 1000, "scale_hardtanh_gelu", "tf32", "pair=1 swap=0"),
    (300, 2048, 1000, "none", "3xtf32", "pair=1 swap=0"),
    (64, 2048, 75 * 256, "swish_scale", "tf32", "pair=1 swap=1"),
    (100, 2048, 75 * 256 - 93, "scale_hardtanh_gelu", "tf32", "pair=1 swap=1"),
]


@pytest.mark.parametrize("M,K,N,problem,precision,kernel", CASES)
def test_each_finisher_branch_matches_the_oracle(fle, M, K, N, problem, precision, kernel):
    desc = fle.desc_for(problem, precision)
    plan = fle.plan_string(M, K, N, desc)
    assert kernel in plan, plan
    n_split = split_tiles(plan)
    assert n_split > 0, plan
    x, W, b = synth.linear_inputs(M, K, N, seed=M + K + N, device="cuda")
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), **oracle.PROBLEMS[problem])
    outs = {}
    for mode in (FINISH_OWN, FINISH_LAST, FINISH_AUTO):
        with finisher(fle, mode):
            finish_counts(fle, reset=True)
            out = fle.linear_epilogue(x, W, b, problem, precision)
            torch.cuda.synchronize()
            assert fle.device_status() == 0
            own, last = finish_counts(fle, reset=True)
        # every split tile (each CTA's half of a pair tile) is finished once,
        # by the branch the mode pins
        assert own + last == n_split, (mode, own, last, plan)
        if mode == FINISH_OWN:
            assert (own, last) == (n_split, 0), plan
        elif mode == FINISH_LAST:
            assert (own, last) == (0, n_split), plan
        assert_close(out.cpu().numpy(), ref, precision, f"mode {mode} {problem} {M}x{K}x{N} {plan}")
        outs[mode] = out
    # the partials are added in contributor order either way
    assert torch.equal(outs[FINISH_OWN], outs[FINISH_LAST])
    assert torch.equal(outs[FINISH_OWN], outs[FINISH_AUTO])


def test_unknown_finisher_mode_is_refused(fle):
    lib = fle.load()
    assert lib.fle_test_set_finisher(7) == -1
    assert lib.fle_test_set_finisher(FINISH_AUTO) == FINISH_AUTO


# A schedule that spreads every k-block evenly over all CTAs (FLE_SCHED=sk,
# read once per process, hence the subprocess): split units are short and
# many CTAs hold two shared tiles, the tail of one and the head of the next,
# so their epilogue warps raise the shared "finish here" flag twice per
# launch.  Repeated launches must give bitwise-equal results that match the
# oracle.
_STRESS_SCRIPT = r"""
import sys, numpy as np, torch
import oracle
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import synth
fle.load()
sms = torch.cuda.get_device_properties(0).multi_processor_count
bad = []
for (M, K, N, problem, precision) in [(300, 4096, 2000, "scale_hardtanh_gelu", "tf32"),
                                      (64, 4096, 4096, "swish_scale", "tf32"),
                                      (64, 4096, 4096, "none", "3xtf32"),
                                      (520, 2080, 1500, "avgpool_gelu_scale_rowmax", "3xtf32")]:
    desc = fle.desc_for(problem, precision)
    plan = fle.plan_string(M, K, N, desc)
    grid = int(plan.split("grid=")[1].split()[0])
    units_per_cta = [fle.plan_units(M, K, N, desc, sms, c)[1] for c in range(grid)]
    twice = sum(1 for u in units_per_cta if int(u[:, 5].sum()) >= 2 and (u[u[:, 5] == 1][:, 3] == 0).any())
    if twice == 0:
        bad.append(("no CTA holds two shared tiles", M, K, N, plan))
        continue
    x, W, b = synth.linear_inputs(M, K, N, seed=11, device="cuda")
    first = fle.linear_epilogue(x, W, b, problem, precision)
    torch.cuda.synchronize()
    rows = synth.sample_rows(M, 64, seed=4)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows,
                              **oracle.PROBLEMS[problem]).astype(np.float64)
    atol, rtol = {"tf32": (5e-3, 5e-3), "3xtf32": (1e-4, 1e-4)}[precision]
    got = first.cpu().numpy()[rows].astype(np.float64)
    if not (np.abs(got - ref) <= atol + rtol * np.abs(ref)).all():
        bad.append(("oracle", M, K, N, problem, precision))
    out = torch.empty_like(first)
    for _ in range(40):
        fle.forward(x, W, b, out, desc, workspace=torch.empty(max(fle.workspace_size(M, K, N, desc), 1),
                                                             dtype=torch.uint8, device="cuda"))
        torch.cuda.synchronize()
        if not torch.equal(out, first):
            bad.append(("repeat differs", M, K, N, problem, precision))
            break
    if fle.device_status() != 0:
        bad.append(("device status", M, K, N))
    print("PLAN", plan, "ctas with two shared tiles:", twice)
print("BAD", bad)
sys.exit(1 if bad else 0)
"""


def test_short_split_units_repeated(fle):
    env = dict(os.environ, FLE_SCHED="sk", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", _STRESS_SCRIPT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
