"""GPU parity of the 512-wide pair tile.

A 512-wide tile is two 256-wide tcgen05 MMAs (cta_group::2, M = 256) per
k-step that share the A tile (the x rows): each CTA of the pair loads its 128
rows of both 256-wide halves of the weight tile, and the accumulator fills
all 512 TMEM columns (one buffer).  The planner takes it in single-pass TF32
when it is cheaper than 256 or 224 columns per tile (2048, 4096 and 1024 x
8192 x 8192).  Covered here: default plans that take it, whole and split
along K; and, with the width forced (FLE_PAIR_BN=512, read once per process,
hence the subprocess), small ragged shapes of every epilogue kind, both
finisher branches of split tiles (bitwise equal) and the oracle.

The same kernel runs the mixed-width plans: one wave of 512-wide tiles and
one of 384-wide tiles (a 256-wide and a 128-wide MMA sharing the A tile,
whose 64 weight rows per CTA come through a second tensor map), cut per
256-row panel.  Covered: ragged M, K and N, 8 to 16 panels, every epilogue
kind, against the oracle on rows from every panel, and bitwise against the
uniform 512-wide plan of the same inputs (FLE_MIX=0): an output element gets
the same MMA chain over the same k-blocks in either plan.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import reduction_epilogue_b200 as m
    from reduction_epilogue_b200 import build
    build.build()
    m.load()
    return m


def _close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert (err <= 5e-3 + 5e-3 * np.abs(ref)).all(), f"{what}: max err {err.max():.3e}"


@pytest.mark.parametrize("M,K,N,problem,split", [
    (1024, 2048, 8192, "avgpool_gelu_scale_rowmax", False),   # 64 wide tiles, one wave
    (1024, 2048, 8192, "scale_hardtanh_gelu", False),
    (4096, 2048, 8192, "none", True),                         # 3 waves + 34 tiles split in two
])
def test_default_plans_with_wide_tiles(fle, M, K, N, problem, split):
    d = fle.desc_for(problem, "tf32")
    plan = fle.plan_string(M, K, N, d)
    assert "tile=256x512 pair=1" in plan, plan
    assert ("sk_tiles=0 " not in plan) == split, plan
    x, W, b = synth.linear_inputs(M, K, N, seed=M + N, device="cuda")
    out = fle.linear_epilogue(x, W, b, problem, "tf32")
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    rows = synth.sample_rows(M, 64 if problem != "avgpool_gelu_scale_rowmax" else M, seed=6)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows, **oracle.PROBLEMS[problem])
    _close(out.cpu().numpy()[rows], ref, f"{problem} {M}x{K}x{N} {plan}")
    again = fle.linear_epilogue(x, W, b, problem, "tf32")
    torch.cuda.synchronize()
    assert torch.equal(out, again)


_FORCED_SCRIPT = r"""
import ctypes, sys, numpy as np, torch
import oracle
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import synth
lib = fle.load()
bad = []
for (M, K, N, problem) in [(300, 1024, 1100, "scale_hardtanh_gelu"), (520, 2080, 1500, "none"),
                           (257, 3000, 700, "swish_scale"), (1024, 4096, 2048, "avgpool_gelu_scale_rowmax"),
                           (600, 8192, 4096, "none")]:
    d = fle.desc_for(problem, "tf32")
    plan = fle.plan_string(M, K, N, d)
    if "tile=256x512" not in plan:
        bad.append(("not wide", plan))
        continue
    x, W, b = synth.linear_inputs(M, K, N, seed=M + N, device="cuda")
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), **oracle.PROBLEMS[problem])
    outs = []
    for mode in (1, 2, 0):  # FLE_FINISH_OWN, FLE_FINISH_LAST, FLE_FINISH_AUTO
        lib.fle_test_set_finisher(mode)
        out = fle.linear_epilogue(x, W, b, problem, "tf32")
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        ok = fle.device_status() == 0 and (np.abs(got - ref) <= 5e-3 + 5e-3 * np.abs(ref)).all()
        if not ok:
            bad.append(("oracle", M, K, N, problem, mode, plan))
        outs.append(out)
    lib.fle_test_set_finisher(0)
    if not all(torch.equal(outs[0], o) for o in outs[1:]):
        bad.append(("branches differ", M, K, N, problem))
    print("PLAN", plan)
print("BAD", bad)
sys.exit(1 if bad else 0)
"""


def test_forced_wide_tiles_small_shapes(fle):
    # ragged M, N and K, whole and split tiles, every epilogue kind
    env = dict(os.environ, FLE_PAIR_BN="512", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", _FORCED_SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
    assert r.stdout.count("PLAN tile=256x512") == 5


MIXED = [
    (2000, 260, 7000, "scale_hardtanh_gelu"),        # ragged M, K and N: 74 + 52 tiles
    (3584, 128, 4096, "swish_scale"),                # 14 panels
    (4096, 128, 3584, "none"),                       # 16 panels
    (2048, 128, 7000, "avgpool_gelu_scale_rowmax"),  # pool windows across 384-wide tiles
]


def _panel_rows(M, seed):
    # the first and last row of every 256-row panel and 64 more at random
    rows = set()
    for p0 in range(0, M, 256):
        rows.update((p0, min(p0 + 255, M - 1)))
    rows.update(int(r) for r in synth.sample_rows(M, 64, seed=seed))
    return np.array(sorted(rows))


_UNIFORM_SCRIPT = r"""
import sys, numpy as np, torch
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import synth
fle.load()
M, K, N, problem, path = sys.argv[1], sys.argv[2], sys.argv[3], sys.argv[4], sys.argv[5]
M, K, N = int(M), int(K), int(N)
plan = fle.plan_string(M, K, N, fle.desc_for(problem, "tf32"))
assert "mix=" not in plan and "tile=256x512" in plan, plan
x, W, b = synth.linear_inputs(M, K, N, seed=M + N + 7, device="cuda")
out = fle.linear_epilogue(x, W, b, problem, "tf32")
torch.cuda.synchronize()
assert fle.device_status() == 0
np.save(path, out.cpu().numpy())
print("PLAN", plan)
"""


@pytest.mark.parametrize("M,K,N,problem", MIXED)
def test_mixed_width_plans(fle, M, K, N, problem, tmp_path):
    d = fle.desc_for(problem, "tf32")
    plan = fle.plan_string(M, K, N, d)
    assert "tile=256x512 pair=1" in plan and " mix=74x512+" in plan and "sk_tiles=0 " in plan, plan
    x, W, b = synth.linear_inputs(M, K, N, seed=M + N + 7, device="cuda")
    out = fle.linear_epilogue(x, W, b, problem, "tf32")
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    pool = problem == "avgpool_gelu_scale_rowmax"
    rows = np.arange(M) if pool else _panel_rows(M, seed=9)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows, **oracle.PROBLEMS[problem])
    _close(out.cpu().numpy()[rows], ref, f"{problem} {M}x{K}x{N} {plan}")
    # the uniform 512-wide plan of the same inputs, in a fresh process
    path = str(tmp_path / "uniform.npy")
    env = dict(os.environ, FLE_MIX="0", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", _UNIFORM_SCRIPT, str(M), str(K), str(N), problem, path], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert np.array_equal(np.load(path), out.cpu().numpy()), "mixed and uniform plans differ"
