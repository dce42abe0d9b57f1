"""Seeded random shapes against the oracle, whole outputs.

The planner picks the kernel (one CTA or a CTA pair, direct or swapped
operands), the pair tile's width (224, 256 or 512), the ring depth and the
split of K from the shape; the hand-picked cases elsewhere cover each choice
on purpose.  Here a seeded generator draws shapes across those boundaries
(M from 1 to ~1100, K a multiple of 4 up to 4096, ragged N), every epilogue
kind, and both precisions, and every output element is compared with the
fp64 oracle at the precision's tolerance.  The plans the draws reach are
collected and must include every kernel and both whole and split tiles.
"""
import random

import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = {"3xtf32": (1e-4, 1e-4), "tf32": (5e-3, 5e-3)}
PROBLEMS = ["scale_hardtanh_gelu", "swish_scale", "avgpool_gelu_scale_rowmax", "none"]


def _draw(n, seed=2026):
    rng = random.Random(seed)
    shapes = []
    while len(shapes) < n:
        band = rng.random()
        if band < 0.3:
            M = rng.randint(1, 128)
        elif band < 0.8:
            M = rng.randint(129, 640)
        else:
            M = rng.randint(641, 1100)
        K = 4 * rng.randint(1, 1024)
        N = rng.randint(16, 3000)
        if M * N * K > 2.5e9:
            continue
        shapes.append((M, K, N, PROBLEMS[len(shapes) % len(PROBLEMS)]))
    return shapes


SHAPES = _draw(40)


@pytest.fixture(scope="module")
def fle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import reduction_epilogue_b200 as m
    from reduction_epilogue_b200 import build
    build.build()
    m.load()
    return m


def test_random_shapes_match_the_oracle(fle):
    plans, bad = [], []
    for i, (M, K, N, problem) in enumerate(SHAPES):
        x, W, b = synth.linear_inputs(M, K, N, seed=1000 + i, device="cuda")
        ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(),
                                  **oracle.PROBLEMS[problem]).astype(np.float64)
        for precision in ("tf32", "3xtf32"):
            plan = fle.plan_string(M, K, N, fle.desc_for(problem, precision))
            plans.append(plan)
            out = fle.linear_epilogue(x, W, b, problem, precision)
            torch.cuda.synchronize()
            st = fle.device_status()
            got = out.cpu().numpy().astype(np.float64)
            atol, rtol = TOL[precision]
            err = np.abs(got - ref)
            if st != 0 or not np.isfinite(got).all() or (err > atol + rtol * np.abs(ref)).any():
                bad.append((M, K, N, problem, precision, st, float(np.nanmax(err)), plan))
    assert not bad, bad
    # the draws reach every kernel, both operand orders and both whole and split tiles
    assert any("pair=1 swap=0" in p for p in plans)
    assert any("pair=0 swap=1" in p for p in plans)
    assert any("pair=0 swap=0" in p for p in plans)
    assert any("sk_tiles=0 " not in p for p in plans)
    assert any("dp_tiles=0 " not in p for p in plans)
    assert len({p.split()[0] for p in plans}) >= 4  # tile shapes
