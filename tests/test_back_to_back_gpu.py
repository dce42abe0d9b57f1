"""CTA-pair kernels of different shapes launched back to back.

A pair CTA must not exit while a signal from the other CTA of its pair can
still reach its shared memory (the exit drain of the pair kernel): such a
late arrival would land in whichever CTA the SM runs next, in the middle of
another launch's barriers, flags or tiles.  Here launches of different pair
kernels (224-wide split tiles with one k-block per stage, the pool kind,
512-wide tiles, swapped tiles split along K, 224-wide tiles of two k-blocks
per stage, a plan of mixed 512- and 384-wide tiles) follow one another without pauses, many times over, so that each
launch's successor on an SM has a different shared-memory layout.  Every
repeat must end with a clean status and be bitwise equal to the first run of
the same shape, which matches the oracle.
"""
import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [
    (300, 2048, 1000, "none", "tile=256x224"),
    (512, 2048, 2560, "avgpool_gelu_scale_rowmax", "tile=256x224"),
    (1024, 2048, 8192, "scale_hardtanh_gelu", "tile=256x512"),
    (64, 2048, 75 * 256, "swish_scale", "pair=1 swap=1"),
    (2560, 1024, 4096, "none", "kps=2"),
    (2000, 260, 7000, "scale_hardtanh_gelu", "mix=74x512"),
]


@pytest.fixture(scope="module")
def fle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import reduction_epilogue_b200 as m
    from reduction_epilogue_b200 import build
    build.build()
    m.load()
    return m


def test_pair_kernels_back_to_back(fle):
    runs = []
    for i, (M, K, N, problem, kernel) in enumerate(SHAPES):
        desc = fle.desc_for(problem, "tf32")
        plan = fle.plan_string(M, K, N, desc)
        assert kernel in plan and "pair=1" in plan, plan
        x, W, b = synth.linear_inputs(M, K, N, seed=50 + i, device="cuda")
        out = torch.empty((M,) if problem.startswith("avgpool") else (M, N), device="cuda")
        wsb = fle.workspace_size(M, K, N, desc)
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
        runs.append((x, W, b, out, desc, ws, wsb, problem, plan))
    # first results, against the oracle
    first = []
    for x, W, b, out, desc, ws, wsb, problem, plan in runs:
        fle.forward(x, W, b, out, desc, workspace=ws, workspace_bytes=wsb)
        torch.cuda.synchronize()
        assert fle.device_status() == 0, plan
        got = out.cpu().numpy().astype(np.float64)
        M = x.shape[0]
        rows = synth.sample_rows(M, M if problem.startswith("avgpool") else 64, seed=3)
        ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows,
                                  **oracle.PROBLEMS[problem])
        err = np.abs(got[rows] - ref)
        assert np.isfinite(got).all() and (err <= 5e-3 + 5e-3 * np.abs(ref)).all(), plan
        first.append(out.clone())
    # then many rounds of every shape in turn, no pauses, one check per round
    for r in range(25):
        for x, W, b, out, desc, ws, wsb, problem, plan in runs:
            fle.forward(x, W, b, out, desc, workspace=ws, workspace_bytes=wsb)
        torch.cuda.synchronize()
        assert fle.device_status() == 0, r
        for (x, W, b, out, desc, ws, wsb, problem, plan), ref in zip(runs, first):
            assert torch.equal(out, ref), (r, plan)
