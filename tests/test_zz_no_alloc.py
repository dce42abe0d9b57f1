"""fle_forward_noalloc: the allocation-free entry point.

Some callers cannot allocate device memory where they run the layer (a
server that fixes each model's HBM budget up front, or a hot loop where
cudaMalloc/cudaFree would synchronise the device).  fle_forward_noalloc takes
its scratch from a static device array inside the library instead of a
caller workspace.  This test calls it through the C ABI twice in a row per
case and checks each result against fle_forward (the entry point that takes
a caller workspace) on the same inputs, within the parity tolerances used by
the other GPU tests.  The cases include plans that use the scratch (stream-K
over every SM, and a split last wave) and one that needs none.

This file is collected last on purpose, and it builds and loads the library
itself, so it passes alone in a fresh process as well as after the others.
"""
import numpy as np
import pytest

from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = {"3xtf32": (1e-4, 1e-4), "tf32": (5e-3, 5e-3)}

# (M, K, N, problem, precision, plan uses scratch)
CASES = [
    (16, 8192, 8192, "scale_hardtanh_gelu", "tf32", True),         # each weight tile split in two
    (256, 8192, 8192, "swish_scale", "tf32", True),                # split last wave, ~33.5 MB
    (300, 2048, 2000, "avgpool_gelu_scale_rowmax", "3xtf32", True),
    (7, 36, 33, "none", "tf32", False),                            # plan needs no scratch
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


@pytest.mark.parametrize("M,K,N,problem,precision,uses_scratch", CASES)
def test_noalloc_matches_workspace_entry_point(fle, M, K, N, problem, precision, uses_scratch):
    x, W, b = synth.linear_inputs(M, K, N, seed=M + K + N, device="cuda")
    desc = fle.desc_for(problem, precision)
    pool = desc.kind == fle.EPI_AVGPOOL_GELU_SCALE_ROWMAX
    shape = (M,) if pool else (M, N)

    ref = torch.empty(shape, device="cuda")
    ws_bytes = fle.workspace_size(M, K, N, desc)
    assert (ws_bytes > 0) == uses_scratch
    assert ws_bytes <= 40 << 20
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    fle.forward(x, W, b, ref, desc, workspace=ws, workspace_bytes=ws_bytes)
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    ref = ref.cpu().numpy().astype(np.float64)

    atol, rtol = TOL[precision]
    for call in range(2):
        out = torch.full(shape, float("nan"), device="cuda")
        fle.forward_noalloc(x, W, b, out, desc)
        torch.cuda.synchronize()
        assert fle.device_status() == 0
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), f"call {call}: non-finite output"
        err = np.abs(got - ref)
        assert (err <= atol + rtol * np.abs(ref)).all(), f"call {call}: max err {err.max():.3e}"


def test_noalloc_scratch_covers_every_plan(fle):
    # fle.h states that on a 148-SM B200 no plan needs more than the 40 MiB
    # static scratch once 3xTF32 computes x's low parts inside the GEMM (the
    # plan the no-alloc call falls back to).  Ask the library for that least
    # workspace of every benchmark workload and of seeded random shapes, in
    # both precisions and every epilogue kind, on this device.
    import random
    kinds = ["scale_hardtanh_gelu", "swish_scale", "avgpool_gelu_scale_rowmax", "none"]
    shapes = [(128, 1024, 1024), (2048, 8192, 8192), (1024, 8192, 8192), (128, 32768, 32768),
              (16, 8192, 8192), (64, 8192, 8192), (256, 8192, 8192), (1024, 8192, 8192),
              (4096, 8192, 8192), (65536, 32768, 65536)]
    rng = random.Random(1234)
    shapes += [(rng.randint(1, 70000), 4 * rng.randint(1, 16384), rng.randint(16, 70000)) for _ in range(300)]
    worst = 0
    for M, K, N in shapes:
        for problem in kinds:
            for precision in ("tf32", "3xtf32"):
                need = fle.workspace_size_min(M, K, N, fle.desc_for(problem, precision))
                assert need <= fle.workspace_size(M, K, N, fle.desc_for(problem, precision))
                worst = max(worst, need)
                assert need <= 40 << 20, (M, K, N, problem, precision, need)
    assert worst > 0
