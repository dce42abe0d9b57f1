"""3xTF32 with the low parts of x in memory.

In 3xTF32 each operand is split into a TF32 high part (the raw fp32 value,
which the tensor core truncates) and a low part lo = v - hi.  With the
workspace of fle_workspace_size(), a pre-pass writes x's low parts once per
call and the GEMM copies them with its tiles, so its split warps split only
W's tiles; with fle_workspace_size_min() bytes the split warps compute both,
as every CTA's tiles arrive.  The tensor core then reads identical operands,
so the two must agree bit for bit, and both must meet the 3xTF32 bound
against the oracle.  Covered: direct tiles on CTA pairs (whole, split along
K, ragged, large M), the row-max kind, the swapped one-CTA kernel, and a
skinny shape (M <= 64) whose plan keeps the split inside the GEMM.
"""
import numpy as np
import pytest

import oracle
from reduction_epilogue_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [
    (300, 2048, 1000, "scale_hardtanh_gelu", True),        # pair tiles, ragged M and N
    (2048, 1024, 4096, "none", True),                      # pairs, several waves
    (520, 2084, 1500, "avgpool_gelu_scale_rowmax", True),  # row max, ragged K
    (100, 1056, 520, "swish_scale", True),                 # swapped one-CTA tiles
    (128, 8192, 4096, "scale_hardtanh_gelu", True),        # swapped, tiles split along K
    (48, 4096, 3000, "none", False),                       # M <= 64: split inside the GEMM
    (2048, 1024, 2048, "scale_hardtanh_gelu", True),       # large M on pairs
    (2100, 1028, 1500, "swish_scale", True),               # the same, ragged M, K and N
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


@pytest.mark.parametrize("M,K,N,problem,lo_mem", SHAPES)
def test_low_parts_in_memory_match_the_split_in_the_gemm(fle, M, K, N, problem, lo_mem):
    d = fle.desc_for(problem, "3xtf32")
    plan = fle.plan_string(M, K, N, d)
    assert (" xlo=mem" in plan) == lo_mem, plan
    full, least = fle.workspace_size(M, K, N, d), fle.workspace_size_min(M, K, N, d)
    if lo_mem:
        assert full >= least + 4 * M * K, (full, least)
    else:
        assert full == least
    sizes = [full, least]
    x, W, b = synth.linear_inputs(M, K, N, seed=M + K + N + 3, device="cuda")
    shape = (M,) if problem.startswith("avgpool") else (M, N)
    outs = []
    for ws_bytes in sizes:
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
        out = torch.full(shape, float("nan"), device="cuda")
        fle.forward(x, W, b, out, d, workspace=ws, workspace_bytes=ws_bytes)
        torch.cuda.synchronize()
        assert fle.device_status() == 0, (ws_bytes, plan)
        outs.append(out)
    assert all(torch.equal(outs[0], o) for o in outs[1:]), plan
    rows = synth.sample_rows(M, M if problem.startswith("avgpool") else 24, seed=8)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows, **oracle.PROBLEMS[problem])
    got = outs[0].cpu().numpy()[rows].astype(np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all() and (err <= 1e-4 + 1e-4 * np.abs(ref)).all(), (float(err.max()), plan)


def test_workspace_below_the_least_is_refused(fle):
    M, K, N = 300, 2048, 1000
    d = fle.desc_for("scale_hardtanh_gelu", "3xtf32")
    least = fle.workspace_size_min(M, K, N, d)
    x, W, b = synth.linear_inputs(M, K, N, seed=1, device="cuda")
    out = torch.empty((M, N), device="cuda")
    if least == 0:
        pytest.skip("this plan needs no workspace")
    ws = torch.empty(least, dtype=torch.uint8, device="cuda")
    with pytest.raises(fle.FleError):
        fle.forward(x, W, b, out, d, workspace=ws, workspace_bytes=least - 256)
