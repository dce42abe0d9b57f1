"""GPU checks of epilogue (c) through pooled weights (fle_pool_weights,
fle_forward_pooled).  The pooled weights are the mean of each window of
pool_k weight rows (page "Kimi-K2.6 l2_p98", derivation of pre-averaged
weights); the pooled result must match the CPU oracle of the unpooled
definition within the usual tolerances."""
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


def _close(got, ref, precision):
    atol, rtol = TOL[precision]
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert (err <= atol + rtol * np.abs(ref)).all(), float(err.max())


@pytest.mark.parametrize("N,K,k", [(64, 8, 16), (1000, 36, 16), (8192, 256, 16), (96, 12, 32), (40, 4, 1)])
def test_pool_weights_is_the_window_mean(fle, N, K, k):
    _, W, b = synth.linear_inputs(2, K, N, seed=N + K, device="cuda")
    Wp, bp = fle.pool_weights(W, b, k)
    torch.cuda.synchronize()
    P = N // k
    Wn = W.cpu().numpy().astype(np.float64)[: P * k].reshape(P, k, K).mean(axis=1)
    bn = b.cpu().numpy().astype(np.float64)[: P * k].reshape(P, k).mean(axis=1)
    np.testing.assert_allclose(Wp.cpu().numpy(), Wn, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(bp.cpu().numpy(), bn, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M,K,N", [(7, 36, 33), (130, 68, 300), (257, 260, 1000), (300, 1024, 2048)])
def test_pooled_matches_oracle_small(fle, M, K, N, precision):
    x, W, b = synth.linear_inputs(M, K, N, seed=M * K + N, device="cuda")
    desc = fle.desc_for("avgpool_gelu_scale_rowmax", precision)
    out = torch.empty(M, device="cuda")
    ws = torch.empty(max(fle.workspace_size_pooled(M, K, N, desc), 1), dtype=torch.uint8, device="cuda")
    fle.forward_pooled(x, W, b, out, desc, workspace=ws)
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(),
                              **oracle.PROBLEMS["avgpool_gelu_scale_rowmax"])
    _close(out.cpu().numpy(), ref, precision)


def test_one_call_equals_pool_then_forward(fle):
    M, K, N = 300, 512, 4096
    x, W, b = synth.linear_inputs(M, K, N, seed=3, device="cuda")
    desc = fle.desc_for("avgpool_gelu_scale_rowmax", "tf32")
    out1 = torch.empty(M, device="cuda")
    ws = torch.empty(fle.workspace_size_pooled(M, K, N, desc), dtype=torch.uint8, device="cuda")
    fle.forward_pooled(x, W, b, out1, desc, workspace=ws)
    Wp, bp = fle.pool_weights(W, b, 16)
    out2 = fle.linear_epilogue(x, Wp, bp, "avgpool_gelu_scale_rowmax", "tf32", pool_k=1)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
def test_pooled_full_size(fle, precision):
    M, K, N = 1024, 8192, 8192
    x, W, b = synth.linear_inputs(M, K, N, seed=0, device="cuda")
    desc = fle.desc_for("avgpool_gelu_scale_rowmax", precision)
    out = torch.empty(M, device="cuda")
    ws = torch.empty(fle.workspace_size_pooled(M, K, N, desc), dtype=torch.uint8, device="cuda")
    fle.forward_pooled(x, W, b, out, desc, workspace=ws)
    torch.cuda.synchronize()
    assert fle.device_status() == 0
    rows = synth.sample_rows(M, 64, seed=1)
    ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows,
                              **oracle.PROBLEMS["avgpool_gelu_scale_rowmax"])
    _close(out.cpu().numpy()[rows], ref, precision)


def test_pooled_rejects_other_kinds(fle):
    x, W, b = synth.linear_inputs(4, 8, 32, seed=1, device="cuda")
    desc = fle.desc_for("swish_scale", "tf32")
    out = torch.empty(4, 32, device="cuda")
    with pytest.raises(fle.FleError) as e:
        fle.forward_pooled(x, W, b, out.view(-1)[:4], desc)
    assert e.value.status == 4
