"""The barrier-checking build on the GPU.

libfle_check.so is the library compiled with -DFLE_CHECK_BARRIERS.  In both
kernels every ring stage and every TMEM accumulator carries a tag naming the
work (tile, first k-block) its producer put there, and each consumer compares
it, after its barrier wait, with the work its own walk of the schedule
expects; in the CTA-pair kernel the leader's MMA also reads the peer CTA's
stage tags, and the peer's epilogue the leader's accumulator tags, through
distributed shared memory.  A mismatch, or a producer re-arming a stage whose
phase already completed, records FLE_ERR_PROTOCOL in the device status word.
These checks stand in for a race detector (compute-sanitizer is not
available here).  Variants: the default plans (both kernels, a plan of
mixed 512- and 384-wide pair tiles among them), the one-CTA
kernel alone (FLE_PAIR=0) and under an even stream-K spread (FLE_SCHED=sk:
short units, CTAs holding two shared tiles), the pair kernel under the same
spread, and 256-wide pair tiles of one k-block per stage (FLE_PAIR_BN=256
FLE_KPS=1).  Each variant runs in a fresh process (the planner overrides are
read once per process) and must end with a clean status and results that
match the oracle.
"""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r"""
import sys, numpy as np, torch
import oracle
import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import build, synth
lib = fle.load()
assert fle.library_path().endswith("libfle_check.so"), fle.library_path()
assert lib.fle_source_hash().decode() == build.source_hash(check=True)
bad, plans = [], []
shapes = [(7, 36, 33, "none"), (100, 1056, 520, "swish_scale"), (16, 8192, 4096, "scale_hardtanh_gelu"),
          (300, 2048, 1000, "scale_hardtanh_gelu"), (520, 2080, 1500, "avgpool_gelu_scale_rowmax"),
          (1024, 1024, 8192, "avgpool_gelu_scale_rowmax"), (64, 2048, 75 * 256, "swish_scale"),
          (600, 4096, 2300, "none"), (2000, 260, 7000, "scale_hardtanh_gelu")]
for M, K, N, problem in shapes:
    for precision in ("tf32", "3xtf32"):
        x, W, b = synth.linear_inputs(M, K, N, seed=M + N, device="cuda")
        out = fle.linear_epilogue(x, W, b, problem, precision)
        torch.cuda.synchronize()
        st = fle.device_status()
        plans.append(fle.plan_string(M, K, N, fle.desc_for(problem, precision)))
        rows = synth.sample_rows(M, 16, seed=2)
        ref = oracle.forward_rows(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), rows=rows,
                                  **oracle.PROBLEMS[problem]).astype(np.float64)
        got = out.cpu().numpy()[rows].astype(np.float64)
        atol, rtol = {"tf32": (5e-3, 5e-3), "3xtf32": (1e-4, 1e-4)}[precision]
        if st != 0 or not (np.abs(got - ref) <= atol + rtol * np.abs(ref)).all():
            bad.append((M, K, N, problem, precision, st))
for p in sorted(set(plans)):
    print("PLAN", p)
print("BAD", bad)
sys.exit(1 if bad else 0)
"""

# planner overrides: the default plans, one-CTA tiles only, an even stream-K
# spread on one-CTA tiles and on pair tiles, and 256-wide pair tiles of one
# k-block per stage
VARIANTS = [{}, {"FLE_PAIR": "0"}, {"FLE_PAIR": "0", "FLE_SCHED": "sk"}, {"FLE_SCHED": "sk"},
            {"FLE_PAIR_BN": "256", "FLE_KPS": "1"}]


@pytest.fixture(scope="module")
def built():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from reduction_epilogue_b200 import build
    build.build()
    assert not build.needs_build(check=True)


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: ",".join(f"{k}={x}" for k, x in v.items()) or "default")
def test_protocol_checks_stay_clean(built, variant):
    env = dict(os.environ, FLE_BUILD="check", PYTHONPATH=ROOT, **variant)
    r = subprocess.run([sys.executable, "-c", _SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
