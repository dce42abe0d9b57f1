"""Host-side checks of the C ABI: the library loads, exports every entry
point include/fle.h declares, and rejects bad arguments on the host before
anything reaches a GPU (these run without one)."""
import ctypes
import os
import re

import pytest

import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import build as fle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fle_build.build()
    return fle.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(fle_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ["fle_forward", "fle_workspace_size", "fle_status_string", "fle_device_status",
                 "fle_plan_string", "fle_version", "fle_source_hash", "fle_forward_noalloc",
                 "fle_test_bounded_wait", "fle_test_epilogue_math", "fle_test_set_finisher",
                 "fle_test_finisher_counts"]:
        assert want in names


def test_test_hooks_live_in_the_testing_header():
    # the product header declares no test hook; fle_testing.h holds them all
    inc = os.path.join(ROOT, "include")
    product = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, "fle.h")).read(), flags=re.S)
    testing = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, "fle_testing.h")).read(), flags=re.S)
    assert "fle_test_" not in product
    assert set(re.findall(r"\b(fle_test_\w+)\s*\(", testing)) == {
        "fle_test_bounded_wait", "fle_test_epilogue_math", "fle_test_set_finisher", "fle_test_finisher_counts"}


def test_library_is_built_from_these_sources(lib):
    # the library carries the hash of the sources and flags it was built from
    assert lib.fle_source_hash().decode() == fle_build.source_hash()
    assert not fle_build.needs_build()


def test_load_refuses_a_library_of_other_sources(monkeypatch):
    # a library whose hash does not match the sources beside it is not used
    monkeypatch.setattr(fle_build, "source_hash", lambda check=False: "0" * 64)
    monkeypatch.setattr(fle, "_lib", None)
    with pytest.raises(RuntimeError, match="not built from the sources"):
        fle.load()


def test_finisher_mode_hook_without_a_device(lib):
    # the mode is host state: set, read back, refuse unknown values
    assert lib.fle_test_set_finisher(2) == 0
    assert lib.fle_test_set_finisher(1) == 2
    assert lib.fle_test_set_finisher(9) == -1
    assert lib.fle_test_set_finisher(0) == 1


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(0, 10):
        s = lib.fle_status_string(code)
        assert s and len(s) > 1
    assert lib.fle_status_string(12345) == b"unknown status"
    assert lib.fle_version() >= 100


def _call(lib, M, K, N, desc, x=16, W=16, b=None, out=16):
    # Fake, aligned, non-null "device" addresses: every case below must be
    # rejected on the host before any pointer is used.
    return lib.fle_forward(x, W, b, M, K, N, ctypes.byref(desc) if desc is not None else None,
                           out, None, 0, None)


def test_null_and_descriptor_errors(lib):
    d = fle.desc_for("scale_hardtanh_gelu")
    assert _call(lib, 4, 8, 8, None) == 1  # FLE_ERR_NULL
    bad = fle.desc_for("scale_hardtanh_gelu"); bad.kind = 9
    assert _call(lib, 4, 8, 8, bad) == 4
    bad = fle.desc_for("scale_hardtanh_gelu"); bad.precision = 5
    assert _call(lib, 4, 8, 8, bad) == 4
    bad = fle.desc_for("scale_hardtanh_gelu"); bad.clamp_lo, bad.clamp_hi = 1.0, -1.0
    assert _call(lib, 4, 8, 8, bad) == 4
    bad = fle.desc_for("swish_scale"); bad.scale = float("inf")
    assert _call(lib, 4, 8, 8, bad) == 4
    bad = fle.desc_for("avgpool_gelu_scale_rowmax"); bad.pool_k = 3; bad.pool_stride = 3
    assert _call(lib, 4, 8, 64, bad) == 4
    bad = fle.desc_for("avgpool_gelu_scale_rowmax"); bad.pool_stride = 8
    assert _call(lib, 4, 8, 64, bad) == 4
    bad = fle.desc_for("scale_hardtanh_gelu"); bad.flags = 4  # unknown option bit
    assert _call(lib, 4, 8, 8, bad) == 4
    # the option bits mirror include/fle.h
    ok = fle.desc_for("scale_hardtanh_gelu", gelu="tanh", fold_scale=True)
    assert ok.flags == fle.FLAG_GELU_TANH | fle.FLAG_FOLD_SCALE == 3
    with pytest.raises(ValueError):
        fle.desc_for("scale_hardtanh_gelu", gelu="sigmoid")


def test_shape_and_alignment_errors(lib):
    d = fle.desc_for("scale_hardtanh_gelu")
    assert _call(lib, -1, 8, 8, d) == 2       # FLE_ERR_SHAPE
    assert _call(lib, 4, 8, 2**31, d) == 2
    assert _call(lib, 4, 6, 8, d) == 3        # K % 4 != 0 -> FLE_ERR_ALIGN
    p = fle.desc_for("avgpool_gelu_scale_rowmax")
    assert _call(lib, 4, 8, 15, p) == 2       # N < pool_k
    assert _call(lib, 4, 8, 8, d, x=17) == 3  # x not 16-byte aligned
    assert _call(lib, 4, 8, 8, d, W=24) == 3
    assert _call(lib, 4, 8, 8, d, out=18) == 3
    assert _call(lib, 4, 8, 8, d, out=None) == 1
    assert _call(lib, 4, 8, 8, d, x=None) == 1


def test_absurd_output_sizes_are_rejected(lib):
    # M * N >= 2^40 outputs is rejected before anything else happens
    d = fle.desc_for("scale_hardtanh_gelu")
    assert _call(lib, 1 << 20, 8, 1 << 20, d) == 2  # FLE_ERR_SHAPE


def test_empty_sizes_enqueue_nothing(lib):
    d = fle.desc_for("scale_hardtanh_gelu")
    # M == 0, or N == 0 for an elementwise kind, is valid and returns before
    # touching the device (no device exists here).
    assert _call(lib, 0, 8, 8, d, x=None, W=None, out=None) == 0
    assert _call(lib, 4, 8, 0, d, x=None, W=None, out=None) == 0
    assert lib.fle_workspace_size(0, 8, 8, ctypes.byref(d)) == 0
    assert lib.fle_workspace_size(4, 6, 8, ctypes.byref(d)) == 0
    lib.fle_workspace_size_min.restype = ctypes.c_size_t
    assert lib.fle_workspace_size_min(0, 8, 8, ctypes.byref(d)) == 0
    assert lib.fle_workspace_size_min(4, 6, 8, ctypes.byref(d)) == 0
    assert lib.fle_workspace_size_min(-1, 8, 8, ctypes.byref(d)) == 0  # invalid: 0, fle_forward reports it


def test_binding_raises_with_status():
    d = fle.desc_for("scale_hardtanh_gelu")
    with pytest.raises(fle.FleError) as e:
        fle.forward(16, 16, None, 16, d, M=-1, K=8, N=8, stream=0)
    assert e.value.status == 2


def test_polynomial_gelu_table_is_the_generator_output():
    # The coefficients in gelu_poly2() are what gen_gelu_poly.py fits (least
    # squares on Chebyshev nodes, fp64 math.erf), and that fit is within 1e-8
    # of the exact-form GELU on [-2, 2].
    import importlib.util
    import re
    csrc = os.path.join(ROOT, "reduction_epilogue_b200", "csrc")
    spec = importlib.util.spec_from_file_location("gen_gelu_poly", os.path.join(csrc, "gen_gelu_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c = gen.fit()
    assert gen.check(c) < 1e-8
    src = open(os.path.join(csrc, "fle_kernel.cuh")).read()
    body = src[src.index("constexpr float kGeluPolyQ[8] = {"):]
    body = body[: body.index("};")]
    table = [float(v) for v in re.findall(r"(-?\d\.\d+e[-+]\d+)f", body)]
    assert len(table) == len(c) == 8
    assert all(abs(a - b) <= 1e-6 * abs(b) for a, b in zip(table, c))
