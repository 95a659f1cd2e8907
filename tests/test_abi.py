"""The C-ABI library: it builds, loads without a GPU, exports every entry point
that include/bra.h declares, and rejects bad arguments on the host before
any CUDA call (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

import dynamic_sparse_attention_bra_b200 as bra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for path in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(bra_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("bra_route", "bra_attend", "bra_forward", "bra_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bra.library_path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(bra.EXPORTED_SYMBOLS) <= set(declared_functions())


def test_debug_build_exports_the_same_symbols():
    """The -DBRA_DEBUG build (output-index checks) is a drop-in for the library."""
    lib = ctypes.CDLL(bra.debug_library_path)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_strings():
    assert bra._lib.bra_version() >= 100
    assert bra.bra_status_string(0) == "ok"
    assert "range" in bra.bra_status_string(5)
    assert "debug" in bra.bra_status_string(bra.BRA_ERR_BOUNDS)


S1 = dict(B=64, H=56, W=56, C=64, heads=2, S=7, topk=1, dtype="bf16")


def shp(**kw):
    a = dict(S1)
    a.update(kw)
    return bra.shape_for(a["B"], a["H"], a["W"], a["C"], a["heads"], a["S"], a["topk"], a["dtype"])


def test_workspace_bytes():
    s = shp()
    means = 64 * 2 * 49 * 32 * 4
    means = (means + 255) // 256 * 256
    assert bra.bra_workspace_bytes(s) == 2 * means + 256
    assert bra.bra_workspace_bytes(shp(B=0)) == 256


@pytest.mark.parametrize("bad,code", [
    (dict(S=5), bra.BRA_ERR_INVALID_ARG),        # S does not divide 56
    (dict(H=57), bra.BRA_ERR_INVALID_ARG),
    (dict(topk=0), bra.BRA_ERR_INVALID_ARG),
    (dict(topk=50), bra.BRA_ERR_INVALID_ARG),
    (dict(heads=3), bra.BRA_ERR_INVALID_ARG),     # C % heads
    (dict(B=-1), bra.BRA_ERR_INVALID_ARG),
    (dict(C=0), bra.BRA_ERR_INVALID_ARG),
    (dict(heads=1), bra.BRA_ERR_UNSUPPORTED),     # d = 64
    (dict(C=128, heads=8), bra.BRA_ERR_UNSUPPORTED),  # d = 16
    (dict(H=64, W=64, S=32, topk=1), bra.BRA_ERR_UNSUPPORTED),  # 1024 regions
])
def test_bad_shapes_rejected_before_launch(bad, code):
    s = shp(**bad)
    p = 1 << 20  # never dereferenced: the shape check fails first
    assert bra._lib.bra_forward(ctypes.byref(s), p, p, p, p, p, p, None) == code
    assert bra._lib.bra_route(ctypes.byref(s), p, p, p, p, None) == code
    assert bra._lib.bra_attend(ctypes.byref(s), p, p, p, p, p, p, None) == code
    assert bra._lib.bra_lce(ctypes.byref(s), p, p, p, p, None) == code
    assert bra._lib.bra_attend_backward(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == code
    assert bra._lib.bra_qkv_project(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == code
    assert bra._lib.bra_forward_qkv(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == code
    assert bra._lib.bra_forward_lce(ctypes.byref(s), p, p, p, p, p, p, p, p, None) == code
    assert bra.bra_workspace_bytes(s) == 0


def test_bad_dtype_and_null_shape():
    s = shp()
    s.dtype = 7
    assert bra._lib.bra_forward(ctypes.byref(s), 16, 16, 16, 16, 16, 16, None) == bra.BRA_ERR_INVALID_ARG
    assert bra._lib.bra_forward(None, 16, 16, 16, 16, 16, 16, None) == bra.BRA_ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(6))
def test_null_and_misaligned_pointers(which):
    s = shp()
    good = [1 << 20] * 6
    for bad in (0, (1 << 20) + 8):
        ptrs = list(good)
        ptrs[which] = bad
        q, k, v, o, idx, ws = ptrs
        assert bra._lib.bra_forward(ctypes.byref(s), q, k, v, o, idx, ws, None) == bra.BRA_ERR_INVALID_ARG
        assert bra._lib.bra_attend(ctypes.byref(s), q, k, v, idx, o, ws, None) == bra.BRA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding has no fallback: a missing library is an ImportError."""
    import importlib.util
    src = os.path.join(os.path.dirname(bra.__file__), "__init__.py")
    pkg = tmp_path / "fakepkg"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("fakepkg", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


@pytest.mark.parametrize("which", range(4))
def test_lce_null_and_misaligned_pointers(which):
    """v, weight, o must be non-null and 16-byte aligned; bias may be null but
    not misaligned.  Every case is rejected on the host, before any launch."""
    s = shp()
    good = [1 << 20] * 4
    for bad in ((0, (1 << 20) + 4) if which != 2 else ((1 << 20) + 4,)):
        ptrs = list(good)
        ptrs[which] = bad
        v, w, b, o = ptrs
        assert bra._lib.bra_lce(ctypes.byref(s), v, w, b, o, None) == bra.BRA_ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(8))
def test_forward_lce_null_and_misaligned_pointers(which):
    """q, k, v, weight, o, idx and the workspace must be non-null and 16-byte
    aligned; bias may be null but not misaligned.  Rejected on the host."""
    s = shp()
    good = [1 << 20] * 8
    for bad in ((0, (1 << 20) + 4) if which != 4 else ((1 << 20) + 4,)):
        ptrs = list(good)
        ptrs[which] = bad
        q, k, v, w, b, o, idx, ws = ptrs
        assert bra._lib.bra_forward_lce(ctypes.byref(s), q, k, v, w, b, o, idx, ws, None) == bra.BRA_ERR_INVALID_ARG


def test_selftest_rejects_bad_arguments_before_launch():
    s = shp()
    ws = 1 << 20
    assert bra._lib.bra_selftest_bounded_wait(ctypes.byref(s), ws, 0, 0, None) == bra.BRA_ERR_INVALID_ARG
    assert bra._lib.bra_selftest_bounded_wait(ctypes.byref(s), ws, (1 << 24) + 1, 0, None) == bra.BRA_ERR_INVALID_ARG
    assert bra._lib.bra_selftest_bounded_wait(ctypes.byref(s), None, 10, 0, None) == bra.BRA_ERR_INVALID_ARG
    assert bra._lib.bra_selftest_bounded_wait(ctypes.byref(s), ws + 8, 10, 0, None) == bra.BRA_ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(9))
def test_backward_null_and_misaligned_pointers(which):
    s = shp()
    good = [1 << 20] * 9
    for bad in (0, (1 << 20) + 8):
        ptrs = list(good)
        ptrs[which] = bad
        assert bra._lib.bra_attend_backward(ctypes.byref(s), *ptrs, None) == bra.BRA_ERR_INVALID_ARG


def test_backward_rejects_what_it_cannot_stage():
    """256-token regions with 1024 routed keys need more shared memory than a CTA has."""
    s = bra.shape_for(2, 128, 128, 64, 2, 8, 4, "bf16")
    p = 1 << 20
    assert bra._lib.bra_attend_backward(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == bra.BRA_ERR_UNSUPPORTED


# Pointer order of bra_qkv_project after the shape: x, w_qkv, b_qkv, q, k, v,
# q_r, k_r, workspace; b_qkv may be NULL (no bias) but not misaligned.
@pytest.mark.parametrize("which", range(9))
def test_projection_null_and_misaligned_pointers(which):
    s = bra.shape_for(2, 56, 56, 64, 2, 7, 1, "bf16")
    good = [1 << 20] * 9
    for bad in (0, (1 << 20) + 8):
        if which == 2 and bad == 0:
            continue
        ptrs = list(good)
        ptrs[which] = bad
        assert bra._lib.bra_qkv_project(ctypes.byref(s), *ptrs, None) == bra.BRA_ERR_INVALID_ARG
        # bra_forward_qkv: x, w, b, q, k, v, o, idx, workspace
        assert bra._lib.bra_forward_qkv(ctypes.byref(s), *ptrs, None) == bra.BRA_ERR_INVALID_ARG


@pytest.mark.parametrize("args", [
    (64, 14, 14, 256, 8, 7, 16, "bf16"),   # C = 256: weights do not stay resident in shared memory
    (2, 128, 128, 64, 2, 8, 4, "bf16"),    # 256-token regions exceed one 128-row tile
    (2, 56, 56, 64, 2, 7, 1, "f32"),       # the projection runs on bf16 tensor cores only
    (2, 56, 56, 96, 3, 7, 1, "bf16"),      # C not a multiple of 64
])
def test_projection_rejects_what_it_does_not_cover(args):
    s = bra.shape_for(*args)
    p = 1 << 20
    assert bra._lib.bra_qkv_project(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == bra.BRA_ERR_UNSUPPORTED
    assert bra._lib.bra_forward_qkv(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None) == bra.BRA_ERR_UNSUPPORTED


@pytest.mark.parametrize("dims", [
    dict(B=4, H=14, W=14, C=256, heads=8, S=7, topk=16),   # regions of 4 tokens (stage 3)
    dict(B=2, H=128, W=128, C=64, heads=2, S=8, topk=4),   # regions of 256 tokens (high resolution)
    dict(B=1, H=16, W=16, C=64, heads=2, S=4, topk=16),    # 256 keys per query
], ids=["n4", "n256", "keys256"])
def test_backward_mma_pin_rejects_uncovered_shapes_on_the_host(dims, monkeypatch):
    """With BRA_BACKWARD_KERNEL=mma a shape the tensor-core backward does not
    cover is refused before any CUDA call (so this runs without a GPU)."""
    monkeypatch.setenv("BRA_BACKWARD_KERNEL", "mma")
    s = shp(**dims)
    p = 1 << 20
    rc = bra._lib.bra_attend_backward(ctypes.byref(s), p, p, p, p, p, p, p, p, p, None)
    assert rc == bra.BRA_ERR_UNSUPPORTED, rc
