"""The C ABI library loads, exports every symbol include/mad.h declares, and
rejects bad arguments on the host before touching the GPU (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mad():
    import hessian_assembly_b200 as m
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mad.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mad_[a-z_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("mad_create", "mad_eval", "mad_hvp", "mad_add_pairs", "mad_pattern",
              "mad_edges", "mad_status_sync", "mad_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(mad):
    lib = mad.load_library()
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", mad.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (mad_\w+)", out))
    assert set(declared_functions()) <= exported
    assert set(mad.EXPORTS) == set(declared_functions())


def test_default_opts(mad):
    o = mad.mad_opts()
    mad.load_library().mad_default_opts(ctypes.byref(o))
    assert o.patch_faces == 512
    assert abs(o.slack - 0.10) < 1e-7
    assert o.max_pairs == 0 and not o.part_xyz


def _create(mad, V, F, dof=3, dt=0, opts=None):
    lib = mad.load_library()
    F = np.ascontiguousarray(np.asarray(F, np.int32).reshape(-1, 3))
    h = ctypes.c_void_p()
    st = lib.mad_create(V, F.shape[0], F.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), dof, dt,
                        opts, None, ctypes.byref(h))
    return st, h, lib.mad_last_error(None).decode()


@pytest.mark.parametrize("F,V,dof,dt", [
    ([[0, 1, 3]], 3, 3, 0),      # index out of range
    ([[0, 1, 1]], 3, 3, 0),      # repeated corner
    ([[0, -1, 2]], 3, 3, 0),     # negative index
    ([[0, 1, 2]], 3, 4, 0),      # bad dof
    ([[0, 1, 2]], 3, 3, 7),      # bad dtype
    ([[0, 1, 2]], -1, 3, 0),     # bad V
])
def test_create_rejects_bad_arguments_on_host(mad, F, V, dof, dt):
    st, h, msg = _create(mad, V, F, dof, dt)
    assert st == mad.MAD_ERR_INVALID_ARG
    assert not h.value
    assert msg


def test_create_rejects_bad_partition_dim(mad):
    o = mad.mad_opts()
    mad.load_library().mad_default_opts(ctypes.byref(o))
    xyz = np.zeros((3, 4))
    o.part_xyz = xyz.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    o.part_dim = 4
    st, h, msg = _create(mad, 3, [[0, 1, 2]], opts=ctypes.byref(o))
    assert st == mad.MAD_ERR_INVALID_ARG and "part_dim" in msg


def test_null_context_calls_are_rejected(mad):
    lib = mad.load_library()
    t = mad.mad_terms()
    assert lib.mad_eval(None, None, ctypes.byref(t), None, None, None, None) == mad.MAD_ERR_INVALID_ARG
    assert lib.mad_hvp(None, None, ctypes.byref(t), None, None, None) == mad.MAD_ERR_INVALID_ARG
    assert lib.mad_add_pairs(None, 0, None, None, None) == mad.MAD_ERR_INVALID_ARG
    assert lib.mad_info(None, None) == mad.MAD_ERR_INVALID_ARG
    assert lib.mad_last_error(None) is not None
    lib.mad_destroy(None)  # no-op


def test_product_path_has_no_oracle_dependency():
    """The CUDA library and its binding never reference the oracle."""
    pkg = os.path.join(ROOT, "hessian_assembly_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in text.lower(), f
