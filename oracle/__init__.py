"""fp64 CPU oracle for mesh gradient / block-CSR Hessian assembly.

TEST INFRASTRUCTURE ONLY.  The product library never imports, links or calls
this package; only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg (``bench.py`` ``cpu_baseline`` and ``--impl reference``) use
it.  It shares no code, header, table or helper with the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, closed forms, COO ->
sort -> merge -> CSR); this module only builds it with gcc and marshals numpy
arrays through ctypes.  It follows the page "Locality-Aware Automatic
Differentiation on the GPU for Mesh-Based Computations", section 方法
(method): g = sum_j S_j^T g_j, H = sum_j S_j^T H_j S_j, with the CSR pattern
preallocated from mesh topology (key design 3) plus runtime pair blocks (key
design 4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import shutil
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MASK_SPRING = 1
MASK_INERTIA = 2
MASK_SYMDIR = 4
MASK_PAIR = 8

_CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math"]


def build(out: str = _LIB, mutant: int = 0) -> str:
    """Compile oracle.c with gcc into ``out`` (a planted mistake when mutant>0)."""
    cmd = ["gcc", *_CFLAGS, f"-DOR_MUTANT={int(mutant)}", "-o", out, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(path: str) -> bool:
    return (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)


_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f64p = ctypes.POINTER(ctypes.c_double)


def _p32(a):
    return None if a is None else a.ctypes.data_as(_i32p)


def _pf(a):
    return None if a is None else a.ctypes.data_as(_f64p)


class Oracle:
    """ctypes handle on one build of oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.or_spring_local.argtypes = [ctypes.c_int, _f64p, _f64p, ctypes.c_double,
                                        ctypes.c_double, _f64p, _f64p, _f64p]
        lib.or_inertia_local.argtypes = [ctypes.c_int, _f64p, _f64p, ctypes.c_double,
                                         _f64p, _f64p, _f64p]
        lib.or_symdir_local.argtypes = [_f64p, _f64p, _f64p, _f64p, ctypes.c_double,
                                        _f64p, _f64p, _f64p]
        lib.or_pattern.argtypes = [ctypes.c_int32, ctypes.c_int32, _i32p, ctypes.c_int32,
                                   _i32p, _i32p, _i32p, ctypes.c_int64, _i64p]
        lib.or_pattern.restype = ctypes.c_int
        lib.or_edges.argtypes = [ctypes.c_int32, ctypes.c_int32, _i32p, _i32p,
                                 ctypes.c_int64, _i64p]
        lib.or_edges.restype = ctypes.c_int
        lib.or_eval.argtypes = [ctypes.c_int32, ctypes.c_int, _f64p, ctypes.c_uint,
                                ctypes.c_int32, _i32p, _f64p, ctypes.c_double,
                                _f64p, ctypes.c_double,
                                ctypes.c_int32, _i32p, _f64p, _f64p,
                                ctypes.c_int32, _i32p, _f64p, ctypes.c_double,
                                _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.or_eval.restype = ctypes.c_int
        lib.or_eval3.argtypes = [ctypes.c_int32, ctypes.c_int, _f64p, ctypes.c_uint,
                                 ctypes.c_int32, _i32p, _f64p, ctypes.c_double, _f64p,
                                 ctypes.c_double, ctypes.c_int32, _i32p, _f64p, _f64p,
                                 ctypes.c_int32, _i32p, _f64p, ctypes.c_double, ctypes.c_double,
                                 ctypes.c_int32, _i32p, _f64p, ctypes.c_double,
                                 _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.or_eval3.restype = ctypes.c_int
        lib.or_eval2.argtypes = [ctypes.c_int32, ctypes.c_int, _f64p, ctypes.c_uint,
                                 ctypes.c_int32, _i32p, _f64p, ctypes.c_double, _f64p,
                                 ctypes.c_double, ctypes.c_int32, _i32p, _f64p, _f64p,
                                 ctypes.c_int32, _i32p, _f64p, ctypes.c_double, ctypes.c_double,
                                 _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.or_eval2.restype = ctypes.c_int
        lib.or_area_local.argtypes = [_f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_double,
                                      _f64p, _f64p, _f64p]
        lib.or_area_local.restype = None
        lib.or_arap_local.argtypes = [_f64p, _f64p, _f64p, _f64p, ctypes.c_double, _f64p,
                                      _f64p, _f64p]
        lib.or_arap_local.restype = None
        lib.or_vf_local.argtypes = [_f64p, _f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_double,
                                    _f64p, _f64p, _f64p]
        lib.or_vf_local.restype = None
        lib.or_bsr_mv.argtypes = [ctypes.c_int32, ctypes.c_int, _i32p, _i32p, _f64p,
                                  _f64p, _f64p]
        lib.or_bsr_mv.restype = ctypes.c_int
        lib.or_spring_res.argtypes = [ctypes.c_int, _f64p, _f64p, ctypes.c_double,
                                      ctypes.c_double, _f64p, _f64p]
        lib.or_spring_res.restype = None
        lib.or_symdir_res.argtypes = [_f64p, _f64p, _f64p, _f64p, ctypes.c_double, _f64p,
                                      _f64p]
        lib.or_symdir_res.restype = None
        lib.or_jacobian_shape.argtypes = [ctypes.c_int32, ctypes.c_int, ctypes.c_uint,
                                          ctypes.c_int32, ctypes.c_int32, _i64p, _i64p]
        lib.or_jacobian_shape.restype = ctypes.c_int
        lib.or_jacobian.argtypes = [ctypes.c_int32, ctypes.c_int, _f64p, ctypes.c_uint,
                                    ctypes.c_int32, _i32p, _f64p, ctypes.c_double, _f64p,
                                    ctypes.c_double, ctypes.c_int32, _i32p, _f64p, _f64p,
                                    _f64p, _i64p, _i32p, _f64p]
        lib.or_jacobian.restype = ctypes.c_int
        self.lib = lib

    # ---- local terms ----------------------------------------------------
    def spring_local(self, xi, xj, L0, k):
        xi = np.ascontiguousarray(xi, np.float64)
        xj = np.ascontiguousarray(xj, np.float64)
        dof = xi.size
        E = np.zeros(1)
        g = np.zeros(2 * dof)
        H = np.zeros((2 * dof, 2 * dof))
        self.lib.or_spring_local(dof, _pf(xi), _pf(xj), float(L0), float(k), _pf(E),
                                 _pf(g), _pf(H))
        return E[0], g, H

    def inertia_local(self, xi, xt, w):
        xi = np.ascontiguousarray(xi, np.float64)
        xt = np.ascontiguousarray(xt, np.float64)
        dof = xi.size
        E = np.zeros(1)
        g = np.zeros(dof)
        H = np.zeros((dof, dof))
        self.lib.or_inertia_local(dof, _pf(xi), _pf(xt), float(w), _pf(E), _pf(g), _pf(H))
        return E[0], g, H

    def symdir_local(self, u0, u1, u2, Minv, area):
        u = [np.ascontiguousarray(a, np.float64) for a in (u0, u1, u2)]
        M = np.ascontiguousarray(Minv, np.float64).reshape(4)
        E = np.zeros(1)
        g = np.zeros(6)
        H = np.zeros((6, 6))
        self.lib.or_symdir_local(_pf(u[0]), _pf(u[1]), _pf(u[2]), _pf(M), float(area),
                                 _pf(E), _pf(g), _pf(H))
        return E[0], g, H

    # ---- topology ---------------------------------------------------------
    def pattern(self, V, F, pairs=None):
        F = np.ascontiguousarray(F, np.int32).reshape(-1, 3)
        P = None if pairs is None else np.ascontiguousarray(pairs, np.int32).reshape(-1, 2)
        nP = 0 if P is None else P.shape[0]
        cap = V + 6 * F.shape[0] + 2 * nP
        rp = np.zeros(V + 1, np.int32)
        ci = np.zeros(max(cap, 1), np.int32)
        need = np.zeros(1, np.int64)
        r = self.lib.or_pattern(V, F.shape[0], _p32(F), nP, _p32(P), _p32(rp), _p32(ci),
                                cap, need.ctypes.data_as(_i64p))
        if r < 0:
            raise ValueError(f"or_pattern failed: {r}")
        return rp, ci[:r].copy()

    def edges(self, V, F):
        F = np.ascontiguousarray(F, np.int32).reshape(-1, 3)
        cap = 3 * F.shape[0]
        ij = np.zeros((max(cap, 1), 2), np.int32)
        need = np.zeros(1, np.int64)
        r = self.lib.or_edges(V, F.shape[0], _p32(F), _p32(ij), cap,
                              need.ctypes.data_as(_i64p))
        if r < 0:
            raise ValueError(f"or_edges failed: {r}")
        return ij[:r].copy()

    # ---- assembly -------------------------------------------------------
    def eval(self, V, dof, x, mask, row_ptr, col_idx, *, edges=None, L0=None, k=0.0,
             xt=None, w=0.0, F=None, Minv=None, area=None, pairs=None, prest=None,
             kp=0.0, ka=0.0, vf=None, vf_rest=None, kc=0.0):
        """Assemble g [V][dof], H_vals [nnzb][dof][dof] and the energy (fp64).
        vf: int [nVF][2] (vertex, face) vertex-face terms (mask bit 64)."""
        f64 = lambda a: None if a is None else np.ascontiguousarray(a, np.float64)  # noqa: E731
        i32 = lambda a: None if a is None else np.ascontiguousarray(a, np.int32)  # noqa: E731
        x = f64(x).reshape(-1)
        row_ptr, col_idx = i32(row_ptr), i32(col_idx)
        edges, F, pairs, vf = i32(edges), i32(F), i32(pairs), i32(vf)
        L0, xt, Minv, area, prest = f64(L0), f64(xt), f64(Minv), f64(area), f64(prest)
        vf_rest = f64(vf_rest)
        nVF = 0 if vf is None else vf.reshape(-1, 2).shape[0]
        nE = 0 if edges is None else edges.reshape(-1, 2).shape[0]
        nF = 0 if F is None else F.reshape(-1, 3).shape[0]
        nP = 0 if pairs is None else pairs.reshape(-1, 2).shape[0]
        nnzb = int(row_ptr[V])
        g = np.zeros(V * dof)
        H = np.zeros(nnzb * dof * dof)
        E = np.zeros(1)
        r = self.lib.or_eval3(V, dof, _pf(x), mask, nE, _p32(edges), _pf(L0), float(k),
                              _pf(xt), float(w), nF, _p32(F), _pf(Minv), _pf(area),
                              nP, _p32(pairs), _pf(prest), float(kp), float(ka),
                              nVF, _p32(vf), _pf(vf_rest), float(kc),
                              _p32(row_ptr), _p32(col_idx), _pf(g), _pf(H), _pf(E))
        if r != 0:
            raise ValueError(f"or_eval failed: {r}")
        return g.reshape(V, dof), H.reshape(nnzb, dof, dof), float(E[0])

    def bsr_mv(self, V, dof, row_ptr, col_idx, H_vals, v):
        row_ptr = np.ascontiguousarray(row_ptr, np.int32)
        col_idx = np.ascontiguousarray(col_idx, np.int32)
        H = np.ascontiguousarray(H_vals, np.float64).reshape(-1)
        v = np.ascontiguousarray(v, np.float64).reshape(-1)
        y = np.zeros(V * dof)
        self.lib.or_bsr_mv(V, dof, _p32(row_ptr), _p32(col_idx), _pf(H), _pf(v), _pf(y))
        return y.reshape(V, dof)


    def arap_local(self, u0, u1, u2, M, A):
        """Energy, gradient [6] and Hessian [6][6] of one ARAP face (UV)."""
        E = np.zeros(1)
        g = np.zeros(6)
        H = np.zeros(36)
        f = lambda a: np.ascontiguousarray(a, np.float64).reshape(-1)  # noqa: E731
        self.lib.or_arap_local(_pf(f(u0)), _pf(f(u1)), _pf(f(u2)), _pf(f(M)), float(A), _pf(E),
                               _pf(g), _pf(H))
        return float(E[0]), g, H.reshape(6, 6)

    def vf_local(self, p, a, b, c, r, k):
        """Energy, gradient [12] and Hessian [12][12] of one vertex-face term."""
        E = np.zeros(1)
        g = np.zeros(12)
        H = np.zeros(144)
        f = lambda v: np.ascontiguousarray(v, np.float64).reshape(-1)  # noqa: E731
        self.lib.or_vf_local(_pf(f(p)), _pf(f(a)), _pf(f(b)), _pf(f(c)), float(r), float(k),
                             _pf(E), _pf(g), _pf(H))
        return float(E[0]), g, H.reshape(12, 12)

    def area_local(self, x0, x1, x2, A0, k):
        """Energy, gradient [9] and Hessian [9][9] of one area-preservation face."""
        E = np.zeros(1)
        g = np.zeros(9)
        H = np.zeros(81)
        f = lambda a: np.ascontiguousarray(a, np.float64)  # noqa: E731
        self.lib.or_area_local(_pf(f(x0)), _pf(f(x1)), _pf(f(x2)), float(A0), float(k), _pf(E),
                               _pf(g), _pf(H))
        return float(E[0]), g, H.reshape(9, 9)

    def spring_res(self, dof, xi, xj, L0, k):
        """Residual [1] and 1 x 2dof Jacobian of one spring."""
        r = np.zeros(1)
        J = np.zeros(2 * dof)
        self.lib.or_spring_res(dof, _pf(np.ascontiguousarray(xi, np.float64)),
                               _pf(np.ascontiguousarray(xj, np.float64)), float(L0), float(k),
                               _pf(r), _pf(J))
        return r, J.reshape(1, 2 * dof)

    def symdir_res(self, u0, u1, u2, M, A):
        """Residuals [8] and 8 x 6 Jacobian of one symmetric Dirichlet face."""
        r = np.zeros(8)
        J = np.zeros(48)
        f = lambda a: np.ascontiguousarray(a, np.float64).reshape(-1)  # noqa: E731
        self.lib.or_symdir_res(_pf(f(u0)), _pf(f(u1)), _pf(f(u2)), _pf(f(M)), float(A), _pf(r),
                               _pf(J))
        return r, J.reshape(8, 6)

    def jacobian(self, V, dof, x, mask, *, edges=None, L0=None, k=0.0, xt=None, w=0.0,
                 F=None, Minv=None, area=None):
        """Residuals r and the CSR Jacobian (row_ptr int64, col_idx, vals) in fp64."""
        f64 = lambda a: None if a is None else np.ascontiguousarray(a, np.float64)  # noqa: E731
        i32 = lambda a: None if a is None else np.ascontiguousarray(a, np.int32)  # noqa: E731
        x = f64(x).reshape(-1)
        edges, F = i32(edges), i32(F)
        L0, xt, Minv, area = f64(L0), f64(xt), f64(Minv), f64(area)
        nE = 0 if edges is None else edges.reshape(-1, 2).shape[0]
        nF = 0 if F is None else F.reshape(-1, 3).shape[0]
        nr = np.zeros(1, np.int64)
        nz = np.zeros(1, np.int64)
        if self.lib.or_jacobian_shape(V, dof, mask, nE, nF, nr.ctypes.data_as(_i64p),
                                      nz.ctypes.data_as(_i64p)) != 0:
            raise ValueError("or_jacobian_shape failed")
        rows, nnz = int(nr[0]), int(nz[0])
        r = np.zeros(max(rows, 1))
        rp = np.zeros(rows + 1, np.int64)
        ci = np.zeros(max(nnz, 1), np.int32)
        vals = np.zeros(max(nnz, 1))
        st = self.lib.or_jacobian(V, dof, _pf(x), mask, nE, _p32(edges), _pf(L0), float(k),
                                  _pf(xt), float(w), nF, _p32(F), _pf(Minv), _pf(area), _pf(r),
                                  rp.ctypes.data_as(_i64p), _p32(ci), _pf(vals))
        if st != 0:
            raise ValueError(f"or_jacobian failed: {st}")
        return r[:rows], rp, ci[:nnz], vals[:nnz]


_DEFAULT: Oracle | None = None


def load() -> Oracle:
    """The oracle as built from oracle.c (built on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        if _needs_build(_LIB):
            build(_LIB)
        _DEFAULT = Oracle(_LIB)
    return _DEFAULT


def load_mutant(mutant: int) -> Oracle:
    """A build of oracle.c with planted mistake number ``mutant`` (tests only).
    The library stays mapped once loaded, so its build folder is removed."""
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        return Oracle(build(os.path.join(d, f"liboracle_m{mutant}.so"), mutant))
    finally:
        shutil.rmtree(d, ignore_errors=True)
