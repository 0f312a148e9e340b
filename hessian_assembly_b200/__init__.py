"""Python binding of libmad, the B200 mesh-autodiff assembly library.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels behind include/mad.h.  PyTorch supplies device memory and streams.
The functions mirror the C entry points (mad_create, mad_eval, mad_hvp,
mad_add_pairs, mad_pattern, mad_edges, mad_status_sync, mad_eval_host,
mad_destroy); ``Context`` wraps one mad_ctx.

The library implements the hot path of the page "Locality-Aware Automatic
Differentiation on the GPU for Mesh-Based Computations" (section 方法):
per-term forward-mode AD of local energies on a triangle mesh, assembled into
g = sum_j S_j^T g_j and a block-CSR H = sum_j S_j^T H_j S_j, plus a
matrix-free Hessian-vector product and GPU insertion of runtime pair blocks.

If libmad.so is missing this module raises at import; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# an alternative build of the same library can be selected for experiments
LIB_PATH = os.environ.get("HESSIAN_ASSEMBLY_B200_LIB", os.path.join(_HERE, "libmad.so"))

MAD_OK = 0
MAD_ERR_INVALID_ARG = 1
MAD_ERR_CUDA = 2
MAD_ERR_OOM = 3
MAD_ERR_CAPACITY = 4
MAD_ERR_INDEX = 5
MAD_ERR_TIMEOUT = 6
MAD_ERR_UNIMPLEMENTED = 7
MAD_ERR_STATE = 8
MAD_F32 = 0
MAD_F64 = 1
MAD_TERM_SPRING = 1
MAD_TERM_INERTIA = 2
MAD_TERM_SYMDIR = 4
MAD_TERM_PAIR = 8
MAD_TERM_AREA = 16
MAD_TERM_ARAP = 32
MAD_TERM_VF = 64
MAD_EVAL_FULL_STENCIL_AD = 1
MAD_EVAL_EDGE_SCATTER = 2
MAD_EVAL_PATCH_STAGED = 4

STATUS_NAMES = {0: "MAD_OK", 1: "MAD_ERR_INVALID_ARG", 2: "MAD_ERR_CUDA", 3: "MAD_ERR_OOM",
                4: "MAD_ERR_CAPACITY", 5: "MAD_ERR_INDEX", 6: "MAD_ERR_TIMEOUT",
                7: "MAD_ERR_UNIMPLEMENTED", 8: "MAD_ERR_STATE"}

# every symbol include/mad.h declares
EXPORTS = ("mad_default_opts", "mad_create", "mad_info", "mad_edges", "mad_pattern",
           "mad_eval", "mad_hvp", "mad_add_pairs", "mad_status_sync", "mad_eval_host",
           "mad_last_error", "mad_destroy", "mad_selftest_dual", "mad_energy_noalloc",
           "mad_jacobian_shape", "mad_jacobian_pattern", "mad_jacobian", "mad_shard_plan",
           "mad_shard_halo", "mad_eval_shard", "mad_add_vf")


class mad_opts(ctypes.Structure):
    _fields_ = [("patch_faces", ctypes.c_int32), ("slack", ctypes.c_float),
                ("max_pairs", ctypes.c_int32), ("part_xyz", ctypes.POINTER(ctypes.c_double)),
                ("part_dim", ctypes.c_int32), ("smem_budget", ctypes.c_int32)]


class mad_terms(ctypes.Structure):
    _fields_ = [("mask", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("spring_rest", ctypes.c_void_p), ("spring_k", ctypes.c_double),
                ("inertia_xt", ctypes.c_void_p), ("inertia_w", ctypes.c_double),
                ("face_Minv", ctypes.c_void_p), ("face_area", ctypes.c_void_p),
                ("pair_k", ctypes.c_double), ("area_k", ctypes.c_double),
                ("vf_n", ctypes.c_int32), ("vf", ctypes.c_void_p), ("vf_rest", ctypes.c_void_p),
                ("vf_k", ctypes.c_double)]


class mad_info_t(ctypes.Structure):
    _fields_ = [("V", ctypes.c_int32), ("nF", ctypes.c_int32), ("E", ctypes.c_int32),
                ("dof", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("nnzb_base", ctypes.c_int32), ("capacity_blocks", ctypes.c_int32),
                ("max_pairs", ctypes.c_int32), ("n_patches", ctypes.c_int32),
                ("max_patch_vertices", ctypes.c_int32), ("max_patch_owned", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("device_bytes", ctypes.c_int64),
                ("row_slot_bytes", ctypes.c_int32)]


class MadError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """ctypes handle on libmad.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmad.so not found at {path}; build it with "
                          "`python hessian_assembly_b200/build.py` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    vp, i32, i32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)
    lib.mad_default_opts.argtypes = [ctypes.POINTER(mad_opts)]
    lib.mad_default_opts.restype = None
    lib.mad_create.argtypes = [i32, i32, i32p, i32, ctypes.c_int, ctypes.POINTER(mad_opts), vp,
                               ctypes.POINTER(vp)]
    lib.mad_create.restype = ctypes.c_int
    lib.mad_info.argtypes = [vp, ctypes.POINTER(mad_info_t)]
    lib.mad_info.restype = ctypes.c_int
    lib.mad_edges.argtypes = [vp, ctypes.POINTER(vp), i32p]
    lib.mad_edges.restype = ctypes.c_int
    lib.mad_pattern.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp)]
    lib.mad_pattern.restype = ctypes.c_int
    lib.mad_eval.argtypes = [vp, vp, ctypes.POINTER(mad_terms), vp, vp, vp, vp]
    lib.mad_eval.restype = ctypes.c_int
    lib.mad_hvp.argtypes = [vp, vp, ctypes.POINTER(mad_terms), vp, vp, vp]
    lib.mad_hvp.restype = ctypes.c_int
    lib.mad_add_pairs.argtypes = [vp, i32, vp, vp, vp]
    lib.mad_add_pairs.restype = ctypes.c_int
    lib.mad_status_sync.argtypes = [vp, vp]
    lib.mad_status_sync.restype = ctypes.c_int
    lib.mad_eval_host.argtypes = [vp, vp, ctypes.POINTER(mad_terms), vp, vp, vp, vp]
    lib.mad_eval_host.restype = ctypes.c_int
    lib.mad_last_error.argtypes = [vp]
    lib.mad_last_error.restype = ctypes.c_char_p
    lib.mad_destroy.argtypes = [vp]
    lib.mad_destroy.restype = None
    lib.mad_selftest_dual.argtypes = [i32, vp, vp]
    lib.mad_selftest_dual.restype = ctypes.c_int
    lib.mad_add_vf.argtypes = [vp, i32, vp, vp]
    lib.mad_add_vf.restype = ctypes.c_int
    lib.mad_shard_plan.argtypes = [i32, i32, i32p, i32, i32p, ctypes.POINTER(ctypes.c_int64)]
    lib.mad_shard_plan.restype = ctypes.c_int
    lib.mad_shard_halo.argtypes = [i32, i32, i32p, i32, i32, i32p, i32p, i32]
    lib.mad_shard_halo.restype = ctypes.c_int
    lib.mad_eval_shard.argtypes = [vp, i32, i32p, ctypes.POINTER(vp), i32,
                                   ctypes.POINTER(mad_terms), vp, vp, vp, vp]
    lib.mad_eval_shard.restype = ctypes.c_int
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.mad_jacobian_shape.argtypes = [vp, ctypes.c_uint32, i64p, i64p]
    lib.mad_jacobian_shape.restype = ctypes.c_int
    lib.mad_jacobian_pattern.argtypes = [vp, ctypes.c_uint32, vp, vp, vp]
    lib.mad_jacobian_pattern.restype = ctypes.c_int
    lib.mad_jacobian.argtypes = [vp, vp, ctypes.POINTER(mad_terms), vp, vp, vp]
    lib.mad_jacobian.restype = ctypes.c_int
    lib.mad_energy_noalloc.argtypes = [i32, i32, ctypes.c_int, vp, ctypes.POINTER(mad_terms), i32,
                                       vp, i32, vp, i32, vp, vp, vp, vp]
    lib.mad_energy_noalloc.restype = ctypes.c_int
    _lib = lib
    return lib


# ---------------------------------------------------------------- helpers


def _torch():
    import torch
    return torch


def _stream_ptr(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev_ptr(t, dtype=None, name="tensor", allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


class _DevView:
    """Zero-copy view of borrowed device memory via __cuda_array_interface__."""

    def __init__(self, ptr: int, shape, typestr: str, owner):
        self.__cuda_array_interface__ = {"data": (int(ptr), False), "shape": tuple(shape),
                                         "typestr": typestr, "version": 2, "strides": None}
        self._owner = owner


@dataclass
class Terms:
    """Term set for mad_eval / mad_hvp (mirrors mad_terms); arrays are CUDA tensors."""
    mask: int = 0
    flags: int = 0
    spring_rest: object = None
    spring_k: float = 0.0
    inertia_xt: object = None
    inertia_w: float = 0.0
    face_Minv: object = None
    face_area: object = None
    pair_k: float = 0.0
    area_k: float = 0.0
    vf: object = None        # int32 [n][2] (vertex, face)
    vf_rest: object = None
    vf_k: float = 0.0

    def to_c(self, dtype) -> mad_terms:
        torch = _torch()
        p = lambda t, n: None if t is None else _dev_ptr(t, dtype, n)  # noqa: E731
        # without vf, the installed set (mad_add_vf): its size from vf_rest
        nvf = (int(self.vf.shape[0]) if self.vf is not None else
               int(self.vf_rest.shape[0]) if self.vf_rest is not None else 0)
        return mad_terms(self.mask, self.flags, p(self.spring_rest, "spring_rest"),
                         float(self.spring_k), p(self.inertia_xt, "inertia_xt"),
                         float(self.inertia_w), p(self.face_Minv, "face_Minv"),
                         p(self.face_area, "face_area"), float(self.pair_k),
                         float(self.area_k), nvf,
                         None if self.vf is None else _dev_ptr(self.vf, torch.int32, "vf"),
                         p(self.vf_rest, "vf_rest"), float(self.vf_k))


class Context:
    """One mad_ctx: mesh topology, patches, CSR buffers (see include/mad.h)."""

    def __init__(self, V: int, F, dof: int, dtype="float32", *, patch_faces: int = 512,
                 slack: float = 0.10, max_pairs: int = 0, part_xyz=None,
                 smem_budget: int = 0, stream=None):
        lib = load_library()
        torch = _torch()
        self.lib = lib
        self.torch_dtype = {"float32": torch.float32, "float64": torch.float64}[str(dtype).replace("torch.", "")]
        self.dt = MAD_F32 if self.torch_dtype == torch.float32 else MAD_F64
        self.dof = int(dof)
        F = np.ascontiguousarray(np.asarray(F, np.int32).reshape(-1, 3))
        o = mad_opts()
        lib.mad_default_opts(ctypes.byref(o))
        o.patch_faces = int(patch_faces)
        o.slack = float(slack)
        o.max_pairs = int(max_pairs)
        o.smem_budget = int(smem_budget)
        self._part = None
        if part_xyz is not None:
            self._part = np.ascontiguousarray(np.asarray(part_xyz, np.float64))
            o.part_xyz = self._part.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
            o.part_dim = int(self._part.shape[1])
        h = ctypes.c_void_p()
        st = lib.mad_create(int(V), F.shape[0], F.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                            self.dof, self.dt, ctypes.byref(o), _stream_ptr(stream),
                            ctypes.byref(h))
        if st != MAD_OK:
            raise MadError(st, lib.mad_last_error(None).decode())
        self.h = h
        self.info = self._info()

    # ---- lifetime -----------------------------------------------------
    def close(self):
        if getattr(self, "h", None) is not None and self.h.value:
            self.lib.mad_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != MAD_OK:
            raise MadError(st, self.lib.mad_last_error(self.h).decode())

    def _info(self) -> mad_info_t:
        i = mad_info_t()
        self._check(self.lib.mad_info(self.h, ctypes.byref(i)))
        return i

    # ---- topology -----------------------------------------------------
    def mad_edges(self):
        torch = _torch()
        p = ctypes.c_void_p()
        E = ctypes.c_int32()
        self._check(self.lib.mad_edges(self.h, ctypes.byref(p), ctypes.byref(E)))
        if E.value == 0:
            return torch.zeros((0, 2), dtype=torch.int32, device="cuda")
        return torch.as_tensor(_DevView(p.value, (E.value, 2), "<i4", self), device="cuda")

    def mad_pattern(self):
        """(row_ptr, col_idx[:capacity], nnzb_dev) as zero-copy CUDA tensors."""
        torch = _torch()
        rp, ci, nz = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        self._check(self.lib.mad_pattern(self.h, ctypes.byref(rp), ctypes.byref(ci),
                                         ctypes.byref(nz)))
        V = self.info.V
        row_ptr = torch.as_tensor(_DevView(rp.value, (V + 1,), "<i4", self), device="cuda")
        col_idx = torch.as_tensor(_DevView(ci.value, (max(self.info.capacity_blocks, 1),), "<i4", self),
                                  device="cuda")
        nnzb = torch.as_tensor(_DevView(nz.value, (1,), "<i4", self), device="cuda")
        return row_ptr, col_idx, nnzb

    # ---- hot path -----------------------------------------------------
    def mad_eval(self, x, terms: Terms, g, H_vals, energy=None, stream=None):
        torch = _torch()
        t = terms.to_c(self.torch_dtype)
        st = self.lib.mad_eval(self.h, _dev_ptr(x, self.torch_dtype, "x"), ctypes.byref(t),
                               _dev_ptr(g, self.torch_dtype, "g"),
                               _dev_ptr(H_vals, self.torch_dtype, "H_vals"),
                               _dev_ptr(energy, torch.float64, "energy", allow_none=True),
                               _stream_ptr(stream))
        self._check(st)

    def mad_add_vf(self, vf, stream=None):
        """Install vertex-face terms: vf a CUDA int32 tensor [n][2] (p, f)."""
        torch = _torch()
        n = int(vf.shape[0]) if vf is not None else 0
        st = self.lib.mad_add_vf(self.h, n, _dev_ptr(vf, torch.int32, "vf") if n else None,
                                 _stream_ptr(stream))
        self._check(st)

    def mad_eval_shard(self, row_begin, x_parts, rank, terms: Terms, g_part, H_part,
                       energy=None, stream=None):
        """Rows of shard `rank` (see include/mad.h).  row_begin: int array
        [nranks+1]; x_parts: per shard a CUDA tensor [rows][dof] or a raw
        device address (int) readable from this device."""
        torch = _torch()
        rb = np.ascontiguousarray(np.asarray(row_begin, np.int32))
        n = rb.shape[0] - 1
        ptrs = (ctypes.c_void_p * max(n, 1))()
        for r, xp in enumerate(x_parts):
            if isinstance(xp, int):
                ptrs[r] = xp
            elif rb[r + 1] > rb[r]:
                ptrs[r] = _dev_ptr(xp, self.torch_dtype, f"x_parts[{r}]")
        t = terms.to_c(self.torch_dtype)
        st = self.lib.mad_eval_shard(
            self.h, n, rb.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), ptrs, int(rank),
            ctypes.byref(t), _dev_ptr(g_part, self.torch_dtype, "g_part", allow_none=True),
            _dev_ptr(H_part, self.torch_dtype, "H_part", allow_none=True),
            _dev_ptr(energy, torch.float64, "energy", allow_none=True), _stream_ptr(stream))
        self._check(st)

    def mad_hvp(self, x, terms: Terms, v, y, stream=None):
        t = terms.to_c(self.torch_dtype)
        st = self.lib.mad_hvp(self.h, _dev_ptr(x, self.torch_dtype, "x"), ctypes.byref(t),
                              _dev_ptr(v, self.torch_dtype, "v"), _dev_ptr(y, self.torch_dtype, "y"),
                              _stream_ptr(stream))
        self._check(st)

    def mad_jacobian_shape(self, mask: int):
        """(rows, nonzeros) of the Jacobian of the terms in `mask`."""
        nr, nz = ctypes.c_int64(0), ctypes.c_int64(0)
        self._check(self.lib.mad_jacobian_shape(self.h, mask, ctypes.byref(nr), ctypes.byref(nz)))
        return nr.value, nz.value

    def mad_jacobian_pattern(self, mask: int, row_ptr, col_idx, stream=None):
        torch = _torch()
        st = self.lib.mad_jacobian_pattern(self.h, mask, _dev_ptr(row_ptr, torch.int64, "row_ptr"),
                                           _dev_ptr(col_idx, torch.int32, "col_idx",
                                                    allow_none=True),
                                           _stream_ptr(stream))
        self._check(st)

    def mad_jacobian(self, x, terms: Terms, r, J_vals, stream=None):
        t = terms.to_c(self.torch_dtype)
        st = self.lib.mad_jacobian(self.h, _dev_ptr(x, self.torch_dtype, "x"), ctypes.byref(t),
                                   _dev_ptr(r, self.torch_dtype, "r", allow_none=True),
                                   _dev_ptr(J_vals, self.torch_dtype, "J_vals", allow_none=True),
                                   _stream_ptr(stream))
        self._check(st)

    def mad_add_pairs(self, ij, rest, stream=None):
        torch = _torch()
        n = 0 if ij is None else int(ij.shape[0])
        st = self.lib.mad_add_pairs(self.h, n,
                                    _dev_ptr(ij, torch.int32, "ij", allow_none=True) if n else None,
                                    _dev_ptr(rest, self.torch_dtype, "rest", allow_none=True) if n else None,
                                    _stream_ptr(stream))
        self._check(st)

    def mad_status_sync(self, stream=None) -> int:
        """Synchronise and return (and clear) the device status (MAD_OK or an error code)."""
        return int(self.lib.mad_status_sync(self.h, _stream_ptr(stream)))

    def mad_eval_host(self, x, terms: Terms, g, H_vals, energy=None, stream=None):
        """x, g, H_vals (and energy) are CPU tensors; pinned memory is fastest."""
        torch = _torch()
        for name, t in (("x", x), ("g", g), ("H_vals", H_vals)):
            if t.is_cuda or not t.is_contiguous() or t.dtype != self.torch_dtype:
                raise ValueError(f"{name} must be a contiguous CPU tensor of {self.torch_dtype}")
        if energy is not None and (energy.is_cuda or energy.dtype != torch.float64):
            raise ValueError("energy must be a CPU float64 tensor")
        tc = terms.to_c(self.torch_dtype)
        st = self.lib.mad_eval_host(self.h, ctypes.c_void_p(x.data_ptr()), ctypes.byref(tc),
                                    ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(H_vals.data_ptr()),
                                    None if energy is None else ctypes.c_void_p(energy.data_ptr()),
                                    _stream_ptr(stream))
        self._check(st)


load_library()  # fail loudly at import when the CUDA library is missing


def mad_create(V, F, dof, dtype="float32", **kw) -> Context:
    return Context(V, F, dof, dtype, **kw)


def _faces_arg(F):
    F = np.ascontiguousarray(np.asarray(F, np.int32).reshape(-1, 3))
    return F, F.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def mad_shard_plan(V: int, F, nranks: int):
    """(row_begin int32 [nranks+1], block_begin int64 [nranks+1]): contiguous
    row ranges balanced by block count (host only, see include/mad.h)."""
    lib = load_library()
    F, fp = _faces_arg(F)
    rb = np.zeros(nranks + 1, np.int32)
    bb = np.zeros(nranks + 1, np.int64)
    st = lib.mad_shard_plan(int(V), F.shape[0], fp, int(nranks),
                            rb.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                            bb.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    if st != MAD_OK:
        raise MadError(st, "mad_shard_plan")
    return rb, bb


def mad_shard_halo(V: int, F, row_lo: int, row_hi: int) -> np.ndarray:
    """Sorted vertices outside [row_lo, row_hi) that its rows couple to."""
    lib = load_library()
    F, fp = _faces_arg(F)
    n = ctypes.c_int32(0)
    st = lib.mad_shard_halo(int(V), F.shape[0], fp, int(row_lo), int(row_hi), ctypes.byref(n),
                            None, 0)
    if st != MAD_OK:
        raise MadError(st, "mad_shard_halo")
    out = np.zeros(max(n.value, 1), np.int32)
    st = lib.mad_shard_halo(int(V), F.shape[0], fp, int(row_lo), int(row_hi), ctypes.byref(n),
                            out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), out.shape[0])
    if st != MAD_OK:
        raise MadError(st, "mad_shard_halo")
    return out[:n.value]


def mad_selftest_dual(ab: np.ndarray) -> np.ndarray:
    """Device HyperDual self-test (see include/mad.h); returns [n][4][6]."""
    lib = load_library()
    ab = np.ascontiguousarray(np.asarray(ab, np.float64).reshape(-1, 2))
    out = np.zeros((ab.shape[0], 4, 6))
    st = lib.mad_selftest_dual(ab.shape[0], ctypes.c_void_p(ab.ctypes.data),
                               ctypes.c_void_p(out.ctypes.data))
    if st != MAD_OK:
        raise MadError(st, lib.mad_last_error(None).decode())
    return out


def mad_energy_noalloc(V, dof, x, terms: Terms, energy, *, edges=None, F=None, pairs=None,
                       pair_rest=None, stream=None) -> int:
    """Energy of the given terms without a context and without any allocation
    (see include/mad.h).  Tensors are CUDA tensors; `energy` is a float64 [1]
    CUDA tensor.  Returns the mad_status code."""
    torch = _torch()
    lib = load_library()
    dt = MAD_F64 if x.dtype == torch.float64 else MAD_F32
    tc = terms.to_c(x.dtype)
    n = lambda a: 0 if a is None else int(a.shape[0])  # noqa: E731
    p = lambda a, d, nm: None if a is None else _dev_ptr(a, d, nm)  # noqa: E731
    return int(lib.mad_energy_noalloc(int(V), int(dof), dt, _dev_ptr(x, x.dtype, "x"),
                                      ctypes.byref(tc), n(edges), p(edges, torch.int32, "edges"),
                                      n(F), p(F, torch.int32, "F"), n(pairs),
                                      p(pairs, torch.int32, "pairs"),
                                      p(pair_rest, x.dtype, "pair_rest"),
                                      _dev_ptr(energy, torch.float64, "energy"),
                                      _stream_ptr(stream)))
