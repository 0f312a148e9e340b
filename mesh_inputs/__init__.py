"""Seeded synthetic inputs for mesh gradient / Hessian assembly workloads.

This module only MAKES INPUTS: grid meshes, noisy positions, rest lengths,
rest-shape inverses, runtime vertex pairs and probe vectors.  It holds none of
the assembly arithmetic (no energies, derivatives, patterns or merges), and it
is the only code that both the CUDA path's tests/benchmarks and the CPU oracle
share.

Workloads (the page "Locality-Aware Automatic Differentiation on the GPU for
Mesh-Based Computations", section 实验结果 (results): mass-spring cloth at
10^2 ... 1000^2 vertices; the parameterization application with a
matrix-free Hessian-vector product; the contact shell's runtime vertex pairs).
The pages do not print meshes or parameters, so these are synthetic stand-ins:

* grid: unit square, spacing s = 1/(n-1); vertex (i, j) has index j*n + i and
  rest position (i*s, j*s, 0); quad (i, j) is split along its v00-v11
  diagonal into the counter-clockwise triangles (v00, v10, v11) and
  (v00, v11, v01); faces are quad-major, row-major.
* cloth: x = rest + N(0, (0.01 s)^2) on every coordinate, drawn afresh per
  step around the flat grid; springs on all mesh edges with rest length from
  the flat grid; k = 1e4; inertia target x~ = flat grid, w = m/h^2 with
  m = 1/V, h = 1e-2.
* pairs: per step, P uniform random vertex pairs (i, j), rejecting i == j,
  mesh-adjacent pairs and repeated unordered pairs; rest = 0.9 * |xi - xj|
  at the step's x; k_p = 1e3.
* parameterization: 2D rest grid, UV = rest + N(0, (0.05 s)^2); a triangle
  whose UV orientation is not positive has the noise of its three vertices
  redrawn from the same stream until no triangle is inverted; per-face
  Dm^-1 and area 1/2 |det Dm| from the rest triangle.
* probe vectors: N(0, 1) per DOF.

Every array is produced with numpy from an explicit seed.
"""
from __future__ import annotations

import numpy as np

CLOTH_K = 1.0e4
CLOTH_H = 1.0e-2
PAIR_K = 1.0e3


def _rng(*seed):
    return np.random.default_rng(np.random.SeedSequence([int(s) for s in seed]))


def grid_mesh(n: int, dim: int = 3):
    """Rest positions [V][dim] (fp64) and faces [2(n-1)^2][3] (int32)."""
    if n < 1:
        raise ValueError("n >= 1")
    s = 1.0 / (n - 1) if n > 1 else 1.0
    jj, ii = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    X = np.zeros((n * n, dim), np.float64)
    X[:, 0] = (ii * s).reshape(-1)
    X[:, 1] = (jj * s).reshape(-1)
    if n < 2:
        return X, np.zeros((0, 3), np.int32)
    qj, qi = np.meshgrid(np.arange(n - 1), np.arange(n - 1), indexing="ij")
    v00 = (qj * n + qi).reshape(-1)
    v10, v01, v11 = v00 + 1, v00 + n, v00 + n + 1
    F = np.empty((2 * (n - 1) ** 2, 3), np.int32)
    F[0::2] = np.stack([v00, v10, v11], 1)
    F[1::2] = np.stack([v00, v11, v01], 1)
    return X, F


def grid_spacing(n: int) -> float:
    return 1.0 / (n - 1) if n > 1 else 1.0


def grid_edges(n: int):
    """Unique undirected edges (i < j) of the grid, sorted by (i, j), built
    from the grid's structure (right, up and up-right neighbours of each
    vertex), not from the face list."""
    a = np.arange(n * n)
    i, j = a % n, a // n
    parts = []
    for di, dj in ((1, 0), (0, 1), (1, 1)):
        ok = (i + di < n) & (j + dj < n)
        parts.append(np.stack([a[ok], a[ok] + dj * n + di], 1))
    E = np.concatenate(parts, 0) if parts else np.zeros((0, 2), np.int64)
    order = np.lexsort((E[:, 1], E[:, 0]))
    return E[order].astype(np.int32)


def grid_adjacent(n: int, a, b):
    """True where grid vertices a and b share a mesh edge (closed form)."""
    a, b = np.asarray(a), np.asarray(b)
    di = b % n - a % n
    dj = b // n - a // n
    axis = (np.abs(di) + np.abs(dj)) == 1
    diag = (di == dj) & (np.abs(di) == 1)
    return axis | diag


def cloth_static(n: int, dtype=np.float32):
    """Topology and per-term parameters of the n x n cloth (step-independent)."""
    X, F = grid_mesh(n, 3)
    E = grid_edges(n)
    L0 = np.linalg.norm(X[E[:, 0]] - X[E[:, 1]], axis=1)
    V = n * n
    return {
        "n": n, "V": V, "X": X, "F": F, "edges": E,
        "L0": L0.astype(dtype), "xt": X.astype(dtype),
        "k": CLOTH_K, "w": (1.0 / V) / CLOTH_H ** 2, "dtype": np.dtype(dtype),
    }


def cloth_x(n: int, seed: int, step: int, dtype=np.float32):
    """Positions of one step: flat grid + N(0, (0.01 s)^2) on x, y, z."""
    X, _ = grid_mesh(n, 3)
    sig = 0.01 * grid_spacing(n)
    return (X + sig * _rng(seed, step, 1).standard_normal(X.shape)).astype(dtype)


def random_pairs(n: int, P: int, seed: int, step: int):
    """P distinct unordered, non-adjacent vertex pairs of the n x n grid, in
    draw order (int32 [P][2])."""
    V = n * n
    rng = _rng(seed, step, 2)
    out = np.zeros((0, 2), np.int64)
    seen_keys = np.zeros(0, np.int64)
    while out.shape[0] < P:
        m = max(2 * (P - out.shape[0]), 64)
        c = rng.integers(0, V, size=(m, 2))
        ok = (c[:, 0] != c[:, 1]) & ~grid_adjacent(n, c[:, 0], c[:, 1])
        c = c[ok]
        key = np.minimum(c[:, 0], c[:, 1]) * V + np.maximum(c[:, 0], c[:, 1])
        _, first = np.unique(key, return_index=True)
        first.sort()
        c, key = c[first], key[first]
        fresh = ~np.isin(key, seen_keys)
        c, key = c[fresh], key[fresh]
        need = P - out.shape[0]
        c, key = c[:need], key[:need]
        out = np.concatenate([out, c], 0)
        seen_keys = np.concatenate([seen_keys, key])
    return out.astype(np.int32)


def pair_rest(x, pairs, dtype=np.float32):
    """0.9 x the pair distance at the step's (stored) positions."""
    x = np.asarray(x, np.float64)
    d = np.linalg.norm(x[pairs[:, 0]] - x[pairs[:, 1]], axis=1)
    return (0.9 * d).astype(dtype)


def random_vf(n: int, nvf: int, seed: int, step: int):
    """nvf vertex-face terms (vertex, face) of the n x n grid, int32 [nvf][2]:
    a uniform face, and a vertex within two grid steps of the face's first
    corner that is not one of its corners (a contact-like neighbourhood)."""
    _, F = grid_mesh(n, 3)
    rng = _rng(seed, step, 5)
    out = []
    while len(out) < nvf:
        m = 2 * (nvf - len(out)) + 64
        f = rng.integers(0, F.shape[0], size=m)
        a = F[f, 0]
        di = rng.integers(-2, 3, size=m)
        dj = rng.integers(-2, 3, size=m)
        i, j = a % n + di, a // n + dj
        ok = (i >= 0) & (i < n) & (j >= 0) & (j < n)
        p = j * n + i
        ok &= (p != F[f, 0]) & (p != F[f, 1]) & (p != F[f, 2])
        for pp, ff in zip(p[ok], f[ok]):
            out.append((pp, ff))
            if len(out) == nvf:
                break
    return np.array(out, np.int32)


def vf_pairs(vf, F):
    """The (vertex, corner) pairs whose blocks vertex-face terms need."""
    F = np.asarray(F)
    return np.stack([np.repeat(vf[:, 0], 3), F[vf[:, 1]].reshape(-1)], axis=1).astype(np.int32)


def param_static(n: int, seed: int, dtype=np.float32):
    """The n x n parameterization problem: 2D rest grid, faces, per-face
    Dm^-1 [F][2][2] and area [F], and non-inverted noisy UV [V][2]."""
    X, F = grid_mesh(n, 2)
    s = grid_spacing(n)
    P0, P1, P2 = X[F[:, 0]], X[F[:, 1]], X[F[:, 2]]
    Dm = np.stack([P1 - P0, P2 - P0], axis=2)  # columns: edge vectors
    det = Dm[:, 0, 0] * Dm[:, 1, 1] - Dm[:, 0, 1] * Dm[:, 1, 0]
    Minv = np.empty_like(Dm)
    Minv[:, 0, 0] = Dm[:, 1, 1] / det
    Minv[:, 0, 1] = -Dm[:, 0, 1] / det
    Minv[:, 1, 0] = -Dm[:, 1, 0] / det
    Minv[:, 1, 1] = Dm[:, 0, 0] / det
    area = 0.5 * np.abs(det)
    rng = _rng(seed, 0, 3)
    sig = 0.05 * s
    noise = sig * rng.standard_normal(X.shape)
    redraws = 0
    while True:
        UV = (X + noise).astype(dtype).astype(np.float64)
        e1 = UV[F[:, 1]] - UV[F[:, 0]]
        e2 = UV[F[:, 2]] - UV[F[:, 0]]
        orient = e1[:, 0] * e2[:, 1] - e1[:, 1] * e2[:, 0]
        bad = np.nonzero(orient <= 0)[0]
        if bad.size == 0:
            break
        vb = np.unique(F[bad].reshape(-1))
        noise[vb] = sig * rng.standard_normal((vb.size, 2))
        redraws += 1
    return {
        "n": n, "V": n * n, "X": X, "F": F, "UV": (X + noise).astype(dtype),
        "Minv": Minv.astype(dtype), "area": area.astype(dtype),
        "redraws": redraws, "dtype": np.dtype(dtype),
    }


def probe_vector(V: int, dof: int, seed: int, dtype=np.float32):
    """HVP direction v ~ N(0, 1) per DOF."""
    return _rng(seed, 0, 4).standard_normal((V, dof)).astype(dtype)
