"""CPU oracle for exact Lloyd k-means -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library: the two share no code.

The arithmetic lives in ``fk_oracle.c`` (fp64, direct-difference distance,
first-minimum argmin, per-cluster mean, empty cluster keeps its previous
centroid), following the problem statement of "Flash-KMeans: Fast and
Memory-Efficient Exact K-Means" (arXiv 2603.09229, abstract: assignment stage
plus centroid-update stage, exact).  This module adds numpy marshalling, the
rounding of centroids to the input dtype and the Lloyd loop.

Readings taken where the pages are silent:
  * ties go to the lowest centroid index;
  * an empty cluster keeps its previous centroid;
  * centroids are kept in fp32 between iterations (the library's master copy)
    and rounded to the input dtype (round-to-nearest-even) for the next
    assignment, so both sides assign against the same rounded values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fk_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, openmp: bool = True) -> str:
    """Compile the C oracle into a shared library (gcc, -O2, OpenMP).  Every
    multiply and add is rounded on its own: no contraction into fused
    multiply-adds, which the plain definition does not perform."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-shared", "-fPIC", src, "-o", out, "-lm"]
    if openmp:
        cmd.insert(1, "-fopenmp")
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lp = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_assign.argtypes = [dp, ctypes.c_int64, ctypes.c_int, dp, ctypes.c_int, ip, dp, dp]
    lib.oracle_assign.restype = None
    lib.oracle_update.argtypes = [dp, ip, ctypes.c_int64, ctypes.c_int, ctypes.c_int, dp, dp, lp]
    lib.oracle_update.restype = ctypes.c_int
    lib.oracle_top2.argtypes = [dp, ctypes.c_int64, ctypes.c_int, dp, ctypes.c_int, ip, ip, dp, dp]
    lib.oracle_top2.restype = None
    lib.oracle_label_dist.argtypes = [dp, ip, ctypes.c_int64, ctypes.c_int, dp, dp]
    lib.oracle_label_dist.restype = None
    lib.oracle_gauss_sum.argtypes = [dp, ctypes.c_int64, ctypes.c_int, dp, ctypes.c_int, dp, ctypes.c_double, dp, dp]
    lib.oracle_gauss_sum.restype = None
    lib.oracle_kmeanspp.argtypes = [dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, dp, ip]
    lib.oracle_kmeanspp.restype = ctypes.c_int
    lib.oracle_objective.argtypes = [dp, ip, ctypes.c_int64, ctypes.c_int, dp]
    lib.oracle_objective.restype = ctypes.c_double
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def load(path: str = _LIB_PATH):
    """Load (building first if needed) an oracle library; returns the ctypes handle."""
    global _lib
    if path == _LIB_PATH and _lib is not None:
        return _lib
    if not os.path.exists(path) or (path == _LIB_PATH and
                                    os.path.getmtime(path) < os.path.getmtime(_SRC)):
        build(out=path)
    lib = _bind(ctypes.CDLL(path))
    if path == _LIB_PATH:
        _lib = lib
    return lib


def _p(a, t):
    return a.ctypes.data_as(ctypes.POINTER(t))


def num_threads() -> int:
    return load().oracle_num_threads()


def assign(X, C, lib=None):
    """Nearest centroid per row.  Returns (labels int32, mindist f64, second f64)."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    N, D = X.shape
    K = C.shape[0]
    assert C.shape[1] == D and K >= 1
    labels = np.zeros(N, np.int32)
    mind = np.zeros(N, np.float64)
    second = np.zeros(N, np.float64)
    if N:
        lib.oracle_assign(_p(X, ctypes.c_double), N, D, _p(C, ctypes.c_double), K,
                          _p(labels, ctypes.c_int32), _p(mind, ctypes.c_double),
                          _p(second, ctypes.c_double))
    return labels, mind, second


def top2(X, C, lib=None):
    """The two nearest centroids per row (oracle_top2): (label1, label2, d1, d2),
    labels int32 (label2 = -1 when K == 1), distances fp64."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    N, D = X.shape
    K = C.shape[0]
    assert C.shape[1] == D and K >= 1
    l1 = np.zeros(N, np.int32)
    l2 = np.zeros(N, np.int32)
    d1 = np.zeros(N, np.float64)
    d2 = np.zeros(N, np.float64)
    if N:
        lib.oracle_top2(_p(X, ctypes.c_double), N, D, _p(C, ctypes.c_double), K, _p(l1, ctypes.c_int32),
                        _p(l2, ctypes.c_int32), _p(d1, ctypes.c_double), _p(d2, ctypes.c_double))
    return l1, l2, d1, d2


def label_dist(X, labels, C, lib=None):
    """|x_i - c_{labels[i]}|^2 per row, the sum oracle_assign forms (fp64)."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    C = np.ascontiguousarray(C, dtype=np.float64)
    out = np.zeros(X.shape[0], np.float64)
    if X.shape[0]:
        lib.oracle_label_dist(_p(X, ctypes.c_double), _p(labels, ctypes.c_int32), X.shape[0], X.shape[1],
                              _p(C, ctypes.c_double), _p(out, ctypes.c_double))
    return out


def assign_screened(X, C, lib=None, block_elems=1 << 25, margin: float = 4.0):
    """``assign`` reached faster on large inputs, with the same labels and
    mindist.

    A library matrix product (torch on the CPU, fp32) gives every expanded
    distance e_k = |c_k|^2 - 2<x, c_k> (the |x|^2 term is common to a row) to
    within delta = margin (D + 8) 2^-24 (|x|^2 + max_k |c_k|^2), margin = 4: a
    generous form of
    the classical bound on the rounding of a length-D dot product and of the
    sums of squares.  A centroid whose e_k exceeds the row minimum by more
    than 2 delta is farther than the nearest one, so it cannot be the
    answer.  A row with one centroid left gets it, and its distance from
    ``label_dist`` (the oracle's own sum); every row with more left goes
    whole through ``assign``.  ``second`` is ``assign``'s for those rows and
    the second-smallest screened distance (|x|^2 added back) otherwise."""
    import torch
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    N, D = X.shape
    K = C.shape[0]
    labels = np.zeros(N, np.int32)
    mind = np.zeros(N, np.float64)
    second = np.full(N, np.inf)
    if N == 0:
        return labels, mind, second
    C32 = torch.from_numpy(C.astype(np.float32))
    cn = (C * C).sum(1)
    cn32 = torch.from_numpy(cn.astype(np.float32))
    cmax = float(cn.max())
    xn_all = np.einsum("ij,ij->i", X, X)
    rows = max(1, min(N, block_elems // max(K, 1)))
    multi = []
    Ebuf = torch.empty((rows, K), dtype=torch.float32)  # reused: fresh pages for every block cost more than the product
    for r0 in range(0, N, rows):
        r1 = min(N, r0 + rows)
        Xb = torch.from_numpy(X[r0:r1].astype(np.float32))
        E = torch.addmm(cn32.unsqueeze(0), Xb, C32.t(), beta=1.0, alpha=-2.0, out=Ebuf[: r1 - r0])
        delta = margin * (D + 8) * 2.0 ** -24 * (xn_all[r0:r1] + cmax)
        if K > 1:
            v, i = torch.topk(E, 2, dim=1, largest=False)
            v = v.double().numpy()
            labels[r0:r1] = i[:, 0].numpy()
            second[r0:r1] = v[:, 1] + xn_all[r0:r1]
            # more than one centroid within 2 delta of the row minimum
            multi.append(np.nonzero(v[:, 1] <= v[:, 0] + 2.0 * delta)[0] + r0)
    multi = np.concatenate(multi) if multi else np.zeros(0, np.int64)
    mind[:] = label_dist(X, labels, C, lib)  # rows with several candidates are redone below
    if len(multi):
        lm, dm, sm = assign(X[multi], C, lib)
        labels[multi] = lm
        mind[multi] = dm
        second[multi] = sm
    return labels, mind, second


def update(X, labels, K, C_prev, lib=None):
    """Per-cluster mean (fp64); empty clusters keep C_prev.  Returns (C_out, counts)."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    C_prev = np.ascontiguousarray(C_prev, dtype=np.float64)
    N, D = X.shape
    out = np.zeros((K, D), np.float64)
    counts = np.zeros(K, np.int64)
    rc = lib.oracle_update(_p(X, ctypes.c_double), _p(labels, ctypes.c_int32), N, D, K,
                           _p(C_prev, ctypes.c_double), _p(out, ctypes.c_double),
                           _p(counts, ctypes.c_int64))
    if rc != 0:
        raise ValueError("oracle_update: label out of range" if rc == -1 else "oracle_update failed")
    return out, counts


def gauss_sum(X, C, beta: float, w=None, lib=None):
    """Weighted Gauss sums G[i] = sum_k w[k] exp(-beta |x_i - c_k|^2) and
    ln G (NaN where G <= 0), fp64.  Returns (G, logG)."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    N, D = X.shape
    K = C.shape[0]
    G = np.zeros(N, np.float64)
    L = np.zeros(N, np.float64)
    wp = None
    if w is not None:
        w = np.ascontiguousarray(w, dtype=np.float64)
        wp = _p(w, ctypes.c_double)
    if N:
        lib.oracle_gauss_sum(_p(X, ctypes.c_double), N, D, _p(C, ctypes.c_double), K, wp, float(beta),
                             _p(G, ctypes.c_double), _p(L, ctypes.c_double))
    return G, L


def kmeanspp(X, K: int, u, lib=None) -> np.ndarray:
    """k-means++ centre indices (int32 K) drawn with the uniforms u (K in [0, 1))."""
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    assert u.shape == (K,) and X.shape[0] >= 1
    out = np.zeros(K, np.int32)
    rc = lib.oracle_kmeanspp(_p(X, ctypes.c_double), X.shape[0], X.shape[1], K, _p(u, ctypes.c_double),
                             _p(out, ctypes.c_int32))
    if rc != 0:
        raise MemoryError("oracle_kmeanspp")
    return out


def objective(X, labels, C, lib=None) -> float:
    lib = lib or load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    C = np.ascontiguousarray(C, dtype=np.float64)
    return lib.oracle_objective(_p(X, ctypes.c_double), _p(labels, ctypes.c_int32),
                                X.shape[0], X.shape[1], _p(C, ctypes.c_double))


# ---------------------------------------------------------------- rounding --
def to_f32(a) -> np.ndarray:
    """fp64 -> fp32, round to nearest even (the C cast numpy performs)."""
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def bf16_bits_from_f32(a) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns, round to nearest even on the dropped 16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to(dtype: str, a) -> np.ndarray:
    """Value of ``a`` stored in ``dtype`` ("f64", "f32", "f16", "bf16"), as fp64.

    fp16/bf16 round from fp32 (the library keeps fp32 master centroids)."""
    a = np.asarray(a, dtype=np.float64)
    if dtype == "f64":
        return a.copy()
    f32 = to_f32(a)
    if dtype == "f32":
        return f32.astype(np.float64)
    if dtype == "f16":
        return f32.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(bf16_bits_from_f32(f32))
    raise ValueError(dtype)


# ------------------------------------------------------------------ Lloyd --
def lloyd_step(X, C_master, dtype: str, lib=None, screened: bool = False):
    """One Lloyd iteration from fp32 (or fp64 when dtype == "f64") master centroids.

    Assignment uses the master rounded to ``dtype``; the update's empty-cluster
    rule keeps the master value.  ``screened`` takes the assignment from
    ``assign_screened`` (same labels, faster on large inputs).  Returns
    (C_next master, labels, mindist, second, counts)."""
    Cr = round_to(dtype, C_master)
    labels, mind, second = (assign_screened if screened else assign)(X, Cr, lib)
    Cn, counts = update(X, labels, Cr.shape[0], np.asarray(C_master, np.float64), lib)
    Cn = Cn if dtype == "f64" else to_f32(Cn).astype(np.float64)
    return Cn, labels, mind, second, counts


def lloyd(X, C0, iters: int, dtype: str, lib=None):
    """``iters`` Lloyd iterations.  Returns dict with final C, last labels /
    mindist / counts and the objective of every assignment (list of floats)."""
    C = np.asarray(C0, dtype=np.float64)
    if dtype != "f64":
        C = to_f32(C).astype(np.float64)
    hist = []
    labels = mind = counts = None
    for _ in range(iters):
        C, labels, mind, _, counts = lloyd_step(X, C, dtype, lib)
        hist.append(float(mind.sum()))
    return {"C": C, "labels": labels, "mindist": mind, "counts": counts, "objective": hist}
