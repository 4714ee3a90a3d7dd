"""Python binding of libfk: exact Lloyd k-means on B200 (Flash-KMeans method).

Argument marshalling only.  Every step runs in the CUDA kernels of
``libfk.so`` (built in-tree by ``_build.py``); PyTorch supplies device memory,
pinned host memory and streams.  Importing this module without the built
library raises ``ImportError``: there is no fallback of any kind.

The functions carry the C names (see ``include/fk.h``) and take torch tensors:

* ``fk_assign(X, C, labels=None, mindist=None, want_mindist=False)``
* ``fk_update(X, labels, C, counts=None)``            (C updated in place)
* ``fk_lloyd(X, C, iters, labels=None, mindist=None, counts=None)``
* ``fk_lloyd_ooc(X_host, C_host, iters, chunk_rows, labels_host=None, counts_host=None)``

A 3-D ``X`` (B x N x D) selects the batched entry points.  Failures raise
``FKError`` carrying the status code and the library's message.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfk.so")

FK_F32, FK_F16, FK_BF16 = 0, 1, 2
FK_OK = 0
FK_ERR_INVALID_ARG, FK_ERR_UNSUPPORTED, FK_ERR_CUDA = -1, -2, -3
FK_ERR_OOM, FK_ERR_TIMEOUT, FK_ERR_HOST_IO, FK_ERR_BAD_LABEL = -4, -5, -6, -7

_DT = {torch.float32: FK_F32, torch.float16: FK_F16, torch.bfloat16: FK_BF16}


class FKError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libfk status {status}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python distance_argmin_flashassign_b200/_build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    V, I64, I, U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64
    sig = {
        "fk_assign": [V, I64, I, I, V, I, V, V, V],
        "fk_assign_batched": [V, I, I64, I, I, V, I, V, V, V],
        "fk_update": [V, V, I64, I, I, I, V, V, V],
        "fk_update_batched": [V, V, I, I64, I, I, I, V, V, V],
        "fk_update_noalloc": [V, V, I64, I, I, I, V, V, V],
        "fk_lloyd": [V, I64, I, I, V, I, V, V, V, I, V],
        "fk_lloyd_fused": [V, I64, I, I, V, I, V, V, V, I, V],
        "fk_assign_top2": [V, I64, I, I, V, I, V, V, V, V, V],
        "fk_lloyd_batched": [V, I, I64, I, I, V, I, V, V, V, I, V],
        "fk_lloyd_ooc": [V, I64, I, I, V, I, V, V, I, I64, V],
        "fk_bias_len": [I, I],
        "fk_prepare_centroids": [V, I, I, I, I, V, V, V],
        "fk_prepare_points": [V, I, I64, I, I, V, V],
        "fk_assign_prepared": [V, I, I64, I, I, V, I, V, V, V, V, V],
        "fk_sync": [V],
        "fk_status_string": [I],
        "fk_get_last_error": [],
        "fk_last_error_message": [],
        "fk_launch_count": [],
        "fk_assign_path": [I64, I, I, I, I],
        "fk_set_assign_path": [I],
        "fk_set_wait_timeout_ns": [U64],
        "fk_debug_wait_timeout": [U64, V],
        "fk_release_workspace": [],
        "fk_debug_inject": [I, I64],
        "fk_gauss_sum": [V, I64, I, I, V, I, V, I, ctypes.c_float, V, V, V],
        "fk_seed_kmeanspp": [V, I64, I, I, I, V, V, V],
        "fk_version": [],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.fk_status_string.restype = ctypes.c_char_p
    lib.fk_last_error_message.restype = ctypes.c_char_p
    lib.fk_launch_count.restype = ctypes.c_uint64
    lib.fk_bias_len.restype = ctypes.c_int64
    return lib


lib = _load()

# names declared in include/fk.h (the C ABI this binding mirrors)
ABI_NAMES = ("fk_bias_len", "fk_prepare_centroids", "fk_prepare_points", "fk_assign_prepared", "fk_assign", "fk_assign_batched", "fk_update", "fk_update_batched", "fk_update_noalloc", "fk_lloyd",
             "fk_lloyd_fused", "fk_assign_top2", "fk_lloyd_batched", "fk_lloyd_ooc", "fk_sync", "fk_status_string", "fk_get_last_error",
             "fk_last_error_message", "fk_launch_count", "fk_assign_path", "fk_set_assign_path",
             "fk_set_wait_timeout_ns", "fk_debug_wait_timeout", "fk_release_workspace", "fk_debug_inject",
             "fk_gauss_sum", "fk_seed_kmeanspp", "fk_version")


def _check(status: int) -> None:
    if status != FK_OK:
        msg = lib.fk_last_error_message().decode(errors="replace")
        raise FKError(status, msg or lib.fk_status_string(status).decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dtype(X: torch.Tensor) -> int:
    if X.dtype not in _DT:
        raise TypeError(f"unsupported dtype {X.dtype}")
    return _DT[X.dtype]


def _need(t: torch.Tensor, name: str, dtype, shape, device) -> None:
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")


def _dims(X: torch.Tensor):
    if X.dim() == 2:
        return 1, X.shape[0], X.shape[1], False
    if X.dim() == 3:
        return X.shape[0], X.shape[1], X.shape[2], True
    raise ValueError("X must be N x D or B x N x D")


# ------------------------------------------------------------------ calls --
def fk_assign(X, C, labels=None, mindist=None, want_mindist=False, stream=None):
    """Nearest centroid per point (ties to the lowest index).  C in X's dtype."""
    B, N, D, bat = _dims(X)
    K = C.shape[-2]
    lead = (B, N) if bat else (N,)
    _need(X, "X", X.dtype, X.shape, X.device)
    _need(C, "C", X.dtype, ((B, K, D) if bat else (K, D)), X.device)
    if labels is None:
        labels = torch.empty(lead, dtype=torch.int32, device=X.device)
    if mindist is None and want_mindist:
        mindist = torch.empty(lead, dtype=torch.float32, device=X.device)
    _need(labels, "labels", torch.int32, lead, X.device)
    if mindist is not None:
        _need(mindist, "mindist", torch.float32, lead, X.device)
    if bat:
        _check(lib.fk_assign_batched(_ptr(X), B, N, D, _dtype(X), _ptr(C), K, _ptr(labels), _ptr(mindist),
                                     _stream(stream)))
    else:
        _check(lib.fk_assign(_ptr(X), N, D, _dtype(X), _ptr(C), K, _ptr(labels), _ptr(mindist), _stream(stream)))
    return labels, mindist


def fk_prepare_centroids(C, dtype, C_dt=None, bias=None, stream=None):
    """Round fp32 centroids (K x D or B x K x D) to ``dtype`` and compute the
    padded bias -|c|^2/2.  Returns (C_dt, bias)."""
    bat = C.dim() == 3
    B, K, D = (C.shape if bat else (1,) + tuple(C.shape))
    _need(C, "C", torch.float32, C.shape, C.device)
    if C_dt is None:
        C_dt = C if dtype == torch.float32 else torch.empty(C.shape, dtype=dtype, device=C.device)
    _need(C_dt, "C_dt", dtype, C.shape, C.device)
    n = int(lib.fk_bias_len(B, K))
    if bias is None:
        bias = torch.empty(n, dtype=torch.float32, device=C.device)
    _need(bias, "bias", torch.float32, (n,), C.device)
    _check(lib.fk_prepare_centroids(_ptr(C), B, K, D, _DT[dtype], _ptr(C_dt), _ptr(bias), _stream(stream)))
    return C_dt, bias


def fk_prepare_points(X, xnorm=None, stream=None):
    """Row norms |x|^2 (fp32) of X (N x D or B x N x D), for fk_assign_prepared."""
    B, N, D, bat = _dims(X)
    lead = (B, N) if bat else (N,)
    if xnorm is None:
        xnorm = torch.empty(lead, dtype=torch.float32, device=X.device)
    _need(xnorm, "xnorm", torch.float32, lead, X.device)
    _check(lib.fk_prepare_points(_ptr(X), B, N, D, _dtype(X), _ptr(xnorm), _stream(stream)))
    return xnorm


def fk_assign_prepared(X, C_dt, bias, labels, mindist=None, xnorm=None, stream=None):
    """Assignment against the output of ``fk_prepare_centroids`` (and
    optionally of ``fk_prepare_points``): the assignment kernel and the exact
    re-decision of near-ties."""
    B, N, D, bat = _dims(X)
    K = C_dt.shape[-2]
    _check(lib.fk_assign_prepared(_ptr(X), B, N, D, _dtype(X), _ptr(C_dt), K, _ptr(bias), _ptr(xnorm),
                                  _ptr(labels), _ptr(mindist), _stream(stream)))
    return labels, mindist


def fk_update(X, labels, C, counts=None, stream=None):
    """Cluster means into fp32 ``C`` (in place; empty clusters keep their row)."""
    B, N, D, bat = _dims(X)
    K = C.shape[-2]
    _need(labels, "labels", torch.int32, ((B, N) if bat else (N,)), X.device)
    _need(C, "C", torch.float32, ((B, K, D) if bat else (K, D)), X.device)
    if counts is not None:
        _need(counts, "counts", torch.int32, ((B, K) if bat else (K,)), X.device)
    if bat:
        _check(lib.fk_update_batched(_ptr(X), _ptr(labels), B, N, D, _dtype(X), K, _ptr(C), _ptr(counts),
                                     _stream(stream)))
    else:
        _check(lib.fk_update(_ptr(X), _ptr(labels), N, D, _dtype(X), K, _ptr(C), _ptr(counts), _stream(stream)))
    return C, counts


def fk_update_noalloc(X, labels, C, counts=None, stream=None):
    """fk_update without any device allocation by the library: its scratch is a
    fixed 32 MiB array inside libfk (about 1.55 M points at D = 128 and
    K = 1,024, 0.41 M at D = 1,024).  For
    callers that cannot let a library allocate (stream capture, a framework
    that owns all device memory, allocation-free loops).  Calls sharing that
    array must not overlap on the GPU."""
    B, N, D, bat = _dims(X)
    if bat:
        raise ValueError("fk_update_noalloc takes one problem (N x D)")
    K = C.shape[-2]
    _need(labels, "labels", torch.int32, (N,), X.device)
    _need(C, "C", torch.float32, (K, D), X.device)
    if counts is not None:
        _need(counts, "counts", torch.int32, (K,), X.device)
    _check(lib.fk_update_noalloc(_ptr(X), _ptr(labels), N, D, _dtype(X), K, _ptr(C), _ptr(counts),
                                 _stream(stream)))
    return C, counts


def fk_assign_top2(X, C, label1=None, label2=None, dist1=None, dist2=None, want_dist=False, stream=None):
    """The two nearest centroids of every row of X (N x D): (label1, label2,
    dist1, dist2); C K x D in X's dtype.  Asynchronous on ``stream``."""
    N, D = X.shape
    K = C.shape[0]
    _need(C, "C", X.dtype, (K, D), X.device)
    if label1 is None:
        label1 = torch.empty(N, dtype=torch.int32, device=X.device)
    if label2 is None:
        label2 = torch.empty(N, dtype=torch.int32, device=X.device)
    if want_dist:
        dist1 = torch.empty(N, dtype=torch.float32, device=X.device) if dist1 is None else dist1
        dist2 = torch.empty(N, dtype=torch.float32, device=X.device) if dist2 is None else dist2
    _need(label1, "label1", torch.int32, (N,), X.device)
    _need(label2, "label2", torch.int32, (N,), X.device)
    _check(lib.fk_assign_top2(_ptr(X), N, D, _dtype(X), _ptr(C), K, _ptr(label1), _ptr(label2), _ptr(dist1),
                              _ptr(dist2), _stream(stream)))
    return label1, label2, dist1, dist2


def fk_lloyd(X, C, iters, labels=None, mindist=None, counts=None, want_mindist=False, stream=None, fused=False):
    """``iters`` Lloyd iterations; fp32 ``C`` is updated in place.  Synchronous.
    ``fused``: one pass over X per iteration (fk_lloyd_fused; single problem,
    centroids that fit in shared memory)."""
    B, N, D, bat = _dims(X)
    K = C.shape[-2]
    lead = (B, N) if bat else (N,)
    _need(C, "C", torch.float32, ((B, K, D) if bat else (K, D)), X.device)
    if labels is None:
        labels = torch.empty(lead, dtype=torch.int32, device=X.device)
    if mindist is None and want_mindist:
        mindist = torch.empty(lead, dtype=torch.float32, device=X.device)
    if counts is None:
        counts = torch.empty(((B, K) if bat else (K,)), dtype=torch.int32, device=X.device)
    _need(labels, "labels", torch.int32, lead, X.device)
    if fused:
        if bat:
            raise ValueError("the single-pass Lloyd step takes one problem")
        _check(lib.fk_lloyd_fused(_ptr(X), N, D, _dtype(X), _ptr(C), K, _ptr(labels), _ptr(mindist),
                                  _ptr(counts), iters, _stream(stream)))
    elif bat:
        _check(lib.fk_lloyd_batched(_ptr(X), B, N, D, _dtype(X), _ptr(C), K, _ptr(labels), _ptr(mindist),
                                    _ptr(counts), iters, _stream(stream)))
    else:
        _check(lib.fk_lloyd(_ptr(X), N, D, _dtype(X), _ptr(C), K, _ptr(labels), _ptr(mindist), _ptr(counts),
                            iters, _stream(stream)))
    return C, labels, mindist, counts


def fk_lloyd_ooc(X_host, C_host, iters, chunk_rows, labels_host=None, counts_host=None, stream=None):
    """Out-of-core Lloyd: ``X_host`` (N x D, CPU, pinned for overlap) is streamed
    in chunks; fp32 ``C_host`` (CPU) is updated in place.  Synchronous."""
    if X_host.device.type != "cpu" or C_host.device.type != "cpu":
        raise ValueError("fk_lloyd_ooc takes host tensors")
    N, D = X_host.shape
    K = C_host.shape[0]
    _need(X_host, "X_host", X_host.dtype, X_host.shape, X_host.device)
    _need(C_host, "C_host", torch.float32, (K, D), X_host.device)
    if labels_host is not None:
        _need(labels_host, "labels_host", torch.int32, (N,), X_host.device)
    if counts_host is not None:
        _need(counts_host, "counts_host", torch.int32, (K,), X_host.device)
    _check(lib.fk_lloyd_ooc(_ptr(X_host), N, D, _dtype(X_host), _ptr(C_host), K, _ptr(labels_host),
                            _ptr(counts_host), iters, chunk_rows, _stream(stream)))
    return C_host, labels_host, counts_host


def fk_gauss_sum(X, C, beta, w=None, signed=False, G=None, logG=None, want=("G", "logG"), stream=None):
    """Weighted Gauss sums G[i] = sum_k w[k] exp(-beta |x_i - c_k|^2) (C in
    X's dtype; w fp32 K or None).  Returns (G, logG); pass C = X for Kv."""
    N, D = X.shape
    K = C.shape[0]
    _need(C, "C", X.dtype, (K, D), X.device)
    if w is not None:
        _need(w, "w", torch.float32, (K,), X.device)
    if G is None and "G" in want:
        G = torch.empty(N, dtype=torch.float32, device=X.device)
    if logG is None and "logG" in want:
        logG = torch.empty(N, dtype=torch.float32, device=X.device)
    _check(lib.fk_gauss_sum(_ptr(X), N, D, _dtype(X), _ptr(C), K, _ptr(w), int(bool(signed)), float(beta), _ptr(G),
                            _ptr(logG), _stream(stream)))
    return G, logG


def fk_seed_kmeanspp(X, K, u, centers=None, stream=None):
    """k-means++ seeding: row indices (device int32 K) of K centres of X
    (N x D) drawn with the caller's uniforms u (K floats in [0, 1))."""
    import numpy as np
    N, D = X.shape
    u = np.ascontiguousarray(np.asarray(u, dtype=np.float64))
    if u.shape != (K,):
        raise ValueError("u must hold K draws")
    if centers is None:
        centers = torch.empty(K, dtype=torch.int32, device=X.device)
    _need(centers, "centers", torch.int32, (K,), X.device)
    _check(lib.fk_seed_kmeanspp(_ptr(X), N, D, _dtype(X), K, ctypes.c_void_p(u.ctypes.data), _ptr(centers),
                                _stream(stream)))
    return centers


def fk_sync(stream=None) -> None:
    _check(lib.fk_sync(_stream(stream)))


def fk_status_string(status: int) -> str:
    return lib.fk_status_string(status).decode()


def fk_launch_count() -> int:
    return int(lib.fk_launch_count())


def fk_assign_path(N: int, D: int, dtype: torch.dtype, K: int, B: int = 1) -> int:
    return int(lib.fk_assign_path(N, D, _DT[dtype], K, B))


def fk_set_assign_path(path: int) -> None:
    _check(lib.fk_set_assign_path(path))


def fk_set_wait_timeout_ns(ns: int) -> None:
    _check(lib.fk_set_wait_timeout_ns(ns))


def fk_debug_wait_timeout(ns: int, stream=None) -> int:
    """Returns the status of the timeout self-test (FK_ERR_TIMEOUT when it works)."""
    return int(lib.fk_debug_wait_timeout(ns, _stream(stream)))


def fk_release_workspace() -> None:
    _check(lib.fk_release_workspace())


FK_INJECT_NONE, FK_INJECT_CHUNK_COPY, FK_INJECT_SCRATCH_ALLOC = 0, 1, 2


def fk_debug_inject(what: int, at: int = -1) -> None:
    """Arm one host-side test fault (see include/fk.h): FK_INJECT_CHUNK_COPY
    at chunk copy `at` of the next fk_lloyd_ooc, or FK_INJECT_SCRATCH_ALLOC."""
    _check(lib.fk_debug_inject(what, at))


def fk_version() -> int:
    return int(lib.fk_version())
