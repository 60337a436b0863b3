"""fp64 CPU oracle for exact Lloyd's k-means (assign + centroid update).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
leg may import this package; the CUDA product path in exact_lloyd_means_b200/ never does.
It shares no code with that path and never takes a value computed by it as an input.

The arithmetic lives in lloyd_oracle.c (plain C loops in fp64, compiled with gcc); this
module only marshals numpy arrays and strings the steps together in the order the
Flash-KMeans article gives them (section "为什么"快"这件事被拖了这么久": assign every point
to a cluster, then recompute the centroids).  Precision handling between iterations
(rounding the centroids to the storage type the GPU keeps) uses torch CPU dtype casts,
a library primitive.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)

# Tie window of the parity rule: a point is a tie point when its fp64 top-2 distance gap
# is below TIE_TAU * (||x||^2 + max_k ||c_k||^2).
TIE_TAU = 1e-4


def lib():
    """Load (building first if needed) the compiled oracle.  FK_ORACLE_LIB, when set,
    names another build of the same sources to load instead: the mutation test points the
    pins at deliberately broken copies with it."""
    global _lib
    if _lib is None:
        path = os.environ.get("FK_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        L.orc_max_threads.restype = ctypes.c_int
        L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_normalize_rows.argtypes = [_dp, ctypes.c_int64, ctypes.c_int]
        L.orc_assign.argtypes = [_dp, ctypes.c_int64, ctypes.c_int, _dp, ctypes.c_int,
                                 _ip, _dp, _dp]
        L.orc_objective.argtypes = [_dp, ctypes.c_int64, ctypes.c_int, _dp, _ip]
        L.orc_objective.restype = ctypes.c_double
        L.orc_csr.argtypes = [_ip, ctypes.c_int64, ctypes.c_int, _ip, _ip, _ip]
        L.orc_csr.restype = ctypes.c_int
        L.orc_update.argtypes = [_dp, ctypes.c_int64, ctypes.c_int, _ip, _dp,
                                 ctypes.c_int, _dp]
        L.orc_ivf_search.argtypes = [_dp, ctypes.c_int64, ctypes.c_int, _dp, ctypes.c_int,
                                     _dp, ctypes.c_int64, _ip, ctypes.c_int, ctypes.c_int,
                                     _ip, _ip, _dp]
        L.orc_ivf_search.restype = ctypes.c_int
        _lib = L
    return _lib


def threads() -> int:
    return lib().orc_max_threads()


def set_threads(n: int) -> None:
    """Threads for the oracle's parallel per-point loops (its results do not depend on
    the count)."""
    lib().orc_set_threads(int(n))


def _f64(a) -> np.ndarray:
    """Exact widening of fp32 / bf16 / fp64 data (numpy or torch) to a C-contiguous fp64
    array."""
    if hasattr(a, "detach"):  # torch tensor (CPU): bf16 has no numpy dtype
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, p):
    return a.ctypes.data_as(p)


def normalize_rows(X) -> np.ndarray:
    """Return X / ||x_i|| row by row in fp64 (zero-norm rows divided by 1)."""
    Y = _f64(X).copy()
    n, d = Y.shape
    lib().orc_normalize_rows(_ptr(Y, _dp), n, d)
    return Y


def assign(X, C):
    """Labels (first-occurrence argmin of the squared L2 distance, difference form, fp64),
    the minimum distance and the second-smallest distance of every point."""
    X = _f64(X)
    C = _f64(C)
    n, d = X.shape
    K = C.shape[0]
    assert C.shape[1] == d and K >= 1
    labels = np.empty(n, dtype=np.int32)
    dmin = np.empty(n, dtype=np.float64)
    d2nd = np.empty(n, dtype=np.float64)
    lib().orc_assign(_ptr(X, _dp), n, d, _ptr(C, _dp), K, _ptr(labels, _ip),
                     _ptr(dmin, _dp), _ptr(d2nd, _dp))
    return labels, dmin, d2nd


def objective(X, C, labels) -> float:
    X = _f64(X)
    C = _f64(C)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    n, d = X.shape
    return lib().orc_objective(_ptr(X, _dp), n, d, _ptr(C, _dp), _ptr(labels, _ip))


def csr(labels, K: int):
    """counts[K], offsets[K+1] and the stable permutation sorted by cluster id."""
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    n = labels.shape[0]
    counts = np.empty(K, dtype=np.int32)
    offsets = np.empty(K + 1, dtype=np.int32)
    perm = np.empty(max(n, 1), dtype=np.int32)
    rc = lib().orc_csr(_ptr(labels, _ip), n, K, _ptr(counts, _ip), _ptr(offsets, _ip),
                       _ptr(perm, _ip))
    if rc != 0:
        raise ValueError("label outside [0, K)")
    return counts, offsets, perm[:n]


def update(X, labels, C_old) -> np.ndarray:
    """Mean of each cluster's points in fp64; empty clusters keep C_old."""
    X = _f64(X)
    C_old = _f64(C_old)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    n, d = X.shape
    K = C_old.shape[0]
    if n and (labels.min() < 0 or labels.max() >= K):
        raise ValueError("label outside [0, K)")
    C_new = np.empty_like(C_old)
    lib().orc_update(_ptr(X, _dp), n, d, _ptr(labels, _ip), _ptr(C_old, _dp), K,
                     _ptr(C_new, _dp))
    return C_new


def ivf_search(Q, C, X, labels, nprobe: int, k: int):
    """IVF-Flat search in fp64 (ivf_search_oracle.c): for every query, the nprobe cells
    with the nearest centroids (ascending (distance, cell)), then the k nearest points of
    those cells (ascending (distance, point index); missing slots -1 / +inf).

    Returns (probes int32 [nq, nprobe], ids int32 [nq, k], dist fp64 [nq, k]).  `labels`
    gives every point's cell; X is in the original point order.
    """
    Q = _f64(Q)
    C = _f64(C)
    X = _f64(X)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    nq, d = Q.shape
    nlist = C.shape[0]
    n = X.shape[0]
    assert C.shape[1] == d and X.shape[1] == d and labels.shape == (n,)
    probes = np.empty((nq, nprobe), dtype=np.int32)
    ids = np.empty((nq, k), dtype=np.int32)
    dist = np.empty((nq, k), dtype=np.float64)
    rc = lib().orc_ivf_search(_ptr(Q, _dp), nq, d, _ptr(C, _dp), nlist, _ptr(X, _dp), n,
                              _ptr(labels, _ip), nprobe, k, _ptr(probes, _ip),
                              _ptr(ids, _ip), _ptr(dist, _dp))
    if rc != 0:
        raise ValueError("ivf_search: label outside [0, nlist) or nprobe/k out of range")
    return probes, ids, dist


def tie_mask(X, C, dmin, d2nd, tau: float = TIE_TAU) -> np.ndarray:
    """True where the fp64 top-2 gap is below tau * (||x_i||^2 + max_k ||c_k||^2)."""
    X = _f64(X)
    C = _f64(C)
    s = (X * X).sum(axis=1) + (C * C).sum(axis=1).max()
    return (d2nd - dmin) < tau * s


def round_f32(A) -> np.ndarray:
    """Round fp64 values to fp32 (round to nearest even), returned widened to fp64."""
    return np.asarray(A, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(A) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest even, via torch's CPU cast), returned
    widened to fp64."""
    import torch
    t = torch.from_numpy(np.asarray(A, dtype=np.float32).copy())
    return t.to(torch.bfloat16).double().numpy()


def lloyd(X, C0, niter: int, metric: str = "l2", precision: str = "f32"):
    """Run `niter` exact Lloyd iterations from C0 and record every step.

    precision "f32": the centroids are kept as fp32 between iterations (each new fp64
    mean is rounded to fp32), the storage type of the GPU's centroids.
    precision "bf16": the fp32 master is kept as above and the assignment sees its bf16
    rounding (the MMA operand of the bf16 data path).
    metric "cosine": X and C0 are L2-normalised first (zero norm -> divide by 1).

    Returns a dict of per-iteration lists: C_used (centroids the assignment saw),
    labels, ties (tie-point mask), J (objective of the labels against C_used),
    counts/offsets/perm, C_next (fp32 master after the update), plus X (the fp64 points
    actually clustered).
    """
    if metric not in ("l2", "cosine"):
        raise ValueError(metric)
    if precision not in ("f32", "bf16"):
        raise ValueError(precision)
    Xd = _f64(X)
    Cm = _f64(C0)
    if metric == "cosine":
        Xd = normalize_rows(Xd)
        Cm = normalize_rows(Cm)
    Cm = round_f32(Cm)
    K = Cm.shape[0]
    out = {k: [] for k in ("C_used", "labels", "ties", "J", "counts", "offsets",
                           "perm", "C_next", "dmin", "d2nd")}
    out["X"] = Xd
    for _ in range(niter):
        Cu = round_bf16(Cm) if precision == "bf16" else Cm
        labels, dmin, d2nd = assign(Xd, Cu)
        counts, offsets, perm = csr(labels, K)
        J = objective(Xd, Cu, labels)
        Cnew = round_f32(update(Xd, labels, Cm))
        for k, v in (("C_used", Cu), ("labels", labels), ("J", J), ("counts", counts),
                     ("offsets", offsets), ("perm", perm), ("C_next", Cnew),
                     ("dmin", dmin), ("d2nd", d2nd),
                     ("ties", tie_mask(Xd, Cu, dmin, d2nd))):
            out[k].append(v)
        Cm = Cnew
    return out
