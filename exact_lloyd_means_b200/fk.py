"""ctypes binding of libfk.so, the C-ABI CUDA library (include/fk.h).

Argument marshalling only: every function here checks tensor dtypes, shapes, devices and
contiguity, passes raw device pointers, sizes and the current CUDA stream to the function
of the same name in libfk.so, and raises FkError on a non-zero status.  All arithmetic
runs in the library's sm_100a kernels; PyTorch only provides device memory and streams.
Importing this module fails loudly when libfk.so has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfk.so")

FK_OK, FK_ERR_INVALID_ARG, FK_ERR_UNSUPPORTED, FK_ERR_WORKSPACE = 0, 1, 2, 3
FK_ERR_CUDA, FK_ERR_TIMEOUT, FK_ERR_DEVICE = 4, 5, 6
FK_F32, FK_BF16, FK_BF16X2 = 0, 1, 2
FK_L2, FK_COSINE = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python -c 'import __graft_entry__; __graft_entry__.build()' or "
        "python exact_lloyd_means_b200/build.py)")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class FkTiming(ctypes.Structure):
    _fields_ = [("ms_setup", ctypes.c_double), ("ms_prep", ctypes.c_double),
                ("ms_assign", ctypes.c_double), ("ms_sort", ctypes.c_double),
                ("ms_update", ctypes.c_double), ("iterations", ctypes.c_int),
                ("launches", ctypes.c_int), ("ms_assign_mma", ctypes.c_double),
                ("screened", ctypes.c_int), ("empty_clusters", ctypes.c_int),
                ("max_cluster", ctypes.c_int), ("fallback_rows", ctypes.c_int),
                ("kernel_only", ctypes.c_int), ("mma_timed", ctypes.c_int)]


class FkSearchTiming(ctypes.Structure):
    _fields_ = [("ms_coarse", ctypes.c_double), ("ms_sort", ctypes.c_double),
                ("ms_fine", ctypes.c_double), ("ms_merge", ctypes.c_double),
                ("screened_coarse", ctypes.c_int), ("screened_fine", ctypes.c_int),
                ("fallback_queries", ctypes.c_int)]


FK_SEARCH_FP64_COARSE, FK_SEARCH_FP64_FINE = 1, 2


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_lib.fk_status_string.argtypes = [ctypes.c_int]
_lib.fk_status_string.restype = ctypes.c_char_p
_sig("fk_version", [])
_sig("fk_launch_count", [], ctypes.c_int64)
_sig("fk_workspace_size", [_i64, _int, _int, _int, _int, ctypes.POINTER(_sz)])
_sig("fk_normalize_rows", [_vp, _vp, _i64, _int, _vp])
_sig("fk_split_points", [_vp, _i64, _int, _vp, _vp])
_sig("fk_centroid_norms", [_vp, _int, _int, _int, _vp, _vp])
_sig("fk_assign", [_vp, _int, _i64, _int, _vp, _int, _vp, _vp, _vp, _sz, _vp])
_sig("fk_assign_split", [_vp, _vp, _i64, _int, _vp, _int, _vp, _vp, _vp, _sz, _vp])
_sig("fk_update", [_vp, _int, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                   _sz, _vp])
_sig("fk_lloyd", [_vp, _int, _i64, _int, _int, _int, _int, _vp, _vp, _vp, _vp,
                  ctypes.POINTER(ctypes.c_double), ctypes.POINTER(FkTiming), _vp, _sz, _vp])
_sig("fk_get_device_error", [_vp, _sz, ctypes.POINTER(ctypes.c_int), _vp])
_sig("fk_selftest_timeout", [_vp, _sz, ctypes.c_uint64, _vp])
_sig("fk_assign_noalloc", [_vp, _int, _i64, _int, _vp, _int, _vp, _vp])
_sig("fk_update_partial", [_vp, _int, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                           _vp])
_sig("fk_finalize_shards", [_vp, _vp, _vp, _int, _int, _int, _vp, _vp, _vp, _vp, _vp])
_sig("fk_ivf_lists", [_vp, _int, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("fk_lloyd_streamed", [_vp, _int, _i64, _int, _int, _int, _int, _vp, _vp,
                           ctypes.POINTER(ctypes.c_double), _i64, _vp, _sz, _vp])
_sig("fk_streamed_workspace_size", [_i64, _int, _int, _int, _int, ctypes.POINTER(_sz)])
_sig("fk_ivf_norms", [_vp, _i64, _int, _vp, _vp])
_sig("fk_ivf_search_workspace_size", [_i64, _int, _int, _i64, _int, _int, ctypes.POINTER(_sz)])
_sig("fk_ivf_search", [_vp, _i64, _int, _vp, _int, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _int,
                       _int, _int, _vp, _vp, _vp, _vp, _sz, ctypes.POINTER(FkSearchTiming),
                       _vp])
_sig("fk_ivf_radii", [_vp, _int, _vp, _vp, _int, _vp, _vp])

EXPORTED = ["fk_status_string", "fk_version", "fk_workspace_size", "fk_normalize_rows",
            "fk_centroid_norms", "fk_assign", "fk_update", "fk_lloyd",
            "fk_get_device_error", "fk_selftest_timeout", "fk_assign_noalloc",
            "fk_update_partial", "fk_finalize_shards", "fk_split_points",
            "fk_launch_count", "fk_ivf_lists", "fk_lloyd_streamed",
            "fk_streamed_workspace_size", "fk_ivf_norms", "fk_ivf_search_workspace_size",
            "fk_ivf_search", "fk_ivf_radii", "fk_assign_split"]

# Bytes of the static device array fk_assign_noalloc takes its scratch from.
NOALLOC_SCRATCH_BYTES = 8 << 20


class FkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.fk_status_string(status).decode()}")


def _check(status: int, where: str):
    if status != FK_OK:
        raise FkError(status, where)


def status_string(status: int) -> str:
    return _lib.fk_status_string(status).decode()


def version() -> int:
    return _lib.fk_version()


def launch_count() -> int:
    """Kernels libfk has launched from this host thread so far."""
    return _lib.fk_launch_count()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return FK_F32
    if t.dtype == torch.bfloat16:
        return FK_BF16
    raise TypeError(f"unsupported point dtype {t.dtype}")


def _metric_code(metric) -> int:
    if metric in ("l2", FK_L2):
        return FK_L2
    if metric in ("cosine", FK_COSINE):
        return FK_COSINE
    raise ValueError(metric)


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _opt(t, name, dtype=None, shape=None):
    return None if t is None else _dev(t, name, dtype, shape)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def fk_workspace_size(N: int, d: int, K: int, dtype=torch.float32, metric="l2") -> int:
    code = dtype if isinstance(dtype, int) else (FK_F32 if dtype == torch.float32 else
                                                 FK_BF16 if dtype == torch.bfloat16 else -1)
    out = _sz(0)
    _check(_lib.fk_workspace_size(N, d, K, code, _metric_code(metric), ctypes.byref(out)),
           "fk_workspace_size")
    return out.value


def workspace(N: int, d: int, K: int, dtype=torch.float32, metric="l2", device="cuda"):
    """A zeroed uint8 workspace tensor of the size libfk asks for (256-byte aligned by the
    CUDA caching allocator)."""
    nbytes = fk_workspace_size(N, d, K, dtype, metric)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
    if ws.data_ptr() % 256:
        raise RuntimeError("workspace is not 256-byte aligned")
    return ws


def fk_normalize_rows(X_in: torch.Tensor, X_out: torch.Tensor, stream=None):
    N, d = X_in.shape
    _check(_lib.fk_normalize_rows(_dev(X_in, "X_in", torch.float32),
                                  _dev(X_out, "X_out", torch.float32, (N, d)), N, d,
                                  _stream(stream)), "fk_normalize_rows")


def fk_centroid_norms(C: torch.Tensor, cn: torch.Tensor, dtype=torch.float32, stream=None):
    K, d = C.shape
    code = FK_F32 if dtype == torch.float32 else FK_BF16
    _check(_lib.fk_centroid_norms(_dev(C, "C", torch.float32), K, d, code,
                                  _dev(cn, "cn", torch.float32, (K,)), _stream(stream)),
           "fk_centroid_norms")


class SplitPoints:
    """fp32 points already split by fk_split_points: one buffer holding the bf16 hi/lo
    planes ([2, N, d_p] bf16, d_p = d rounded up to 64) followed by ||x||^2 per row ([N]
    fp32).  fk_assign takes it in place of the fp32 tensor and skips its per-call split:
    with the fp32 rows it was made from (`source`) through fk_assign_split, else as
    FK_BF16X2 planes alone."""

    def __init__(self, buf: torch.Tensor, N: int, d: int, source: torch.Tensor | None = None):
        dp = (d + 63) // 64 * 64
        self.buf, self.N, self.d, self.source = buf, N, d, source
        self.planes = buf[:2 * N * dp].view(2, N, dp)
        self.norms = buf[2 * N * dp:].view(torch.float32)

    @property
    def shape(self):
        return (self.N, self.d)


def split_points_buffer(N: int, d: int, device="cuda") -> torch.Tensor:
    """A buffer of the size fk_split_points writes (4 N d_p + 4 N bytes, as bf16)."""
    dp = (d + 63) // 64 * 64
    return torch.empty(2 * N * dp + 2 * N, dtype=torch.bfloat16, device=device)


def fk_split_points(X: torch.Tensor, out: torch.Tensor | None = None,
                    stream=None) -> SplitPoints:
    """Split fp32 points into bf16 hi/lo planes (and their squared norms) once; `out`
    (from split_points_buffer) is allocated when not given."""
    N, d = X.shape
    dp = (d + 63) // 64 * 64
    if out is None:
        out = split_points_buffer(N, d, X.device)
    _check(_lib.fk_split_points(_dev(X, "X", torch.float32), N, d,
                                _dev(out, "out", torch.bfloat16, (2 * N * dp + 2 * N,)),
                                _stream(stream)), "fk_split_points")
    return SplitPoints(out, N, d, source=X)


def fk_assign(X, C: torch.Tensor, labels: torch.Tensor, ws: torch.Tensor,
              mind: torch.Tensor | None = None, stream=None):
    N, d = X.shape
    K = C.shape[0]
    if isinstance(X, SplitPoints) and X.source is not None:
        _check(_lib.fk_assign_split(_dev(X.source, "X.source", torch.float32, (N, d)),
                                    _dev(X.buf, "X.buf", torch.bfloat16), N, d,
                                    _dev(C, "C", torch.float32, (K, d)), K,
                                    _dev(labels, "labels", torch.int32, (N,)),
                                    _opt(mind, "mind", torch.float32, (N,)),
                                    _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
               "fk_assign_split")
        return
    if isinstance(X, SplitPoints):
        xptr, code = _dev(X.buf, "X.buf", torch.bfloat16), FK_BF16X2
    else:
        xptr, code = _dev(X, "X"), _dtype_code(X)
    _check(_lib.fk_assign(xptr, code, N, d,
                          _dev(C, "C", torch.float32, (K, d)), K,
                          _dev(labels, "labels", torch.int32, (N,)),
                          _opt(mind, "mind", torch.float32, (N,)),
                          _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "fk_assign")


def fk_update(X: torch.Tensor, labels: torch.Tensor, C_old: torch.Tensor,
              C_new: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
              ws: torch.Tensor, perm: torch.Tensor | None = None,
              objective: torch.Tensor | None = None, stream=None):
    N, d = X.shape
    K = C_old.shape[0]
    _check(_lib.fk_update(_dev(X, "X"), _dtype_code(X), N, d, K,
                          _dev(labels, "labels", torch.int32, (N,)),
                          _dev(C_old, "C_old", torch.float32, (K, d)),
                          _dev(C_new, "C_new", torch.float32, (K, d)),
                          _dev(counts, "counts", torch.int32, (K,)),
                          _dev(offsets, "offsets", torch.int32, (K + 1,)),
                          _opt(perm, "perm", torch.int32, (N,)),
                          _opt(objective, "objective", torch.float64, (1,)),
                          _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "fk_update")


def fk_lloyd(X: torch.Tensor, C: torch.Tensor, niter: int, labels: torch.Tensor,
             ws: torch.Tensor, metric="l2", counts: torch.Tensor | None = None,
             offsets: torch.Tensor | None = None, timing: bool | str = False, stream=None):
    """Run niter iterations in place on C.  Returns (objectives list, timing dict|None).
    timing: True times every phase; "kernel" only the assignment's tensor-core kernel of
    every iteration; "kernel_last" only that of the last iteration."""
    N, d = X.shape
    K = C.shape[0]
    obj = (ctypes.c_double * max(niter, 1))()
    tm = FkTiming() if timing else None
    if tm is not None:
        tm.kernel_only = {"kernel": 1, "kernel_last": 2}.get(timing, 0)
    _check(_lib.fk_lloyd(_dev(X, "X"), _dtype_code(X), N, d, K, _metric_code(metric), niter,
                         _dev(C, "C", torch.float32, (K, d)),
                         _dev(labels, "labels", torch.int32, (N,)),
                         _opt(counts, "counts", torch.int32, (K,)),
                         _opt(offsets, "offsets", torch.int32, (K + 1,)), obj,
                         ctypes.byref(tm) if tm is not None else None,
                         _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "fk_lloyd")
    t = None
    if tm is not None:
        t = {f: getattr(tm, f) for f, _ in FkTiming._fields_}
    return [obj[i] for i in range(niter)], t


def fk_get_device_error(ws: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int(0)
    _check(_lib.fk_get_device_error(_dev(ws, "ws", torch.uint8), ws.numel(),
                                    ctypes.byref(code), _stream(stream)),
           "fk_get_device_error")
    return code.value


def fk_selftest_timeout(ws: torch.Tensor, limit_ns: int, stream=None):
    _check(_lib.fk_selftest_timeout(_dev(ws, "ws", torch.uint8), ws.numel(), int(limit_ns),
                                    _stream(stream)), "fk_selftest_timeout")


def fk_assign_noalloc(X: torch.Tensor, C: torch.Tensor, labels: torch.Tensor, stream=None):
    """fk_assign without a workspace: scratch comes from the library's static device array
    (for callers that cannot allocate device memory).  Synchronous."""
    N, d = X.shape
    K = C.shape[0]
    _check(_lib.fk_assign_noalloc(_dev(X, "X"), _dtype_code(X), N, d,
                                  _dev(C, "C", torch.float32, (K, d)), K,
                                  _dev(labels, "labels", torch.int32, (N,)), _stream(stream)),
           "fk_assign_noalloc")


def fk_update_partial(X: torch.Tensor, labels: torch.Tensor, C_old: torch.Tensor,
                      sums: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
                      ws: torch.Tensor, objective: torch.Tensor | None = None, stream=None):
    """One shard's fp64 per-cluster sums, counts, CSR offsets and objective."""
    N, d = X.shape
    K = C_old.shape[0]
    _check(_lib.fk_update_partial(_dev(X, "X"), _dtype_code(X), N, d, K,
                                  _dev(labels, "labels", torch.int32, (N,)),
                                  _dev(C_old, "C_old", torch.float32, (K, d)),
                                  _dev(sums, "sums", torch.float64, (K, d)),
                                  _dev(counts, "counts", torch.int32, (K,)),
                                  _dev(offsets, "offsets", torch.int32, (K + 1,)),
                                  _opt(objective, "objective", torch.float64, (1,)),
                                  _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "fk_update_partial")


def fk_finalize_shards(sums: torch.Tensor, counts_w: torch.Tensor, C_old: torch.Tensor,
                       C_new: torch.Tensor, objectives_w: torch.Tensor | None = None,
                       counts: torch.Tensor | None = None,
                       objective: torch.Tensor | None = None, stream=None):
    """Combine W gathered shards ([W][K][d] sums, [W][K] int64 counts) in shard order."""
    W, K, d = sums.shape
    _check(_lib.fk_finalize_shards(_dev(sums, "sums", torch.float64),
                                   _dev(counts_w, "counts_w", torch.int64, (W, K)),
                                   _opt(objectives_w, "objectives_w", torch.float64, (W,)),
                                   W, K, d, _dev(C_old, "C_old", torch.float32, (K, d)),
                                   _dev(C_new, "C_new", torch.float32, (K, d)),
                                   _opt(counts, "counts", torch.int64, (K,)),
                                   _opt(objective, "objective", torch.float64, (1,)),
                                   _stream(stream)), "fk_finalize_shards")


def fk_ivf_lists(X: torch.Tensor, labels: torch.Tensor, K: int, offsets: torch.Tensor,
                 row_ids: torch.Tensor, ws: torch.Tensor, X_lists: torch.Tensor | None = None,
                 stream=None):
    """Inverted lists of a clustering: CSR offsets per cell, row ids in cell order and
    (optionally) the points gathered in that order."""
    N, d = X.shape
    _check(_lib.fk_ivf_lists(_dev(X, "X"), _dtype_code(X), N, d, K,
                             _dev(labels, "labels", torch.int32, (N,)),
                             _dev(offsets, "offsets", torch.int32, (K + 1,)),
                             _dev(row_ids, "row_ids", torch.int32, (N,)),
                             _opt(X_lists, "X_lists", X.dtype, (N, d)),
                             _dev(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "fk_ivf_lists")


def streamed_workspace(chunk_rows: int, d: int, K: int, dtype=torch.float32, metric="l2",
                       device="cuda"):
    """A workspace tensor for fk_lloyd_streamed with this chunk size."""
    code = FK_F32 if dtype == torch.float32 else FK_BF16
    out = _sz(0)
    _check(_lib.fk_streamed_workspace_size(chunk_rows, d, K, code, _metric_code(metric),
                                           ctypes.byref(out)), "fk_streamed_workspace_size")
    return torch.zeros(out.value, dtype=torch.uint8, device=device)


def fk_lloyd_streamed(X_host: torch.Tensor, C: torch.Tensor, niter: int, ws: torch.Tensor,
                      chunk_rows: int, metric="l2", labels: torch.Tensor | None = None,
                      stream=None):
    """Lloyd's iterations over points in host memory (pin them for overlap), streamed in
    chunks.  C (device) is updated in place; returns the objectives; `labels` (host int32)
    receives the last iteration's labels."""
    if X_host.device.type != "cpu" or not X_host.is_contiguous():
        raise ValueError("X_host must be a contiguous CPU tensor")
    N, d = X_host.shape
    K = C.shape[0]
    obj = (ctypes.c_double * max(niter, 1))()
    lab_ptr = None
    if labels is not None:
        if labels.device.type != "cpu" or labels.dtype != torch.int32 or \
                tuple(labels.shape) != (N,) or not labels.is_contiguous():
            raise ValueError("labels must be a contiguous CPU int32 tensor of N entries")
        lab_ptr = labels.data_ptr()
    _check(_lib.fk_lloyd_streamed(X_host.data_ptr(), _dtype_code(X_host), N, d, K,
                                  _metric_code(metric), niter,
                                  _dev(C, "C", torch.float32, (K, d)), lab_ptr, obj,
                                  chunk_rows, _dev(ws, "ws", torch.uint8), ws.numel(),
                                  _stream(stream)), "fk_lloyd_streamed")
    return [obj[i] for i in range(niter)]


def fk_ivf_norms(V: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp64 squared norms of the fp32 rows of V (for fk_ivf_search: V = X_lists)."""
    n, d = V.shape
    if out is None:
        out = torch.empty(n, dtype=torch.float64, device=V.device)
    _check(_lib.fk_ivf_norms(_dev(V, "V", torch.float32), n, d,
                             _dev(out, "out", torch.float64, (n,)), _stream(stream)),
           "fk_ivf_norms")
    return out


def ivf_search_workspace(nq: int, d: int, nlist: int, N: int, nprobe: int, k: int,
                         device="cuda") -> torch.Tensor:
    out = _sz(0)
    _check(_lib.fk_ivf_search_workspace_size(nq, d, nlist, N, nprobe, k, ctypes.byref(out)),
           "fk_ivf_search_workspace_size")
    return torch.empty(out.value, dtype=torch.uint8, device=device)


def fk_ivf_search(Q: torch.Tensor, C: torch.Tensor, X_lists: torch.Tensor,
                  X_norms: torch.Tensor, offsets: torch.Tensor, row_ids: torch.Tensor,
                  nprobe: int, k: int, ws: torch.Tensor | None = None,
                  distances: torch.Tensor | None = None, ids: torch.Tensor | None = None,
                  probes: torch.Tensor | None = None, timing: dict | None = None,
                  fp64_coarse: bool = False, X_planes=None, fp64_fine: bool = False,
                  cell_radius: torch.Tensor | None = None, stream=None):
    """IVF-Flat search: returns (distances fp32 [nq, k], ids int32 [nq, k]); `probes`
    (int32 [nq, nprobe]) receives the probed cells when given.  A `timing` dict receives
    the per-phase device times in ms (the call then synchronises its stream).
    X_planes: fk_split_points of X_lists (a SplitPoints or its buffer), which enables the
    tensor-core fine pass; cell_radius: fk_ivf_radii of the index, which lets that pass
    skip the points that cannot be among a query's k nearest.  fp64_coarse / fp64_fine compute every coarse / fine distance
    in fp64 (FK_SEARCH_FP64_COARSE / FK_SEARCH_FP64_FINE)."""
    nq, d = Q.shape
    nlist = C.shape[0]
    N = X_lists.shape[0]
    if ws is None:
        ws = ivf_search_workspace(nq, d, nlist, N, nprobe, k, Q.device)
    if distances is None:
        distances = torch.empty((nq, k), dtype=torch.float32, device=Q.device)
    if ids is None:
        ids = torch.empty((nq, k), dtype=torch.int32, device=Q.device)
    tm = FkSearchTiming() if timing is not None else None
    if isinstance(X_planes, SplitPoints):
        if X_planes.N != N or X_planes.d != d:
            raise ValueError("X_planes must split X_lists")
        X_planes = X_planes.buf
    dp = (d + 63) // 64 * 64
    planes_ptr = _opt(X_planes, "X_planes", torch.bfloat16, (2 * N * dp + 2 * N,))
    flags = (FK_SEARCH_FP64_COARSE if fp64_coarse else 0) | \
        (FK_SEARCH_FP64_FINE if fp64_fine else 0)
    _check(_lib.fk_ivf_search(_dev(Q, "Q", torch.float32), nq, d,
                              _dev(C, "C", torch.float32, (nlist, d)), nlist,
                              _dev(X_lists, "X_lists", torch.float32, (N, d)),
                              _dev(X_norms, "X_norms", torch.float64, (N,)), planes_ptr,
                              _opt(cell_radius, "cell_radius", torch.float32, (nlist,)),
                              _dev(offsets, "offsets", torch.int32, (nlist + 1,)),
                              _dev(row_ids, "row_ids", torch.int32, (N,)), N, nprobe, k,
                              flags,
                              _dev(distances, "distances", torch.float32, (nq, k)),
                              _dev(ids, "ids", torch.int32, (nq, k)),
                              _opt(probes, "probes", torch.int32, (nq, nprobe)),
                              _dev(ws, "ws", torch.uint8), ws.numel(),
                              ctypes.byref(tm) if tm is not None else None, _stream(stream)),
           "fk_ivf_search")
    if tm is not None:
        timing.update({f: getattr(tm, f) for f, _ in FkSearchTiming._fields_})
    return distances, ids


def fk_ivf_radii(C: torch.Tensor, X_lists: torch.Tensor, offsets: torch.Tensor,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Per cell, an upper bound on the distance of its points to its centroid."""
    nlist, d = C.shape
    if out is None:
        out = torch.empty(nlist, dtype=torch.float32, device=C.device)
    _check(_lib.fk_ivf_radii(_dev(C, "C", torch.float32), nlist,
                             _dev(X_lists, "X_lists", torch.float32),
                             _dev(offsets, "offsets", torch.int32, (nlist + 1,)), d,
                             _dev(out, "out", torch.float32, (nlist,)), _stream(stream)),
           "fk_ivf_radii")
    return out


class IvfFlatIndex:
    """An IVF-Flat index: centroids, cell-contiguous points with their original ids, CSR
    offsets, fp64 norms, and for the tensor-core fine pass the bf16 planes of the points
    and the cell radii.  `build` and `search` only sequence libfk calls
    (fk_normalize_rows, fk_lloyd, fk_ivf_lists, fk_ivf_norms, fk_split_points,
    fk_ivf_radii, fk_ivf_search)."""

    def __init__(self, C, X_lists, X_norms, offsets, row_ids, metric="l2", X_planes=None,
                 cell_radius=None):
        self.C, self.X_lists, self.X_norms = C, X_lists, X_norms
        self.offsets, self.row_ids, self.metric = offsets, row_ids, metric
        self.X_planes, self.cell_radius = X_planes, cell_radius

    @classmethod
    def build(cls, X: torch.Tensor, C0: torch.Tensor, niter: int, metric="l2", stream=None):
        """Cluster X (fp32, N x d) from the initial centroids C0 with niter Lloyd iterations
        and lay out the cells.  metric "cosine" L2-normalises X and C0 first."""
        N, d = X.shape
        K = C0.shape[0]
        C = C0.clone()
        if metric == "cosine":
            Xn = torch.empty_like(X)
            fk_normalize_rows(X, Xn, stream)
            fk_normalize_rows(C0, C, stream)
            X = Xn
        labels = torch.empty(N, dtype=torch.int32, device=X.device)
        ws = workspace(N, d, K, X.dtype, "l2", X.device)
        fk_lloyd(X, C, niter, labels, ws, "l2", stream=stream)
        offsets = torch.empty(K + 1, dtype=torch.int32, device=X.device)
        row_ids = torch.empty(N, dtype=torch.int32, device=X.device)
        X_lists = torch.empty_like(X)
        fk_ivf_lists(X, labels, K, offsets, row_ids, ws, X_lists, stream)
        del ws
        X_norms = fk_ivf_norms(X_lists, stream=stream)
        X_planes = fk_split_points(X_lists, stream=stream)
        radius = fk_ivf_radii(C, X_lists, offsets, stream=stream)
        return cls(C, X_lists, X_norms, offsets, row_ids, metric, X_planes, radius)

    def search(self, Q: torch.Tensor, k: int, nprobe: int, ws=None, distances=None,
               ids=None, probes=None, timing=None, fp64_coarse=False, fp64_fine=False,
               stream=None):
        """(distances, ids) of the k nearest indexed points of every query, probing nprobe
        cells; a cosine index L2-normalises the queries first."""
        if self.metric == "cosine":
            Qn = torch.empty_like(Q)
            fk_normalize_rows(Q, Qn, stream)
            Q = Qn
        return fk_ivf_search(Q, self.C, self.X_lists, self.X_norms, self.offsets,
                             self.row_ids, nprobe, k, ws=ws, distances=distances, ids=ids,
                             probes=probes, timing=timing, fp64_coarse=fp64_coarse,
                             X_planes=self.X_planes, fp64_fine=fp64_fine,
                             cell_radius=self.cell_radius, stream=stream)
