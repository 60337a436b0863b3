"""Exact Lloyd's k-means on B200 (sm_100a): a C-ABI CUDA library (libfk.so, declared in
include/fk.h) plus a thin Python binding in the `fk` submodule.

    from exact_lloyd_means_b200 import fk
    ws = fk.workspace(N, d, K, X.dtype, "l2")
    objs, _ = fk.fk_lloyd(X, C, niter, labels, ws)

The package itself imports nothing, so building the library (build.py) does not need it.
"""
