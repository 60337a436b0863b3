"""GPU parity of fk_ivf_search (IVF-Flat search) against the fp64 oracle.

The index is laid out on the GPU by fk_ivf_lists / fk_ivf_norms from labels that come from
the generator or the oracle, never from the GPU.  Parity rule: probes and ids equal the
oracle's; where a row differs, the GPU's selection must be an equally valid one in fp64
(its oracle distances equal the oracle's sorted list within NEAR of the squared norms: the
rounding of the fp64 expansion the kernels evaluate), and such rows must stay rare.
Distances are the fp32 rounding of an fp64 value: within 2^-23 relative (plus NEAR of the
norms, absolute) of the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import gaussian_mixture, init_indices, mixture_queries

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
NEAR = 1e-12  # relative to ||q||^2 + max ||x||^2


def fk():
    from exact_lloyd_means_b200 import fk as m
    return m


def _index(X, labels, nlist):
    m = fk()
    N, d = X.shape
    Xg = X.to(DEV)
    offsets = torch.empty(nlist + 1, dtype=torch.int32, device=DEV)
    row_ids = torch.empty(N, dtype=torch.int32, device=DEV)
    X_lists = torch.empty_like(Xg)
    ws = m.workspace(N, d, nlist, Xg.dtype, "l2")
    m.fk_ivf_lists(Xg, torch.as_tensor(labels).to(DEV), nlist, offsets, row_ids, ws,
                   X_lists=X_lists)
    assert m.fk_get_device_error(ws) == m.FK_OK
    return X_lists, m.fk_ivf_norms(X_lists), offsets, row_ids, m.fk_split_points(X_lists)


def _search(Q, C, idx, nprobe, k, fp64_coarse=False, fp64_fine=False, timing=None,
            radius=True):
    m = fk()
    X_lists, X_norms, offsets, row_ids, planes = idx
    nq = Q.shape[0]
    Cd = C.to(DEV)
    rad = m.fk_ivf_radii(Cd, X_lists, offsets) if radius else None
    probes = torch.full((nq, nprobe), -7, dtype=torch.int32, device=DEV)
    dist, ids = m.fk_ivf_search(Q.to(DEV), Cd, X_lists, X_norms, offsets, row_ids,
                                nprobe, k, probes=probes, fp64_coarse=fp64_coarse,
                                X_planes=planes, fp64_fine=fp64_fine, timing=timing,
                                cell_radius=rad)
    torch.cuda.synchronize()
    return probes.cpu().numpy(), ids.cpu().numpy(), dist.cpu().numpy()


# (fp64 coarse, fp64 fine, cell radii)
MODES = [(False, False, True), (True, False, True), (False, True, True), (True, True, True),
         (False, False, False)]


def _sqd(A, B):
    """fp64 difference-form squared distances of the rows of A to the rows of B."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return ((A[:, None, :] - B[None, :, :]) ** 2).sum(axis=2)


def check_search(Q, C, X, got, ref, max_bad_frac=0.01):
    probes, ids, dist = got
    rp, ri, rd = ref
    Q64, X64, C64 = (np.asarray(a, dtype=np.float64) for a in (Q, X, C))
    scale = (Q64 ** 2).sum(1) + max((X64 ** 2).sum(1).max(), (C64 ** 2).sum(1).max())
    bad = 0
    for r in np.nonzero((probes != rp).any(axis=1))[0]:
        bad += 1
        dc = _sqd(Q64[r:r + 1], C64)[0]
        assert np.allclose(np.sort(dc[probes[r]]), np.sort(dc[rp[r]]), rtol=0,
                           atol=NEAR * scale[r]), f"query {r}: probes {probes[r]} vs {rp[r]}"
    for r in np.nonzero((ids != ri).any(axis=1))[0]:
        bad += 1
        real = ids[r] >= 0
        assert (real == (ri[r] >= 0)).all(), f"query {r}: padding differs"
        dg = _sqd(Q64[r:r + 1], X64[ids[r][real]])[0]
        assert np.allclose(dg, rd[r][real], rtol=0, atol=NEAR * scale[r]), \
            f"query {r}: ids {ids[r]} vs {ri[r]}"
    assert bad <= max_bad_frac * len(Q64) + 0.5, f"{bad} rows differ"
    fin = np.isfinite(rd)
    assert np.array_equal(np.isfinite(dist), fin)
    assert np.array_equal(ids[~fin], np.full((~fin).sum(), -1))
    err = np.abs(dist[fin].astype(np.float64) - rd[fin])
    tol = 2.0 ** -23 * np.abs(rd[fin]) + NEAR * np.broadcast_to(scale[:, None], rd.shape)[fin]
    assert (err <= tol).all(), float((err - tol).max())
    return bad


CASES = [
    # N, d, nlist, nq, nprobe, k, weights, labels
    (20000, 64, 64, 100, 4, 10, "equal", "assign"),
    (30011, 100, 97, 77, 7, 32, "equal", "assign"),     # ragged d, nq and tiles
    (50000, 768, 256, 64, 16, 10, "equal", "assign"),   # the guide's d
    (4000, 128, 50, 33, 50, 5, "equal", "assign"),      # nprobe = nlist: exact kNN
    (2000, 16, 40, 40, 1, 1, "equal", "assign"),
    (60000, 32, 100, 300, 8, 10, "zipf", "comp"),       # cells of thousands, many items/cell
    (3000, 24, 300, 50, 3, 20, "equal", "comp"),        # tiny cells: padded lists
]


@pytest.mark.parametrize("N,d,nlist,nq,nprobe,k,weights,labels_from", CASES)
def test_ivf_search_matches_oracle(N, d, nlist, nq, nprobe, k, weights, labels_from):
    X, comp, _ = gaussian_mixture(N, d, nlist, centers="normal", sigma=0.4, weights=weights,
                                  seed=N + d)
    C = X[init_indices(N, nlist, N + d)].float().contiguous()
    if labels_from == "assign":
        labels, _, _ = oracle.assign(X, C)
    else:
        labels = comp.numpy().astype(np.int32)
    Q = mixture_queries(nq, d, nlist, centers="normal", sigma=0.4, weights=weights,
                        seed=N + d, stream=1)
    ref = oracle.ivf_search(Q, C, X, labels, nprobe, k)
    idx = _index(X, labels, nlist)
    for f64c, f64f, rad in MODES:
        tm = {}
        got = _search(Q, C, idx, nprobe, k, fp64_coarse=f64c, fp64_fine=f64f, timing=tm,
                      radius=rad)
        assert tm["screened_coarse"] == (0 if f64c else 1)
        assert tm["screened_fine"] == (0 if (f64f or k > 16) else 1)
        check_search(Q, C, X, got, ref)


def test_ivf_search_empty_cells_and_few_candidates():
    """Centroids with no points (probed and returning nothing) and fewer candidates than
    k: padded slots are -1 / +inf, exactly as the oracle's."""
    N, d, K = 500, 32, 20
    X, comp, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.2, seed=7)
    labels = comp.numpy().astype(np.int32)
    extra = torch.randn(12, d, generator=torch.Generator().manual_seed(3))
    C = torch.cat([X[init_indices(N, K, 7)].float(), extra]).contiguous()
    nlist = C.shape[0]
    Q = torch.cat([extra[:4] + 0.01, mixture_queries(40, d, K, sigma=0.2, seed=7, stream=1)])
    for nprobe, k in ((1, 32), (3, 32), (nlist, 8)):
        ref = oracle.ivf_search(Q, C, X, labels, nprobe, k)
        assert (ref[1] == -1).any() or nprobe == nlist
        idx = _index(X, labels, nlist)
        for f64c, f64f, rad in MODES:
            got = _search(Q, C, idx, nprobe, k, fp64_coarse=f64c, fp64_fine=f64f, radius=rad)
            check_search(Q, C, X, got, ref, max_bad_frac=0.0)


def test_ivf_search_duplicates_and_self_queries():
    """Exact duplicate points tie at every query: the lower original index comes first.
    Queries that are data points find themselves at distance 0."""
    N, d, K = 6000, 48, 30
    X, comp, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, seed=9)
    X[N // 2:N // 2 + 200] = X[100:300]   # 200 duplicated rows
    C = X[init_indices(N, K, 9)].float().contiguous()
    labels, _, _ = oracle.assign(X, C)
    sel = np.r_[np.arange(100, 140), np.arange(4000, 4030)]
    Q = X[sel].clone()
    ref = oracle.ivf_search(Q, C, X, labels, 2, 6)
    idx = _index(X, labels, K)
    for f64c, f64f, rad in MODES:
        got = _search(Q, C, idx, 2, 6, fp64_coarse=f64c, fp64_fine=f64f, radius=rad)
        check_search(Q, C, X, got, ref, max_bad_frac=0.0)
        ids = got[1]
        assert (ids[:, 0] == sel).all()
        assert (ids[:40, 1] == sel[:40] + N // 2 - 100).all()   # the duplicate, second


def test_ivf_search_built_index_exhaustive_is_exact_knn():
    """IvfFlatIndex.build (GPU Lloyd, cosine) then search with every cell probed: the result
    is the exact k nearest neighbours of the normalised corpus, whatever the partition."""
    m = fk()
    N, d, K = 40000, 96, 64
    X, _, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.5, seed=11)
    C0 = X[init_indices(N, K, 11)].float().contiguous()
    index = m.IvfFlatIndex.build(X.to(DEV), C0.to(DEV), 5, metric="cosine")
    Q = mixture_queries(64, d, K, sigma=0.5, seed=11, stream=2)
    dist, ids = index.search(Q.to(DEV), 10, K)
    torch.cuda.synchronize()
    Xn = oracle.normalize_rows(X)
    Qn = oracle.normalize_rows(Q)
    # one cell holding every point: the oracle's search is then the brute-force kNN
    _, ri, rd = oracle.ivf_search(Qn, Xn[:1], Xn, np.zeros(N, dtype=np.int32), 1, 10)
    ids = ids.cpu().numpy()
    assert (ids == ri).mean() > 0.999
    np.testing.assert_allclose(dist.cpu().numpy(), rd, rtol=1e-6, atol=1e-6)


def test_ivf_search_deterministic_and_batched_coarse():
    """Two calls give the same bits; a query set larger than one coarse batch (nlist large
    enough that the coarse matrix is cut) gives the same answers as per-batch calls."""
    m = fk()
    N, d, K = 70000, 16, 20000
    X, comp, _ = gaussian_mixture(N, d, 4000, centers="normal", sigma=0.3, seed=13)
    C = X[init_indices(N, K, 13)].float().contiguous()
    labels = torch.randint(0, K, (N,), generator=torch.Generator().manual_seed(5)).numpy()
    labels = labels.astype(np.int32)
    idx = _index(X, labels, K)
    nq = 4000   # coarse batch: 512 MiB / (20000 * 8 B) = 3328 rows -> two batches
    Q = mixture_queries(nq, d, 4000, sigma=0.3, seed=13, stream=3)
    a = _search(Q, C, idx, 5, 7)
    b = _search(Q, C, idx, 5, 7)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    c = [_search(Q[i:i + 1000], C, idx, 5, 7) for i in range(0, nq, 1000)]
    for t in range(3):
        assert np.array_equal(a[t], np.concatenate([z[t] for z in c]))
    sub = np.arange(0, nq, 97)
    ref = oracle.ivf_search(Q[sub], C, X, labels, 5, 7)
    check_search(Q[sub], C, X, tuple(x[sub] for x in a), ref)


def test_ivf_search_argument_errors():
    m = fk()
    N, d, K = 1000, 16, 10
    X, comp, _ = gaussian_mixture(N, d, K, seed=17)
    C = X[:K].contiguous().to(DEV)
    idx = _index(X, comp.numpy().astype(np.int32), K)
    Q = X[:5].to(DEV)
    for nprobe, k in ((K + 1, 3), (0, 3), (2, 0), (2, 33)):
        with pytest.raises(m.FkError) as e:
            m.fk_ivf_search(Q, C, *idx[:4], nprobe, k)
        assert e.value.status == m.FK_ERR_INVALID_ARG
    ws = m.ivf_search_workspace(5, d, K, N, 2, 3)
    with pytest.raises(m.FkError) as e:
        m.fk_ivf_search(Q, C, *idx[:4], 2, 3, ws=ws[:1024])
    assert e.value.status == m.FK_ERR_WORKSPACE


def test_ivf_search_equal_centroid_distances():
    """Thousands of identical centroids: every coarse distance of a query ties, so one
    histogram bin holds more entries than the staged selection sorts and the radix path
    decides; the probes are the lowest cell indices, as in the oracle."""
    N, d, nlist = 4000, 16, 3000
    X, _, _ = gaussian_mixture(N, d, 10, centers="normal", sigma=0.3, seed=21)
    C = X[:1].expand(nlist, d).contiguous()
    labels = (np.arange(N) % nlist).astype(np.int32)
    Q = mixture_queries(40, d, 10, sigma=0.3, seed=21, stream=1)
    idx = _index(X, labels, nlist)
    for nprobe, k in ((5, 4), (700, 32)):
        ref = oracle.ivf_search(Q, C, X, labels, nprobe, k)
        for f64 in (False, True):
            got = _search(Q, C, idx, nprobe, k, fp64_coarse=f64)
            assert (got[0] == np.arange(nprobe)).all()
            check_search(Q, C, X, got, ref, max_bad_frac=0.0)


def test_ivf_search_coarse_paths_agree_and_large_nlist_uses_fp64():
    """The screened and the fp64 coarse pass give the same probes and results bit for bit
    on a cosine workload at the guide's d; above 8192 cells the fp64 pass runs."""
    N, d, K = 60000, 768, 512
    X, _, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, seed=23)
    Xn = torch.nn.functional.normalize(X, dim=1)
    labels = torch.randint(0, K, (N,), generator=torch.Generator().manual_seed(2)).numpy()
    idx = _index(Xn, labels.astype(np.int32), K)
    C = Xn[init_indices(N, K, 23)].contiguous()
    Q = torch.nn.functional.normalize(mixture_queries(1000, d, K, sigma=0.3, seed=23,
                                                      stream=1), dim=1)
    for nprobe in (1, 16, 128):
        ta, tb = {}, {}
        a = _search(Q, C, idx, nprobe, 10, timing=ta)
        b = _search(Q, C, idx, nprobe, 10, fp64_coarse=True, timing=tb)
        assert ta["screened_coarse"] == 1 and tb["screened_coarse"] == 0
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        assert np.array_equal(a[2], b[2])
    tm = {}
    Cbig = Xn[init_indices(N, 9000, 24)].contiguous()
    lab = torch.randint(0, 9000, (N,), generator=torch.Generator().manual_seed(3)).numpy()
    _search(Q[:50], Cbig, _index(Xn, lab.astype(np.int32), 9000), 4, 5, timing=tm)
    assert tm["screened_coarse"] == 0


def test_ivf_search_screened_fine_fallback_on_tied_candidates():
    """100 copies of one point in a cell tie at every query, so a pair list (32 entries)
    drops copies inside the re-ranking window and the query is recomputed exactly: the
    lowest original indices of the copies come first, as in the oracle."""
    N, d, K = 5000, 64, 20
    X, comp, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, seed=29)
    dup = np.arange(1000, 1100)
    X[dup] = X[7].clone()
    C = X[init_indices(N, K, 29)].float().contiguous()
    labels, _, _ = oracle.assign(X, C)
    Q = torch.cat([X[7:8] + 0.01, mixture_queries(30, d, K, sigma=0.3, seed=29, stream=1)])
    idx = _index(X, labels, K)
    for k in (10, 16):
        ref = oracle.ivf_search(Q, C, X, labels, 3, k)
        tm = {}
        got = _search(Q, C, idx, 3, k, timing=tm)
        assert tm["screened_fine"] == 1 and tm["fallback_queries"] >= 1
        check_search(Q, C, X, got, ref, max_bad_frac=0.0)
        assert (got[1][0] == np.r_[7, dup][:k]).all()


def test_ivf_radii_bound_every_cell():
    """fk_ivf_radii: each radius is at least the largest distance of a cell's points to its
    centroid (fp64 on the CPU), and within fp32 rounding of it; empty cells give 0."""
    m = fk()
    N, d, K = 20000, 48, 64
    X, comp, _ = gaussian_mixture(N, d, K - 3, centers="normal", sigma=0.4, seed=31)
    labels = comp.numpy().astype(np.int32)          # cells K-3 .. K-1 stay empty
    C = torch.randn(K, d, generator=torch.Generator().manual_seed(4))
    idx = _index(X, labels, K)
    rad = m.fk_ivf_radii(C.to(DEV), idx[0], idx[2]).cpu().numpy().astype(np.float64)
    X64, C64 = X.double().numpy(), C.double().numpy()
    for c in range(K):
        pts = X64[labels == c]
        if len(pts) == 0:
            assert rad[c] == 0.0
            continue
        r = np.sqrt(((pts - C64[c]) ** 2).sum(1).max())
        assert r <= rad[c] <= r * (1 + 1e-6)


@pytest.mark.parametrize("seed", range(12))
def test_ivf_search_random_shapes(seed):
    """Seeded random shapes: small and odd d, nlist down to 1, cells of every size, k up to
    32, nprobe up to nlist; every path against the oracle."""
    r = np.random.default_rng(1000 + seed)
    d = int(r.choice([4, 8, 12, 36, 64, 100, 132]))
    nlist = int(r.choice([1, 2, 7, 33, 100]))
    N = int(r.integers(max(nlist, 20), 3000))
    nq = int(r.integers(1, 70))
    k = int(r.integers(1, 33))
    nprobe = int(r.integers(1, nlist + 1))
    X, _, _ = gaussian_mixture(N, d, max(nlist, 2), centers="normal", sigma=float(r.uniform(0.05, 1.0)),
                               weights=str(r.choice(["equal", "zipf"])), seed=seed)
    C = X[init_indices(N, nlist, seed)].float().contiguous()
    labels = (oracle.assign(X, C)[0] if r.random() < 0.5 else
              r.integers(0, nlist, N).astype(np.int32))
    Q = mixture_queries(nq, d, max(nlist, 2), seed=seed, stream=3)
    ref = oracle.ivf_search(Q, C, X, labels, nprobe, k)
    idx = _index(X, labels, nlist)
    for f64c, f64f, rad in MODES:
        got = _search(Q, C, idx, nprobe, k, fp64_coarse=f64c, fp64_fine=f64f, radius=rad)
        check_search(Q, C, X, got, ref, max_bad_frac=0.05)
