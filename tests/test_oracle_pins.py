"""Pins for the fp64 oracle: checks against what the mathematics fixes, never against the
oracle's own formula retyped.

Each test names the mistake it would catch (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie rule, an unstable sort, ...).
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _J_loops(X, C, labels):
    """Objective by explicit Python loops (small cases only)."""
    tot = 0.0
    for i in range(len(X)):
        for j in range(X.shape[1]):
            t = X[i, j] - C[labels[i], j]
            tot += t * t
    return tot


# --------------------------------------------------------------------------- assign


@pytest.mark.parametrize("seed", range(6))
def test_assign_minimises_objective_over_all_labelings(seed):
    """Brute force: among all K^N labelings, the oracle's labels reach the minimum of J
    (catches a wrong sign, a dropped coordinate or a max instead of a min)."""
    r = _rng(seed)
    n, d, K = 6, 3, 3
    X = r.normal(size=(n, d))
    C = r.normal(size=(K, d))
    labels, dmin, _ = oracle.assign(X, C)
    best = min(_J_loops(X, C, lab) for lab in itertools.product(range(K), repeat=n))
    assert abs(_J_loops(X, C, labels) - best) <= 1e-12 * max(1.0, best)
    assert abs(dmin.sum() - best) <= 1e-12 * max(1.0, best)


def test_assign_identity_when_centroids_are_the_points():
    """K = N with C = X: every point is its own cluster at distance 0."""
    X = _rng(1).normal(size=(17, 5))
    labels, dmin, d2nd = oracle.assign(X, X)
    assert (labels == np.arange(17)).all()
    assert (dmin == 0).all() and (d2nd > 0).all()


def test_assign_tie_goes_to_lowest_index():
    """A duplicated centroid: the lower index wins and the gap is exactly 0."""
    X = _rng(2).normal(size=(50, 4))
    C = _rng(3).normal(size=(3, 4))
    C = np.vstack([C, C[1:2]])  # centroid 3 duplicates centroid 1
    labels, dmin, d2nd = oracle.assign(X, C)
    assert not (labels == 3).any()
    on1 = labels == 1
    assert on1.any() and (d2nd[on1] == dmin[on1]).all()


def test_assign_single_centroid():
    X = _rng(4).normal(size=(20, 3))
    labels, dmin, d2nd = oracle.assign(X, X[:1])
    assert (labels == 0).all() and np.isinf(d2nd).all()


def test_assign_recovers_components_of_a_tight_mixture():
    """sigma -> 0 and C = the true centers: labels equal the component ids (catches a
    transposed operand: with K != d the wrong layout gives different labels)."""
    r = _rng(5)
    K, d, n = 7, 5, 400
    cen = r.uniform(-1, 1, size=(K, d))
    comp = r.integers(0, K, size=n)
    X = cen[comp] + 1e-6 * r.normal(size=(n, d))
    labels, _, _ = oracle.assign(X, cen)
    assert (labels == comp).all()


def test_assign_translation_invariant():
    r = _rng(6)
    X = r.normal(size=(300, 6))
    C = r.normal(size=(9, 6))
    t = r.normal(size=(1, 6))
    l0, dmin, d2nd = oracle.assign(X, C)
    l1, _, _ = oracle.assign(X + t, C + t)
    keep = ~oracle.tie_mask(X, C, dmin, d2nd)
    assert (l0[keep] == l1[keep]).all()


def test_distance_is_formed_from_differences():
    """The squared distance is sum_j (x_j - c_j)^2 formed from the differences (Flash-KMeans
    article, "它不是银弹，但切中了一个真痛点": squared L2).  On a dyadic grid, a shift of every
    coordinate by 2^24 is exact in fp64 and so is each difference, so distances, labels, the
    objective and the search's distances must be bit-identical before and after the shift.
    Expanding the square (|x|^2 + |c|^2 - 2 x.c) loses about half a unit to cancellation at
    this offset and fails this."""
    r = _rng(16)
    X = np.round(r.normal(size=(200, 8)) * 1024) / 1024
    C = np.round(r.normal(size=(12, 8)) * 1024) / 1024
    t = float(2 ** 24)
    l0, dmin0, d2nd0 = oracle.assign(X, C)
    l1, dmin1, d2nd1 = oracle.assign(X + t, C + t)
    assert np.array_equal(dmin0, dmin1) and np.array_equal(d2nd0, d2nd1)
    assert np.array_equal(l0, l1)
    assert oracle.objective(X, C, l0) == oracle.objective(X + t, C + t, l0)
    Q = X[:20]
    p0, i0, g0 = oracle.ivf_search(Q, C, X, l0, nprobe=3, k=5)
    p1, i1, g1 = oracle.ivf_search(Q + t, C + t, X + t, l0, nprobe=3, k=5)
    assert np.array_equal(p0, p1) and np.array_equal(i0, i1) and np.array_equal(g0, g1)


def test_tie_mask_definition():
    """A point exactly between two centroids is a tie point; one far from the bisector
    is not."""
    C = np.array([[-1.0, 0.0], [1.0, 0.0]])
    X = np.array([[0.0, 3.0], [0.9, 0.0]])
    labels, dmin, d2nd = oracle.assign(X, C)
    m = oracle.tie_mask(X, C, dmin, d2nd)
    assert m.tolist() == [True, False]
    assert labels.tolist() == [0, 1]


# --------------------------------------------------------------------------- update


def test_update_single_cluster_is_numpy_mean():
    X = _rng(7).normal(size=(1000, 8))
    C = oracle.update(X, np.zeros(1000, np.int32), np.zeros((1, 8)))
    np.testing.assert_allclose(C[0], np.mean(X, axis=0), rtol=0, atol=1e-14)


def test_update_matches_per_cluster_numpy_mean_and_keeps_empty():
    r = _rng(8)
    X = r.normal(size=(500, 4))
    labels = r.integers(0, 6, size=500).astype(np.int32)
    labels[labels == 4] = 5  # cluster 4 empty
    C_old = r.normal(size=(6, 4))
    C = oracle.update(X, labels, C_old)
    for k in range(6):
        if k == 4:
            assert (C[k] == C_old[k]).all()
        else:
            np.testing.assert_allclose(C[k], np.mean(X[labels == k], axis=0), atol=1e-14)


@pytest.mark.parametrize("seed", range(3))
def test_update_is_first_order_optimal(seed):
    """Moving any coordinate of any updated centroid by +-delta raises J (the mean
    minimises the within-cluster sum of squares)."""
    r = _rng(seed + 10)
    X = r.normal(size=(60, 3))
    labels = r.integers(0, 4, size=60).astype(np.int32)
    C = oracle.update(X, labels, np.zeros((4, 3)))
    J0 = _J_loops(X, C, labels)
    for k in range(4):
        for j in range(3):
            for delta in (1e-3, -1e-3):
                Cp = C.copy()
                Cp[k, j] += delta
                assert _J_loops(X, Cp, labels) > J0


def test_objective_parallel_axis_identity():
    """J = sum_k [ sum_{i in k} ||x_i||^2 - n_k ||mu_k||^2 + n_k ||mu_k - c_k||^2 ]
    (a different computation from the direct sum)."""
    r = _rng(11)
    X = r.normal(size=(400, 5))
    K = 7
    labels = r.integers(0, K, size=400).astype(np.int32)
    C = r.normal(size=(K, 5))
    J = oracle.objective(X, C, labels)
    alt = 0.0
    for k in range(K):
        M = X[labels == k]
        mu = M.mean(axis=0)
        alt += (M * M).sum() - len(M) * (mu @ mu) + len(M) * ((mu - C[k]) @ (mu - C[k]))
    assert abs(J - alt) <= 1e-10 * J


# --------------------------------------------------------------------------- CSR


def test_csr_matches_stable_argsort_and_invariants():
    r = _rng(12)
    K = 37
    labels = r.integers(0, K, size=5000).astype(np.int32)
    labels[labels == 5] = 6
    counts, offsets, perm = oracle.csr(labels, K)
    assert (perm == np.argsort(labels, kind="stable")).all()
    assert counts.sum() == 5000 and offsets[0] == 0 and offsets[K] == 5000
    assert (np.diff(offsets) == counts).all() and counts[5] == 0
    assert (np.bincount(labels, minlength=K) == counts).all()
    for k in range(K):
        seg = perm[offsets[k]:offsets[k + 1]]
        assert (labels[seg] == k).all() and (np.diff(seg) > 0).all()


def test_csr_rejects_out_of_range_label():
    with pytest.raises(ValueError):
        oracle.csr(np.array([0, 3], np.int32), 3)


# --------------------------------------------------------------------------- normalise


def test_normalize_rows_unit_norm_and_zero_guard():
    r = _rng(13)
    X = r.normal(size=(100, 9)) * r.uniform(0.01, 100, size=(100, 1))
    X[7] = 0.0
    Y = oracle.normalize_rows(X)
    nrm = np.linalg.norm(Y, axis=1)
    keep = np.arange(100) != 7
    np.testing.assert_allclose(nrm[keep], 1.0, atol=1e-15)
    assert (Y[7] == 0).all()
    np.testing.assert_allclose(Y[keep], X[keep] / np.linalg.norm(X[keep], axis=1,
                                                                 keepdims=True),
                               rtol=1e-15)


def test_cosine_labels_invariant_to_row_scaling():
    r = _rng(14)
    X = r.normal(size=(300, 6))
    C0 = X[:5].copy()
    s = 2.0 ** r.integers(-4, 5, size=(300, 1))
    a = oracle.lloyd(X, C0, 2, metric="cosine")
    b = oracle.lloyd(X * s, C0, 2, metric="cosine")
    for t in range(2):
        keep = ~a["ties"][t]
        assert (a["labels"][t][keep] == b["labels"][t][keep]).all()


# --------------------------------------------------------------------------- Lloyd


def test_golden_line4_hand_derived():
    g = json.load(open(os.path.join(GOLDEN, "line4_hand.json")))
    X = np.array(g["X"])
    C = np.array(g["C0"])
    for it in g["iterations"]:
        labels, dmin, _ = oracle.assign(X, C)
        assert labels.tolist() == it["labels"]
        J = oracle.objective(X, C, labels)
        assert abs(J - it["J"]) <= 1e-12 * it["J"]
        counts, _, _ = oracle.csr(labels, len(C))
        assert counts.tolist() == it["counts"]
        C = oracle.update(X, labels, C)
        np.testing.assert_allclose(C, np.array(it["C_next"]), rtol=1e-15, atol=0)


def test_lloyd_objective_non_increasing():
    r = _rng(15)
    cen = r.uniform(-1, 1, size=(12, 8))
    X = cen[r.integers(0, 12, size=3000)] + 0.2 * r.normal(size=(3000, 8))
    out = oracle.lloyd(X, X[:12], 8)
    J = out["J"]
    for t in range(1, len(J)):
        assert J[t] <= J[t - 1] * (1 + 1e-6)
    # the objective against the updated centroids sits between consecutive J's
    for t in range(len(J) - 1):
        Jp = oracle.objective(out["X"], out["C_next"][t], out["labels"][t])
        assert J[t + 1] <= Jp * (1 + 1e-6) and Jp <= J[t] * (1 + 1e-6)


def test_lloyd_bf16_precision_feeds_rounded_centroids():
    r = _rng(16)
    X = r.normal(size=(200, 16)).astype(np.float32)
    out = oracle.lloyd(X, X[:4], 2, precision="bf16")
    Cu = out["C_used"][1]
    assert (oracle.round_bf16(Cu) == Cu).all()
    assert (oracle.round_f32(out["C_next"][0]) == out["C_next"][0]).all()


def test_lloyd_objective_is_against_the_centroids_used():
    """J of an iteration is sum_i ||x_i - c_{l_i}||^2 against the centroids that
    iteration's assignment used: with bf16 centroids, their bf16 roundings, not the fp32
    master.  Formed here with numpy from the recorded labels; the master gives a J the test
    can tell apart."""
    r = _rng(17)
    X = r.normal(size=(300, 16)).astype(np.float32)
    out = oracle.lloyd(X, X[:5], 2, precision="bf16")
    for t in range(2):
        Cu, lab = out["C_used"][t], out["labels"][t]
        J_np = float(((out["X"] - Cu[lab]) ** 2).sum())
        assert abs(out["J"][t] - J_np) <= 1e-12 * J_np
        master = out["C_next"][t - 1] if t else X[:5].astype(np.float64)
        J_master = float(((out["X"] - master[lab]) ** 2).sum())
        assert abs(J_master - J_np) > 1e-9 * J_np


def test_lloyd_cosine_normalises_initial_centroids():
    """Cosine mode L2-normalises the points and the initial centroids (LEANN FlashLib
    guide, "距离度量只有 squared L2如何支持 mips / cosine"), so the first assignment sees
    unit-norm centroids (rounded to fp32) and unit-norm points."""
    r = _rng(18)
    X = r.normal(size=(100, 8)) * 3.0
    C0 = X[:4] * np.array([[0.5], [2.0], [7.0], [1.0]])
    out = oracle.lloyd(X, C0, 1, metric="cosine")
    assert np.abs(np.linalg.norm(out["C_used"][0], axis=1) - 1.0).max() <= 1e-6
    assert np.abs(np.linalg.norm(out["X"], axis=1) - 1.0).max() <= 1e-12


def test_tie_window_scales_with_the_largest_centroid_norm():
    """The tie window is tau * (||x||^2 + max_k ||c_k||^2) (the parity rule's reading): a
    far centroid of large norm widens it for every point.  Here the top-2 gap is 0.04:
    inside the window with the far centroid (about 1.0), outside it without (about 1e-4)."""
    C = np.array([[-1.0, 0.0], [1.0, 0.0], [100.0, 0.0]])
    X = np.array([[0.01, 0.0]])
    labels, dmin, d2nd = oracle.assign(X, C)
    assert labels.tolist() == [1]
    assert oracle.tie_mask(X, C, dmin, d2nd).tolist() == [True]
    _, dmin2, d2nd2 = oracle.assign(X, C[:2])
    assert oracle.tie_mask(X, C[:2], dmin2, d2nd2).tolist() == [False]


def test_round_bf16_is_nearest_even():
    ulp = 2.0 ** -7  # bf16 spacing on [1, 2)
    v = np.array([1 + ulp / 2, 1 + 1.5 * ulp, 1 + 0.75 * ulp, -(1 + ulp / 2)])
    assert oracle.round_bf16(v).tolist() == [1.0, 1 + 2 * ulp, 1 + ulp, -1.0]


# --------------------------------------------------------------------------- IVF-Flat search


def _sq_loop(u, v):
    # sequential fp64 sum (the builtin sum() of floats is compensated since Python 3.12)
    s = 0.0
    for a, b in zip(u, v):
        s += (a - b) * (a - b)
    return s


def _search_python_loops(Q, C, X, labels, nprobe, k):
    """Brute force in pure Python on tiny inputs: sorted() over (distance, index) tuples."""
    probes, ids, dist = [], [], []
    for q in Q.tolist():
        cd = [(_sq_loop(q, c), j) for j, c in enumerate(C.tolist())]
        cells = [j for _, j in sorted(cd)[:nprobe]]
        cand = [(_sq_loop(q, x), i) for i, x in enumerate(X.tolist()) if labels[i] in cells]
        best = sorted(cand)[:k]
        probes.append(cells)
        ids.append([i for _, i in best] + [-1] * (k - len(best)))
        dist.append([v for v, _ in best] + [np.inf] * (k - len(best)))
    return np.array(probes), np.array(ids), np.array(dist)


def test_ivf_search_golden_hand_derived():
    g = json.load(open(os.path.join(GOLDEN, "ivf_search_hand.json")))
    C, X = np.array(g["C"]), np.array(g["X"])
    labels = np.array(g["labels"], dtype=np.int32)
    for case in g["cases"]:
        probes, ids, dist = oracle.ivf_search(np.array(case["Q"]), C, X, labels,
                                              case["nprobe"], case["k"])
        assert probes.tolist() == case["probes"]
        assert ids.tolist() == case["ids"]
        want = np.array([[np.inf if v is None else v for v in row] for row in case["dist"]])
        assert np.array_equal(dist, want)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ivf_search_matches_python_brute_force(seed):
    r = _rng(40 + seed)
    X = np.round(r.normal(size=(70, 3)), 1)   # one decimal: exact ties occur
    C = np.round(r.normal(size=(6, 3)), 1)
    Q = np.round(r.normal(size=(9, 3)), 1)
    labels = r.integers(0, 6, size=70).astype(np.int32)
    for nprobe, k in ((1, 3), (2, 5), (6, 7), (3, 40)):
        got = oracle.ivf_search(Q, C, X, labels, nprobe, k)
        want = _search_python_loops(Q, C, X, labels, nprobe, k)
        for a, b in zip(got, want):
            assert np.array_equal(a, b)


def test_ivf_search_all_cells_is_exact_knn():
    """nprobe = nlist probes every cell: the result is the exact k-nearest-neighbour list of
    scikit-learn's brute-force search."""
    from sklearn.neighbors import NearestNeighbors
    r = _rng(50)
    X = r.normal(size=(3000, 16))
    C = X[:40].copy()
    labels, _, _ = oracle.assign(X, C)
    Q = r.normal(size=(25, 16))
    _, ids, dist = oracle.ivf_search(Q, C, X, labels, 40, 10)
    nn = NearestNeighbors(n_neighbors=10, algorithm="brute").fit(X)
    d_ref, i_ref = nn.kneighbors(Q)
    assert np.array_equal(ids, i_ref)
    np.testing.assert_allclose(dist, d_ref ** 2, rtol=1e-10)


def test_ivf_probes_are_nearest_centroids_by_cdist():
    from scipy.spatial.distance import cdist
    r = _rng(51)
    C = r.normal(size=(64, 12))
    X = r.normal(size=(500, 12))
    labels = r.integers(0, 64, size=500).astype(np.int32)
    Q = r.normal(size=(30, 12))
    probes, _, _ = oracle.ivf_search(Q, C, X, labels, 9, 1)
    D = cdist(Q, C, "sqeuclidean")
    want = np.argsort(D, axis=1, kind="stable")[:, :9]
    assert np.array_equal(probes, want)


def test_ivf_search_self_query_finds_itself():
    """With labels from the assignment against the same centroids, a point used as a query
    probes its own cell first and is its own nearest neighbour at distance 0."""
    r = _rng(52)
    X = r.normal(size=(800, 10))
    C = X[r.choice(800, 20, replace=False)]
    labels, _, _ = oracle.assign(X, C)
    sel = r.choice(800, 40, replace=False)
    probes, ids, dist = oracle.ivf_search(X[sel], C, X, labels, 1, 3)
    assert np.array_equal(probes[:, 0], labels[sel])
    assert np.array_equal(ids[:, 0], sel)
    assert np.all(dist[:, 0] == 0.0)
    assert np.all(np.diff(dist, axis=1) >= 0)


def test_ivf_search_kth_distance_non_increasing_in_nprobe():
    r = _rng(53)
    X = r.normal(size=(2000, 8))
    C = r.normal(size=(32, 8))
    labels, _, _ = oracle.assign(X, C)
    Q = r.normal(size=(20, 8))
    prev = None
    for nprobe in (1, 2, 4, 8, 16, 32):
        probes, _, dist = oracle.ivf_search(Q, C, X, labels, nprobe, 5)
        if prev is not None:
            assert np.all(dist[:, -1] <= prev[1][:, -1])
            assert np.array_equal(probes[:, :prev[0].shape[1]], prev[0])  # nested probe lists
        prev = (probes, dist)


def test_ivf_search_rejects_bad_arguments():
    X = np.zeros((4, 2))
    C = np.zeros((2, 2))
    with pytest.raises(ValueError):
        oracle.ivf_search(X, C, X, np.array([0, 1, 2, 0], dtype=np.int32), 1, 1)
    with pytest.raises(ValueError):
        oracle.ivf_search(X, C, X, np.zeros(4, dtype=np.int32), 3, 1)
