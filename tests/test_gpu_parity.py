"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element
on the same seeded inputs, at sizes spanning several tiles with ragged tails.

Parity rules (written here, applied in every test):
  labels   bit-exact except at tie points (oracle top-2 gap < 1e-4 (||x||^2 + max||c||^2));
  counts, offsets, perm  bit-exact;
  centroids (given identical labels)  max |dc| <= 1e-5 max |c_ref| per centroid;
  objective  relative error <= 1e-5.
Inputs reach the GPU from the generator or from the oracle (lockstep); nothing computed on
the GPU is ever handed to the oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
from synth import adversarial_rows, gaussian_mixture, init_indices
from tests.gpu_helpers import (CENTROID_TOL, OBJECTIVE_TOL, centroid_rel_err, fk, gpu_assign,
                               gpu_update, label_mismatches)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _mixture(N, d, K, dtype="f32", seed=0, centers="uniform", sigma=0.1, weights="equal"):
    X, comp, cen = gaussian_mixture(N, d, K, centers=centers, sigma=sigma, weights=weights,
                                    dtype=dtype, seed=seed)
    C0 = X[init_indices(N, K, seed)].float().contiguous()
    return X, C0, comp


ASSIGN_SHAPES = [(1000, 64, 10), (4097, 128, 256), (3001, 96, 300), (5000, 8, 7),
                 (777, 768, 513), (300, 128, 1), (129, 16, 129), (20000, 128, 1000)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,K", ASSIGN_SHAPES)
def test_assign_matches_oracle(N, d, K, dtype):
    X, C0, _ = _mixture(N, d, K, dtype, seed=N + d + K)
    Cref = oracle.round_bf16(C0.numpy()) if dtype == "bf16" else C0.numpy()
    ref, dmin, d2nd = oracle.assign(X, Cref)
    ties = oracle.tie_mask(X, Cref, dmin, d2nd)
    lab, mind = gpu_assign(X.to(DEV), C0.to(DEV), with_mind=True)
    assert (lab >= 0).all() and (lab < K).all()
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"
    # mind is the expansion form: within the same window the tie rule uses
    Xd = X.double().numpy()
    s = (Xd * Xd).sum(1) + (Cref.astype(np.float64) ** 2).sum(1).max()
    assert (np.abs(mind.astype(np.float64) - dmin) <= 1e-4 * s).all()


def test_assign_points_as_centroids():
    X, _, _ = _mixture(1000, 64, 50, seed=3)
    lab, _ = gpu_assign(X.to(DEV), X.to(DEV).clone())
    assert (lab == np.arange(1000)).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_assign_duplicate_centroid_lowest_index(dtype):
    X, C0, _ = _mixture(3000, 128, 40, dtype, seed=4)
    C = torch.cat([C0, C0[5:6], C0[17:18]])  # 40 duplicates 5, 41 duplicates 17
    lab, _ = gpu_assign(X.to(DEV), C.to(DEV))
    assert not np.isin(lab, [40, 41]).any()
    assert (lab == 5).any() and (lab == 17).any()


def test_assign_tight_mixture_recovers_components():
    X, comp, cen = gaussian_mixture(5000, 128, 300, centers="uniform", sigma=1e-3, seed=5)
    lab, _ = gpu_assign(X.to(DEV), cen.float().to(DEV))
    assert (lab == comp.numpy()).all()


UPDATE_SHAPES = [(1000, 64, 10, "equal"), (20000, 128, 37, "equal"), (70000, 128, 3, "equal"),
                 (5000, 768, 50, "equal"), (3000, 1032, 20, "equal"), (200000, 16, 2, "equal"),
                 (150000, 128, 4096, "zipf"), (777, 8, 700, "equal"),
                 (60000, 96, 500, "zipf"), (40960, 64, 1000, "zipf")]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,K,weights", UPDATE_SHAPES)
def test_update_matches_oracle(N, d, K, weights, dtype):
    if dtype == "bf16" and d % 8:
        pytest.skip("bf16 needs d % 8 == 0")
    X, C0, comp = _mixture(N, d, K, dtype, seed=N + K, weights=weights, centers="normal")
    labels = comp.numpy().astype(np.int32)  # generator labels: Zipf gives huge clusters
    labels[labels == K // 2] = (K // 2 + 1) % K  # force an empty cluster
    C_old = torch.randn(K, d, generator=torch.Generator().manual_seed(1))
    counts, offsets, perm = oracle.csr(labels, K)
    C_ref = oracle.update(X, labels, C_old.numpy())
    C_used = oracle.round_bf16(C_old.numpy()) if dtype == "bf16" else C_old.numpy()
    J_ref = oracle.objective(X, C_used, labels)

    g = gpu_update(X.to(DEV), labels, C_old.to(DEV))
    assert (g["counts"] == counts).all()
    assert (g["offsets"] == offsets).all()
    assert (g["perm"] == perm).all()
    nonempty = counts > 0
    assert centroid_rel_err(g["C_new"][nonempty], C_ref[nonempty]) <= CENTROID_TOL
    # an empty cluster keeps its previous centroid bit for bit
    assert (g["C_new"][~nonempty] == C_old.numpy()[~nonempty].astype(np.float64)).all()
    assert abs(g["J"] - J_ref) <= OBJECTIVE_TOL * J_ref


def test_update_single_cluster_is_global_mean():
    X, _, _ = _mixture(50000, 128, 1, seed=9)
    g = gpu_update(X.to(DEV), np.zeros(50000, np.int32), torch.zeros(1, 128, device=DEV))
    mean = X.double().numpy().mean(axis=0)
    assert centroid_rel_err(g["C_new"], mean[None]) <= 1e-6
    assert (g["perm"] == np.arange(50000)).all() and g["offsets"].tolist() == [0, 50000]


@pytest.mark.parametrize("K", [256, 300, 65536])
def test_update_sort_large_input_tiles(K):
    """Inputs above 4M keys take the radix sort's large tiles (8 keys per thread); N leaves
    a ragged last tile.  K = 256 sorts in one 8-bit pass, 300 in two 5-bit passes, 65536
    in two 8-bit passes.  perm, counts and offsets against the oracle's stable CSR (a long
    run of one label and an empty cluster included), centroids against its means."""
    N, d = (1 << 22) + 12345, 4
    rng = np.random.default_rng(K)
    labels = rng.integers(0, K, N, dtype=np.int32)
    labels[1000:300000] = 7
    labels[labels == K - 1] = 0
    X = torch.randn(N, d, generator=torch.Generator().manual_seed(K))
    C_old = torch.randn(K, d, generator=torch.Generator().manual_seed(K + 1))
    counts, offsets, perm = oracle.csr(labels, K)
    C_ref = oracle.update(X, labels, C_old.numpy())
    g = gpu_update(X.to(DEV), labels, C_old.to(DEV))
    assert (g["counts"] == counts).all()
    assert (g["offsets"] == offsets).all()
    assert (g["perm"] == perm).all()
    nonempty = counts > 0
    assert not nonempty.all()
    assert centroid_rel_err(g["C_new"][nonempty], C_ref[nonempty]) <= CENTROID_TOL


@pytest.mark.parametrize("case", ["tiny_f32", "tiny_bf16", "cosine_768"])
def test_lockstep_lloyd_matches_oracle(case):
    """Lockstep: each iteration the GPU assigns with the oracle's centroids and updates
    with the oracle's labels; every output is compared with the oracle's."""
    if case == "tiny_f32":
        # the 65,536 x 128, K = 256 workload, all five of its iterations
        X, C0, _ = _mixture(65536, 128, 256, "f32", seed=0, sigma=0.1)
        niter, prec, metric = 5, "f32", "l2"
    elif case == "tiny_bf16":
        X, C0, _ = _mixture(30000, 128, 500, "bf16", seed=1, centers="normal", sigma=0.25)
        niter, prec, metric = 3, "bf16", "l2"
    else:
        X, C0, _ = _mixture(20000, 768, 64, "f32", seed=2, centers="normal", sigma=0.3)
        niter, prec, metric = 3, "f32", "cosine"
    ref = oracle.lloyd(X, C0, niter, metric=metric, precision=prec)
    Xg = X.to(DEV)
    if metric == "cosine":
        Xn = torch.empty_like(Xg)
        fk().fk_normalize_rows(Xg, Xn)
        dn = np.abs(Xn.cpu().double().numpy() - ref["X"])
        assert (dn <= 2 ** -23 * np.abs(ref["X"]) + 1e-30).all()  # <= 1 ulp of fp32
        Xg = Xn
    C_master = [C0.double().numpy()] + ref["C_next"]
    if metric == "cosine":
        C_master[0] = oracle.round_f32(oracle.normalize_rows(C0.numpy()))
    total_ties = 0
    for t in range(niter):
        Cm = torch.as_tensor(C_master[t], dtype=torch.float32)
        lab, _ = gpu_assign(Xg, Cm.to(DEV))
        ties = ref["ties"][t]
        total_ties += int(ties.sum())
        assert label_mismatches(lab, ref["labels"][t], ties) == 0, f"iteration {t}"
        g = gpu_update(Xg, ref["labels"][t], Cm.to(DEV))
        assert (g["counts"] == ref["counts"][t]).all()
        assert (g["offsets"] == ref["offsets"][t]).all()
        assert (g["perm"] == ref["perm"][t]).all()
        assert centroid_rel_err(g["C_new"], ref["C_next"][t]) <= CENTROID_TOL
        assert abs(g["J"] - ref["J"][t]) <= OBJECTIVE_TOL * ref["J"][t]
    print(f"{case}: tie points over {niter} iterations: {total_ties}")


@pytest.mark.parametrize("metric", ["l2", "cosine"])
def test_fk_lloyd_free_running_objective(metric):
    """fk_lloyd end to end from the same C0 as the oracle's own free-running Lloyd.

    Iteration 0 sees identical centroids, so its objective must agree to 1e-5.  Later
    iterations may legitimately drift: a point inside the tie window may take the other
    label (allowed by the parity rule), which moves two centroids by |x - c| / n_k and
    changes the rest of the trajectory; the lockstep test above is the parity gate for
    every later iteration.  Here the later objectives are held to 1e-3 and the run's own
    invariants are checked exactly."""
    X, C0, _ = _mixture(40000, 64 if metric == "l2" else 256, 100, seed=7, centers="normal",
                        sigma=0.3)
    niter = 4
    ref = oracle.lloyd(X, C0, niter, metric=metric)
    m = fk()
    C = C0.to(DEV).clone()
    labels = torch.empty(X.shape[0], dtype=torch.int32, device=DEV)
    counts = torch.empty(100, dtype=torch.int32, device=DEV)
    offsets = torch.empty(101, dtype=torch.int32, device=DEV)
    ws = m.workspace(X.shape[0], X.shape[1], 100, torch.float32, metric)
    objs, tm = m.fk_lloyd(X.to(DEV), C, niter, labels, ws, metric=metric, counts=counts,
                          offsets=offsets, timing=True)
    assert abs(objs[0] - ref["J"][0]) <= OBJECTIVE_TOL * ref["J"][0]
    for t in range(1, niter):
        assert abs(objs[t] - ref["J"][t]) <= 1e-3 * ref["J"][t], t
    assert tm["iterations"] == niter and tm["ms_assign"] > 0 and tm["launches"] > 4 * niter
    lab = labels.cpu().numpy()
    assert (np.bincount(lab, minlength=100) == counts.cpu().numpy()).all()
    assert offsets.cpu().numpy()[-1] == X.shape[0]
    # objective never increases (beyond fp32 rounding of the centroids)
    for t in range(1, niter):
        assert objs[t] <= objs[t - 1] * (1 + 1e-6)


def test_fk_lloyd_deterministic_and_resumable():
    X, C0, _ = _mixture(30000, 128, 200, seed=8, centers="normal", sigma=0.3)
    m = fk()
    Xg = X.to(DEV)
    ws = m.workspace(30000, 128, 200, torch.float32, "l2")

    def run(C, n):
        labels = torch.empty(30000, dtype=torch.int32, device=DEV)
        objs, _ = m.fk_lloyd(Xg, C, n, labels, ws)
        return C, labels, objs

    a = run(C0.to(DEV).clone(), 5)
    b = run(C0.to(DEV).clone(), 5)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and a[2] == b[2]
    # checkpoint/resume: 2 iterations then 3 more from the saved centroids == 5 at once
    c = run(C0.to(DEV).clone(), 2)
    d = run(c[0].clone(), 3)
    assert torch.equal(d[0], a[0]) and torch.equal(d[1], a[1]) and d[2] == a[2][2:]


def test_fk_lloyd_repeated_calls_replay_identically():
    """A call that repeats the previous one replays its iteration loop from a CUDA graph
    (captured on the second call): every call gives the eager call's result bit for bit,
    new centroid values reach the replayed loop, and timing still works on a replay."""
    N, d, K = 20000, 128, 200
    X, C0, _ = _mixture(N, d, K, seed=12, centers="normal", sigma=0.3)
    m = fk()
    Xg = X.to(DEV)
    ws = m.workspace(N, d, K, torch.float32, "l2")
    C = torch.empty(K, d, dtype=torch.float32, device=DEV)
    labels = torch.empty(N, dtype=torch.int32, device=DEV)
    counts = torch.empty(K, dtype=torch.int32, device=DEV)

    def run(Cinit, lab=labels, timing=False):
        C.copy_(Cinit)
        objs, tm = m.fk_lloyd(Xg, C, 4, lab, ws, counts=counts, timing=timing)
        return C.clone(), lab.clone(), counts.clone(), objs, tm

    C0g = C0.to(DEV)
    ref = run(C0g)
    for _ in range(3):
        r = run(C0g)
        assert all(torch.equal(a, b) for a, b in zip(r[:3], ref[:3])) and r[3] == ref[3]
    timed = [run(C0g, timing=True) for _ in range(3)]
    for r in timed:
        assert all(torch.equal(a, b) for a, b in zip(r[:3], ref[:3])) and r[3] == ref[3]
        tm = r[4]
        assert tm["iterations"] == 4 and tm["launches"] == timed[0][4]["launches"] > 0
        for k in ("ms_prep", "ms_assign", "ms_sort", "ms_update", "ms_assign_mma"):
            assert tm[k] > 0, k
    # kernel-only timing: the assignment kernel's time alone (every iteration's, or the
    # last iteration's), the same results
    for mode, code, n in (("kernel", 1, 4), ("kernel_last", 2, 1)):
        for r in [run(C0g, timing=mode) for _ in range(3)]:
            assert all(torch.equal(a, b) for a, b in zip(r[:3], ref[:3])) and r[3] == ref[3]
            tm = r[4]
            assert tm["kernel_only"] == code and tm["iterations"] == 4
            assert tm["mma_timed"] == n and tm["ms_assign_mma"] > 0
            assert tm["ms_assign"] == 0 and tm["ms_update"] == 0 and tm["max_cluster"] == 0
            assert tm["launches"] == timed[0][4]["launches"] - 1  # no statistics kernel
    # other initial centroids: the eager result (another labels buffer, so another call)
    # equals the replay of the cached loop with the original buffers
    C1g = C0g[torch.randperm(K, generator=torch.Generator().manual_seed(5)).to(DEV)]
    other = torch.empty_like(labels)
    e = run(C1g, lab=other)
    run(C0g)  # make the cached call the previous one again
    r = run(C1g)
    assert torch.equal(r[0], e[0]) and torch.equal(r[1], e[1]) and r[3] == e[3]
    assert not torch.equal(r[0], ref[0])


def test_fk_lloyd_objective_ring_wraps():
    """More iterations than the device's objective ring (4096 entries): the full ring is
    handed to the host before it wraps, and the run equals the same run in two calls."""
    N, d, K = 2000, 16, 8
    X, C0, _ = _mixture(N, d, K, seed=13, centers="normal", sigma=0.5)
    m = fk()
    Xg = X.to(DEV)
    ws = m.workspace(N, d, K, torch.float32, "l2")
    labels = torch.empty(N, dtype=torch.int32, device=DEV)
    Ca = C0.to(DEV).clone()
    oa, _ = m.fk_lloyd(Xg, Ca, 4099, labels, ws)
    Cb = C0.to(DEV).clone()
    ob1, _ = m.fk_lloyd(Xg, Cb, 4096, labels, ws)
    ob2, _ = m.fk_lloyd(Xg, Cb, 3, labels, ws)
    assert len(oa) == 4099 and oa == ob1 + ob2 and torch.equal(Ca, Cb)
    assert all(o > 0 for o in oa)


def test_fk_lloyd_k_equals_one_and_k_equals_n():
    m = fk()
    X, _, _ = _mixture(513, 32, 4, seed=10)
    Xg = X.to(DEV)
    for K, C in [(1, X[:1].clone()), (513, X.clone())]:
        ws = m.workspace(513, 32, K, torch.float32, "l2")
        labels = torch.empty(513, dtype=torch.int32, device=DEV)
        Cg = C.to(DEV).contiguous()
        objs, _ = m.fk_lloyd(Xg, Cg, 1, labels, ws)
        lab = labels.cpu().numpy()
        if K == 1:
            assert (lab == 0).all()
            assert centroid_rel_err(Cg.cpu().numpy(), X.double().numpy().mean(0)[None]) < 1e-6
        else:
            assert (lab == np.arange(513)).all() and objs[0] == 0.0
            assert torch.equal(Cg.cpu(), X)


def test_device_error_paths_without_fault():
    """A wait that nothing ends expires and is reported; a bad label is reported; the
    context stays usable afterwards."""
    m = fk()
    ws = m.workspace(1000, 64, 10, torch.float32, "l2")
    assert m.fk_get_device_error(ws) == m.FK_OK
    m.fk_selftest_timeout(ws, 20_000_000)  # 20 ms
    assert m.fk_get_device_error(ws) == m.FK_ERR_TIMEOUT
    assert m.fk_get_device_error(ws) == m.FK_OK  # read clears it
    X, C0, _ = _mixture(1000, 64, 10, seed=11)
    labels = np.zeros(1000, np.int32)
    labels[7] = 10  # == K: out of range
    m2 = fk()
    Xg = X.to(DEV)
    lab = torch.as_tensor(labels).to(DEV)
    C_new = torch.empty(10, 64, device=DEV)
    counts = torch.empty(10, dtype=torch.int32, device=DEV)
    offsets = torch.empty(11, dtype=torch.int32, device=DEV)
    m2.fk_update(Xg, lab, C0.to(DEV), C_new, counts, offsets, ws)
    assert m2.fk_get_device_error(ws) == m2.FK_ERR_DEVICE
    lab2, _ = gpu_assign(Xg, C0.to(DEV))  # still works
    assert (lab2 >= 0).all()


def test_update_partial_and_shard_finalize_match_fk_update():
    """Two shards through fk_update_partial + fk_finalize_shards give fk_update's result
    on all the points (same fp64 sums, combined in shard order)."""
    m = fk()
    X, C0, comp = _mixture(30000, 128, 300, seed=21, centers="normal", sigma=0.3)
    Xg = X.to(DEV)
    lab = comp.to(DEV)
    K, d = 300, 128
    full = gpu_update(Xg, comp.numpy(), C0.to(DEV), want_perm=False)
    sums_w = torch.empty(2, K, d, dtype=torch.float64, device=DEV)
    cnt_w = torch.empty(2, K, dtype=torch.int64, device=DEV)
    obj_w = torch.empty(2, dtype=torch.float64, device=DEV)
    for w, (a, b) in enumerate([(0, 13001), (13001, 30000)]):
        ws = m.workspace(b - a, d, K, torch.float32, "l2")
        cnt = torch.empty(K, dtype=torch.int32, device=DEV)
        off = torch.empty(K + 1, dtype=torch.int32, device=DEV)
        obj = torch.empty(1, dtype=torch.float64, device=DEV)
        m.fk_update_partial(Xg[a:b].contiguous(), lab[a:b].contiguous(), C0.to(DEV),
                            sums_w[w], cnt, off, ws, objective=obj)
        cnt_w[w] = cnt.to(torch.int64)
        obj_w[w] = obj[0]
    C_new = torch.empty(K, d, device=DEV)
    counts = torch.empty(K, dtype=torch.int64, device=DEV)
    objective = torch.empty(1, dtype=torch.float64, device=DEV)
    m.fk_finalize_shards(sums_w, cnt_w, C0.to(DEV), C_new, objectives_w=obj_w, counts=counts,
                         objective=objective)
    assert (counts.cpu().numpy() == full["counts"]).all()
    assert centroid_rel_err(C_new.cpu().numpy(), full["C_new"]) <= 1e-6
    # The objective's per-row terms are fp32 and are summed in fp32 within a batch of at most
    # 16 rows before going to fp64. Shard boundaries move those batches, so the two sums
    # can differ by up to 16 fp32 roundings of the objective's size (16 * 2^-24 < 1e-6).
    assert abs(objective.item() - full["J"]) <= 1e-6 * full["J"]


def test_lloyd_sharded_one_rank_equals_fk_lloyd():
    """The data-parallel loop on one NCCL rank reproduces fk_lloyd bit for bit."""
    import os
    import socket
    import torch.distributed as dist
    from exact_lloyd_means_b200.dist import gpu_ops, lloyd_sharded
    m = fk()
    X, C0, _ = _mixture(40000, 128, 200, seed=22, centers="normal", sigma=0.3)
    Xg = X.to(DEV)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1)
    try:
        C1 = C0.to(DEV).clone()
        objs1, counts1 = lloyd_sharded(Xg, C1, 4, gpu_ops(40000, 128, 200,
                                                            torch.float32, DEV))
    finally:
        dist.destroy_process_group()
    C2 = C0.to(DEV).clone()
    labels = torch.empty(40000, dtype=torch.int32, device=DEV)
    counts2 = torch.empty(200, dtype=torch.int32, device=DEV)
    objs2, _ = m.fk_lloyd(Xg, C2, 4, labels, m.workspace(40000, 128, 200), counts=counts2)
    assert torch.equal(C1, C2)
    assert objs1 == objs2
    assert torch.equal(counts1.cpu(), counts2.cpu().to(torch.int64))


@pytest.mark.parametrize("N,d", [(1000, 64), (4097, 100), (300, 768)])
def test_split_points_planes_are_rounded_hi_lo(N, d):
    """fk_split_points: hi = RN_bf16(x), lo = RN_bf16(x - hi), zero padding to d_p = 64k,
    compared with PyTorch's own round-to-nearest-even casts."""
    m = fk()
    g = torch.Generator().manual_seed(N + d)
    X = torch.randn(N, d, generator=g) * torch.logspace(-3, 3, d)
    sp = m.fk_split_points(X.to(DEV))
    P = sp.planes.cpu()
    dp = (d + 63) // 64 * 64
    assert tuple(P.shape) == (2, N, dp)
    hi = X.to(torch.bfloat16)
    lo = (X - hi.float()).to(torch.bfloat16)
    assert torch.equal(P[0, :, :d].view(torch.int16), hi.view(torch.int16))
    assert torch.equal(P[1, :, :d].view(torch.int16), lo.view(torch.int16))
    assert not P[:, :, d:].float().any()
    norms = sp.norms.cpu().double()
    assert torch.allclose(norms, (X.double() ** 2).sum(1), rtol=1e-6, atol=0)


@pytest.mark.parametrize("N,d,K", [(20000, 128, 300), (5000, 768, 1000), (3001, 64, 37),
                                   (40000, 256, 300), (20000, 1024, 500)])
def test_assign_pre_split_points_equals_fp32_assign(N, d, K):
    """fk_assign_split (the fp32 rows plus their fk_split_points planes) gives the fp32
    call's labels and minimum distances bit for bit, on the three-product route, the
    screened route (40000 x 256) and the deep route (d = 1024)."""
    m = fk()
    X, C0, _ = _mixture(N, d, K, seed=N + K, centers="normal", sigma=0.3)
    Xg, Cg = X.to(DEV), C0.to(DEV)
    ws = m.workspace(N, d, K)
    l1 = torch.empty(N, dtype=torch.int32, device=DEV)
    l2 = torch.empty(N, dtype=torch.int32, device=DEV)
    d1 = torch.empty(N, dtype=torch.float32, device=DEV)
    d2 = torch.empty(N, dtype=torch.float32, device=DEV)
    m.fk_assign(Xg, Cg, l1, ws, mind=d1)
    sp = m.fk_split_points(Xg)
    assert sp.source is not None  # through fk_assign_split
    m.fk_assign(sp, Cg, l2, ws, mind=d2)
    assert torch.equal(l1, l2) and torch.equal(d1, d2)


@pytest.mark.parametrize("N,d,K", [(40000, 256, 300), (30000, 768, 1024), (3001, 64, 37)])
def test_assign_planes_only_matches_oracle(N, d, K):
    """FK_BF16X2 planes without the fp32 rows: the screened route re-ranks from hi + lo
    (within 2^-16 |x| of x), which must still match the oracle outside the tie window, at
    screened shapes (N >= 18,944, d >= 256) and on the three-product route."""
    m = fk()
    X, C0, _ = _mixture(N, d, K, seed=N + K + 1, centers="normal", sigma=0.3)
    sp = m.fk_split_points(X.to(DEV))
    planes_only = m.SplitPoints(sp.buf, N, d)  # no source rows: dtype FK_BF16X2
    ref, dmin, d2nd = oracle.assign(X, C0.numpy())
    ties = oracle.tie_mask(X, C0.numpy(), dmin, d2nd)
    labels = torch.full((N,), -7, dtype=torch.int32, device=DEV)
    ws = m.workspace(N, d, K)
    m.fk_assign(planes_only, C0.to(DEV), labels, ws)
    assert m.fk_get_device_error(ws) == m.FK_OK
    lab = labels.cpu().numpy()
    assert (lab >= 0).all() and (lab < K).all()
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,d", [(1000, 96), (257, 768), (1, 8)])
def test_centroid_norms_match_oracle(K, d, dtype):
    """fk_centroid_norms: ||c||^2 of the values the tensor cores consume (bf16-rounded for
    bf16), against the oracle's fp64 distance of each centroid to the origin, rounded once
    to fp32: within one fp32 ulp (the two fp64 sums differ only in order)."""
    m = fk()
    g = torch.Generator().manual_seed(K + d)
    C = torch.randn(K, d, generator=g) * torch.logspace(-2, 2, K).unsqueeze(1)
    cn = torch.full((K,), float("nan"), dtype=torch.float32, device=DEV)
    m.fk_centroid_norms(C.to(DEV), cn, torch.bfloat16 if dtype == "bf16" else torch.float32)
    Cref = oracle.round_bf16(C.numpy()) if dtype == "bf16" else C.numpy()
    _, n2, _ = oracle.assign(Cref, np.zeros((1, d)))  # ||c - 0||^2 in fp64
    ref = n2.astype(np.float32)
    got = cn.cpu().numpy()
    ulp = np.spacing(np.abs(ref))
    assert (np.abs(got.astype(np.float64) - ref) <= ulp).all()


# Deep fp32 points (d rounded up to 64 above 768): no label is decided by the three-product
# form.  At any N every row is screened and re-ranked in fp64, and rows whose candidates
# overflow get an exact fp64 scan over all centroids.
DEEP_CASES = [(6000, 1024, 500, "normal", 0.3), (3001, 1032, 257, "normal", 0.3),
              (25000, 1024, 2000, "normal", 0.3), (700, 1536, 40, "uniform", 0.2),
              (200, 832, 1, "normal", 0.3)]


@pytest.mark.parametrize("N,d,K,centers,sigma", DEEP_CASES)
def test_deep_fp32_assign_matches_oracle(N, d, K, centers, sigma):
    X, _, _ = gaussian_mixture(N, d, K, centers=centers, sigma=sigma, seed=N + d)
    C0 = X[init_indices(N, K, N + d)].float().contiguous()
    ref, dmin, d2nd = oracle.assign(X, C0.numpy())
    ties = oracle.tie_mask(X, C0.numpy(), dmin, d2nd)
    lab, mind = gpu_assign(X.to(DEV), C0.to(DEV), with_mind=True)
    assert (lab >= 0).all() and (lab < K).all()
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"
    # mind is the fp64 difference form rounded to fp32 on this route
    assert (np.abs(mind.astype(np.float64) - dmin) <= 2 ** -23 * dmin + 1e-30).all()


def test_deep_fp32_overflow_rows_take_the_exact_scan():
    """d = 1024: 30 distinct centroids, each present 20 times, so every row's nearest
    value is shared by 20 columns and its 16-slot candidate list overflows: every label
    comes from the exact fp64 scan, which must pick the lowest of the copies."""
    N, d = 4000, 1024
    X, _, _ = gaussian_mixture(N, d, 30, centers="normal", sigma=0.3, seed=77)
    base = X[init_indices(N, 30, 77)].float()
    C = base.repeat(20, 1).contiguous()  # column 30 * r + j is a copy of base[j]
    lab, mind = gpu_assign(X.to(DEV), C.to(DEV), with_mind=True)
    ref, dmin, d2nd = oracle.assign(X, base.numpy())
    ties = oracle.tie_mask(X, base.numpy(), dmin, d2nd)
    assert label_mismatches(lab, ref, ties) == 0
    assert (lab[~ties] < 30).all()
    assert (np.abs(mind.astype(np.float64) - dmin) <= 2 ** -23 * dmin + 1e-30).all()


@pytest.mark.parametrize("N,d,K", [(40000, 256, 300), (4000, 256, 300), (3000, 1024, 200),
                                   (20000, 128, 1000)])
def test_assign_adversarial_roundings_match_oracle(N, d, K):
    """The near-worst-case operands of the window bounds, on the hardware: the screened
    route (40000 x 256), the three-product route (4000 x 256 and 20000 x 128) and the deep
    route (d = 1024) must all match the oracle outside the tie window."""
    X = adversarial_rows(N, d, seed=N + d + K)
    C0 = X[init_indices(N, K, 5)].contiguous()
    C = (C0 * 1.0001).contiguous()  # centroids near, not on, their rows
    ref, dmin, d2nd = oracle.assign(X, C.numpy())
    ties = oracle.tie_mask(X, C.numpy(), dmin, d2nd)
    lab, _ = gpu_assign(X.to(DEV), C.to(DEV))
    assert (lab >= 0).all() and (lab < K).all()
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"
    print(f"adversarial {N}x{d}, K={K}: {int(ties.sum())} tie points")


# Screened fp32 assignment: for fp32 points with d >= 256 or K * d >= 2^22 at CTA-pair
# sizes (N >= 2 * 128 * 148 / 2) the single-product pass keeps the columns inside a proven error window, the candidates
# are re-ranked exactly, and rows whose candidates do not fit are assigned by the
# three-product pass.  These cases drive each branch: ordinary mixtures (few candidates),
# components that received several initial centroids (several candidates), exact
# duplicates (ties resolved to the lowest index), and a Zipf mixture whose heavy
# components hold hundreds of nearly equidistant centroids (the overflow path).
SCREEN_CASES = [
    ("normal", 40000, 256, 300, "equal", 0.3),
    ("normal", 30000, 768, 1024, "equal", 0.3),
    ("uniform", 50001, 320, 4100, "equal", 0.2),
    ("normal", 40000, 256, 2000, "zipf", 0.15),
    ("normal", 20000, 1032, 700, "equal", 0.3),
    ("normal", 40000, 128, 32768, "equal", 0.25),
]


@pytest.mark.parametrize("centers,N,d,K,weights,sigma", SCREEN_CASES)
def test_screened_assign_matches_oracle(centers, N, d, K, weights, sigma):
    X, comp, _ = gaussian_mixture(N, d, K, centers=centers, sigma=sigma, weights=weights,
                                  seed=N + K)
    C0 = X[init_indices(N, K, N + K)].float().contiguous()
    ref, dmin, d2nd = oracle.assign(X, C0.numpy())
    ties = oracle.tie_mask(X, C0.numpy(), dmin, d2nd)
    lab, mind = gpu_assign(X.to(DEV), C0.to(DEV), with_mind=True)
    assert (lab >= 0).all() and (lab < K).all()
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"
    Xd = X.double().numpy()
    s = (Xd * Xd).sum(1) + (C0.double().numpy() ** 2).sum(1).max()
    assert (np.abs(mind.astype(np.float64) - dmin) <= 1e-4 * s).all()


def test_screened_assign_duplicates_take_lowest_index():
    """30 distinct centroids, each present 10 times at scattered columns: every row's
    nearest value is shared by 10 columns, which overflows some column groups; the label
    must be the lowest of the 10 (bit-identical values), whichever pass decides it."""
    N, d = 40000, 256
    X, _, _ = gaussian_mixture(N, d, 30, centers="normal", sigma=0.3, seed=31)
    base = X[init_indices(N, 30, 31)].float()
    C = base.repeat(10, 1).contiguous()  # column 30 * r + j is a copy of base[j]
    lab, _ = gpu_assign(X.to(DEV), C.to(DEV))
    ref, dmin, d2nd = oracle.assign(X, base.numpy())
    ties = oracle.tie_mask(X, base.numpy(), dmin, d2nd)
    assert label_mismatches(lab, ref, ties) == 0  # and so the lowest copy, column < 30
    assert (lab[~ties] < 30).all()


def test_screened_lloyd_lockstep_heavy_components():
    """Lockstep iterations on a Zipf mixture (many centroids per heavy component)."""
    X, _, _ = gaussian_mixture(40000, 256, 1500, centers="normal", sigma=0.15,
                               weights="zipf", seed=33)
    C0 = X[init_indices(40000, 1500, 33)].float().contiguous()
    ref = oracle.lloyd(X, C0, 2)
    Xg = X.to(DEV)
    C_master = [C0.double().numpy()] + ref["C_next"]
    for t in range(2):
        Cm = torch.as_tensor(C_master[t], dtype=torch.float32)
        lab, _ = gpu_assign(Xg, Cm.to(DEV))
        assert label_mismatches(lab, ref["labels"][t], ref["ties"][t]) == 0, t


def test_screened_lloyd_deterministic_and_resumable():
    """The screened route gives the same bits run to run (its fallback queue's order
    varies with scheduling, the labels do not), and 2 + 2 iterations equal 4."""
    X, _, _ = gaussian_mixture(40000, 256, 600, centers="normal", sigma=0.3, seed=41)
    C0 = X[init_indices(40000, 600, 41)].float().contiguous()
    m = fk()
    Xg = X.to(DEV)
    ws = m.workspace(40000, 256, 600, torch.float32, "l2")

    def run(C, n):
        labels = torch.empty(40000, dtype=torch.int32, device=DEV)
        objs, tm = m.fk_lloyd(Xg, C, n, labels, ws, timing=True)
        assert tm["screened"] == n  # the screened route was taken
        return C, labels, objs

    a = run(C0.to(DEV).clone(), 4)
    b = run(C0.to(DEV).clone(), 4)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and a[2] == b[2]
    c = run(C0.to(DEV).clone(), 2)
    d = run(c[0].clone(), 2)
    assert torch.equal(d[0], a[0]) and torch.equal(d[1], a[1]) and d[2] == a[2][2:]


IVF_CASES = [(1000, 64, 10, "equal"), (70001, 128, 1024, "zipf"), (20000, 768, 300, "equal"),
             (5000, 8, 1, "equal"), (3000, 1032, 2500, "equal")]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,K,weights", IVF_CASES)
def test_ivf_lists_match_oracle(N, d, K, weights, dtype):
    """fk_ivf_lists: offsets and row ids bit-exact against the oracle's stable CSR, and the
    gathered rows bit-exact against X[row_ids] (empty cells included)."""
    m = fk()
    X, comp, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, weights=weights,
                                  dtype=dtype, seed=N + K)
    lab = comp.numpy().astype(np.int32)
    _, off_ref, perm_ref = oracle.csr(lab, K)
    Xg = X.to(DEV)
    offsets = torch.full((K + 1,), -1, dtype=torch.int32, device=DEV)
    row_ids = torch.full((N,), -1, dtype=torch.int32, device=DEV)
    X_lists = torch.empty_like(Xg)
    ws = m.workspace(N, d, K, Xg.dtype, "l2")
    m.fk_ivf_lists(Xg, torch.as_tensor(lab).to(DEV), K, offsets, row_ids, ws, X_lists=X_lists)
    assert m.fk_get_device_error(ws) == m.FK_OK
    assert (offsets.cpu().numpy() == off_ref).all()
    assert (row_ids.cpu().numpy() == perm_ref).all()
    assert torch.equal(X_lists.cpu().view(torch.int16 if dtype == "bf16" else torch.int32),
                       X[perm_ref].view(torch.int16 if dtype == "bf16" else torch.int32))
    # without the gather: the same ids
    row2 = torch.empty_like(row_ids)
    m.fk_ivf_lists(Xg, torch.as_tensor(lab).to(DEV), K, offsets, row2, ws)
    assert torch.equal(row2, row_ids)


@pytest.mark.parametrize("dtype,metric,d", [("f32", "l2", 128), ("f32", "cosine", 256),
                                            ("bf16", "l2", 128), ("f32", "l2", 768)])
def test_lloyd_streamed_matches_oracle_and_fk_lloyd(dtype, metric, d):
    """fk_lloyd_streamed (points in pinned host memory, 4 chunks with a ragged last one)
    against the oracle on the first iteration (labels outside ties, centroids, objective)
    and against fk_lloyd on the same data (objectives and centroids)."""
    m = fk()
    N, K = 150001, 500
    X, _, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, dtype=dtype, seed=51)
    C0 = X[init_indices(N, K, 51)].float().contiguous()
    prec = "bf16" if dtype == "bf16" else "f32"
    ref = oracle.lloyd(X, C0, 1, metric=metric, precision=prec)
    Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
    Xh.copy_(X)
    labels = torch.empty(N, dtype=torch.int32, pin_memory=True)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = m.streamed_workspace(40000, d, K, tdt, metric)
    C = C0.to(DEV).clone()
    objs = m.fk_lloyd_streamed(Xh, C, 1, ws, 40000, metric=metric, labels=labels)
    lab = labels.numpy()
    assert label_mismatches(lab, ref["labels"][0], ref["ties"][0]) == 0
    assert abs(objs[0] - ref["J"][0]) <= OBJECTIVE_TOL * ref["J"][0]
    if not ref["ties"][0].any():
        assert centroid_rel_err(C.cpu().numpy(), ref["C_next"][0]) <= CENTROID_TOL
    # three iterations against fk_lloyd on the device copy
    C1 = C0.to(DEV).clone()
    objs1 = m.fk_lloyd_streamed(Xh, C1, 3, ws, 40000, metric=metric)
    C2 = C0.to(DEV).clone()
    lab2 = torch.empty(N, dtype=torch.int32, device=DEV)
    objs2, _ = m.fk_lloyd(X.to(DEV), C2, 3, lab2, m.workspace(N, d, K, tdt, metric),
                          metric=metric)
    for a, b in zip(objs1, objs2):
        assert abs(a - b) <= 1e-6 * b
    assert centroid_rel_err(C1.cpu().numpy(), C2.cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("case", ["threshold_rows", "ragged_d", "k_equals_n", "zero_rows"])
def test_screened_assign_edge_cases(case):
    """Screened-route edges: N exactly at the CTA-pair threshold (2 * 128 * 148 / 2 rows),
    d not a multiple of 64 (padded operand columns), K = N (every point its own centroid,
    256-column tiles full of near-ties), and all-zero rows (every centroid at distance
    ||c||^2: ties resolved to the lowest index of the smallest norm)."""
    g = torch.Generator().manual_seed(61)
    if case == "threshold_rows":
        X, _, _ = gaussian_mixture(18944, 256, 300, centers="normal", sigma=0.3, seed=61)
        C = X[init_indices(18944, 300, 61)].float().contiguous()
    elif case == "ragged_d":
        X, _, _ = gaussian_mixture(30001, 260, 700, centers="normal", sigma=0.3, seed=62)
        C = X[init_indices(30001, 700, 62)].float().contiguous()
    elif case == "k_equals_n":
        X, _, _ = gaussian_mixture(20000, 256, 20000, centers="normal", sigma=0.3, seed=63)
        C = X.clone()
    else:
        X, _, _ = gaussian_mixture(20000, 256, 400, centers="normal", sigma=0.3, seed=64)
        X[::7] = 0.0
        C = X[init_indices(20000, 400, 64)].float().contiguous()
    ref, dmin, d2nd = oracle.assign(X, C.numpy())
    ties = oracle.tie_mask(X, C.numpy(), dmin, d2nd)
    lab, _ = gpu_assign(X.to(DEV), C.to(DEV))
    assert label_mismatches(lab, ref, ties) == 0, f"ties={int(ties.sum())}"
    if case == "k_equals_n":
        assert (lab == np.arange(20000)).all()


def test_fk_lloyd_reports_cluster_statistics():
    """fk_timing's last-iteration statistics: empty clusters and the largest cluster agree
    with the returned counts; the screened route's fallback count is within [0, N]."""
    m = fk()
    N, d, K = 40000, 256, 300
    X, _, _ = gaussian_mixture(N, d, 200, centers="normal", sigma=0.3, seed=61)
    C0 = X[init_indices(N, K, 61)].float().contiguous()
    C0[:5] = 1e3  # far away: these clusters stay empty
    Xg, C = X.to(DEV), C0.to(DEV)
    labels = torch.empty(N, dtype=torch.int32, device=DEV)
    counts = torch.empty(K, dtype=torch.int32, device=DEV)
    ws = m.workspace(N, d, K, torch.float32, "l2")
    _, tm = m.fk_lloyd(Xg, C, 3, labels, ws, counts=counts, timing=True)
    c = counts.cpu().numpy()
    assert tm["empty_clusters"] == int((c == 0).sum()) >= 5
    assert tm["max_cluster"] == int(c.max())
    assert 0 <= tm["fallback_rows"] <= N
    assert tm["screened"] in (0, 3)
    if tm["screened"] == 0:
        assert tm["fallback_rows"] == 0


def test_fault_injection_launch_fails_before_device_work():
    """FK_FAULT=launch (in a child process): fk_lloyd and fk_ivf_search return FK_ERR_CUDA
    and launch nothing."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, torch\n"
        f"sys.path.insert(0, {root!r})\n"
        "from exact_lloyd_means_b200 import fk\n"
        "X = torch.randn(4096, 64, device='cuda'); C = X[:16].clone()\n"
        "lab = torch.empty(4096, dtype=torch.int32, device='cuda')\n"
        "ws = fk.workspace(4096, 64, 16)\n"
        "n0 = fk.launch_count()\n"
        "try:\n"
        "    fk.fk_lloyd(X, C, 2, lab, ws)\n"
        "    print('no error')\n"
        "except fk.FkError as e:\n"
        "    print(e.status, fk.launch_count() - n0)\n")
    env = dict(os.environ, FK_FAULT="launch")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr
    status, launched = (int(x) for x in out.stdout.split())
    assert status == fk().FK_ERR_CUDA and launched == 0
