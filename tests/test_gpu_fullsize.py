"""Parity at the workloads' full sizes, in the launch configuration bench.py times
(fk_assign / fk_update / fk_lloyd run exactly the kernels and grids of a bench step).

The oracle cannot assign 10^7..10^8 points against 10^3..10^4 centroids in test time, so:
  * assign: every label is computed on the GPU; a seeded sample of rows is recomputed by
    the oracle one by one and must match outside the tie window;
  * update: the generator's component ids serve as labels (an input, so the cluster-size
    distribution is the workload's, Zipf included); counts and offsets are checked in full
    (numpy bincount on the same labels), centroids for a sample of clusters that always
    includes the largest one, and the objective over all N rows in chunks;
  * fk_lloyd: invariants that hold at any size (non-increasing objective, counts sum to N).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, IVF, LARGE, MID, ZIPF, gaussian_mixture, init_indices
from tests.gpu_helpers import CENTROID_TOL, OBJECTIVE_TOL, centroid_rel_err, fk

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLE_ROWS = {IVF: 1024, MID: 4096, ZIPF: 1024, LARGE: 768}


def _data(cfg):
    spec = CONFIGS[cfg]
    X, comp, _ = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers,
                                  sigma=spec.sigma, weights=spec.weights, zipf_s=spec.zipf_s,
                                  dtype=spec.dtype, seed=spec.seed, device="cuda")
    C0 = X[init_indices(spec.n, spec.k, spec.seed, device="cuda")].float().contiguous()
    return spec, X, comp, C0


def _rows64(X, idx):
    return X[torch.as_tensor(idx, device=X.device)].double().cpu().numpy()


def _oracle_normalized_f32(X, chunk=1 << 17):
    """The oracle's normalisation of every row, rounded to fp32 (in chunks), as a CPU
    tensor: an input both sides can share."""
    out = torch.empty(X.shape, dtype=torch.float32)
    for r0 in range(0, X.shape[0], chunk):
        r1 = min(X.shape[0], r0 + chunk)
        out[r0:r1] = torch.from_numpy(
            oracle.round_f32(oracle.normalize_rows(X[r0:r1].cpu())).astype(np.float32))
    return out


@pytest.mark.parametrize("cfg", [IVF, MID, ZIPF, LARGE])
def test_fullsize_assign_sampled_rows(cfg):
    spec, X, _, C0 = _data(cfg)
    m = fk()
    Xa = X
    if spec.metric == "cosine":
        # the product path normalises the points (fk_normalize_rows); the centroids both
        # sides assign with are the oracle's normalisation of C0, rounded to fp32
        Xa = torch.empty_like(X)
        m.fk_normalize_rows(X, Xa)
        C0 = _oracle_normalized_f32(C0).to("cuda")
    labels = torch.empty(spec.n, dtype=torch.int32, device="cuda")
    ws = m.workspace(spec.n, spec.d, spec.k, X.dtype, "l2")
    m.fk_assign(Xa, C0, labels, ws)
    assert m.fk_get_device_error(ws) == m.FK_OK
    lab = labels.cpu().numpy()
    assert lab.min() >= 0 and lab.max() < spec.k
    del ws
    rng = np.random.default_rng(len(cfg))
    idx = np.sort(rng.choice(spec.n, SAMPLE_ROWS[cfg], replace=False))
    Xs = _rows64(X, idx)
    C = C0.double().cpu().numpy()
    if spec.metric == "cosine":
        Xs = oracle.normalize_rows(Xs)  # the oracle normalises the raw rows itself
    if spec.dtype == "bf16":
        C = oracle.round_bf16(C)
    ref, dmin, d2nd = oracle.assign(Xs, C)
    ties = oracle.tie_mask(Xs, C, dmin, d2nd)
    bad = int(((lab[idx] != ref) & ~ties).sum())
    print(f"{cfg}: {len(idx)} sampled rows, {int(ties.sum())} tie points, {bad} bad")
    assert bad == 0


@pytest.mark.parametrize("cfg", [IVF, MID, ZIPF, LARGE])
def test_fullsize_update_given_labels(cfg):
    spec, X, comp, C0 = _data(cfg)
    m = fk()
    K = spec.k
    if spec.metric == "cosine":
        # the update of the cosine workload sees normalised points: both sides take the
        # oracle's normalisation, rounded to fp32
        X = _oracle_normalized_f32(X).to("cuda")
        C0 = _oracle_normalized_f32(C0).to("cuda")
    labels = comp.to("cuda")
    C_new = torch.empty_like(C0)
    counts = torch.empty(K, dtype=torch.int32, device="cuda")
    offsets = torch.empty(K + 1, dtype=torch.int32, device="cuda")
    obj = torch.empty(1, dtype=torch.float64, device="cuda")
    ws = m.workspace(spec.n, spec.d, K, X.dtype, "l2")
    m.fk_update(X, labels, C0, C_new, counts, offsets, ws, objective=obj)
    assert m.fk_get_device_error(ws) == m.FK_OK
    del ws
    lab = comp.cpu().numpy()
    cnt_ref = np.bincount(lab, minlength=K)
    assert (counts.cpu().numpy() == cnt_ref).all()
    off_ref = np.concatenate([[0], np.cumsum(cnt_ref)])
    assert (offsets.cpu().numpy() == off_ref).all()

    # centroids of sampled clusters (the largest always among them)
    rng = np.random.default_rng(100 + len(cfg))
    nonempty = np.flatnonzero(cnt_ref)
    pick = np.unique(np.concatenate([[int(np.argmax(cnt_ref))],
                                     rng.choice(nonempty, min(64, len(nonempty)),
                                                replace=False)]))
    sel = np.flatnonzero(np.isin(lab, pick))
    Xs = _rows64(X, sel)
    remap = {k: j for j, k in enumerate(pick)}
    lab_s = np.array([remap[k] for k in lab[sel]], dtype=np.int32)
    C_ref = oracle.update(Xs, lab_s, np.zeros((len(pick), spec.d)))
    Cg = C_new.cpu().double().numpy()[pick]
    assert centroid_rel_err(Cg, C_ref) <= CENTROID_TOL
    empty = cnt_ref == 0
    if empty.any():
        assert torch.equal(C_new[torch.as_tensor(np.flatnonzero(empty), device="cuda")],
                           C0[torch.as_tensor(np.flatnonzero(empty), device="cuda")])

    # objective over all rows, oracle in chunks of the same labels
    Cu = C0.double().cpu().numpy()
    if spec.dtype == "bf16":
        Cu = oracle.round_bf16(Cu)
    J = 0.0
    step = 1 << 21
    for r0 in range(0, spec.n, step):
        r1 = min(spec.n, r0 + step)
        J += oracle.objective(X[r0:r1].double().cpu().numpy(), Cu, lab[r0:r1])
    assert abs(obj.item() - J) <= OBJECTIVE_TOL * J


@pytest.mark.parametrize("cfg", [MID, ZIPF])
def test_fullsize_lloyd_invariants(cfg):
    spec, X, _, C0 = _data(cfg)
    m = fk()
    labels = torch.empty(spec.n, dtype=torch.int32, device="cuda")
    counts = torch.empty(spec.k, dtype=torch.int32, device="cuda")
    offsets = torch.empty(spec.k + 1, dtype=torch.int32, device="cuda")
    ws = m.workspace(spec.n, spec.d, spec.k, X.dtype, spec.metric)
    C = C0.clone()
    objs, _ = m.fk_lloyd(X, C, 3, labels, ws, metric=spec.metric, counts=counts,
                         offsets=offsets)
    for t in range(1, len(objs)):
        assert objs[t] <= objs[t - 1] * (1 + 1e-6)
    cnt = counts.cpu().numpy()
    off = offsets.cpu().numpy()
    assert cnt.sum() == spec.n and off[0] == 0 and off[-1] == spec.n
    assert (np.diff(off) == cnt).all()
    assert (np.bincount(labels.cpu().numpy(), minlength=spec.k) == cnt).all()
    assert torch.isfinite(C).all()
