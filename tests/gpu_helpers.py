"""Shared helpers for the GPU parity tests: call the C ABI, compare with the oracle under
the parity rules (labels bit-exact outside tie points, centroids within a normwise
relative tolerance, objective within a relative tolerance)."""
import numpy as np
import torch

CENTROID_TOL = 1e-5   # given identical labels, per-centroid max |dc| / max |c_ref|
OBJECTIVE_TOL = 1e-5  # relative


def fk():
    from exact_lloyd_means_b200 import fk as m
    return m


def gpu_assign(X, C, with_mind=False):
    """X on the GPU (fp32 or bf16), C fp32 on the GPU -> labels (and mind) on the CPU."""
    m = fk()
    N, d = X.shape
    K = C.shape[0]
    labels = torch.full((N,), -7, dtype=torch.int32, device=X.device)
    mind = torch.empty(N, dtype=torch.float32, device=X.device) if with_mind else None
    ws = m.workspace(N, d, K, X.dtype, "l2")
    m.fk_assign(X, C, labels, ws, mind=mind)
    assert m.fk_get_device_error(ws) == m.FK_OK
    return labels.cpu().numpy(), (mind.cpu().numpy() if with_mind else None)


def gpu_update(X, labels, C_old, want_perm=True):
    """Returns dict of counts, offsets, perm, C_new (fp32, CPU numpy) and objective."""
    m = fk()
    N, d = X.shape
    K = C_old.shape[0]
    dev = X.device
    lab = torch.as_tensor(np.asarray(labels, dtype=np.int32)).to(dev)
    C_new = torch.full((K, d), float("nan"), dtype=torch.float32, device=dev)
    counts = torch.full((K,), -1, dtype=torch.int32, device=dev)
    offsets = torch.full((K + 1,), -1, dtype=torch.int32, device=dev)
    perm = torch.full((N,), -1, dtype=torch.int32, device=dev) if want_perm else None
    obj = torch.full((1,), float("nan"), dtype=torch.float64, device=dev)
    ws = m.workspace(N, d, K, X.dtype, "l2")
    m.fk_update(X, lab, C_old, C_new, counts, offsets, ws, perm=perm, objective=obj)
    assert m.fk_get_device_error(ws) == m.FK_OK
    return {"counts": counts.cpu().numpy(), "offsets": offsets.cpu().numpy(),
            "perm": perm.cpu().numpy() if want_perm else None,
            "C_new": C_new.cpu().numpy().astype(np.float64), "J": obj.item()}


def label_mismatches(gpu_labels, ref_labels, ties):
    """Number of points outside the tie set whose labels differ."""
    return int(((np.asarray(gpu_labels) != np.asarray(ref_labels)) & ~ties).sum())


def centroid_rel_err(C, C_ref):
    C = np.asarray(C, dtype=np.float64)
    C_ref = np.asarray(C_ref, dtype=np.float64)
    scale = np.abs(C_ref).max(axis=1)
    err = np.abs(C - C_ref).max(axis=1)
    return float((err / np.maximum(scale, 1e-300)).max())
