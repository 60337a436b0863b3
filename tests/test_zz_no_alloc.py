"""fk_assign_noalloc: the assignment step for callers that cannot allocate device memory
(code under another framework's memory manager, or on a path where cudaMalloc would
synchronise the device).  Its scratch lives in a static device array inside libfk, so it
must give the same labels as fk_assign, which takes its scratch from a caller workspace.

Collected last on purpose (file name), so a run that stops at the first failure has run
every other test first; it also passes alone in a fresh process.  Labels are integers
decided by the same kernel arithmetic on both paths, so the check is bit-exact."""
import numpy as np
import pytest
import torch

from synth import gaussian_mixture, init_indices

pytestmark = pytest.mark.gpu

CASES = [(5000, 128, 300, "f32"), (3001, 96, 257, "bf16"), (20000, 128, 1000, "bf16"),
         (1200, 64, 40, "f32")]


def _reference_labels(fk, X, C):
    N, d = X.shape
    labels = torch.empty(N, dtype=torch.int32, device=X.device)
    ws = fk.workspace(N, d, C.shape[0], X.dtype, "l2")
    fk.fk_assign(X, C, labels, ws)
    torch.cuda.synchronize()
    return labels.cpu().numpy()


def test_noalloc_assign_matches_workspace_assign_twice_in_a_row():
    from exact_lloyd_means_b200 import fk
    for N, d, K, dtype in CASES:
        X, _, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, dtype=dtype,
                                   seed=N + K)
        C = X[init_indices(N, K, 1)].float().contiguous()
        Xg, Cg = X.cuda(), C.cuda()
        ref = _reference_labels(fk, Xg, Cg)
        for call in range(2):  # the static array keeps the previous call's contents
            labels = torch.full((N,), -1, dtype=torch.int32, device="cuda")
            fk.fk_assign_noalloc(Xg, Cg, labels)
            got = labels.cpu().numpy()
            assert np.array_equal(got, ref), (N, d, K, dtype, call)


def test_noalloc_rejects_problems_beyond_the_static_limit():
    from exact_lloyd_means_b200 import fk
    N, d, K = 20000, 128, 256  # fp32 X planes alone need 4 * N * 128 = 10 MB > 8 MiB
    X = torch.randn(N, d, device="cuda")
    C = X[:K].clone()
    labels = torch.empty(N, dtype=torch.int32, device="cuda")
    with pytest.raises(fk.FkError) as e:
        fk.fk_assign_noalloc(X, C, labels)
    assert e.value.status == fk.FK_ERR_WORKSPACE
    # a problem that fits still works after the rejection
    small = X[:4000].contiguous()
    labels = torch.empty(4000, dtype=torch.int32, device="cuda")
    fk.fk_assign_noalloc(small, C, labels)
    assert np.array_equal(labels.cpu().numpy(), _reference_labels(fk, small, C))
