"""fk_assign_noalloc: the assignment step for callers that cannot allocate device memory
(code under another framework's memory manager, or on a path where cudaMalloc would
synchronise the device).  Its scratch lives in a static device array inside libfk, so it
must give the same labels as fk_assign, which takes its scratch from a caller workspace,
and, like it, the oracle's labels outside the parity tie window.

Collected last on purpose (file name), so a run that stops at the first failure has run
every other test first; it also passes alone in a fresh process.  Labels are integers
decided by the same kernel arithmetic on both paths, so the comparison with fk_assign is
bit-exact."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from synth import gaussian_mixture, init_indices

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

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


def test_noalloc_assign_matches_oracle_outside_the_tie_window():
    """Against the fp64 oracle (labels outside the tie window), twice in a row, for fp32
    (three-product route) and bf16 points (the oracle assigns with the bf16-rounded
    centroids the kernel uses)."""
    from exact_lloyd_means_b200 import fk
    for N, d, K, dtype in CASES:
        X, _, _ = gaussian_mixture(N, d, K, centers="normal", sigma=0.3, dtype=dtype,
                                   seed=N + K)
        C = X[init_indices(N, K, 1)].float().contiguous()
        Cref = oracle.round_bf16(C.numpy()) if dtype == "bf16" else C.numpy()
        ref, dmin, d2nd = oracle.assign(X, Cref)
        ties = oracle.tie_mask(X, Cref, dmin, d2nd)
        for call in range(2):
            labels = torch.full((N,), -1, dtype=torch.int32, device="cuda")
            fk.fk_assign_noalloc(X.cuda(), C.cuda(), labels)
            got = labels.cpu().numpy()
            bad = int(((got != ref) & ~ties).sum())
            assert bad == 0, (N, d, K, dtype, call, int(ties.sum()))


def test_noalloc_refuses_deep_fp32_points():
    """fp32 points deeper than 768 (rounded up to 64) always take fk_assign's screened
    route, whose buffers the static array does not hold: refused, nothing launched."""
    from exact_lloyd_means_b200 import fk
    X = torch.randn(500, 1024, device="cuda")
    labels = torch.empty(500, dtype=torch.int32, device="cuda")
    n0 = fk.launch_count()
    with pytest.raises(fk.FkError) as e:
        fk.fk_assign_noalloc(X, X[:20].clone(), labels)
    assert e.value.status == fk.FK_ERR_UNSUPPORTED
    assert fk.launch_count() == n0


def test_noalloc_injected_launch_failure():
    """FK_FAULT=launch (read when the library is first used, so in a child process): the
    call fails as a failed launch would, FK_ERR_CUDA, and launches nothing."""
    code = (
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "from exact_lloyd_means_b200 import fk\n"
        "X = torch.randn(1000, 64, device='cuda')\n"
        "labels = torch.empty(1000, dtype=torch.int32, device='cuda')\n"
        "n0 = fk.launch_count()\n"
        "try:\n"
        "    fk.fk_assign_noalloc(X, X[:10].clone(), labels)\n"
        "    print(0, fk.launch_count() - n0)\n"
        "except fk.FkError as e:\n"
        "    print(e.status, fk.launch_count() - n0)\n")
    env = dict(os.environ, FK_FAULT="launch")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    from exact_lloyd_means_b200 import fk
    status, launched = (int(x) for x in out.stdout.split())
    assert status == fk.FK_ERR_CUDA and launched == 0


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
