"""The data-parallel (N > 1 ranks) path on CPU: two gloo ranks, each holding half of the
points, run exact_lloyd_means_b200.dist.lloyd_sharded with stand-in local steps (the fp64
oracle for the assignment, per-cluster sums for the partial update, and a rank-order
combine rounded once to fp32 like the GPU's).  The result must equal the single-process
oracle Lloyd on all the points: the exchange (gather order, combine, counts, objective)
is what is under test."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _data():
    from synth import gaussian_mixture, init_indices
    X, _, _ = gaussian_mixture(3001, 16, 7, centers="normal", sigma=0.4, seed=5)
    C0 = X[init_indices(3001, 7, 5)].clone()
    return X, C0


def _stand_in_ops():
    import oracle
    from exact_lloyd_means_b200.dist import LocalOps

    def assign(X, C):
        lab, _, _ = oracle.assign(X.numpy(), C.numpy())
        return torch.from_numpy(lab)

    def partial(X, lab, C):
        K, d = C.shape
        Xd = X.double().numpy()
        lab = lab.numpy()
        sums = np.zeros((K, d))
        for k in range(K):
            sums[k] = Xd[lab == k].sum(axis=0)
        cnt = np.bincount(lab, minlength=K).astype(np.int64)
        obj = oracle.objective(Xd, C.double().numpy(), lab)
        return (torch.from_numpy(sums), torch.from_numpy(cnt),
                torch.tensor([obj], dtype=torch.float64))

    def finalize(sums_w, counts_w, objs_w, C_old):
        S = torch.zeros_like(sums_w[0])
        n = torch.zeros_like(counts_w[0])
        for w in range(sums_w.shape[0]):  # rank order
            S += sums_w[w]
            n += counts_w[w]
        C_new = C_old.clone()
        nz = n > 0
        C_new[nz] = (S[nz] / n[nz].double()[:, None]).float()
        return C_new, n, objs_w.sum().reshape(1)

    return LocalOps(assign, partial, finalize)


def _rank(rank, world, port, niter, out):
    os.environ["OMP_NUM_THREADS"] = "1"
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    from exact_lloyd_means_b200.dist import lloyd_sharded
    X, C0 = _data()
    bounds = np.linspace(0, X.shape[0], world + 1).astype(int)
    Xl = X[bounds[rank]:bounds[rank + 1]].contiguous()
    C = C0.clone()
    objs, counts = lloyd_sharded(Xl, C, niter, _stand_in_ops())
    out.put((rank, C.numpy(), objs, counts.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_sharded_lloyd_equals_single_process_oracle(world):
    import oracle
    niter = 4
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, niter, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda t: t[0])
    X, C0 = _data()
    ref = oracle.lloyd(X.numpy(), C0.numpy(), niter)
    for rank, C, objs, counts in res:
        # every rank holds the same centroids: the oracle's, up to the order of fp64 sums
        scale = np.abs(ref["C_next"][-1]).max(axis=1, keepdims=True)
        assert (np.abs(C - ref["C_next"][-1]) <= 1e-6 * scale).all()
        for t in range(niter):
            assert abs(objs[t] - ref["J"][t]) <= 1e-9 * ref["J"][t]
        assert (counts == ref["counts"][-1]).all()
    assert np.array_equal(res[0][1], res[1][1])  # bit-identical across ranks


def _failing_rank(rank, world, port, out, mode):
    """Rank 1 fails in its local step of the second iteration, between exchanges (no
    collective in flight): mode "raise" leaves (its process ends), mode "stall" stays alive
    but never reaches the exchange.  Rank 0 carries on into its next exchange."""
    os.environ["OMP_NUM_THREADS"] = "1"
    import sys
    import time
    from datetime import timedelta
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=10))
    from exact_lloyd_means_b200.dist import LocalOps, lloyd_sharded
    X, C0 = _data()
    bounds = np.linspace(0, X.shape[0], world + 1).astype(int)
    Xl = X[bounds[rank]:bounds[rank + 1]].contiguous()
    ops = _stand_in_ops()
    calls = {"n": 0}

    def assign(Xa, C):
        calls["n"] += 1
        if rank == 1 and calls["n"] == 2:
            if mode == "stall":
                time.sleep(25.0)
            raise RuntimeError("injected: rank 1 lost its device")
        return ops.assign(Xa, C)

    t0 = time.monotonic()
    try:
        lloyd_sharded(Xl, C0.clone(), 4, LocalOps(assign, ops.partial, ops.finalize))
        out.put((rank, "finished", time.monotonic() - t0))
    except Exception as e:  # noqa: BLE001 - what ended the rank is the result
        out.put((rank, type(e).__name__ + ": " + str(e)[:120], time.monotonic() - t0))
    # no destroy_process_group: the peer is gone, and a collective would wait on it


@pytest.mark.parametrize("mode", ["raise", "stall"])
def test_sharded_lloyd_lost_rank_ends_peer_with_error(mode):
    """Failure detection on the data-parallel path without a GPU: when one rank leaves or
    stalls between steps, the other's next exchange ends with an error (a closed
    connection, or the process group's 10 s timeout) instead of waiting for good, and the
    survivor reports no result."""
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_rank, args=(r, world, port, out, mode))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, what, secs = out.get(timeout=120)
        res[rank] = (what, secs)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    print(res)
    assert res[1][0].startswith("RuntimeError: injected")
    assert res[0][0] != "finished"      # the survivor did not carry on alone
    assert res[0][1] < 22.0            # it gave up before the stalled peer woke (25 s)
