"""The update's one-launch combine for small problems (wide_combine_kernel, csrc/update.cu)
must form the same fp64 sums as the level-by-level combine it replaces (seg_pieces_kernel
levels, then the tail's last level): the centroids of a small problem are then the same
bits whichever path a size takes.  Both walks are written out here on the host, each the
way its kernel walks the data, and must agree exactly over random cluster layouts (huge
clusters, single-row clusters, empty clusters, ragged last units).  The level-1 pieces are
random fp64 values: both paths read the same pieces, and the level-1 kernel that writes
them is shared.  The host walk also pins the one-launch kernel's rule for where a unit
holds a cluster's piece (slot 0 when the cluster holds the unit's first position)."""
import numpy as np
import pytest

GROUP = 16  # units of one combine level per unit of the next


def level1_pieces(offsets, N, R, rng):
    """Slot keys and pieces per unit of R sorted positions, as the level-1 kernel leaves
    them: a cluster that continues outside the unit leaves a piece, in slot 0 if it is the
    unit's first cluster, else in slot 1 (only the first and last clusters can continue)."""
    lab = np.repeat(np.arange(len(offsets) - 1), np.diff(offsets))
    nunits = -(-N // R)
    keys = np.full((nunits, 2), -1, dtype=np.int64)
    vals = rng.standard_normal((nunits, 2)) * rng.choice([1e-3, 1.0, 1e3], size=(nunits, 2))
    for u in range(nunits):
        p0, p1 = u * R, min(N, u * R + R)
        first, last = lab[p0], lab[p1 - 1]
        before = lab[p0 - 1] if p0 > 0 else -1
        after = lab[p1] if p1 < N else -1
        cont = lambda k: k == before or k == after  # noqa: E731
        if cont(first):
            keys[u, 0] = first
        if last != first and cont(last):
            keys[u, 1] = last
    return keys, vals


def levels_walk(keys, vals, offsets, R):
    """seg_pieces_kernel's walk: each unit of a level reduces the slots of its GROUP units
    of the level below in slot order, finishing a cluster at the first level whose unit
    holds all of it, else leaving a piece (first cluster in slot 0, last in slot 1)."""
    done = {}
    span, units = R, keys.shape[0]
    while units > 1:
        n2 = -(-units // GROUP)
        span *= GROUP
        nk = np.full((n2, 2), -1, dtype=np.int64)
        nv = np.zeros((n2, 2))
        for g in range(n2):
            st = {"cur": -1, "acc": 0.0, "first": -1, "first_done": False, "slot1": -1}

            def flush(k):
                lo, hi = offsets[k], offsets[k + 1]
                fin = lo // span == (hi - 1) // span
                if k == st["first"]:
                    st["first_done"] = fin
                if fin:
                    done[k] = st["acc"]
                else:
                    slot = 0 if k == st["first"] else 1
                    if slot == 1:
                        st["slot1"] = k
                    nv[g, slot] = st["acc"]

            for u in range(g * GROUP, min(units, g * GROUP + GROUP)):
                for s in (0, 1):
                    k = keys[u, s]
                    if k < 0:
                        continue
                    if k != st["cur"]:
                        if st["cur"] >= 0:
                            flush(st["cur"])
                        if st["cur"] < 0:
                            st["first"] = k
                        st["cur"], st["acc"] = k, 0.0
                    st["acc"] += vals[u, s]
            if st["cur"] >= 0:
                flush(st["cur"])
            nk[g, 0] = st["first"] if st["first"] >= 0 and not st["first_done"] else -1
            nk[g, 1] = st["slot1"]
        keys, vals, units = nk, nv, n2
    return done


def wide_walk(keys, vals, offsets, R):
    """wide_combine_kernel's walk: per cluster, its units' pieces (slot chosen from the
    positions alone) added GROUP units at a time in unit order, level after level, until
    the cluster lies in one unit."""
    done = {}
    for k in range(len(offsets) - 1):
        lo, hi = offsets[k], offsets[k + 1]
        if hi == lo:
            continue
        a0, a1 = lo // R, (hi - 1) // R
        if a0 == a1:
            continue  # finished by the level-1 kernel
        items = []
        for u in range(a0, a1 + 1):
            slot = 0 if lo <= u * R else 1
            assert keys[u, slot] == k, (k, u, slot)  # the slot rule
            items.append(vals[u, slot])
        while True:
            g0, g1 = a0 // GROUP, a1 // GROUP
            nxt = []
            for g in range(g0, g1 + 1):
                acc = 0.0
                for i in range(max(a0, g * GROUP), min(a1, g * GROUP + GROUP - 1) + 1):
                    acc += items[i - a0]
                nxt.append(acc)
            if g0 == g1:
                done[k] = nxt[0]
                break
            a0, a1, items = g0, g1, nxt
    return done


def random_offsets(rng, N, K, kind):
    if kind == "zipf":
        w = 1.0 / np.arange(1, K + 1) ** 1.2
    elif kind == "one_huge":
        w = np.full(K, 1e-3)
        w[rng.integers(K)] = 1.0
    else:
        w = np.ones(K)
    counts = rng.multinomial(N, w / w.sum())
    counts[rng.integers(K, size=max(1, K // 10))] = 0  # some empty clusters
    counts[0] += N - counts.sum()
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


@pytest.mark.parametrize("seed", range(12))
def test_one_launch_combine_sums_equal_level_by_level(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 9000))
    K = int(rng.integers(1, min(N, 400) + 1))
    R = int(rng.choice([2, 4, 8]))  # any power of two: small R gives deep trees here
    kind = ["equal", "zipf", "one_huge"][seed % 3]
    offsets = random_offsets(rng, N, K, kind)
    keys, vals = level1_pieces(offsets, N, R, rng)
    a = levels_walk(keys, vals, offsets, R)
    b = wide_walk(keys, vals, offsets, R)
    assert set(a) == set(b)
    assert all(a[k] == b[k] for k in a), [k for k in a if a[k] != b[k]][:5]
    # the walks differ in order from a plain left-to-right sum for deep clusters, so the
    # comparison is not vacuous
    assert len(a) > 0 or -(-N // R) <= 1
