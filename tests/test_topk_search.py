"""The block-selection search of the top-k kernels (topk.cuh), emulated on the
host: the most-significant-bit-first search for the free-th largest key, with
its early stop once exactly `free` keys are >= the candidate, and the rule
that keeps keys > tau plus the lowest-index ties at tau.  It must keep the
same blocks as ranking all keys (descending, ties to the lower index), for
any key multiset -- many ties included."""
import numpy as np


def _bit_search(keys, free, early):
    tau = 0
    for bit in range(31, -1, -1):
        c = tau | (1 << bit)
        cnt = int((keys >= c).sum())
        if cnt >= free:
            tau = c
        if early and cnt == free:
            break
    need_eq = free - int((keys > tau).sum())
    kept = []
    for i, k in enumerate(keys):
        if k > tau:
            kept.append(i)
        elif k == tau and need_eq > 0:
            kept.append(i)
            need_eq -= 1
    return sorted(kept)


def _rank(keys, free):
    order = sorted(range(len(keys)), key=lambda i: (-int(keys[i]), i))
    return sorted(order[:free])


def test_early_stop_keeps_the_same_blocks():
    rng = np.random.default_rng(7)
    for trial in range(400):
        n = int(rng.integers(2, 600))
        free = int(rng.integers(1, n))
        kind = trial % 4
        if kind == 0:    # continuous scores as order-preserving keys
            keys = (rng.random(n).astype(np.float32).view(np.uint32) | np.uint32(0x80000000))
        elif kind == 1:  # few distinct values: ties everywhere
            keys = rng.integers(1, 6, n).astype(np.uint32) << np.uint32(20)
        elif kind == 2:  # one value
            keys = np.full(n, 0x80000001, dtype=np.uint32)
        else:            # wide range of integers
            keys = rng.integers(1, 2**32 - 1, n, dtype=np.uint64).astype(np.uint32)
        keys = keys.astype(np.uint64)
        want = _rank(keys, free)
        assert _bit_search(keys, free, early=False) == want
        assert _bit_search(keys, free, early=True) == want
