"""Shared helpers of the GPU parity tests (no method arithmetic here)."""
import numpy as np

from trainable_block_sparse_compressed_b200 import workloads as wl

# Tolerances (spec contract): selection sets bit-exact outside a 1e-3
# relative score band at the k-th / (k+1)-th boundary; attention output
# max-abs <= 2e-2 for bf16 output; LSE within 1e-3.
SEL_REL_BAND = 1e-3
O_ATOL = 2e-2
LSE_ATOL = 1e-3
O_ATOL_FP32 = 1e-4   # the fp32 validation build's output


def gpu_bf16(bits):
    return wl.to_torch_bf16(bits).cuda()


def f64(t):
    """torch bf16/fp32 GPU tensor -> float64 numpy."""
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def check_selection_row(orow, gpu_row, topk, rel=SEL_REL_BAND):
    """Band rule.  Returns True if the row matched exactly, False if it
    differed only inside the band; raises AssertionError otherwise."""
    gpu_row = [int(x) for x in gpu_row]
    n = sum(1 for x in gpu_row if x >= 0)
    g = gpu_row[:n]
    assert gpu_row[n:] == [-1] * (topk - n), gpu_row
    assert g == sorted(set(g)), g
    o = [int(x) for x in orow.idx if x >= 0]
    assert len(g) == len(o), (g, o)
    assert set(orow.forced) <= set(g), (orow.forced, g)
    if g == o:
        return True
    free, ranked, bs = orow.free_slots, orow.ranked, orow.bs
    assert free < len(ranked), "every candidate fits, the sets must match"
    s_k, s_k1 = bs[ranked[free - 1]], bs[ranked[free]]
    assert np.isfinite(s_k) and s_k != 0, (s_k, g, o)
    gap = (s_k - s_k1) / abs(s_k)
    assert gap < rel, f"clear gap {gap:.3g} but sets differ: gpu {g} oracle {o}"
    for blk in set(g) ^ set(o):
        assert abs(bs[blk] - s_k) <= rel * abs(s_k), (blk, bs[blk], s_k)
    return False


def sample_rows(T, n, seed, extra=()):
    """Query positions to check at full size: edges, block borders, random."""
    rng = np.random.default_rng(seed)
    base = {0, 1, 30, 31, 32, 47, 63, 64, 65, 127, 128, T - 1, T - 2, T - 64, T - 65}
    base |= {int(x) for x in rng.integers(0, T, n)}
    base |= set(extra)
    return sorted(t for t in base if 0 <= t < T)
