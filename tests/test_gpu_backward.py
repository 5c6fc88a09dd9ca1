"""Gradients of the block-sparse attention with the selection held fixed
(infllmv2_sparse_attn_backward) against the fp64 oracle's backward
(oracle.sparse_attention_backward, itself pinned by finite differences and
by autograd of dense attention).

Tolerance: the kernels round P and dS to bf16 for the tensor-core products
(relative error 2^-9 per factor) and accumulate in fp32, so every gradient
element carries an error of a few bf16 ulps of the largest terms summed into
it: max |gpu - oracle| <= 2e-2 * max |oracle| per tensor, the normwise
counterpart of the forward's 2e-2 output bound (|O| <= 1 there).
"""
import numpy as np
import pytest

from oracle import infllmv2_oracle as orc
from trainable_block_sparse_compressed_b200 import workloads as wl

from _helpers import f64, gpu_bf16, sample_rows

pytestmark = pytest.mark.gpu

G_RTOL = 2e-2


def _close(got, ref, what):
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= G_RTOL * scale, f"{what}: max err {err:.3g} vs {G_RTOL} x {scale:.3g}"


def _run(api, w, data, idx, dO_bits):
    """Forward (for O and lse) then backward on the GPU with the given idx."""
    import torch
    B, T, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    p = api.make_params(B, T, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    Q, K, V = gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"])
    idx_g = torch.from_numpy(idx).cuda()
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    api.sparse_attn(p, Q, K, V, idx_g, O, lse, api.alloc_workspace(p, api.OP_ATTN))
    dO = gpu_bf16(dO_bits)
    dQ = torch.full((B, T, Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
    dK = torch.full((B, T, Hkv, 128), float("nan"), dtype=torch.float32, device="cuda")
    dV = torch.full_like(dK, float("nan"))
    ws = api.alloc_workspace(p, api.OP_BACKWARD)
    api.sparse_attn_backward(p, Q, K, V, idx_g, O, lse, dO, dQ, dK, dV, ws)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return f64(dQ), f64(dK), f64(dV), (p, Q, K, V, idx_g, O, lse, dO, ws)


def _dO(w, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return wl.f32_to_bf16_bits(rng.standard_normal((w.B, w.T, w.Hq, w.d), dtype=np.float32))


CASES = [
    # (B, T, Hq, Hkv, topk, needles, seed)
    (1, 2048, 8, 2, 8, 4, 1),     # the T=2048 workload's shape (groups of 4 heads)
    (2, 1000, 32, 2, 8, 2, 7),    # ragged T, groups of 16, two sequences
    (1, 777, 16, 1, 5, 2, 8),     # a single kv head
    (1, 600, 8, 1, 4, 1, 9),      # groups of 8
    (1, 129, 32, 2, 64, 0, 12),   # topk covers every block: dense gradients
    (1, 33, 32, 2, 8, 0, 13),     # one compressed window
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_Hkv{c[3]}_k{c[4]}" for c in CASES])
def test_sparse_backward_all_elements(cuda_lib, case):
    B, T, Hq, Hkv, topk, needles, seed = case
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=needles, seed=seed)
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    op = orc.Params(topk=topk)
    idx, _ = orc.select_blocks(Q, K, op)
    dO_bits = _dO(w, 100 + seed)
    dQ, dK, dV, _ = _run(cuda_lib, w, data, idx, dO_bits)
    rQ, rK, rV = orc.sparse_attention_backward(Q, K, V, idx, wl.bf16_to_f64(dO_bits), op)
    _close(dQ, rQ, "dQ")
    _close(dK, rK, "dK")
    _close(dV, rV, "dV")


def test_sparse_backward_is_deterministic(cuda_lib):
    """Two calls give bit-identical gradients (dK and dV are summed in a
    fixed order, no atomics)."""
    import torch
    api = cuda_lib
    w = wl.small_workload(B=1, T=3000, Hq=32, Hkv=2, topk=16, needles=2, seed=3)
    data = wl.make_prefill(w)
    Q, K = wl.bf16_to_f64(data["Q"]), wl.bf16_to_f64(data["K"])
    idx, _ = orc.select_blocks(Q, K, orc.Params(topk=16))
    dQ, dK, dV, (p, Qg, Kg, Vg, idx_g, O, lse, dO, ws) = _run(api, w, data, idx, _dO(w, 5))
    dQ2 = torch.empty((1, 3000, 32, 128), dtype=torch.float32, device="cuda")
    dK2 = torch.empty((1, 3000, 2, 128), dtype=torch.float32, device="cuda")
    dV2 = torch.empty_like(dK2)
    api.sparse_attn_backward(p, Qg, Kg, Vg, idx_g, O, lse, dO, dQ2, dK2, dV2, ws)
    torch.cuda.synchronize()
    assert np.array_equal(f64(dQ2), dQ)
    assert np.array_equal(f64(dK2), dK)
    assert np.array_equal(f64(dV2), dV)


def test_sparse_backward_32k_sampled(cuda_lib):
    """The T=32768 workload with the GPU's own selection: dQ on sampled rows
    against the oracle row by row; dK and dV of the last block and of a
    middle block against the oracle over exactly the rows that selected them;
    and, over all keys, sum_keys dV = sum_rows dO per (b, kv head) (each
    softmax row sums to one).  (The companion identity sum_keys dK = 0 holds
    only in exact arithmetic: D is formed from the bf16 output O, and the
    per-row residual dO . (O - bf16(O)) random-walks over the 524288 rows to
    a few tenths, so it is not a check at this size.)"""
    import torch
    api = cuda_lib
    w = wl.WORKLOADS["sparse_prefill_T32768_Hq32_Hkv2"]
    data = wl.make_prefill(w)
    Qg, Kg, Vg = gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"])
    _, _, _, idx = api.prefill(Qg, Kg, Vg, topk=w.topk, threshold=w.threshold)
    idx_np = idx.cpu().numpy()
    del Qg, Kg, Vg
    torch.cuda.empty_cache()
    dO_bits = _dO(w, 77)
    dQ, dK, dV, _ = _run(api, w, data, idx_np, dO_bits)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    dOf = wl.bf16_to_f64(dO_bits)
    op = orc.Params(topk=w.topk)
    sc = op.sm_scale(128)
    G = w.Hq // w.Hkv
    # identities over all keys
    for g in range(w.Hkv):
        hs = slice(g * G, (g + 1) * G)
        sum_dO = dOf[0, :, hs].sum(axis=(0, 1))
        assert np.abs(dV[0, :, g].sum(axis=0) - sum_dO).max() <= G_RTOL * np.abs(sum_dO).max()
    # dQ on sampled rows
    for g in range(w.Hkv):
        hs = slice(g * G, (g + 1) * G)
        errs, scale = [], 0.0
        for t in sample_rows(w.T, 24, 21):
            keys = orc.selected_keys(idx_np[0, g, t], t, op)
            dq, _, _ = orc.attend_backward(Q[0, t, hs], K[0, :, g], V[0, :, g], keys, sc, dOf[0, t, hs])
            errs.append(np.abs(dQ[0, t, hs] - dq).max())
            scale = max(scale, np.abs(dq).max())
        assert max(errs) <= G_RTOL * scale, (max(errs), scale)
    # dK, dV of whole blocks over the rows that selected them
    nb = w.T // 64
    for g in range(w.Hkv):
        hs = slice(g * G, (g + 1) * G)
        for blk in (nb - 1, nb // 2 + 3):
            rows = np.nonzero((idx_np[0, g] == blk).any(axis=-1))[0]
            rK = np.zeros((64, 128))
            rV = np.zeros((64, 128))
            for t in rows:
                if blk > t // 64:
                    continue
                keys = orc.selected_keys(idx_np[0, g, t], int(t), op)
                _, dk, dv = orc.attend_backward(Q[0, t, hs], K[0, :, g], V[0, :, g], keys, sc,
                                                dOf[0, t, hs])
                sel = (keys >= blk * 64) & (keys < blk * 64 + 64)
                rK[keys[sel] - blk * 64] += dk[sel]
                rV[keys[sel] - blk * 64] += dv[sel]
            _close(dK[0, blk * 64:blk * 64 + 64, g], rK, f"dK block {blk}")
            _close(dV[0, blk * 64:blk * 64 + 64, g], rV, f"dV block {blk}")
