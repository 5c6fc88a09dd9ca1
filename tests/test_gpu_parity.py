"""GPU parity against the fp64 oracle, through the C ABI.

Small cases are compared element by element on every row; the full-size
workloads (T = 32768, 131072; decode over a 131072-token cache) on sampled
rows that the oracle computes one by one.  Attention kernels receive the
ORACLE's block indices, so their outputs can be compared exactly against the
oracle; the GPU's own selection is checked with the band rule.
"""
import numpy as np
import pytest

from oracle import infllmv2_oracle as orc
from trainable_block_sparse_compressed_b200 import workloads as wl

from _helpers import (LSE_ATOL, O_ATOL, check_selection_row, f64, gpu_bf16, sample_rows)

pytestmark = pytest.mark.gpu


def _params(api, w, T=None, **kw):
    T = w.T if T is None else T
    d = dict(topk=w.topk, n_init=w.n_init, n_local=w.n_local, switch_threshold=w.threshold)
    d.update(kw)
    return api.make_params(w.B, T, w.Hq, w.Hkv, **d)


def _oparams(w, **kw):
    d = dict(topk=w.topk, n_init=w.n_init, n_local=w.n_local, threshold=w.threshold)
    d.update(kw)
    return orc.Params(**d)


# ---------------------------------------------------------------------------
# compressed keys
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,Hkv,B", [(31, 2, 1), (32, 2, 2), (1000, 2, 2), (4111, 1, 1),
                                     (2048, 4, 1)])
def test_compress_keys(cuda_lib, T, Hkv, B):
    import torch
    api = cuda_lib
    w = wl.small_workload(B=B, T=T, Hq=Hkv * 4, Hkv=Hkv, needles=0, seed=T)
    data = wl.make_prefill(w)
    p = _params(api, w)
    n_c = api.num_compressed(T)
    K = gpu_bf16(data["K"])
    Kc = torch.full((B, max(n_c, 1), Hkv, 2, 128), float("nan"), dtype=torch.bfloat16,
                    device="cuda")
    api.compress_keys(p, K, Kc)
    torch.cuda.synchronize()
    if n_c == 0:
        return
    ref = orc.compress_keys(wl.bf16_to_f64(data["K"]), orc.Params())
    got = f64(Kc[:, :n_c])
    hi, lo = got[..., 0, :], got[..., 1, :]
    # hi is the bf16 rounding of the mean (one ulp at most off, from the fp32 sum)
    ref_hi = wl.bf16_to_f64(wl.f32_to_bf16_bits(ref.astype(np.float32)))
    assert np.all(np.abs(hi - ref_hi) <= np.abs(ref_hi) * 2.0 ** -7 + 1e-30)
    assert np.mean(hi == ref_hi) > 0.999
    # hi + lo carries ~17 significant bits: |hi + lo - mean| <= 2^-16 |mean| (+ fp32 sum error)
    err = np.abs(hi + lo - ref)
    assert np.all(err <= np.abs(ref) * 2.0 ** -16 + 1e-7), (err / (np.abs(ref) + 1e-30)).max()


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------
SMALL = [
    # (B, T, Hq, Hkv, topk, needles, seed)
    (1, 2048, 8, 2, 8, 4, 1),     # the smallest evaluation workload
    (2, 1000, 32, 2, 8, 2, 7),    # ragged T, G = 16, two sequences
    (1, 777, 16, 1, 5, 2, 8),     # G = 16, single kv head
    (1, 600, 8, 1, 4, 1, 9),      # G = 8
    (1, 500, 4, 2, 6, 1, 10),     # G = 2
    (1, 300, 2, 2, 3, 0, 11),     # G = 1, topk == forced count
    (1, 129, 32, 2, 64, 0, 12),   # topk covers every block
    (1, 33, 32, 2, 8, 0, 13),     # a single compressed window
    (1, 20, 32, 2, 8, 0, 14),     # no compressed window at all
]


def _run_select(api, w, data):
    import torch
    p = _params(api, w)
    n_c = api.num_compressed(w.T)
    Q, K = gpu_bf16(data["Q"]), gpu_bf16(data["K"])
    Kc = torch.empty((w.B, max(n_c, 1), w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    if n_c:
        api.compress_keys(p, K, Kc)
    idx = torch.full((w.B, w.Hkv, w.T, w.topk), -7, dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_SELECT)
    api.select_blocks(p, Q, Kc, idx, ws)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return idx.cpu().numpy()


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_Hkv{c[3]}_k{c[4]}" for c in SMALL])
def test_select_blocks_all_rows(cuda_lib, case):
    B, T, Hq, Hkv, topk, needles, seed = case
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=needles, seed=seed)
    data = wl.make_prefill(w)
    got = _run_select(cuda_lib, w, data)
    Q, K = wl.bf16_to_f64(data["Q"]), wl.bf16_to_f64(data["K"])
    _, det = orc.select_blocks(Q, K, _oparams(w))
    exact = 0
    for (b, g, t), r in det.items():
        exact += check_selection_row(r, got[b, g, t], topk)
    assert exact >= 0.8 * len(det), f"only {exact}/{len(det)} rows exact"


TIE_CASES = [(1, 1500, 32, 2, 16), (2, 700, 8, 1, 6), (1, 2111, 32, 2, 12)]


@pytest.mark.parametrize("case", TIE_CASES, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_k{c[4]}" for c in TIE_CASES])
def test_select_exact_ties_go_to_lower_blocks(cuda_lib, case):
    """Every key equal: every visible window scores alike, so all block scores
    with a visible window are exactly equal (on the GPU as in the oracle) and
    the free slots go to the lowest-index free blocks -- compared exactly."""
    B, T, Hq, Hkv, topk = case
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=0, seed=21)
    data = wl.make_prefill(w)
    data["K"][:] = data["K"][:, :1]  # every token carries the first token's key
    got = _run_select(cuda_lib, w, data)
    ref, _ = orc.select_blocks(wl.bf16_to_f64(data["Q"]), wl.bf16_to_f64(data["K"]), _oparams(w))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# attention with the oracle's selection
# ---------------------------------------------------------------------------
SCHEDULES = ["query_tiles", "per_token_packed", "per_token_tensor_map"]


def _run_sparse(api, p, schedule, Q, K, V, idx, O, lse):
    """The block-sparse attention under one of its schedules: query tiles over
    each tile's union of blocks (sparse_attn with its workspace; groups of 8
    or 16 heads, smaller groups fall back to the per-token schedule), one item
    per token gathering packed tiles, or one item per token gathering from K
    and V by tensor maps (no workspace)."""
    if schedule == "query_tiles":
        api.sparse_attn(p, Q, K, V, idx, O, lse, api.alloc_workspace(p, api.OP_ATTN))
    elif schedule == "per_token_packed":
        api.sparse_attn_per_token(p, Q, K, V, idx, O, lse,
                                  api.alloc_workspace(p, api.OP_ATTN_PER_TOKEN))
    else:
        api.sparse_attn_per_token(p, Q, K, V, idx, O, lse, None)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_Hkv{c[3]}_k{c[4]}" for c in SMALL])
def test_sparse_attn_all_rows(cuda_lib, case, schedule):
    import torch
    api = cuda_lib
    B, T, Hq, Hkv, topk, needles, seed = case
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=needles, seed=seed)
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    op = _oparams(w)
    idx, _ = orc.select_blocks(Q, K, op)
    O_ref, L_ref = orc.sparse_attention(Q, K, V, idx, op)
    O = torch.empty((B, T, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    p = _params(api, w)
    _run_sparse(api, p, schedule, gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                torch.from_numpy(idx).cuda(), O, lse)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert np.abs(f64(O) - O_ref).max() <= O_ATOL
    assert np.abs(f64(lse) - L_ref).max() <= LSE_ATOL


@pytest.mark.parametrize("shared", [True, False], ids=["tokens_share_blocks", "tokens_disjoint"])
def test_query_tile_union_extremes(cuda_lib, shared):
    """The query-tile schedule at the two ends of block sharing: every token
    of a tile selecting the same blocks (union = one token's set), and
    neighbouring tokens selecting disjoint blocks (union = 8 x topk)."""
    import torch
    api = cuda_lib
    B, T, Hq, Hkv, topk = 1, 2500, 32, 2, 6
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=0, seed=31)
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    rng = np.random.default_rng(5)
    idx = np.full((B, Hkv, T, topk), -1, dtype=np.int32)
    for g in range(Hkv):
        for t in range(T):
            cur = t // 64
            free = [b for b in range(1, cur - 1)]
            if shared:
                r = np.random.default_rng(1000 * g + t // 8)   # one choice per 8-token tile
            else:
                r = rng
            k = min(topk - 3, len(free))
            pick = sorted(set([0, max(cur - 1, 0), cur] + list(r.choice(free, size=k, replace=False)))) \
                if free else sorted(set([0, max(cur - 1, 0), cur]))
            idx[0, g, t, :len(pick)] = pick
    op = orc.Params(topk=topk)
    O_ref, L_ref = orc.sparse_attention(Q, K, V, idx, op)
    O = torch.empty((B, T, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    p = _params(api, w)
    _run_sparse(api, p, "query_tiles", gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                torch.from_numpy(idx).cuda(), O, lse)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert np.abs(f64(O) - O_ref).max() <= O_ATOL
    assert np.abs(f64(lse) - L_ref).max() <= LSE_ATOL


def test_sparse_attn_unsorted_padding_and_ignored_entries(cuda_lib):
    """Rows shorter than topk (-1 padded) and entries beyond t//64 (ignored)."""
    import torch
    api = cuda_lib
    w = wl.small_workload(B=1, T=400, Hq=32, Hkv=2, topk=6, needles=0, seed=21)
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    idx = np.full((1, 2, 400, 6), -1, dtype=np.int32)
    rng = np.random.default_rng(0)
    for g in range(2):
        for t in range(400):
            cur = t // 64
            n = int(rng.integers(1, min(6, cur + 1) + 1))
            blocks = sorted(rng.choice(cur + 1, size=n, replace=False).tolist())
            row = blocks + ([cur + 1] if cur + 1 <= 6 and n < 6 else [])
            idx[0, g, t, :len(row)] = row
    op = orc.Params(topk=6)
    O_ref, L_ref = orc.sparse_attention(Q, K, V, idx, op)
    O = torch.empty((1, 400, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 32, 400), dtype=torch.float32, device="cuda")
    p = _params(api, w)
    api.sparse_attn(p, gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                    torch.from_numpy(idx).cuda(), O, lse, api.alloc_workspace(p, api.OP_ATTN))
    torch.cuda.synchronize()
    assert np.abs(f64(O) - O_ref).max() <= O_ATOL
    assert np.abs(f64(lse) - L_ref).max() <= LSE_ATOL


# ---------------------------------------------------------------------------
# dense path and the switch
# ---------------------------------------------------------------------------
DENSE = [(1, 300, 32, 2), (2, 130, 8, 2), (1, 1, 16, 1), (1, 1000, 16, 1), (1, 700, 2, 2),
         (2, 333, 16, 2), (1, 517, 4, 2)]


@pytest.mark.parametrize("B,T,Hq,Hkv", DENSE, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_Hkv{c[3]}" for c in DENSE])
def test_dense_attn_all_rows(cuda_lib, B, T, Hq, Hkv):
    import torch
    api = cuda_lib
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, needles=0, seed=T + Hq)
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    O_ref, L_ref = orc.dense_attention(Q, K, V, orc.Params())
    O = torch.empty((B, T, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    p = _params(api, w)
    api.dense_attn(p, gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]), O, lse)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert np.abs(f64(O) - O_ref).max() <= O_ATOL
    assert np.abs(f64(lse) - L_ref).max() <= LSE_ATOL


# ---------------------------------------------------------------------------
# the compressed-attention branch
# ---------------------------------------------------------------------------
CMP = [(1, 700, 32, 2), (1, 1000, 8, 2), (2, 300, 16, 1), (1, 31, 32, 2), (1, 47, 16, 2),
       (1, 1500, 2, 2)]


def _run_compressed(api, w, data):
    import torch
    p = _params(api, w)
    n_c = api.num_compressed(w.T)
    K, V = gpu_bf16(data["K"]), gpu_bf16(data["V"])
    Kc = torch.empty((w.B, max(n_c, 1), w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    if n_c:
        api.compress_keys(p, K, Kc)
        api.compress_keys(p, V, Vc)
    O = torch.full((w.B, w.T, w.Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.Hq, w.T), float("nan"), dtype=torch.float32, device="cuda")
    api.compressed_attn(p, gpu_bf16(data["Q"]), Kc, Vc, O, lse)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return f64(O), f64(lse)


@pytest.mark.parametrize("B,T,Hq,Hkv", CMP, ids=[f"B{c[0]}_T{c[1]}_Hq{c[2]}_Hkv{c[3]}" for c in CMP])
def test_compressed_attn_all_rows(cuda_lib, B, T, Hq, Hkv):
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, needles=2, seed=T + 3 * Hq)
    data = wl.make_prefill(w)
    Og, Lg = _run_compressed(cuda_lib, w, data)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    O_ref, L_ref = orc.compressed_attention(Q, K, V, orc.Params())
    none = np.isneginf(L_ref)            # rows that see no window: O = 0, lse = -inf
    assert np.array_equal(np.isneginf(Lg), none)
    assert np.abs(Og - O_ref).max() <= O_ATOL
    if (~none).any():
        assert np.abs(Lg[~none] - L_ref[~none]).max() <= LSE_ATOL


def test_compressed_attn_32k_sampled(cuda_lib):
    w = wl.WORKLOADS["sparse_prefill_T32768_Hq32_Hkv2"]
    data = wl.make_prefill(w)
    Og, Lg = _run_compressed(cuda_lib, w, data)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    needle_rows = [nd.query_block * 64 + 5 for nd in data["needles"][:8]]
    rows = [(0, g, t) for g in range(w.Hkv) for t in sample_rows(w.T, 40, 9, needle_rows)]
    O_ref, L_ref = orc.compressed_attention(Q, K, V, orc.Params(), rows)
    G = w.Hq // w.Hkv
    for (b, g, t) in rows:
        hs = slice(g * G, (g + 1) * G)
        assert np.abs(Og[b, t, hs] - O_ref[b, t, hs]).max() <= O_ATOL
        if t >= 31:
            assert np.abs(Lg[b, hs, t] - L_ref[b, hs, t]).max() <= LSE_ATOL
        else:
            assert np.all(np.isneginf(Lg[b, hs, t]))


def test_dense_switch_workload_sampled(cuda_lib):
    """B=2, T=4096, Hq=32, Hkv=2 below the 8192 threshold: the switch must
    take the dense path; sampled rows equal exact causal attention."""
    api = cuda_lib
    w = wl.WORKLOADS["dense_switch_B2_T4096_Hq32_Hkv2"]
    data = wl.make_prefill(w)
    O, lse, path, _ = api.prefill(gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                                  topk=w.topk, threshold=w.threshold)
    assert path == api.PATH_DENSE
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    rows = [(b, g, t) for b in range(2) for g in range(2) for t in sample_rows(w.T, 24, 5)]
    O_ref, L_ref = orc.dense_attention(Q, K, V, orc.Params(), rows)
    Og, Lg = f64(O), f64(lse)
    G = w.Hq // w.Hkv
    for (b, g, t) in rows:
        hs = slice(g * G, (g + 1) * G)
        assert np.abs(Og[b, t, hs] - O_ref[b, t, hs]).max() <= O_ATOL
        assert np.abs(Lg[b, hs, t] - L_ref[b, hs, t]).max() <= LSE_ATOL


def test_switch_takes_sparse_above_threshold(cuda_lib):
    api = cuda_lib
    w = wl.small_workload(B=1, T=576, Hq=32, Hkv=2, topk=4, needles=1, seed=3)
    data = wl.make_prefill(w)
    *_, path, idx = api.prefill(gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                                topk=4, threshold=512)
    assert path == api.PATH_SPARSE and idx is not None
    *_, path2, idx2 = api.prefill(gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"]),
                                  topk=4, threshold=576)
    assert path2 == api.PATH_DENSE and idx2 is None


# ---------------------------------------------------------------------------
# full-size prefill workloads, sampled rows
# ---------------------------------------------------------------------------
def _full_prefill_check(api, name, n_rows, seed):
    import torch
    w = wl.WORKLOADS[name]
    data = wl.make_prefill(w)
    Qg, Kg, Vg = gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"])
    O, lse, path, idx = api.prefill(Qg, Kg, Vg, topk=w.topk, threshold=w.threshold)
    torch.cuda.synchronize()
    assert path == api.PATH_SPARSE
    assert api.get_status() == 0
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    op = _oparams(w)
    needle_rows = [nd.query_block * 64 + 17 for nd in data["needles"][:8]]
    ts = sample_rows(w.T, n_rows, seed, needle_rows)
    rows = [(0, g, t) for g in range(w.Hkv) for t in ts]
    oidx, det = orc.select_blocks(Q, K, op, rows)
    gidx = idx.cpu().numpy()
    exact = sum(check_selection_row(det[r], gidx[r], w.topk) for r in rows)
    assert exact >= 0.5 * len(rows)
    # attention at full size with the oracle's selection on the sampled rows
    # (other rows keep the GPU's own selection; they are not compared)
    full_idx = gidx.copy()
    for r in rows:
        full_idx[r] = oidx[r]
    O2 = torch.empty_like(Qg)
    lse2 = torch.empty_like(lse)
    p = api.make_params(w.B, w.T, w.Hq, w.Hkv, topk=w.topk, switch_threshold=w.threshold)
    api.sparse_attn(p, Qg, Kg, Vg, torch.from_numpy(full_idx).cuda(), O2, lse2,
                    api.alloc_workspace(p, api.OP_ATTN))
    torch.cuda.synchronize()
    O_ref, L_ref = orc.sparse_attention(Q, K, V, oidx, op, rows)
    Og, Lg = f64(O2), f64(lse2)
    Of, Lf = f64(O), f64(lse)
    G = w.Hq // w.Hkv
    for (b, g, t) in rows:
        hs = slice(g * G, (g + 1) * G)
        assert np.abs(Og[b, t, hs] - O_ref[b, t, hs]).max() <= O_ATOL
        assert np.abs(Lg[b, hs, t] - L_ref[b, hs, t]).max() <= LSE_ATOL
        # forward()'s own output, over its own selection (band-checked above)
        keys = orc.selected_keys(gidx[b, g, t], t, op)
        o, l = orc.attend(Q[b, t, hs], K[b, :, g], V[b, :, g], keys, op.sm_scale(128))
        assert np.abs(Of[b, t, hs] - o).max() <= O_ATOL
        assert np.abs(Lf[b, hs, t] - l).max() <= LSE_ATOL


def test_prefill_32k_sampled(cuda_lib):
    _full_prefill_check(cuda_lib, "sparse_prefill_T32768_Hq32_Hkv2", 48, 3)


def test_prefill_128k_sampled(cuda_lib):
    _full_prefill_check(cuda_lib, "sparse_prefill_T131072_Hq32_Hkv2", 32, 4)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
def _decode_setup(api, w, L0, steps, B, mutate=None):
    import torch
    data = wl.make_decode(w, L=L0, steps=steps, B=B)
    if mutate is not None:
        mutate(data)
    Lmax = L0 + steps
    p = api.make_params(B, Lmax, w.Hq, w.Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local)
    NC = api.num_compressed(Lmax)
    Kc = torch.zeros((B, Lmax, w.Hkv, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    Kc[:, :L0] = gpu_bf16(data["K0"])
    Vc[:, :L0] = gpu_bf16(data["V0"])
    Kcmp = torch.zeros((B, max(NC, 1), w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    p0 = api.make_params(B, L0, w.Hq, w.Hkv)
    n0 = api.num_compressed(L0)
    if n0:
        tmp = torch.empty((B, n0, w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
        api.compress_keys(p0, gpu_bf16(data["K0"]), tmp)
        Kcmp[:, :n0] = tmp
    seqlens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_DECODE)
    return data, p, Kc, Vc, Kcmp, seqlens, ws



def _check_decode_row(K_seq, V_seq, Kc_seq, q, t, gi, Og, Lg, op, O_ref=None, L_ref=None,
                      i_ref=None):
    """One sequence's decode step, every kv group: the GPU's selection by the
    band rule; its O and LSE against the oracle's attention over the GPU's own
    selection (so rows whose selection differs inside the band are compared
    too), and against the oracle's own result where the selections agree."""
    Hq = q.shape[0]
    Hkv = K_seq.shape[1]
    G = Hq // Hkv
    sc = op.sm_scale(128)
    for g in range(Hkv):
        hs = slice(g * G, (g + 1) * G)
        r = orc.select_query(q[hs], Kc_seq[:, g], t, op)
        check_selection_row(r, gi[g], op.topk)
        keys = orc.selected_keys(gi[g], t, op)
        o, lse = orc.attend(q[hs], K_seq[:, g], V_seq[:, g], keys, sc)
        assert np.abs(Og[hs] - o).max() <= O_ATOL
        assert np.abs(Lg[hs] - lse).max() <= LSE_ATOL
        if i_ref is not None and np.array_equal(gi[g], i_ref[g]):
            assert np.abs(Og[hs] - O_ref[hs]).max() <= O_ATOL
            assert np.abs(Lg[hs] - L_ref[hs]).max() <= LSE_ATOL

def test_decode_steps_small(cuda_lib):
    import torch
    api = cuda_lib
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B, L0, steps = 3, 990, 40
    data, p, Kc, Vc, Kcmp, seqlens, ws = _decode_setup(api, w, L0, steps, B)
    op = orc.Params(topk=w.topk)
    st = orc.DecodeState.from_prefill(wl.bf16_to_f64(data["K0"]), wl.bf16_to_f64(data["V0"]), op)
    O = torch.empty((B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    for s in range(steps):
        q = gpu_bf16(data["q"][s])
        api.decode_step(p, q, gpu_bf16(data["k_new"][s]), gpu_bf16(data["v_new"][s]), Kc, Vc, Kcmp,
                        seqlens, O, lse, idx, ws)
        torch.cuda.synchronize()
        qf = wl.bf16_to_f64(data["q"][s])
        O_ref, L_ref, i_ref = orc.decode_step(st, qf, wl.bf16_to_f64(data["k_new"][s]),
                                              wl.bf16_to_f64(data["v_new"][s]), op)
        gi = idx.cpu().numpy()
        Og, Lg = f64(O), f64(lse)
        t = L0 + s
        for b in range(B):
            _check_decode_row(st.K[b], st.V[b], st.Kc[b], qf[b], t, gi[b], Og[b], Lg[b], op,
                              O_ref[b], L_ref[b], i_ref[b])
    assert api.get_status() == 0
    assert seqlens.cpu().tolist() == [L0 + steps] * B
    # incremental compressed keys == batch compression of the final cache
    Lf = L0 + steps
    nf = api.num_compressed(Lf)
    batch = torch.empty((B, nf, w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    api.compress_keys(api.make_params(B, Lf, w.Hq, w.Hkv), Kc[:, :Lf].contiguous(), batch)
    torch.cuda.synchronize()
    assert torch.equal(batch, Kcmp[:, :nf])


def test_decode_workload_at_length(cuda_lib):
    """The decode workload at its size: B=16 sequences over 131072-token
    caches, 16 consecutive steps.  Afterwards the incrementally built
    compressed-key cache must equal a batch compression of the final K cache
    bit for bit, and on six sequences the first and the last step must match
    the oracle (selection by the band rule; O and LSE of every kv group against
    the oracle's attention over the GPU's own selection)."""
    import torch
    api = cuda_lib
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B, L0, steps = w.B, w.T, 16
    data, p, Kc, Vc, Kcmp, seqlens, ws = _decode_setup(api, w, L0, steps, B)
    O = torch.empty((B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    kept = {}
    for s in range(steps):
        api.decode_step(p, gpu_bf16(data["q"][s]), gpu_bf16(data["k_new"][s]),
                        gpu_bf16(data["v_new"][s]), Kc, Vc, Kcmp, seqlens, O, lse, idx, ws)
        if s in (0, steps - 1):
            torch.cuda.synchronize()
            kept[s] = (idx.cpu().numpy(), f64(O), f64(lse))
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert seqlens.cpu().tolist() == [L0 + steps] * B
    Lf = L0 + steps
    nf = api.num_compressed(Lf)
    batch = torch.empty((B, nf, w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    api.compress_keys(api.make_params(B, Lf, w.Hq, w.Hkv), Kc[:, :Lf].contiguous(), batch)
    torch.cuda.synchronize()
    assert torch.equal(batch, Kcmp[:, :nf])
    op = orc.Params(topk=w.topk, n_init=w.n_init, n_local=w.n_local)
    for b in (0, 3, 7, 11, 14, 15):
        Kseq = np.concatenate([wl.bf16_to_f64(data["K0"][b]),
                               wl.bf16_to_f64(data["k_new"][:steps, b])], axis=0)
        Vseq = np.concatenate([wl.bf16_to_f64(data["V0"][b]),
                               wl.bf16_to_f64(data["v_new"][:steps, b])], axis=0)
        Kc_seq = orc.compress_keys(Kseq[None], op)[0]
        for s, (gi, Og, Lg) in kept.items():
            t = L0 + s
            qf = wl.bf16_to_f64(data["q"][s][b])
            O_ref, L_ref, i_ref = orc.decode_query(Kseq[:t + 1], Vseq[:t + 1], Kc_seq, qf, t, op)
            _check_decode_row(Kseq[:t + 1], Vseq[:t + 1], Kc_seq, qf, t, gi[b], Og[b], Lg[b], op,
                              O_ref, L_ref, i_ref)


def test_decode_full_sequence_is_reported(cuda_lib):
    import torch
    api = cuda_lib
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B, L0 = 2, 200
    data, p, Kc, Vc, Kcmp, seqlens, ws = _decode_setup(api, w, L0, 1, B)
    seqlens[1] = L0 + 1  # == capacity: sequence 1 is full
    O = torch.full((B, w.Hq, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    api.decode_step(p, gpu_bf16(data["q"][0]), gpu_bf16(data["k_new"][0]), gpu_bf16(data["v_new"][0]),
                    Kc, Vc, Kcmp, seqlens, O, lse, None, ws)
    st = api.get_status()
    assert st & api.STATUS_SEQ_FULL
    assert seqlens.cpu().tolist() == [L0 + 1, L0 + 1]
    assert float(O[1].abs().max()) == 0.0


# ---------------------------------------------------------------------------
# bounded waits
# ---------------------------------------------------------------------------
def test_timeout_selftest_reports_and_context_survives(cuda_lib):
    import torch
    api = cuda_lib
    assert api.get_status() == 0
    api.set_wait_limit(1_000_000)  # 1 ms
    try:
        api.selftest_timeout()
        assert api.get_status() & api.STATUS_TIMEOUT
    finally:
        api.set_wait_limit(2_000_000_000)
    assert api.get_status() == 0
    # the context still runs real work
    test_compress_keys(cuda_lib, 1000, 2, 2)


def test_decode_exact_ties_go_to_lower_blocks(cuda_lib):
    """Decode with every cached and appended key equal: the block scores tie
    exactly and the selection must equal the oracle's lowest-index choice."""
    import torch
    api = cuda_lib
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B, L0, steps = 2, 3000, 20

    def same_keys(d):
        d["K0"][:] = d["K0"][:, :1]
        d["k_new"][:] = d["K0"][:, 0][None]

    data, p, Kc, Vc, Kcmp, seqlens, ws = _decode_setup(api, w, L0, steps, B, mutate=same_keys)
    op = orc.Params(topk=w.topk)
    st = orc.DecodeState.from_prefill(wl.bf16_to_f64(data["K0"]), wl.bf16_to_f64(data["V0"]), op)
    O = torch.empty((B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    for s in range(steps):
        api.decode_step(p, gpu_bf16(data["q"][s]), gpu_bf16(data["k_new"][s]),
                        gpu_bf16(data["v_new"][s]), Kc, Vc, Kcmp, seqlens, O, lse, idx, ws)
        torch.cuda.synchronize()
        O_ref, L_ref, i_ref = orc.decode_step(st, wl.bf16_to_f64(data["q"][s]),
                                              wl.bf16_to_f64(data["k_new"][s]),
                                              wl.bf16_to_f64(data["v_new"][s]), op)
        assert np.array_equal(idx.cpu().numpy(), i_ref), s
        assert np.abs(f64(O) - O_ref).max() <= O_ATOL
        assert np.abs(f64(lse) - L_ref).max() <= LSE_ATOL
    assert api.get_status() == 0


@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_small_groups(cuda_lib, G):
    """Decode with GQA groups smaller than 16 heads: the scoring product pads
    the query side to 16 rows and must use only the group's G columns."""
    import torch
    api = cuda_lib
    Hkv = 2
    w = wl.Workload(f"decode_G{G}", B=2, T=2500, Hq=G * Hkv, Hkv=Hkv, topk=12, seed=40 + G,
                    decode_steps=6, needles_per_seq=2)
    B, L0, steps = w.B, w.T, w.decode_steps
    data, p, Kc, Vc, Kcmp, seqlens, ws = _decode_setup(api, w, L0, steps, B)
    op = orc.Params(topk=w.topk)
    st = orc.DecodeState.from_prefill(wl.bf16_to_f64(data["K0"]), wl.bf16_to_f64(data["V0"]), op)
    O = torch.empty((B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, Hkv, w.topk), dtype=torch.int32, device="cuda")
    for s in range(steps):
        api.decode_step(p, gpu_bf16(data["q"][s]), gpu_bf16(data["k_new"][s]),
                        gpu_bf16(data["v_new"][s]), Kc, Vc, Kcmp, seqlens, O, lse, idx, ws)
        torch.cuda.synchronize()
        qf = wl.bf16_to_f64(data["q"][s])
        O_ref, L_ref, i_ref = orc.decode_step(st, qf, wl.bf16_to_f64(data["k_new"][s]),
                                              wl.bf16_to_f64(data["v_new"][s]), op)
        gi, Og, Lg = idx.cpu().numpy(), f64(O), f64(lse)
        for b in range(B):
            _check_decode_row(st.K[b], st.V[b], st.Kc[b], qf[b], L0 + s, gi[b], Og[b], Lg[b], op,
                              O_ref[b], L_ref[b], i_ref[b])
    assert api.get_status() == 0


# ---------------------------------------------------------------------------
# chunked prefill over existing caches
# ---------------------------------------------------------------------------
CHUNKS = [
    # (B, T, Hq, Hkv, topk, q0, threshold)
    (1, 2000, 32, 2, 8, 1000, 0),     # unaligned chunk start, G = 16
    (2, 1400, 8, 2, 6, 640, 0),       # block-aligned start, G = 4, two sequences
    (1, 1100, 16, 1, 5, 1093, 0),     # a 7-token chunk
    (1, 3000, 32, 2, 64, 2048, 8192), # dense: the sequence is below the threshold
]


def _run_chunk(api, B, T, Hq, Hkv, topk, q0, threshold, seed):
    import torch
    w = wl.small_workload(B=B, T=T, Hq=Hq, Hkv=Hkv, topk=topk, needles=2, seed=seed,
                          threshold=threshold)
    data = wl.make_prefill(w)
    p = _params(api, w)
    Q, K, V = gpu_bf16(data["Q"]), gpu_bf16(data["K"]), gpu_bf16(data["V"])
    n_c = api.num_compressed(T)
    Kc = torch.empty((B, max(n_c, 1), Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    if n_c:
        api.compress_keys(p, K, Kc)
    Tq = T - q0
    Qc = Q[:, q0:].contiguous()
    O = torch.empty_like(Qc)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device="cuda")
    idx = torch.full((B, Hkv, Tq, topk), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(api.prefill_chunk_workspace_bytes(p, q0, Tq), dtype=torch.uint8,
                     device="cuda")
    path = api.prefill_chunk(p, q0, Tq, Qc, K, V, Kc, O, lse, idx, ws)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return w, data, (Q, K, V, Kc), path, f64(O), f64(lse), idx.cpu().numpy()


@pytest.mark.parametrize("case", CHUNKS, ids=[f"B{c[0]}_T{c[1]}_q0_{c[5]}_thr{c[6]}" for c in CHUNKS])
def test_prefill_chunk_against_the_oracle(cuda_lib, case):
    B, T, Hq, Hkv, topk, q0, threshold = case
    w, data, _, path, Og, Lg, ig = _run_chunk(cuda_lib, *case, seed=50 + q0)
    Qf, Kf, Vf = (wl.bf16_to_f64(data[x]) for x in "QKV")
    op = _oparams(w)
    O_ref, L_ref, path_ref, idx_ref = orc.chunk_forward(Qf[:, q0:], Kf, Vf, q0, op)
    assert path == (cuda_lib.PATH_DENSE if path_ref == "dense" else cuda_lib.PATH_SPARSE)
    G = Hq // Hkv
    sc = op.sm_scale(128)
    if path_ref == "sparse":
        Kc = orc.compress_keys(Kf, op)
        for b in range(B):
            for g in range(Hkv):
                for i in range(T - q0):
                    t = q0 + i
                    r = orc.select_query(Qf[b, t, g * G:(g + 1) * G], Kc[b, :, g], t, op)
                    check_selection_row(r, ig[b, g, i], topk)
    for b in range(B):
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            for i in range(T - q0):
                t = q0 + i
                if path_ref == "sparse":
                    keys = orc.selected_keys(ig[b, g, i], t, op)  # the GPU's own selection
                else:
                    keys = np.arange(t + 1)
                o, l = orc.attend(Qf[b, t, hs], Kf[b, :, g], Vf[b, :, g], keys, sc)
                assert np.abs(Og[b, i, hs] - o).max() <= O_ATOL
                assert np.abs(Lg[b, hs, i] - l).max() <= LSE_ATOL


@pytest.mark.parametrize("q0", [1336, 1337], ids=["tile_aligned", "unaligned"])
def test_prefill_chunk_equals_the_whole_sequence_rows(cuda_lib, q0):
    """The chunk's selection is bit-identical to the same rows of a
    whole-sequence forward on the GPU.  Its outputs are too when the chunk
    starts on a query-tile boundary (8 tokens for 16-head groups: the tiles,
    their block unions and so every row's arithmetic are the same); from an
    unaligned start the tiles group other tokens, and the rows agree within
    rounding."""
    import torch
    api = cuda_lib
    B, T, Hq, Hkv, topk = 1, 3000, 32, 2, 16
    w, data, (Q, K, V, Kc), path, Og, Lg, ig = _run_chunk(api, B, T, Hq, Hkv, topk, q0, 0, 77)
    p = _params(api, w)
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, Hkv, T, topk), dtype=torch.int32, device="cuda")
    Kc2 = torch.empty_like(Kc)
    ws = api.alloc_workspace(p, api.OP_FORWARD)
    assert api.forward(p, Q, K, V, O, lse, Kc2, idx, ws) == api.PATH_SPARSE
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy()[:, :, q0:], ig)
    if q0 % 8 == 0:
        assert np.array_equal(f64(O)[:, q0:], Og)
        assert np.array_equal(f64(lse)[:, :, q0:], Lg)
    else:
        assert np.abs(f64(O)[:, q0:] - Og).max() <= O_ATOL
        assert np.abs(f64(lse)[:, :, q0:] - Lg).max() <= LSE_ATOL


# ---------------------------------------------------------------------------
# variable-length prefill: a packed batch of ragged sequences
# ---------------------------------------------------------------------------
def test_prefill_varlen_against_the_oracle(cuda_lib):
    """Five sequences of different lengths in one call: full prefills and
    tail chunks, sparse (longer than the threshold) and dense, one with no
    query at all.  Each row against the oracle's chunked forward of its own
    sequence: selection by the band rule, O and LSE over the GPU's own
    selection (dense rows over every key)."""
    import torch
    api = cuda_lib
    Hq, Hkv, topk, thr = 32, 2, 8, 1024
    seqs = [(1500, 1500), (700, 700), (2000, 333), (64, 10), (1200, 0)]  # (k_len, q_len)
    datas = [wl.make_prefill(wl.small_workload(B=1, T=k, Hq=Hq, Hkv=Hkv, topk=topk, needles=1,
                                               seed=90 + i, threshold=thr))
             for i, (k, _) in enumerate(seqs)]
    cu_q, cu_k = [0], [0]
    for k, q in seqs:
        cu_q.append(cu_q[-1] + q)
        cu_k.append(cu_k[-1] + k)
    Qp = torch.cat([gpu_bf16(d["Q"])[0, k - q:] for d, (k, q) in zip(datas, seqs)])
    Kp = torch.cat([gpu_bf16(d["K"])[0] for d in datas])
    Vp = torch.cat([gpu_bf16(d["V"])[0] for d in datas])
    kcs = []
    for d, (k, _) in zip(datas, seqs):
        n_c = api.num_compressed(k)
        Kc = torch.empty((1, max(n_c, 1), Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
        if n_c:
            api.compress_keys(api.make_params(1, k, Hq, Hkv), gpu_bf16(d["K"]), Kc)
        kcs.append(Kc[0, :n_c])
    Kcp = torch.cat(kcs)
    p = api.make_params(1, 1, Hq, Hkv, topk=topk, switch_threshold=thr)
    O = torch.full((cu_q[-1], Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((Hq * cu_q[-1],), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((Hkv * topk * cu_q[-1],), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(api.prefill_varlen_workspace_bytes(p, cu_q, cu_k), 16), dtype=torch.uint8,
                     device="cuda")
    paths = api.prefill_varlen(p, cu_q, cu_k, Qp, Kp, Vp, Kcp, O, lse, idx, ws)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    Og, Lg, ig = f64(O), f64(lse), idx.cpu().numpy()
    G = Hq // Hkv
    for i, (d, (k, q)) in enumerate(zip(datas, seqs)):
        assert paths[i] == (api.PATH_DENSE if k <= thr else api.PATH_SPARSE)
        if q == 0:
            continue
        Qf, Kf, Vf = (wl.bf16_to_f64(d[x])[0] for x in "QKV")
        op = orc.Params(topk=topk, threshold=thr)
        Kc = orc.compress_keys(Kf[None], op)[0]
        q0 = k - q
        Oi = Og[cu_q[i]:cu_q[i + 1]]
        Li = Lg[Hq * cu_q[i]:Hq * cu_q[i + 1]].reshape(Hq, q)
        Ii = ig[Hkv * topk * cu_q[i]:Hkv * topk * cu_q[i + 1]].reshape(Hkv, q, topk)
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            for r in range(q):
                t = q0 + r
                if k > thr:
                    sel = orc.select_query(Qf[t, hs], Kc[:, g], t, op)
                    check_selection_row(sel, Ii[g, r], topk)
                    keys = orc.selected_keys(Ii[g, r], t, op)
                else:
                    keys = np.arange(t + 1)
                o, l = orc.attend(Qf[t, hs], Kf[:, g], Vf[:, g], keys, op.sm_scale(128))
                assert np.abs(Oi[r, hs] - o).max() <= O_ATOL
                assert np.abs(Li[hs, r] - l).max() <= LSE_ATOL
