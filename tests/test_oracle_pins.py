"""Pins for the fp64 oracle: checks against things other than itself.

* hand-derived worked examples (``tests/golden``: exact fractions);
* closed forms of the window mean (ramp, constant) and a prefix-sum
  formulation of the same mean;
* brute-force enumeration of window/block overlaps and visibility;
* an exhaustive, independently written ranking of block scores on tiny
  inputs (pure Python loops with ``math.exp``);
* top-k covering every block reduces to dense causal attention, and dense
  causal attention equals torch's ``scaled_dot_product_attention`` in fp64;
* planted needle blocks are selected; structural invariants of the selection;
* decode: incremental compressed keys equal the batch ones, and a decode step
  equals the prefill row at the same position.
"""
import fractions
import itertools
import json
import math
import os
import re

import numpy as np
import pytest

from oracle import infllmv2_oracle as orc
from trainable_block_sparse_compressed_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# golden worked examples
# --------------------------------------------------------------------------
def _num(s):
    """'3/4', '0', 1.0, 'ln(4)', 'ln(4)/2' -> float."""
    if isinstance(s, (int, float)):
        return float(s)
    m = re.fullmatch(r"ln\((\d+)\)(?:/(\d+))?", s)
    if m:
        v = math.log(int(m.group(1)))
        return v / int(m.group(2)) if m.group(2) else v
    return float(fractions.Fraction(s))


def _build_golden(ex):
    sh = ex["shape"]
    B, T, Hq, Hkv, d = sh["B"], sh["T"], sh["Hq"], sh["Hkv"], sh["d"]
    Q = np.zeros((B, T, Hq, d))
    for h, qv in enumerate(ex["q_per_head"]):
        Q[:, :, h, :] = [_num(x) for x in qv]
    K = np.zeros((B, T, Hkv, d))
    V = np.zeros((B, T, Hkv, d))
    for seg in ex["k_segments"]:
        lo, hi = seg["tokens"]
        K[:, lo:hi + 1, :, :] = [_num(x) for x in seg["value"]]
    for seg in ex["v_segments"]:
        lo, hi = seg["tokens"]
        V[:, lo:hi + 1, :, :] = [_num(x) for x in seg["value"]]
    p = orc.Params(**ex["params"])
    return Q, K, V, p


GOLDEN_FILES = sorted(f for f in os.listdir(GOLDEN) if f.endswith(".json"))


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def check_golden(ex, mod=orc):
    Q, K, V, p = _build_golden(ex)
    Kc = mod.compress_keys(K, p)
    for j, vals in ex["expect"]["kc"].items():
        np.testing.assert_allclose(Kc[0, int(j), 0, :], [_num(v) for v in vals],
                                   rtol=0, atol=1e-12)
    for row in ex["expect"]["rows"]:
        t, g = row["t"], row["g"]
        assert mod.visible_windows(t, p) == row["visible"]
        r = mod.select_row(Q, Kc, 0, g, t, p)
        np.testing.assert_allclose(r.bs, [_num(v) for v in row["bs"]], rtol=1e-12, atol=0)
        assert list(r.idx) == row["idx"]
        idx = np.full((1, K.shape[2], Q.shape[1], p.topk), -1, dtype=np.int32)
        idx[0, g, t] = r.idx
        O, L = mod.sparse_attention(Q, K, V, idx, p, rows=[(0, g, t)])
        G = Q.shape[2] // K.shape[2]
        np.testing.assert_allclose(O[0, t, g * G:(g + 1) * G],
                                   [[_num(x) for x in o] for o in row["O"]], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[0, g * G:(g + 1) * G, t], [_num(x) for x in row["lse"]],
                                   rtol=0, atol=1e-12)
        if "dense_O" in row:
            Od, Ld = mod.dense_attention(Q, K, V, p, rows=[(0, g, t)])
            np.testing.assert_allclose(Od[0, t, g * G:(g + 1) * G],
                                       [[_num(x) for x in o] for o in row["dense_O"]],
                                       rtol=0, atol=1e-12)
            np.testing.assert_allclose(Ld[0, g * G:(g + 1) * G, t],
                                       [_num(x) for x in row["dense_lse"]], rtol=0, atol=1e-12)


@pytest.mark.parametrize("name", GOLDEN_FILES)
def test_golden_worked_examples(name):
    check_golden(load_golden(name))


# --------------------------------------------------------------------------
# compression: closed forms and a second formulation
# --------------------------------------------------------------------------
def test_compress_ramp_and_constant_closed_form():
    p = orc.Params()
    T = 200
    K = np.broadcast_to(np.arange(T, dtype=np.float64)[None, :, None, None], (1, T, 2, 3)).copy()
    Kc = orc.compress_keys(K, p)
    n_c = (T - 32) // 16 + 1
    assert Kc.shape == (1, n_c, 2, 3)
    for j in range(n_c):
        assert np.all(Kc[0, j] == 16 * j + 15.5)  # mean of 16j .. 16j+31
    Kc2 = orc.compress_keys(np.full((2, 77, 1, 4), -2.25), p)
    assert Kc2.shape[1] == (77 - 32) // 16 + 1 and np.all(Kc2 == -2.25)
    assert orc.compress_keys(np.zeros((1, 31, 1, 2)), p).shape[1] == 0
    assert orc.compress_keys(np.zeros((1, 32, 1, 2)), p).shape[1] == 1


def test_compress_matches_prefix_sums():
    p = orc.Params()
    rng = np.random.default_rng(0)
    K = rng.standard_normal((2, 517, 3, 8))
    csum = np.concatenate([np.zeros((2, 1, 3, 8)), np.cumsum(K, axis=1)], axis=1)
    n_c = (517 - 32) // 16 + 1
    ref = np.stack([(csum[:, 16 * j + 32] - csum[:, 16 * j]) / 32.0 for j in range(n_c)], axis=1)
    np.testing.assert_allclose(orc.compress_keys(K, p), ref, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# window visibility and block overlap by brute force over token sets
# --------------------------------------------------------------------------
@pytest.mark.parametrize("kernel,stride,block", [(32, 16, 64), (32, 32, 64), (16, 8, 32), (64, 16, 64)])
def test_windows_of_block_bruteforce(kernel, stride, block):
    p = orc.Params(block_size=block, cmp_kernel=kernel, cmp_stride=stride)
    for T in [1, 31, 32, 33, 100, 257, 640]:
        for t in range(T):
            vis = [j for j in range(0, T) if j * stride + kernel - 1 <= t]
            assert orc.visible_windows(t, p) == len(vis)
            for b in range(t // block + 1):
                toks = set(range(b * block, b * block + block))
                want = [j for j in vis if toks & set(range(j * stride, j * stride + kernel))]
                assert orc.windows_of_block(b, len(vis), p) == want


# --------------------------------------------------------------------------
# selection against an independent exhaustive ranking on tiny inputs
# --------------------------------------------------------------------------
def _brute_block_scores(q_heads, kc_rows, t, scale, kernel, stride, block):
    """Independent pure-Python computation of the block scores of one row."""
    vis = [j for j in range(len(kc_rows)) if j * stride + kernel - 1 <= t]
    n_blocks = t // block + 1
    if not vis:
        return [-math.inf] * n_blocks
    S = {j: 0.0 for j in vis}
    for q in q_heads:
        logits = {j: scale * sum(a * b for a, b in zip(q, kc_rows[j])) for j in vis}
        top = max(logits.values())
        z = sum(math.exp(v - top) for v in logits.values())
        for j in vis:
            S[j] += math.exp(logits[j] - top) / z
    out = []
    for b in range(n_blocks):
        toks = set(range(b * block, (b + 1) * block))
        vals = [S[j] for j in vis if toks & set(range(j * stride, j * stride + kernel))]
        out.append(max(vals) if vals else -math.inf)
    return out


def _rank_select(bs, t, k, n_init, n_local, block):
    """b is kept iff forced, or fewer than `free` candidates beat it."""
    cur = t // block
    forced = {b for b in range(cur + 1) if b < n_init or b > cur - n_local}
    cands = [b for b in range(cur + 1) if b not in forced]
    free = k - len(forced)

    def beats(c, b):
        return bs[c] > bs[b] or (bs[c] == bs[b] and c < b)
    chosen = set(forced)
    for b in cands:
        if sum(1 for c in cands if c != b and beats(c, b)) < free:
            chosen.add(b)
    return sorted(chosen)


@pytest.mark.parametrize("seed,G,T,d,k", [(0, 1, 300, 4, 3), (1, 2, 512, 8, 4), (2, 4, 450, 16, 5),
                                          (3, 3, 400, 6, 6), (4, 2, 257, 5, 8)])
def test_selection_equals_exhaustive_ranking(seed, G, T, d, k):
    rng = np.random.default_rng(seed)
    Hkv = 2
    p = orc.Params(topk=k)
    Q = rng.standard_normal((1, T, G * Hkv, d))
    K = rng.standard_normal((1, T, Hkv, d))
    # quantise some keys so that exact ties between windows happen
    K[:, ::3] = np.round(K[:, ::3])
    Kc = orc.compress_keys(K, p)
    for t in list(range(0, T, 7)) + [T - 1]:
        for g in range(Hkv):
            r = orc.select_row(Q, Kc, 0, g, t, p)
            ref = _brute_block_scores(Q[0, t, g * G:(g + 1) * G].tolist(), Kc[0, :, g].tolist(), t,
                                      1 / math.sqrt(d), 32, 16, 64)
            np.testing.assert_allclose(r.bs, ref, rtol=1e-12, atol=1e-15)
            chosen = _rank_select(list(r.bs), t, k, 1, 2, 64)
            want = chosen + [-1] * (k - len(chosen))
            assert list(r.idx) == want, (t, g)


def test_exact_tie_goes_to_lower_block():
    p = orc.Params(topk=4)
    bs = np.array([0.1, 0.5, 0.5, 0.5, 0.2, 0.3, 0.3])
    chosen, ranked = orc.select_from_scores(bs, 6 * 64 + 5, p)   # cur = 6 -> forced {0, 5, 6}
    assert chosen == [0, 1, 5, 6]
    assert ranked[:3] == [1, 2, 3]
    bs2 = np.array([0.1, -np.inf, 0.2, 0.2, 0.0, 0.3])
    chosen2, ranked2 = orc.select_from_scores(bs2, 5 * 64, orc.Params(topk=5))
    assert chosen2 == [0, 2, 3, 4, 5] and ranked2[-1] == 1


# --------------------------------------------------------------------------
# attention: dense reduces to torch SDPA; full top-k reduces to dense
# --------------------------------------------------------------------------
def _torch_causal(Q, K, V):
    import torch
    import torch.nn.functional as F
    B, T, Hq, d = Q.shape
    G = Hq // K.shape[2]
    q = torch.from_numpy(Q).permute(0, 2, 1, 3)
    k = torch.from_numpy(np.repeat(K, G, axis=2)).permute(0, 2, 1, 3)
    v = torch.from_numpy(np.repeat(V, G, axis=2)).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(d)
    mask = torch.triu(torch.ones(T, T, dtype=torch.bool), 1)
    lse = torch.logsumexp(s.masked_fill(mask, -math.inf), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def test_dense_equals_torch_sdpa():
    rng = np.random.default_rng(5)
    Q = rng.standard_normal((2, 150, 4, 16))
    K = rng.standard_normal((2, 150, 2, 16))
    V = rng.standard_normal((2, 150, 2, 16))
    p = orc.Params()
    O, L = orc.dense_attention(Q, K, V, p)
    O_ref, L_ref = _torch_causal(Q, K, V)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, rtol=0, atol=1e-12)


def test_topk_covering_all_blocks_is_dense():
    rng = np.random.default_rng(6)
    T = 700
    Q = rng.standard_normal((1, T, 4, 16))
    K = rng.standard_normal((1, T, 2, 16))
    V = rng.standard_normal((1, T, 2, 16))
    p = orc.Params(topk=(T + 63) // 64, threshold=0)
    O, L, path, idx = orc.forward(Q, K, V, p)
    assert path == "sparse"
    Od, Ld = orc.dense_attention(Q, K, V, p)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


def test_switch_threshold():
    p = orc.Params(threshold=4096)
    assert orc.uses_dense(4096, p) and not orc.uses_dense(4097, p)
    assert orc.uses_dense(1, orc.Params(threshold=8192))
    assert not orc.uses_dense(2048, orc.Params(threshold=0))


# --------------------------------------------------------------------------
# the smallest workload: needles and invariants
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def small_case():
    w = wl.WORKLOADS["sparse_prefill_T2048_Hq8_Hkv2"]
    data = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(data[x]) for x in "QKV")
    p = orc.Params(topk=w.topk, n_init=w.n_init, n_local=w.n_local, threshold=w.threshold)
    idx, det = orc.select_blocks(Q, K, p)
    return w, data, Q, K, V, p, idx, det


def test_needles_are_selected(small_case):
    w, data, Q, K, V, p, idx, det = small_case
    assert len(data["needles"]) == w.needles
    # a needle is kept for nearly every query row of its range; an ordinary
    # candidate block is kept at about the chance rate free/candidates.
    needle_blocks = {nd.block for nd in data["needles"]}
    for nd in data["needles"]:
        hits = [nd.block in idx[nd.batch, g, t]
                for t in range(nd.query_block * 64, nd.query_block * 64 + 64)
                for g in range(w.Hkv)]
        assert np.mean(hits) >= 0.9, (nd, np.mean(hits))
        other = [b for b in range(1, nd.query_block - 1) if b not in needle_blocks]
        rate = np.mean([b in idx[nd.batch, g, t] for b in other
                        for t in range(nd.query_block * 64, nd.query_block * 64 + 64)
                        for g in range(w.Hkv)])
        assert rate < 0.5, (nd, rate)


def test_selection_invariants(small_case):
    w, data, Q, K, V, p, idx, det = small_case
    G = w.Hq // w.Hkv
    Kc = orc.compress_keys(K, p)
    for (b, g, t), r in det.items():
        row = [x for x in r.idx if x >= 0]
        cur = t // 64
        assert row == sorted(set(row))
        assert len(row) == min(p.topk, cur + 1)
        assert all(0 <= x <= cur for x in row)
        assert set(r.forced) <= set(row)
        assert list(r.idx[len(row):]) == [-1] * (p.topk - len(row))
        if t % 97 == 0:
            P = orc.head_probs(Q[b, t, g * G:(g + 1) * G], Kc[b, :, g], t, p)
            if P.shape[1]:
                np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------
def test_decode_incremental_equals_batch_and_prefill_row():
    rng = np.random.default_rng(7)
    B, L0, Hq, Hkv, d, steps = 2, 250, 4, 2, 16, 40
    p = orc.Params(topk=3)
    K0 = rng.standard_normal((B, L0, Hkv, d))
    V0 = rng.standard_normal((B, L0, Hkv, d))
    st = orc.DecodeState.from_prefill(K0, V0, p)
    for s in range(steps):
        q = rng.standard_normal((B, Hq, d))
        kn = rng.standard_normal((B, Hkv, d))
        vn = rng.standard_normal((B, Hkv, d))
        O, Ls, idx = orc.decode_step(st, q, kn, vn, p)
        t = L0 + s
        Kfull = np.stack(st.K)
        Vfull = np.stack(st.V)
        np.testing.assert_allclose(np.stack(st.Kc), orc.compress_keys(Kfull, p), rtol=0, atol=1e-13)
        Qfull = np.zeros((B, t + 1, Hq, d))
        Qfull[:, t] = q
        rows = [(b, g, t) for b in range(B) for g in range(Hkv)]
        idx_p, _ = orc.select_blocks(Qfull, Kfull, p, rows)
        Op, Lp = orc.sparse_attention(Qfull, Kfull, Vfull, idx_p, p, rows)
        assert np.array_equal(idx_p[:, :, t], idx)
        np.testing.assert_allclose(Op[:, t], O, rtol=0, atol=1e-13)
        np.testing.assert_allclose(Lp[:, :, t], Ls, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# planted mistakes: each pin above must catch a plausible oracle bug
# --------------------------------------------------------------------------
def _contained_windows(b, n_visible, p):
    j_lo = -((-(b * p.block_size)) // p.cmp_stride)
    j_hi = min(n_visible - 1, (b * p.block_size + p.block_size - p.cmp_kernel) // p.cmp_stride)
    return list(range(j_lo, j_hi + 1))


def _logit_group_scores(q_group, Kc_g, t, p):
    v = min(p_vis(t, p), Kc_g.shape[0])
    return (p.sm_scale(q_group.shape[1]) * (q_group @ Kc_g[:v].T)).sum(axis=0)


def p_vis(t, p):
    return orc.visible_windows(t, p)


def _reversed_ties(bs, t, p):
    forced = orc.forced_blocks(t, p)
    cands = [b for b in range(t // p.block_size + 1) if b not in forced]
    ranked = sorted(cands, key=lambda b: (-bs[b], -b))
    return sorted(forced + ranked[:p.topk - len(forced)]), ranked


def _no_causal_clip(idx_row, t, p):
    keys = []
    for blk in idx_row:
        if blk >= 0:
            keys.extend(range(int(blk) * p.block_size, int(blk) * p.block_size + p.block_size))
    return np.asarray(sorted(set(keys)))


def _visible_off_by_one(t, p):
    return max(0, (t - p.cmp_kernel) // p.cmp_stride + 1) if t >= p.cmp_kernel else 0


@pytest.mark.parametrize("attr,bad", [
    ("windows_of_block", _contained_windows),
    ("group_scores", _logit_group_scores),
    ("select_from_scores", _reversed_ties),
    ("selected_keys", _no_causal_clip),
    ("visible_windows", _visible_off_by_one),
])
def test_planted_oracle_mistakes_are_caught(monkeypatch, attr, bad):
    monkeypatch.setattr(orc, attr, bad)
    caught = 0
    for name in GOLDEN_FILES:
        try:
            check_golden(load_golden(name))
        except (AssertionError, IndexError, ValueError):
            caught += 1
    assert caught >= 1, f"no golden pin caught a broken {attr}"


@pytest.mark.parametrize("q0,Tq,threshold", [(0, 700, 0), (300, 400, 0), (333, 367, 0),
                                              (640, 60, 0), (500, 200, 8192)])
def test_chunk_forward_equals_the_whole_sequence_rows(q0, Tq, threshold):
    """A chunk of queries over the full caches gives exactly the rows q0..q0+Tq-1
    of the whole-sequence forward (sparse and dense), including the selection."""
    w = wl.small_workload(B=2, T=q0 + Tq, Hq=8, Hkv=2, topk=5, needles=1, seed=31,
                          threshold=threshold)
    d = wl.make_prefill(w)
    Q, K, V = (wl.bf16_to_f64(d[x]) for x in "QKV")
    p = orc.Params(topk=w.topk, n_init=w.n_init, n_local=w.n_local, threshold=threshold)
    O, L, path, idx = orc.forward(Q, K, V, p)
    Oc, Lc, path_c, idx_c = orc.chunk_forward(Q[:, q0:], K, V, q0, p)
    assert path_c == path
    assert np.array_equal(Oc, O[:, q0:]) and np.array_equal(Lc, L[:, :, q0:])
    if idx is not None:
        assert np.array_equal(idx_c, idx[:, :, q0:])


def _tiny_sparse_case(seed=41, T=200, Hq=4, Hkv=2, d=16, topk=3):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((1, T, Hq, d))
    K = rng.standard_normal((1, T, Hkv, d))
    V = rng.standard_normal((1, T, Hkv, d))
    p = orc.Params(topk=topk, n_init=1, n_local=1, threshold=0)
    idx, _ = orc.select_blocks(Q, K, p)
    return Q, K, V, idx, p


def test_sparse_backward_matches_finite_differences():
    """Central differences of L = sum(dO * O) with the selection held fixed."""
    Q, K, V, idx, p = _tiny_sparse_case()
    rng = np.random.default_rng(5)
    dO = rng.standard_normal(Q.shape)
    loss = lambda Q_, K_, V_: float((orc.sparse_attention(Q_, K_, V_, idx, p)[0] * dO).sum())  # noqa: E731
    dQ, dK, dV = orc.sparse_attention_backward(Q, K, V, idx, dO, p)
    eps = 1e-6
    picks = [(0, 150, 1, 3), (0, 70, 0, 0), (0, 199, 3, 15)]
    for (b, t, h, c) in picks:
        Qp, Qm = Q.copy(), Q.copy()
        Qp[b, t, h, c] += eps
        Qm[b, t, h, c] -= eps
        num = (loss(Qp, K, V) - loss(Qm, K, V)) / (2 * eps)
        assert abs(num - dQ[b, t, h, c]) <= 1e-6 * max(1.0, abs(num))
    for (b, t, g, c) in [(0, 3, 0, 2), (0, 130, 1, 7), (0, 64, 1, 0)]:
        for X, dX in ((K, dK), (V, dV)):
            Xp, Xm = X.copy(), X.copy()
            Xp[b, t, g, c] += eps
            Xm[b, t, g, c] -= eps
            args_p = (Q, Xp, V) if X is K else (Q, K, Xp)
            args_m = (Q, Xm, V) if X is K else (Q, K, Xm)
            num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(num - dX[b, t, g, c]) <= 1e-6 * max(1.0, abs(num))


def test_sparse_backward_with_every_block_equals_dense_autograd():
    """top-k covering every block: the gradients equal torch autograd (fp64)
    of exact causal softmax attention."""
    import torch
    Q, K, V, _, _ = _tiny_sparse_case(T=190, topk=3)
    p = orc.Params(topk=8, n_init=1, n_local=1, threshold=0)
    idx, _ = orc.select_blocks(Q, K, p)
    dO = np.random.default_rng(6).standard_normal(Q.shape)
    dQ, dK, dV = orc.sparse_attention_backward(Q, K, V, idx, dO, p)
    G = Q.shape[2] // K.shape[2]
    q = torch.tensor(Q, requires_grad=True)
    k = torch.tensor(K, requires_grad=True)
    v = torch.tensor(V, requires_grad=True)
    kk = k.repeat_interleave(G, dim=2)
    vv = v.repeat_interleave(G, dim=2)
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2), is_causal=True,
        scale=p.sm_scale(Q.shape[-1])).transpose(1, 2)
    (out * torch.tensor(dO)).sum().backward()
    assert np.allclose(dQ, q.grad.numpy(), atol=1e-10)
    assert np.allclose(dK, k.grad.numpy(), atol=1e-10)
    assert np.allclose(dV, v.grad.numpy(), atol=1e-10)


def test_compressed_attention_with_equal_keys_averages_the_window_values():
    """Closed form: with every key equal, all visible windows score alike and
    the output is the plain mean of the visible windows' mean values."""
    rng = np.random.default_rng(12)
    T, d = 300, 16
    Q = rng.standard_normal((1, T, 4, d))
    K = np.broadcast_to(rng.standard_normal((1, 1, 2, d)), (1, T, 2, d)).copy()
    V = rng.standard_normal((1, T, 2, d))
    p = orc.Params()
    O, L = orc.compressed_attention(Q, K, V, p)
    for t in (0, 30, 31, 46, 47, 299):
        v = 0 if t < 31 else (t - 31) // 16 + 1
        for h in range(4):
            g = h // 2
            if v == 0:
                assert np.all(O[0, t, h] == 0) and L[0, h, t] == -np.inf
                continue
            win_means = [V[0, 16 * j:16 * j + 32, g].mean(axis=0) for j in range(v)]
            assert np.allclose(O[0, t, h], np.mean(win_means, axis=0), atol=1e-12)
            s = (Q[0, t, h] @ K[0, 0, g]) / np.sqrt(d)
            assert np.isclose(L[0, h, t], s + np.log(v))


def test_compressed_attention_equals_masked_sdpa():
    """Against torch's fp64 scaled_dot_product_attention over the window
    means with an explicit visibility mask."""
    import torch
    rng = np.random.default_rng(13)
    T, d, Hq, Hkv = 260, 16, 4, 2
    Q = rng.standard_normal((1, T, Hq, d))
    K = rng.standard_normal((1, T, Hkv, d))
    V = rng.standard_normal((1, T, Hkv, d))
    p = orc.Params()
    O, _ = orc.compressed_attention(Q, K, V, p)
    n = (T - 32) // 16 + 1
    Kc = np.stack([K[:, 16 * j:16 * j + 32].mean(axis=1) for j in range(n)], axis=1)
    Vc = np.stack([V[:, 16 * j:16 * j + 32].mean(axis=1) for j in range(n)], axis=1)
    t = np.arange(T)[:, None]
    j = np.arange(n)[None, :]
    mask = torch.tensor(16 * j + 31 <= t)                        # [T, n]
    rows = mask.any(dim=1).numpy()
    q = torch.tensor(Q).transpose(1, 2)
    kk = torch.tensor(Kc).repeat_interleave(Hq // Hkv, dim=2).transpose(1, 2)
    vv = torch.tensor(Vc).repeat_interleave(Hq // Hkv, dim=2).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, :, rows], kk, vv, attn_mask=mask[rows]).transpose(1, 2).numpy()
    assert np.allclose(O[:, rows], ref, atol=1e-12)
    assert np.all(O[:, ~rows] == 0)
