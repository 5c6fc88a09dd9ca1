"""Why the compressed keys carry a second bf16 plane, and what the scoring
kernel's arithmetic does to the selection, checked on the CPU against the
fp64 oracle with the band rule (selection bit-exact unless the k-th and
(k+1)-th block scores are within 1e-3 relative).

The kernels sum a window's 32 bf16 keys in fp32 in token order, round the mean
to hi = bf16(m) and keep lo = bf16(m - hi).  The block scorer takes each
head's log-sum-exp from q . hi alone and the probabilities from q . (hi + lo).
These tests rebuild those quantities in numpy (fp32 window sums, RNE to bf16)
and run the selection rule in fp64 on them.
"""
import numpy as np

from oracle import infllmv2_oracle as orc
from trainable_block_sparse_compressed_b200 import workloads as wl

from _helpers import check_selection_row


def _bf16(x):
    return wl.bf16_to_f64(wl.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _planes(K_bits, p):
    """hi, lo planes of the compressed keys as the kernels compute them."""
    K = wl.bf16_to_f32(K_bits)
    B, T, Hkv, d = K.shape
    n_c = orc.num_windows(T, p)
    m = np.zeros((B, n_c, Hkv, d), dtype=np.float32)
    for j in range(n_c):
        acc = np.zeros((B, Hkv, d), dtype=np.float32)
        for i in range(p.cmp_kernel):             # fp32, token order
            acc = acc + K[:, j * p.cmp_stride + i]
        m[:, j] = acc * np.float32(1.0 / p.cmp_kernel)
    hi = _bf16(m)
    lo = _bf16(m.astype(np.float64) - hi)
    return hi, lo


def _select_with(q_group, kc_lse, kc_prob, t, p):
    """The selection rule with each head's normaliser from kc_lse and its
    probabilities' numerators from kc_prob."""
    v = min(orc.visible_windows(t, p), kc_prob.shape[0])
    sc = p.sm_scale(q_group.shape[1])
    if v == 0:
        S = np.zeros(0)
    else:
        s_l = sc * (q_group @ kc_lse[:v].T)
        s_p = sc * (q_group @ kc_prob[:v].T)
        mx = s_l.max(axis=1, keepdims=True)
        lse = mx + np.log(np.exp(s_l - mx).sum(axis=1, keepdims=True))
        S = np.exp(s_p - lse).sum(axis=0)
    bs = orc.block_scores(S, t, p)
    chosen, _ = orc.select_from_scores(bs, t, p)
    return orc.pad_row(chosen, p.topk)


def _run(name, rows, variant):
    w = wl.WORKLOADS[name]
    d = wl.make_prefill(w)
    p = orc.Params(topk=w.topk, n_init=w.n_init, n_local=w.n_local, threshold=w.threshold)
    Q, K = wl.bf16_to_f64(d["Q"]), wl.bf16_to_f64(d["K"])
    Kc = orc.compress_keys(K, p)
    hi, lo = _planes(d["K"], p)
    G = w.Hq // w.Hkv
    fails = 0
    for (b, g, t) in rows:
        hs = slice(g * G, (g + 1) * G)
        ref = orc.select_query(Q[b, t, hs], Kc[b, :, g], t, p)
        if variant == "hi_only":
            got = _select_with(Q[b, t, hs], hi[b, :, g], hi[b, :, g], t, p)
        else:  # the scoring kernel: normaliser from hi, probabilities from hi + lo
            got = _select_with(Q[b, t, hs], hi[b, :, g], hi[b, :, g] + lo[b, :, g], t, p)
        try:
            check_selection_row(ref, got, p.topk)
        except AssertionError:
            fails += 1
    return fails


C1_ROWS = [(0, g, t) for g in range(2) for t in range(2048)]
# rows of the T=32768 workload where one bf16 plane broke the band rule, plus
# a random sample
C3_ROWS = [(0, 0, 29172), (0, 0, 29274), (0, 0, 30063), (0, 1, 27422)] + \
    [(0, g, int(t)) for g in range(2) for t in np.random.default_rng(1).integers(0, 32768, 150)]


def test_one_bf16_plane_breaks_the_band_rule():
    """Compressed keys rounded once to bf16 move some rows' selection across
    a score gap wider than the 1e-3 band: the second plane is needed."""
    assert _run("sparse_prefill_T2048_Hq8_Hkv2", C1_ROWS, "hi_only") >= 1
    assert _run("sparse_prefill_T32768_Hq32_Hkv2", C3_ROWS[:4], "hi_only") >= 1


def test_scoring_arithmetic_keeps_every_row_in_the_band():
    """hi + lo probabilities over a hi-only normaliser (what the kernel
    computes): every row of the T=2048 workload and the sampled T=32768 rows,
    the four above included, pass the band rule."""
    assert _run("sparse_prefill_T2048_Hq8_Hkv2", C1_ROWS, "kernel") == 0
    assert _run("sparse_prefill_T32768_Hq32_Hkv2", C3_ROWS, "kernel") == 0
