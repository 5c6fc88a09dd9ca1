"""fp64 CPU oracle for InfLLM-V2 dense-sparse switchable attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check and the benchmark's CPU
baseline leg do.  It shares no code with the CUDA library; it reads the same
seeded inputs (bfloat16 bit patterns, widened exactly to float64).

It is deliberately plain and slow: every query row is computed on its own,
in float64, in the order the method states its steps:

1. compressed keys: the mean of each 32-token key window, one window every
   16 tokens (the compressed pattern aggregates tokens hierarchically:
   InfLLM-V2 skill write-up, Core Concept; kernel 32 / stride 16 are the
   method's settings);
2. scores of one query token against the compressed keys it may see, a
   softmax per query head, then a sum over the query heads of each GQA group
   (the group summation the skill write-up's Architecture Overview, Hardware
   Kernel bullet, fuses into its attention loop with an LSE approximation;
   computed here exactly);
3. max-pool of the group score onto 64-token key blocks (block size 64,
   skill write-up, Implementation Step 2);
4. block selection: the initial block and the local (sliding-window) blocks
   are always kept, the other slots go to the highest-scoring blocks (the
   first of two steps picks the relevant key/value blocks: reportify digest,
   Technical Mechanism; the sliding pattern keeps local context: skill
   write-up, Core Concept);
5. causal attention over the keys of the selected blocks only (the second
   step: reportify digest, Technical Mechanism), and exact dense causal
   attention when the sequence is not longer than the switch threshold
   (skill write-up, Architecture Overview, dense pathway bullet, and
   Implementation Step 3, whose switch returns the dense result when the
   length is at most the threshold).

Readings where the pages are silent (each is listed in the design notes):

* A compressed window ``j`` (tokens ``[16j, 16j+31]``) is visible to query
  token ``t`` only when it lies wholly at or before ``t``: ``16j + 31 <= t``
  (causality: the skill write-up's When NOT to Use list warns that the
  sliding window must only look at past tokens).
* The group sum adds per-head softmax *probabilities* (the pages tie the
  group summation to LSE, i.e. to normalised scores).
* Block ``b`` pools every visible window that overlaps its tokens
  ``[64b, 64b+63]``; with kernel 32 / stride 16 that is ``j in [4b-1, 4b+3]``.
  A block with no visible window scores ``-inf``.
* Forced blocks: blocks ``0 .. n_init-1`` and the ``n_local`` most recent
  blocks ``cur-n_local+1 .. cur`` with ``cur = t // 64``, clipped to
  ``[0, cur]`` and de-duplicated.  The remaining ``topk - |forced|`` slots go
  to the other blocks ``b <= cur`` in descending score; equal scores go to the
  lower block index; ``-inf`` ranks last.  Fewer candidates than slots: all
  are taken and the row is padded with ``-1``.  Indices are ascending.
* Softmax scale ``1/sqrt(d)``; LSE is the natural log of the sum of
  ``exp(scale * q.k)`` over the attended keys.
* Decode: the new key/value is appended at position ``pos = seqlen`` first,
  a compressed key is appended when window ``(pos-31)/16`` completes, then the
  new token attends as query row ``t = pos``.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = float("-inf")


@dataclasses.dataclass(frozen=True)
class Params:
    """The method's knobs (skill write-up, Implementation Steps 2-3)."""
    block_size: int = 64
    cmp_kernel: int = 32
    cmp_stride: int = 16
    topk: int = 64
    n_init: int = 1
    n_local: int = 2
    threshold: int = 8192
    scale: Optional[float] = None  # None: 1/sqrt(d)

    def sm_scale(self, d: int) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(d)


# --------------------------------------------------------------------------
# step 1: compressed keys
# --------------------------------------------------------------------------
def num_windows(T: int, p: Params) -> int:
    """Number of complete compression windows in a sequence of T tokens."""
    if T < p.cmp_kernel:
        return 0
    return (T - p.cmp_kernel) // p.cmp_stride + 1


def compress_keys(K: np.ndarray, p: Params) -> np.ndarray:
    """Kc[b, j, g, :] = mean of K[b, i, g, :] over i in [16j, 16j+31].

    K: [B, T, Hkv, d] float64  ->  Kc: [B, n_c, Hkv, d] float64.
    """
    B, T, Hkv, d = K.shape
    n_c = num_windows(T, p)
    Kc = np.zeros((B, n_c, Hkv, d), dtype=np.float64)
    for j in range(n_c):
        start = j * p.cmp_stride
        Kc[:, j] = K[:, start:start + p.cmp_kernel].mean(axis=1)
    return Kc


def visible_windows(t: int, p: Params) -> int:
    """How many windows lie wholly at or before token t (16j + 31 <= t)."""
    if t < p.cmp_kernel - 1:
        return 0
    return (t - (p.cmp_kernel - 1)) // p.cmp_stride + 1


def windows_of_block(b: int, n_visible: int, p: Params) -> List[int]:
    """Visible windows j whose tokens [16j, 16j+31] overlap block b's tokens.

    Window j overlaps [lo, hi] iff 16j <= hi and 16j + 31 >= lo, i.e.
    ceil((lo - 31) / 16) <= j <= floor(hi / 16); with kernel 32, stride 16
    and block 64 that is j in [4b-1, 4b+3].
    """
    lo_tok = b * p.block_size
    hi_tok = lo_tok + p.block_size - 1
    j_lo = max(0, -((p.cmp_kernel - 1 - lo_tok) // p.cmp_stride))
    j_hi = min(n_visible - 1, hi_tok // p.cmp_stride)
    return list(range(j_lo, j_hi + 1))


# --------------------------------------------------------------------------
# steps 2-3: per-head softmax over compressed keys, group sum, block max-pool
# --------------------------------------------------------------------------
def head_probs(q_group: np.ndarray, Kc_g: np.ndarray, t: int, p: Params) -> np.ndarray:
    """Softmax over the visible compressed keys, one row per query head.

    q_group: [G, d]; Kc_g: [n_c, d].  Returns [G, v(t)].
    """
    v = min(visible_windows(t, p), Kc_g.shape[0])
    G, d = q_group.shape
    if v == 0:
        return np.zeros((G, 0))
    s = p.sm_scale(d) * (q_group @ Kc_g[:v].T)          # [G, v]
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def group_scores(q_group: np.ndarray, Kc_g: np.ndarray, t: int, p: Params) -> np.ndarray:
    """S[j] = sum over the group's heads of the per-head probabilities."""
    return head_probs(q_group, Kc_g, t, p).sum(axis=0)


def block_scores(S: np.ndarray, t: int, p: Params) -> np.ndarray:
    """bs[b] = max of S over the visible windows overlapping block b, b <= t//64."""
    cur = t // p.block_size
    bs = np.full(cur + 1, NEG_INF)
    for b in range(cur + 1):
        js = windows_of_block(b, S.shape[0], p)
        if js:
            bs[b] = max(S[j] for j in js)
    return bs


# --------------------------------------------------------------------------
# step 4: block selection
# --------------------------------------------------------------------------
def forced_blocks(t: int, p: Params) -> List[int]:
    """Initial blocks and the local (most recent) blocks of query token t."""
    cur = t // p.block_size
    forced = set(range(0, min(p.n_init, cur + 1)))
    forced |= set(range(max(0, cur - p.n_local + 1), cur + 1))
    return sorted(forced)


def select_from_scores(bs: np.ndarray, t: int, p: Params) -> Tuple[List[int], List[int]]:
    """Returns (selected blocks ascending, ranked free candidates).

    The ranking orders the non-forced blocks b <= t//64 by descending score,
    ties to the lower index, -inf last.
    """
    forced = forced_blocks(t, p)
    cur = t // p.block_size
    free = p.topk - len(forced)
    if free < 0:
        raise ValueError("topk smaller than the forced block count")
    candidates = [b for b in range(cur + 1) if b not in forced]
    ranked = sorted(candidates, key=lambda b: (-bs[b], b))
    chosen = sorted(forced + ranked[:free])
    return chosen, ranked


def pad_row(chosen: Sequence[int], k: int) -> np.ndarray:
    row = np.full(k, -1, dtype=np.int32)
    row[:len(chosen)] = np.asarray(chosen, dtype=np.int32)
    return row


@dataclasses.dataclass
class RowSelection:
    idx: np.ndarray        # [topk] int32 ascending, -1 padded
    bs: np.ndarray         # [t//64 + 1] float64 block scores
    ranked: List[int]      # free candidates, best first
    forced: List[int]
    free_slots: int


def select_query(q_group: np.ndarray, Kc_g: np.ndarray, t: int, p: Params) -> RowSelection:
    """Selection for the heads q_group [G, d] of query token t over Kc_g [n, d]."""
    S = group_scores(q_group, Kc_g, t, p)
    bs = block_scores(S, t, p)
    chosen, ranked = select_from_scores(bs, t, p)
    forced = forced_blocks(t, p)
    return RowSelection(pad_row(chosen, p.topk), bs, ranked, forced,
                        p.topk - len(forced))


def select_row(Q: np.ndarray, Kc: np.ndarray, b: int, g: int, t: int,
               p: Params) -> RowSelection:
    """Selection for one (batch, kv head, query token)."""
    Hq, Hkv = Q.shape[2], Kc.shape[2]
    G = Hq // Hkv
    return select_query(Q[b, t, g * G:(g + 1) * G, :], Kc[b, :, g, :], t, p)


def select_blocks(Q: np.ndarray, K: np.ndarray, p: Params,
                  rows: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Block indices [B, Hkv, T, topk] (or only the listed (b, g, t) rows).

    Returns (idx, details) where details maps (b, g, t) -> RowSelection.
    """
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    Kc = compress_keys(K, p)
    if rows is None:
        rows = [(b, g, t) for b in range(B) for g in range(Hkv) for t in range(T)]
    idx = np.full((B, Hkv, T, p.topk), -1, dtype=np.int32)
    details = {}
    for (b, g, t) in rows:
        r = select_row(Q, Kc, b, g, t, p)
        idx[b, g, t] = r.idx
        details[(b, g, t)] = r
    return idx, details


# --------------------------------------------------------------------------
# step 5: attention
# --------------------------------------------------------------------------
def attend(q_group: np.ndarray, K_g: np.ndarray, V_g: np.ndarray,
           keys: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of the group's heads over the listed key positions.

    Returns (O [G, d], LSE [G]) with LSE = log sum exp(scale * q.k).
    """
    s = scale * (q_group @ K_g[keys].T)                 # [G, n]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    O = (e / z) @ V_g[keys]
    lse = (m + np.log(z))[:, 0]
    return O, lse


def selected_keys(idx_row: np.ndarray, t: int, p: Params) -> np.ndarray:
    """Token positions of the selected blocks, clipped causally to [0, t]."""
    keys = []
    for blk in idx_row:
        if blk < 0:
            continue
        lo = int(blk) * p.block_size
        hi = min(lo + p.block_size - 1, t)
        keys.extend(range(lo, hi + 1))
    return np.asarray(sorted(set(keys)), dtype=np.int64)


def sparse_attention(Q, K, V, idx, p: Params, rows=None):
    """O [B, T, Hq, d], LSE [B, Hq, T] over each row's selected blocks.

    ``rows``: optional list of (b, g, t); other rows are left as NaN.
    """
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    O = np.full((B, T, Hq, d), np.nan)
    L = np.full((B, Hq, T), np.nan)
    if rows is None:
        rows = [(b, g, t) for b in range(B) for g in range(Hkv) for t in range(T)]
    sc = p.sm_scale(d)
    for (b, g, t) in rows:
        keys = selected_keys(idx[b, g, t], t, p)
        o, lse = attend(Q[b, t, g * G:(g + 1) * G], K[b, :, g], V[b, :, g], keys, sc)
        O[b, t, g * G:(g + 1) * G] = o
        L[b, g * G:(g + 1) * G, t] = lse
    return O, L


def attend_backward(q_group, K_g, V_g, keys, scale, dO_group):
    """Gradients of attend() for one row: the softmax attention of the group's
    heads q_group [G, d] over the listed keys, given dO [G, d].

    With s = scale q.k, P = softmax(s), o = P V:
      dV[keys] += P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * o)),
      dq = scale dS K[keys],  dK[keys] += scale dS^T q.
    Returns (dq [G, d], dK_rows [n, d], dV_rows [n, d]) for the listed keys.
    """
    Kk, Vk = K_g[keys], V_g[keys]
    s = scale * (q_group @ Kk.T)                          # [G, n]
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    o = P @ Vk                                            # [G, d]
    dV = P.T @ dO_group                                   # [n, d]
    dP = dO_group @ Vk.T                                  # [G, n]
    dS = P * (dP - (dO_group * o).sum(axis=1, keepdims=True))
    dq = scale * dS @ Kk
    dK = scale * dS.T @ q_group
    return dq, dK, dV


def sparse_attention_backward(Q, K, V, idx, dO, p: Params):
    """Gradients (dQ, dK, dV) of sparse_attention's O with the selection idx
    held fixed (the selection is a discrete choice; training propagates
    through the attention over the chosen blocks), given dO [B, T, Hq, d].
    Keys shared by several rows accumulate their contributions."""
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    sc = p.sm_scale(d)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            for t in range(T):
                keys = selected_keys(idx[b, g, t], t, p)
                dq, dk, dv = attend_backward(Q[b, t, hs], K[b, :, g], V[b, :, g], keys, sc,
                                             dO[b, t, hs])
                dQ[b, t, hs] = dq
                np.add.at(dK[b, :, g], keys, dk)
                np.add.at(dV[b, :, g], keys, dv)
    return dQ, dK, dV


def compressed_attention(Q, K, V, p: Params, rows=None):
    """The compressed-attention branch (skill write-up, Core Concept: the
    compressed pattern aggregates tokens hierarchically): each query row
    attends over the compressed windows it can see, with keys Kc[j] and values
    Vc[j] the means of K and V over window j.  Visibility follows the
    selection's rule (window j visible to t iff 16j+31 <= t); a row with no
    visible window gets O = 0 and LSE = -inf.

    Returns (O [B, T, Hq, d], LSE [B, Hq, T]); ``rows`` as in sparse_attention.
    """
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    Kc, Vc = compress_keys(K, p), compress_keys(V, p)   # the same window means
    O = np.full((B, T, Hq, d), np.nan)
    L = np.full((B, Hq, T), np.nan)
    if rows is None:
        rows = [(b, g, t) for b in range(B) for g in range(Hkv) for t in range(T)]
    sc = p.sm_scale(d)
    for (b, g, t) in rows:
        hs = slice(g * G, (g + 1) * G)
        v = min(visible_windows(t, p), Kc.shape[1])
        if v == 0:
            O[b, t, hs] = 0.0
            L[b, hs, t] = -np.inf
            continue
        o, lse = attend(Q[b, t, hs], Kc[b, :, g], Vc[b, :, g], np.arange(v), sc)
        O[b, t, hs] = o
        L[b, hs, t] = lse
    return O, L


def dense_attention(Q, K, V, p: Params, rows=None):
    """Exact causal softmax attention (every key 0..t)."""
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    O = np.full((B, T, Hq, d), np.nan)
    L = np.full((B, Hq, T), np.nan)
    if rows is None:
        rows = [(b, g, t) for b in range(B) for g in range(Hkv) for t in range(T)]
    sc = p.sm_scale(d)
    for (b, g, t) in rows:
        keys = np.arange(t + 1)
        o, lse = attend(Q[b, t, g * G:(g + 1) * G], K[b, :, g], V[b, :, g], keys, sc)
        O[b, t, g * G:(g + 1) * G] = o
        L[b, g * G:(g + 1) * G, t] = lse
    return O, L


def uses_dense(T: int, p: Params) -> bool:
    """The length switch: dense when T <= threshold (skill write-up, Step 3)."""
    return T <= p.threshold


def forward(Q, K, V, p: Params, rows=None):
    """The switchable attention: dense below the threshold, else sparse.

    Returns (O, LSE, path, idx) with path 'dense' or 'sparse'.
    """
    T = Q.shape[1]
    if uses_dense(T, p):
        O, L = dense_attention(Q, K, V, p, rows)
        return O, L, "dense", None
    idx, _ = select_blocks(Q, K, p, rows)
    O, L = sparse_attention(Q, K, V, idx, p, rows)
    return O, L, "sparse", idx


def chunk_forward(Qc, K, V, q0: int, p: Params, rows=None):
    """Chunked prefill: the queries Qc [B, Tq, Hq, d] are tokens q0 .. q0+Tq-1
    of sequences whose keys and values K, V [B, q0+Tq, Hkv, d] are all known.
    Row i is what forward() gives token q0+i of the whole sequence: the same
    length switch on T = q0+Tq, selection over the compressed keys visible at
    t = q0+i and blocks <= t/64, attention over keys <= t.

    Returns (O [B, Tq, Hq, d], LSE [B, Hq, Tq], path, idx [B, Hkv, Tq, topk]
    or None); ``rows``: optional list of (b, g, i).
    """
    B, Tq, Hq, d = Qc.shape
    T = K.shape[1]
    assert T == q0 + Tq
    Hkv = K.shape[2]
    G = Hq // Hkv
    if rows is None:
        rows = [(b, g, i) for b in range(B) for g in range(Hkv) for i in range(Tq)]
    dense = uses_dense(T, p)
    Kc = None if dense else compress_keys(K, p)
    O = np.full((B, Tq, Hq, d), np.nan)
    L = np.full((B, Hq, Tq), np.nan)
    idx = None if dense else np.full((B, Hkv, Tq, p.topk), -1, dtype=np.int32)
    sc = p.sm_scale(d)
    for (b, g, i) in rows:
        t = q0 + i
        qg = Qc[b, i, g * G:(g + 1) * G]
        if dense:
            keys = np.arange(t + 1)
        else:
            r = select_query(qg, Kc[b, :, g, :], t, p)
            idx[b, g, i] = r.idx
            keys = selected_keys(r.idx, t, p)
        o, lse = attend(qg, K[b, :, g], V[b, :, g], keys, sc)
        O[b, i, g * G:(g + 1) * G] = o
        L[b, g * G:(g + 1) * G, i] = lse
    return O, L, ("dense" if dense else "sparse"), idx


# --------------------------------------------------------------------------
# decode: one new token per sequence
# --------------------------------------------------------------------------
@dataclasses.dataclass
class DecodeState:
    """Per-sequence caches: K, V [T_b, Hkv, d] and compressed keys [n_b, Hkv, d]."""
    K: List[np.ndarray]
    V: List[np.ndarray]
    Kc: List[np.ndarray]

    @staticmethod
    def from_prefill(K0: np.ndarray, V0: np.ndarray, p: Params) -> "DecodeState":
        Kc0 = compress_keys(K0, p)
        B = K0.shape[0]
        return DecodeState([K0[b].copy() for b in range(B)],
                           [V0[b].copy() for b in range(B)],
                           [Kc0[b].copy() for b in range(B)])


def decode_append(state: DecodeState, k_new: np.ndarray, v_new: np.ndarray,
                  p: Params) -> List[int]:
    """Append one key/value per sequence at pos = current length; when the
    window ending at pos completes, append its compressed key.

    k_new, v_new: [B, Hkv, d].  Returns the query positions (the old lengths).
    """
    positions = []
    for b in range(len(state.K)):
        pos = state.K[b].shape[0]
        state.K[b] = np.concatenate([state.K[b], k_new[b][None]], axis=0)
        state.V[b] = np.concatenate([state.V[b], v_new[b][None]], axis=0)
        if pos >= p.cmp_kernel - 1 and (pos - (p.cmp_kernel - 1)) % p.cmp_stride == 0:
            j = (pos - (p.cmp_kernel - 1)) // p.cmp_stride
            assert j == state.Kc[b].shape[0]
            start = j * p.cmp_stride
            new_c = state.K[b][start:start + p.cmp_kernel].mean(axis=0)
            state.Kc[b] = np.concatenate([state.Kc[b], new_c[None]], axis=0)
        positions.append(pos)
    return positions


def decode_query(K_seq: np.ndarray, V_seq: np.ndarray, Kc_seq: np.ndarray,
                 q: np.ndarray, t: int, p: Params):
    """Sparse attention of one sequence's new query (row t) over its caches.

    K_seq, V_seq: [>= t+1, Hkv, d]; Kc_seq: [>= v(t), Hkv, d]; q: [Hq, d].
    Returns (O [Hq, d], LSE [Hq], idx [Hkv, topk]).
    """
    Hq, d = q.shape
    Hkv = K_seq.shape[1]
    G = Hq // Hkv
    O = np.zeros((Hq, d))
    L = np.zeros(Hq)
    idx = np.full((Hkv, p.topk), -1, dtype=np.int32)
    for g in range(Hkv):
        qg = q[g * G:(g + 1) * G]
        idx[g] = select_query(qg, Kc_seq[:, g, :], t, p).idx
        keys = selected_keys(idx[g], t, p)
        o, lse = attend(qg, K_seq[:, g], V_seq[:, g], keys, p.sm_scale(d))
        O[g * G:(g + 1) * G] = o
        L[g * G:(g + 1) * G] = lse
    return O, L, idx


def decode_step(state: DecodeState, q: np.ndarray, k_new: np.ndarray,
                v_new: np.ndarray, p: Params):
    """One decode step for every sequence: append, then attend as row t = pos.

    q: [B, Hq, d]; k_new, v_new: [B, Hkv, d].  Mutates ``state``.
    Returns (O [B, Hq, d], LSE [B, Hq], idx [B, Hkv, topk]).
    """
    positions = decode_append(state, k_new, v_new, p)
    outs = [decode_query(state.K[b], state.V[b], state.Kc[b], q[b], t, p)
            for b, t in enumerate(positions)]
    O = np.stack([o[0] for o in outs])
    L = np.stack([o[1] for o in outs])
    idx = np.stack([o[2] for o in outs])
    return O, L, idx
