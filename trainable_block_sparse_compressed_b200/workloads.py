"""Seeded synthetic inputs for InfLLM-V2 dense-sparse switchable attention.

This module generates inputs only. It holds none of the method's arithmetic
(no compression, scoring, selection or attention), so that the fp64 oracle and
the CUDA path can both consume exactly the same bytes without sharing any code
that computes the method.

Recipe (the pages give shapes and a value distribution, not data):

* Q, K, V are iid N(0, 1) drawn with numpy's PCG64 generator from the
  workload's seed, in the order Q, K, V, as float32, then rounded to bfloat16
  with round-to-nearest-even.  Layout is BSHD: ``[B, T, H, d]``.
* "Planted high-affinity key blocks" (needles): a needle is a 64-token key
  block ``nb_i`` (never block 0 and never one of the last two blocks) paired
  with a later query block ``qb_i >= nb_i + 2`` (so the needle is never a
  forced local block of those queries).  For every KV head ``g`` all 64 keys
  of the needle block are set to ``3 * sqrt(d) * u`` where ``u`` is the unit
  vector of the mean query of the heads of group ``g`` over the 64 tokens of
  the query block, i.e. three times the mean query direction at three times
  the typical key norm.
* Decode: a prefilled cache of ``L`` tokens per sequence plus ``steps``
  pre-generated (q, k_new, v_new) triples; a sequence's needles point along the
  mean of that sequence's pre-generated decode queries.

All tensors are returned as numpy ``uint16`` arrays holding bfloat16 bit
patterns; :func:`bf16_to_f64` widens them exactly for the oracle and
:func:`to_torch_bf16` reinterprets them for the GPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

BLOCK = 64  # key-block size used by the pages' sparse attention


# --------------------------------------------------------------------------
# bfloat16 helpers (pure bit manipulation, no method arithmetic)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u = u.reshape(-1)
    flat_o = out.reshape(-1)
    chunk = 1 << 24
    for s in range(0, flat_u.size, chunk):
        v = flat_u[s:s + chunk]
        nan = (v & 0x7FFFFFFF) > 0x7F800000
        r = ((v >> 16) & 1) + 0x7FFF
        o = ((v + r) >> 16).astype(np.uint16)
        o[nan] = ((v[nan] >> 16) | 0x40).astype(np.uint16)
        flat_o[s:s + chunk] = o
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return bf16_to_f32(bits).astype(np.float64)


def to_torch_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16)


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int = 128
    topk: int = 64
    n_init: int = 1
    n_local: int = 2
    threshold: int = 8192
    needles: int = 0           # prefill: total needles per sequence
    seed: int = 0
    decode_steps: int = 0      # >0: decode workload, T is the prefilled length
    needles_per_seq: int = 0   # decode: needles per sequence

    @property
    def kind(self) -> str:
        if self.decode_steps:
            return "decode"
        return "dense" if self.T <= self.threshold else "sparse"


# The five workloads of the method's evaluation, by what they are.
WORKLOADS = {
    # GQA group 4; threshold 0 forces the sparse path at T = 2048.
    "sparse_prefill_T2048_Hq8_Hkv2": Workload(
        "sparse_prefill_T2048_Hq8_Hkv2", B=1, T=2048, Hq=8, Hkv=2, topk=8,
        threshold=0, needles=4, seed=1),
    # T = 4096 <= 8192: the switch must pick exact dense causal attention.
    "dense_switch_B2_T4096_Hq32_Hkv2": Workload(
        "dense_switch_B2_T4096_Hq32_Hkv2", B=2, T=4096, Hq=32, Hkv=2, topk=64,
        threshold=8192, needles=0, seed=2),
    "sparse_prefill_T32768_Hq32_Hkv2": Workload(
        "sparse_prefill_T32768_Hq32_Hkv2", B=1, T=32768, Hq=32, Hkv=2, topk=64,
        threshold=8192, needles=32, seed=3),
    "sparse_prefill_T131072_Hq32_Hkv2": Workload(
        "sparse_prefill_T131072_Hq32_Hkv2", B=1, T=131072, Hq=32, Hkv=2,
        topk=64, threshold=8192, needles=128, seed=4),
    "sparse_decode_B16_L131072_Hq32_Hkv2": Workload(
        "sparse_decode_B16_L131072_Hq32_Hkv2", B=16, T=131072, Hq=32, Hkv=2,
        topk=64, threshold=8192, seed=5, decode_steps=256, needles_per_seq=4),
}


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 24
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        out[s:s + m] = f32_to_bf16_bits(rng.standard_normal(m, dtype=np.float32))
    return out.reshape(shape)


def _unit(v: np.ndarray) -> np.ndarray:
    nrm = float(np.sqrt(np.dot(v, v)))
    return v / nrm if nrm > 0 else v


@dataclasses.dataclass
class Needle:
    batch: int
    block: int          # planted key block
    query_block: int    # query tokens [64*query_block, 64*query_block+63]


def _choose_needles(rng, n_needles: int, nb: int, batch: int):
    """Needle blocks in [1, nb-3]; each gets a query block >= block + 2."""
    lo, hi = 1, nb - 3
    if n_needles == 0 or hi - lo + 1 <= 0:
        return []
    n = min(n_needles, hi - lo + 1)
    blocks = np.sort(rng.choice(np.arange(lo, hi + 1), size=n, replace=False))
    out = []
    for b in blocks:
        qb = int(rng.integers(int(b) + 2, nb))
        out.append(Needle(batch, int(b), qb))
    return out


def _plant(K: np.ndarray, needle: Needle, direction_by_group, d: int, T: int):
    t0 = needle.block * BLOCK
    t1 = min(t0 + BLOCK, T)
    for g, u in enumerate(direction_by_group):
        key = f32_to_bf16_bits((3.0 * math.sqrt(d) * u).astype(np.float32))
        K[needle.batch, t0:t1, g, :] = key


def make_prefill(w: Workload, T: Optional[int] = None, seed: Optional[int] = None,
                 needles: Optional[int] = None):
    """Returns dict(Q, K, V, needles) for a prefill workload (bf16 bits)."""
    T = w.T if T is None else T
    seed = w.seed if seed is None else seed
    n_needles = w.needles if needles is None else needles
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = _normal_bf16(rng, (w.B, T, w.Hq, w.d))
    K = _normal_bf16(rng, (w.B, T, w.Hkv, w.d))
    V = _normal_bf16(rng, (w.B, T, w.Hkv, w.d))
    G = w.Hq // w.Hkv
    nb = (T + BLOCK - 1) // BLOCK
    planted = []
    for b in range(w.B):
        for nd in _choose_needles(rng, n_needles, nb, b):
            q0 = nd.query_block * BLOCK
            q1 = min(q0 + BLOCK, T)
            qs = bf16_to_f64(Q[b, q0:q1])  # [tq, Hq, d]
            dirs = [_unit(qs[:, g * G:(g + 1) * G, :].reshape(-1, w.d).mean(axis=0))
                    for g in range(w.Hkv)]
            _plant(K, nd, dirs, w.d, T)
            planted.append(nd)
    return dict(Q=Q, K=K, V=V, needles=planted)


def make_decode(w: Workload, L: Optional[int] = None, steps: Optional[int] = None,
                B: Optional[int] = None, seed: Optional[int] = None):
    """Returns dict(K0, V0, q, k_new, v_new, needles) for a decode workload.

    K0/V0: the prefilled cache ``[B, L, Hkv, d]``; q: ``[steps, B, Hq, d]``;
    k_new/v_new: ``[steps, B, Hkv, d]``.
    """
    L = w.T if L is None else L
    steps = w.decode_steps if steps is None else steps
    B = w.B if B is None else B
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    K0 = _normal_bf16(rng, (B, L, w.Hkv, w.d))
    V0 = _normal_bf16(rng, (B, L, w.Hkv, w.d))
    q = _normal_bf16(rng, (steps, B, w.Hq, w.d))
    k_new = _normal_bf16(rng, (steps, B, w.Hkv, w.d))
    v_new = _normal_bf16(rng, (steps, B, w.Hkv, w.d))
    G = w.Hq // w.Hkv
    nb = (L + BLOCK - 1) // BLOCK
    planted = []
    for b in range(B):
        qs = bf16_to_f64(q[:, b])  # [steps, Hq, d]
        dirs = [_unit(qs[:, g * G:(g + 1) * G, :].reshape(-1, w.d).mean(axis=0))
                for g in range(w.Hkv)]
        lo, hi = 1, nb - 3
        n = min(w.needles_per_seq, max(0, hi - lo + 1))
        if n:
            blocks = np.sort(rng.choice(np.arange(lo, hi + 1), size=n, replace=False))
            for blk in blocks:
                nd = Needle(b, int(blk), -1)
                _plant(K0, nd, dirs, w.d, L)
                planted.append(nd)
    return dict(K0=K0, V0=V0, q=q, k_new=k_new, v_new=v_new, needles=planted)


def small_workload(B=1, T=1000, Hq=8, Hkv=2, d=128, topk=8, n_init=1, n_local=2,
                   threshold=0, needles=2, seed=11) -> Workload:
    """A test-sized prefill workload with arbitrary (possibly ragged) T."""
    return Workload(f"prefill_B{B}_T{T}_Hq{Hq}_Hkv{Hkv}", B=B, T=T, Hq=Hq, Hkv=Hkv,
                    d=d, topk=topk, n_init=n_init, n_local=n_local,
                    threshold=threshold, needles=needles, seed=seed)
