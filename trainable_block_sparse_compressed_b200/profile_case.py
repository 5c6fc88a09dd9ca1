"""Runs the prefill path on one workload a few times, for profilers.

    python -m trainable_block_sparse_compressed_b200.profile_case \
        [--workload sparse_prefill_T32768_Hq32_Hkv2] [--iters 2] [--decode-steps 0]

Inputs are the seeded synthetic workload, generated on the host and copied to
the GPU once; each iteration runs compress_keys, select_blocks and
sparse_attn (or, with --decode-steps N, N decode steps over a reduced cache).
Used as the target of ncu captures (kernel filters select what to capture).
"""
from __future__ import annotations

import argparse

import torch

from . import infllmv2 as api
from . import workloads as wl


def prefill(name: str, iters: int):
    w = wl.WORKLOADS[name]
    d = wl.make_prefill(w)
    Q, K, V = (wl.to_torch_bf16(d[x]).cuda() for x in "QKV")
    p = api.make_params(w.B, w.T, w.Hq, w.Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    Kc = torch.empty((w.B, api.num_compressed(w.T), w.Hkv, 2, 128), dtype=torch.bfloat16,
                     device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.T, w.topk), dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_SELECT)
    O = torch.empty_like(Q)
    aws = api.alloc_workspace(p, api.OP_ATTN)
    lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device="cuda")
    for _ in range(iters):
        api.compress_keys(p, K, Kc)
        api.select_blocks(p, Q, Kc, idx, ws)
        api.sparse_attn(p, Q, K, V, idx, O, lse, aws)
    torch.cuda.synchronize()
    assert api.get_status() == 0


def decode(steps: int, L: int):
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B = w.B
    d = wl.make_decode(w, L=L, steps=steps, B=B)
    Lmax = L + steps
    p = api.make_params(B, Lmax, w.Hq, w.Hkv, topk=w.topk)
    Kc = torch.zeros((B, Lmax, w.Hkv, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    Kc[:, :L] = wl.to_torch_bf16(d["K0"]).cuda()
    Vc[:, :L] = wl.to_torch_bf16(d["V0"]).cuda()
    Kcmp = torch.zeros((B, api.num_compressed(Lmax), w.Hkv, 2, 128), dtype=torch.bfloat16,
                       device="cuda")
    n0 = api.num_compressed(L)
    tmp = torch.empty((B, n0, w.Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    api.compress_keys(api.make_params(B, L, w.Hq, w.Hkv), Kc[:, :L].contiguous(), tmp)
    Kcmp[:, :n0] = tmp
    seqlens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    O = torch.empty((B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_DECODE)
    q, kn, vn = (wl.to_torch_bf16(d[x]).cuda() for x in ("q", "k_new", "v_new"))
    for s in range(steps):
        api.decode_step(p, q[s], kn[s], vn[s], Kc, Vc, Kcmp, seqlens, O, lse, None, ws)
    torch.cuda.synchronize()
    assert api.get_status() == 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="sparse_prefill_T32768_Hq32_Hkv2")
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--decode-steps", type=int, default=0)
    ap.add_argument("--decode-len", type=int, default=131072)
    args = ap.parse_args()
    api.load()
    if args.decode_steps:
        decode(args.decode_steps, args.decode_len)
    else:
        prefill(args.workload, args.iters)
    print("done")


if __name__ == "__main__":
    main()
