"""Benchmark of the InfLLM-V2 sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole prefill path (length switch -> compressed
keys -> block scoring + top-k selection -> block-sparse attention) over the
T = 131072 sparse-prefill workload (B=1, Hq=32, Hkv=2, d=128, top-64 with
1 init + 2 local blocks), seeded synthetic bf16 inputs already resident in
HBM.  The L2 cache is flushed (256 MB write) between timed steps, outside the
per-step CUDA events.  Extra keys report the T = 32768 prefill and the decode
workload (B=16 sequences over a 131072-token cache, 256 steps in a CUDA
graph).  With N > 1 (torchrun) every rank runs an independent replica: the
path has no exchange step; value = all ranks' tokens / max-over-ranks time.

--impl reference times the fp64 CPU oracle (the only other implementation of
the method this project has) on a bounded sample of query rows of the same
workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn prefill tokens/s + TFLOP/s at 32k/128k; decode tok/s, HBM GB/s"
MAIN = "sparse_prefill_T131072_Hq32_Hkv2"
SIDE = "sparse_prefill_T32768_Hq32_Hkv2"
SMALL = "sparse_prefill_T2048_Hq8_Hkv2"
DENSE = "dense_switch_B2_T4096_Hq32_Hkv2"
DECODE = "sparse_decode_B16_L131072_Hq32_Hkv2"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; barrier + max over ranks only)
# ---------------------------------------------------------------------------
class Dist:
    """One process per GPU under torchrun.  The step has no exchange, so the
    only collectives are the barrier around the timed region and the max of
    the per-rank times (gloo when CUDA is absent, or when asked for)."""

    def __init__(self, n_gpus: int, backend: str | None = None):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"
        if self.world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            if backend is None:
                backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                self.device = "cuda"
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def main_config(w, world: int) -> dict:
    """The workload description both arms report."""
    return {"workload": MAIN, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": 128,
            "topk": w.topk, "n_init": w.n_init, "n_local": w.n_local,
            "switch_threshold": w.threshold, "needles": w.needles,
            "parallelism": f"replicas x{world}",
            "l2": "flushed between timed steps (256 MB write, outside the events)"}


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_source_hash(name: str) -> str:
    """Hash of a kernel source's code: comments and whitespace removed, so that
    counters taken on a kernel stay attached to it across comment edits."""
    path = os.path.join(ROOT, "trainable_block_sparse_compressed_b200", "csrc", name)
    with open(path, encoding="utf-8") as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = " ".join(src.split())
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def profiled_traffic(kernel_file: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_file, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_hash(kernel_file):
        return None
    return e.get("dram_bytes_per_launch")


def attended_keys(idx_np, T):
    """Keys each (b, g, t) row attends: selected blocks clipped to [0, t]."""
    import numpy as np
    t = np.arange(T)[None, None, :, None]
    valid = (idx_np >= 0) & (idx_np <= (t // 64))
    start = idx_np.astype(np.int64) * 64
    n = np.minimum(start + 63, t) - start + 1
    return np.where(valid, n, 0).sum(axis=-1)  # [B, Hkv, T]


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_prefill(api, wl, w, steps, warmup, dist, flush, time_e2e=True, clocks=None,
                chunk_len=0, measure_gather=False):
    import numpy as np
    import torch
    data = wl.make_prefill(w)
    Qh, Kh, Vh = (wl.to_torch_bf16(data[x]) for x in "QKV")
    Q, K, V = Qh.cuda(), Kh.cuda(), Vh.cuda()
    B, T, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    G = Hq // Hkv
    p = api.make_params(B, T, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    assert T > w.threshold
    n_c = api.num_compressed(T)
    Kc = torch.empty((B, n_c, Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, Hkv, T, w.topk), dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_FORWARD)
    O = torch.empty_like(Q)
    aws = api.alloc_workspace(p, api.OP_ATTN)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(evs=None):
        # the length switch (T > threshold -> sparse), then the three stages
        if evs: evs[0].record(stream)
        api.compress_keys(p, K, Kc)
        if evs: evs[1].record(stream)
        api.select_blocks(p, Q, Kc, idx, ws)
        if evs: evs[2].record(stream)
        api.sparse_attn(p, Q, K, V, idx, O, lse, aws)
        if evs: evs[3].record(stream)

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    assert api.get_status() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    for s in range(steps):
        flush()
        step(evs[s])
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop() if clocks else None
    per = [[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in evs]
    step_ms = [sum(x) for x in per]
    ms = sum(step_ms) / steps
    kern = {name: sum(x[i] for x in per) / steps
            for i, name in enumerate(["compress_keys", "select_blocks", "sparse_attn"])}
    assert api.get_status() == 0
    # useful work of this selection
    nkeys = attended_keys(idx.cpu().numpy(), T)  # noqa: E501
    useful_attn_flops = float(4 * 128 * G * nkeys.sum())
    v = np.array([0 if t < 31 else (t - 31) // 16 + 1 for t in range(T)], dtype=np.int64)
    useful_score_flops = float(2 * 128 * Hq * B * v.sum())
    executed_score_flops = 0.0
    tpt = 128 // G
    # a scoring CTA takes two query tiles (256 rows) and streams the windows
    # its later tile sees; both tiles run both passes over them
    for t0 in range(0, T, 2 * tpt):
        tl = min(t0 + 2 * tpt - 1, T - 1)
        vt = 0 if tl < 31 else min(n_c, (tl - 31) // 16 + 1)
        nt = (vt + 127) // 128
        # pass 1 multiplies the hi plane only (K = 128), pass 2 hi and lo (K = 256)
        executed_score_flops += 2 * (2 * 128 * 128 * 128 + 2 * 128 * 128 * 256) * nt
    executed_score_flops *= B * Hkv
    idx_np = idx.cpu().numpy()
    cur = (np.arange(T) // 64)[None, None, :, None]
    valid = (idx_np >= 0) & (idx_np <= cur)
    if G >= 4:
        # query-tile schedule: each tile of 128/G tokens loads the union of its
        # tokens' blocks once (K and V, 32 KB per block) and runs 128-key
        # tiles of 128 rows (S and P V, 2 FLOP per MAC)
        tpt = 128 // G
        n_t = -(-T // tpt)
        pad = n_t * tpt - T
        u = np.where(valid, idx_np, -1)
        if pad:
            u = np.concatenate([u, np.full(u.shape[:2] + (pad, u.shape[3]), -1, u.dtype)], axis=2)
        u = np.sort(u.reshape(B, Hkv, n_t, tpt * w.topk), axis=-1)
        heads = (u >= 0) & np.concatenate([np.ones(u.shape[:3] + (1,), bool),
                                           u[..., 1:] != u[..., :-1]], axis=-1)
        n_u = heads.sum(axis=-1)
        gathered_bytes = float(n_u.sum()) * 32768
        executed_attn_flops = float(((n_u + 1) // 2).sum()) * 2 * (2 * 128 * 128 * 128)
    else:
        n_valid = valid.sum(axis=-1)
        pairs = int(((n_valid + 1) // 2).sum())
        gathered_bytes = float(pairs) * 65536
        # per gathered pair: S^T (128 keys x 16 heads x 128) and P V, 2 FLOP per MAC
        executed_attn_flops = float(pairs) * 2 * (2 * 128 * 16 * 128)
    gather = None
    if measure_gather:
        gather = gather_roofline(api, aws, gathered_bytes, kern["sparse_attn"])
    out = dict(ms=ms, step_ms=step_ms, kernels=kern, tokens=B * T, gather=gather,
               useful_attn_flops=useful_attn_flops, useful_score_flops=useful_score_flops,
               executed_score_flops=executed_score_flops, executed_attn_flops=executed_attn_flops,
               clocks=clk,
               # compress, score, top-k, (union lists,) pack, attention
               launches_per_step=6 if G >= 4 else 5)
    if chunk_len:
        out["chunk"] = time_chunk(api, p, Q, K, V, Kc, chunk_len, steps, warmup, flush)
    if time_e2e:
        out.update(e2e_prefill(api, p, Qh, Kh, Vh, O.shape, lse.shape, Kc, idx, ws, steps, dist))
    del Q, K, V, Kc, idx, ws, O, lse
    torch.cuda.empty_cache()
    return out


def gather_roofline(api, tiles, per_launch, attn_ms, rounds=2000, reps=5):
    """The attention's L2 -> shared-memory gather (per_launch bytes of K and V
    blocks) against this GPU's ceiling for that movement, measured now by the
    library's gather kernel over the attention's workspace (L2-resident)."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(2):
        api.gather_peak(tiles, rounds)
    torch.cuda.synchronize()
    rates = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moved = api.gather_peak(tiles, rounds)
        e1.record(stream)
        torch.cuda.synchronize()
        rates.append(moved / (e0.elapsed_time(e1) / 1e3) / 1e9)
    assert api.get_status() == 0
    peak = statistics.median(rates)
    achieved = per_launch / (attn_ms / 1e3) / 1e9
    return {"bound": "l2_gather", "kernel": "sparse_attn", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak, "bytes_per_launch": per_launch,
            "peak_source": "measured in this run: infllmv2_gather_peak, 16 KB bulk copies "
                           "from an L2-resident buffer into a 3 x 64 KB ring, one CTA "
                           "per SM, median of 5"}


def time_chunk(api, p, Q, K, V, Kc, n, steps, warmup, flush):
    """Chunked prefill: the last n tokens' queries over the sequence's full
    caches (K, V and the compressed keys the main step computed)."""
    import torch
    B, T, Hq = Q.shape[0], Q.shape[1], Q.shape[2]
    q0 = T - n
    Qc = Q[:, q0:].contiguous()
    O = torch.empty_like(Qc)
    lse = torch.empty((B, Hq, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, p.Hkv, n, p.topk), dtype=torch.int32, device="cuda")
    ws = torch.empty(api.prefill_chunk_workspace_bytes(p, q0, n), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        api.prefill_chunk(p, q0, n, Qc, K, V, Kc, O, lse, idx, ws)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        api.prefill_chunk(p, q0, n, Qc, K, V, Kc, O, lse, idx, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    assert api.get_status() == 0
    return dict(q_offset=q0, q_len=n, ms=sum(ms) / len(ms))


def e2e_prefill(api, p, Qh, Kh, Vh, o_shape, lse_shape, Kc, idx, ws, steps, dist):
    """End to end through the public API (infllmv2_forward) from pinned host
    buffers, as a serving loop would run it: two device buffer sets, the
    host-to-device copy of step i+1 and the device-to-host copy of step i-1
    on their own streams while step i computes.  Every step copies its
    inputs in and its outputs back inside the timed region; the time is from
    the first copy in to the last copy out."""
    import torch
    Qp, Kp, Vp = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
    sets = []
    for _ in range(2):
        sets.append(dict(Q=torch.empty(Qh.shape, dtype=Qh.dtype, device="cuda"),
                         K=torch.empty(Kh.shape, dtype=Kh.dtype, device="cuda"),
                         V=torch.empty(Vh.shape, dtype=Vh.dtype, device="cuda"),
                         O=torch.empty(o_shape, dtype=torch.bfloat16, device="cuda"),
                         lse=torch.empty(lse_shape, dtype=torch.float32, device="cuda"),
                         Op=torch.empty(o_shape, dtype=torch.bfloat16).pin_memory(),
                         Lp=torch.empty(lse_shape, dtype=torch.float32).pin_memory()))
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev(), ev()]
    cmp_done = [ev(), ev()]
    out_done = [ev(), ev()]

    def run(n):
        for i in range(n):
            b = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[i % 2])  # step i-2 has read these inputs
                b["Q"].copy_(Qp, non_blocking=True)
                b["K"].copy_(Kp, non_blocking=True)
                b["V"].copy_(Vp, non_blocking=True)
                in_done[i % 2].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_done[i % 2])
                if i >= 2:
                    s_cmp.wait_event(out_done[i % 2])  # step i-2's outputs are copied out
                api.forward(p, b["Q"], b["K"], b["V"], b["O"], b["lse"], Kc, idx, ws,
                            stream=s_cmp)
                cmp_done[i % 2].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[i % 2])
                b["Op"].copy_(b["O"], non_blocking=True)
                b["Lp"].copy_(b["lse"], non_blocking=True)
                out_done[i % 2].record(s_out)

    run(2)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    run(steps)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    res = dict(e2e_ms=e0.elapsed_time(e1) / steps,
               h2d=sum(x.numel() * x.element_size() for x in (Qp, Kp, Vp)),
               d2h=sum(sets[0][k].numel() * sets[0][k].element_size() for k in ("Op", "Lp")))
    del sets
    torch.cuda.empty_cache()
    return res


def run_decode(api, wl, w, steps, warmup, flush):
    """256 decode steps over B=16 caches of 131072 tokens, captured in a CUDA graph."""
    import torch
    B, L0, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    total = warmup + steps
    data = wl.make_decode(w, L=L0, steps=total, B=B)
    Lmax = L0 + total
    p = api.make_params(B, Lmax, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local)
    Kc = torch.zeros((B, Lmax, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    Kc[:, :L0] = wl.to_torch_bf16(data["K0"]).cuda()
    Vc[:, :L0] = wl.to_torch_bf16(data["V0"]).cuda()
    NC = api.num_compressed(Lmax)
    Kcmp = torch.zeros((B, NC, Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    n0 = api.num_compressed(L0)
    tmp = torch.empty((B, n0, Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    api.compress_keys(api.make_params(B, L0, Hq, Hkv), Kc[:, :L0].contiguous(), tmp)
    Kcmp[:, :n0] = tmp
    del tmp
    seqlens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    q = wl.to_torch_bf16(data["q"]).cuda()
    kn = wl.to_torch_bf16(data["k_new"]).cuda()
    vn = wl.to_torch_bf16(data["v_new"]).cuda()
    O = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_DECODE)
    for s in range(warmup):
        api.decode_step(p, q[s], kn[s], vn[s], Kc, Vc, Kcmp, seqlens, O, lse, None, ws)
    torch.cuda.synchronize()
    # capture the timed steps in one graph (inputs of each step are distinct slices)
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    seq_start = seqlens.clone()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for s in range(warmup, total):
                api.decode_step(p, q[s], kn[s], vn[s], Kc, Vc, Kcmp, seqlens, O, lse, None, ws)
    torch.cuda.synchronize()
    seqlens.copy_(seq_start)
    flush()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert api.get_status() == 0
    assert int(seqlens[0]) == L0 + total
    per_step = ms / steps
    # algorithmic HBM bytes per step: every visible compressed key of every
    # sequence and kv head as one bf16 row, the K and V rows of the selected
    # blocks, the appended K/V rows, q and the outputs.  The library also
    # reads the low bf16 plane of each compressed key (its precision choice,
    # not the method's work): listed apart, not counted.
    nc_vis = (L0 + warmup + steps // 2 - 31) // 16 + 1
    kc_bytes = B * Hkv * nc_vis * 128 * 2
    kv_bytes = B * Hkv * w.topk * 64 * 128 * 2 * 2
    small = B * (Hq * 128 * 2 * 2 + Hkv * 128 * 2 * 2 + Hq * 4)
    bytes_step = kc_bytes + kv_bytes + small
    del g
    return dict(ms_per_step=per_step, tokens_per_s=B / (per_step / 1e3),
                hbm_gbs=bytes_step / (per_step / 1e3) / 1e9, bytes_per_step=bytes_step,
                lo_plane_bytes_per_step=kc_bytes, steps=steps, launches_per_step=6)


def run_compressed(api, wl, w, steps, warmup, flush):
    """The compressed-attention branch on a prefill workload: compress V (the
    keys' compression is the selection's), then every query row over its
    visible window means.  Inputs resident; the compressed keys precomputed."""
    import torch
    data = wl.make_prefill(w)
    Q, K, V = (wl.to_torch_bf16(data[x]).cuda() for x in "QKV")
    B, T, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    p = api.make_params(B, T, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    n_c = api.num_compressed(T)
    Kc = torch.empty((B, n_c, Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    api.compress_keys(p, K, Kc)
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        api.compress_keys(p, V, Vc)
        api.compressed_attn(p, Q, Kc, Vc, O, lse)
    torch.cuda.synchronize()
    ms, ams = [], []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        api.compress_keys(p, V, Vc)
        e[1].record(stream)
        api.compressed_attn(p, Q, Kc, Vc, O, lse)
        e[2].record(stream)
        torch.cuda.synchronize()
        ms.append(e[0].elapsed_time(e[2]))
        ams.append(e[1].elapsed_time(e[2]))
    assert api.get_status() == 0
    v = [0 if t < 31 else min(n_c, (t - 31) // 16 + 1) for t in range(T)]
    flops = 4.0 * 128 * Hq * B * float(sum(v))  # q.Kc and P Vc over the visible windows
    del Q, K, V, Kc, Vc, O, lse
    torch.cuda.empty_cache()
    return dict(ms=sum(ms) / len(ms), attn_ms=sum(ams) / len(ams), tokens=B * T, flops=flops)


def run_backward(api, wl, w, steps, warmup, flush):
    """Gradients of the block-sparse attention with the selection fixed, on a
    prefill workload: the forward (for O, lse and the selection) once, then
    the timed backward.  Inputs and dO resident."""
    import numpy as np
    import torch
    data = wl.make_prefill(w)
    Q, K, V = (wl.to_torch_bf16(data[x]).cuda() for x in "QKV")
    B, T, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    O, lse, _, idx = api.prefill(Q, K, V, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                                 threshold=w.threshold)
    p = api.make_params(B, T, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    g = torch.Generator(device="cuda").manual_seed(7)
    dO = torch.randn(Q.shape, generator=g, device="cuda").to(torch.bfloat16)
    dQ = torch.empty(Q.shape, dtype=torch.float32, device="cuda")
    dK = torch.empty(K.shape, dtype=torch.float32, device="cuda")
    dV = torch.empty_like(dK)
    ws = api.alloc_workspace(p, api.OP_BACKWARD)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        api.sparse_attn_backward(p, Q, K, V, idx, O, lse, dO, dQ, dK, dV, ws)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        api.sparse_attn_backward(p, Q, K, V, idx, O, lse, dO, dQ, dK, dV, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    assert api.get_status() == 0
    nkeys = attended_keys(idx.cpu().numpy(), T)
    G = Hq // Hkv
    # S, dP, dQ, dK, dV: five products of 2 d FLOP per (row, attended key)
    flops = float(10 * 128 * G * nkeys.sum())
    del Q, K, V, O, lse, idx, dO, dQ, dK, dV, ws
    torch.cuda.empty_cache()
    return dict(ms=sum(ms) / len(ms), tokens=B * T, flops=flops)


def run_dense(api, wl, w, steps, warmup, flush):
    """The dense-switch workload through infllmv2_forward (T <= threshold, so
    the switch takes exact dense causal attention), inputs resident."""
    import torch
    data = wl.make_prefill(w)
    Q, K, V = (wl.to_torch_bf16(data[x]).cuda() for x in "QKV")
    B, T, Hq, Hkv = w.B, w.T, w.Hq, w.Hkv
    p = api.make_params(B, T, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local,
                        switch_threshold=w.threshold)
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(p, api.OP_FORWARD)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        assert api.forward(p, Q, K, V, O, lse, ws=ws) == api.PATH_DENSE
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        api.forward(p, Q, K, V, O, lse, ws=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    assert api.get_status() == 0
    # causal attention: row t attends t + 1 keys; QK^T and PV, 2 FLOP per MAC
    flops = 4.0 * 128 * Hq * B * (T * (T + 1) / 2)
    m = sum(ms) / len(ms)
    del Q, K, V, O, lse, ws
    torch.cuda.empty_cache()
    return dict(ms=m, tokens=B * T, flops=flops)


def profile_case(api, wl, name: str, iters: int, decode_steps: int, decode_len: int):
    """A few passes of the path for profilers (kernel filters pick what to
    capture): the prefill stages on one workload, or decode steps over a
    cache of decode_len tokens.  Seeded inputs, copied to the GPU once."""
    import torch
    if decode_steps:
        w = wl.WORKLOADS[DECODE]
        B, L = w.B, decode_len
        d = wl.make_decode(w, L=L, steps=decode_steps, B=B)
        Lmax = L + decode_steps
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
        for s in range(decode_steps):
            api.decode_step(p, q[s], kn[s], vn[s], Kc, Vc, Kcmp, seqlens, O, lse, None, ws)
    else:
        w = wl.WORKLOADS[name]
        d = wl.make_prefill(w)
        Q, K, V = (wl.to_torch_bf16(d[x]).cuda() for x in "QKV")
        p = api.make_params(w.B, w.T, w.Hq, w.Hkv, topk=w.topk, n_init=w.n_init,
                            n_local=w.n_local, switch_threshold=w.threshold)
        O = torch.empty_like(Q)
        lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device="cuda")
        if w.T <= w.threshold:
            ws = api.alloc_workspace(p, api.OP_FORWARD)
            for _ in range(iters):
                api.forward(p, Q, K, V, O, lse, ws=ws)
        else:
            Kc = torch.empty((w.B, api.num_compressed(w.T), w.Hkv, 2, 128), dtype=torch.bfloat16,
                             device="cuda")
            idx = torch.empty((w.B, w.Hkv, w.T, w.topk), dtype=torch.int32, device="cuda")
            ws = api.alloc_workspace(p, api.OP_SELECT)
            aws = api.alloc_workspace(p, api.OP_ATTN)
            for _ in range(iters):
                api.compress_keys(p, K, Kc)
                api.select_blocks(p, Q, Kc, idx, ws)
                api.sparse_attn(p, Q, K, V, idx, O, lse, aws)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    print("profile case done", flush=True)


# --- the fp64 oracle on the host cores (test infrastructure, timed as a baseline) ---
_ORC = {}


def _oracle_worker_init(shm_names, shapes, params, G):
    """Worker of the oracle pool: attaches the shared bf16 inputs and the
    compressed keys, one BLAS thread."""
    import numpy as np
    from multiprocessing import shared_memory
    from threadpoolctl import threadpool_limits
    from oracle import infllmv2_oracle as orc
    threadpool_limits(limits=1)
    arrs = {}
    for name, (sname, shape, dtype) in zip(("Q", "K", "V", "Kc"), zip(shm_names, shapes[0], shapes[1])):
        sh = shared_memory.SharedMemory(name=sname)
        arrs[name] = (sh, np.ndarray(shape, dtype=dtype, buffer=sh.buf))
    _ORC.update(arrs=arrs, p=orc.Params(**params), G=G, orc=orc)


def _oracle_rows(ts):
    """The oracle's selection and attention for query tokens ts (all kv groups)."""
    import numpy as np
    from trainable_block_sparse_compressed_b200 import workloads as wl
    orc, p, G = _ORC["orc"], _ORC["p"], _ORC["G"]
    Qb, Kb, Vb = (_ORC["arrs"][x][1] for x in ("Q", "K", "V"))
    Kc = _ORC["arrs"]["Kc"][1]
    sc = p.sm_scale(128)
    for t in ts:
        for g in range(Kb.shape[2]):
            q = wl.bf16_to_f64(Qb[0, t, g * G:(g + 1) * G])
            sel = orc.select_query(q, Kc[0, :, g], t, p)
            keys = orc.selected_keys(sel.idx, t, p)
            orc.attend(q, wl.bf16_to_f64(Kb[0, keys, g]), wl.bf16_to_f64(Vb[0, keys, g]),
                       np.arange(len(keys)), sc)
    return len(ts)


class OracleBaseline:
    """The fp64 oracle, as it stands, timed on the host's cores: a
    spawn-context process pool (one BLAS thread per worker) runs the oracle's
    selection and attention on random query tokens of the workload, the
    inputs shared read-only, the compressed keys computed once (timed)."""

    def __init__(self, w, workers=None):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        import numpy as np
        from threadpoolctl import threadpool_limits
        from oracle import infllmv2_oracle as orc
        from trainable_block_sparse_compressed_b200 import workloads as wl
        self.w = w
        data = wl.make_prefill(w)
        p = dict(topk=w.topk, n_init=w.n_init, n_local=w.n_local, threshold=w.threshold)
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            Kc = orc.compress_keys(wl.bf16_to_f64(data["K"]), orc.Params(**p))
            self.t_cmp = time.perf_counter() - t0
        self.shms, names, shapes, dtypes = [], [], [], []
        for arr in (data["Q"], data["K"], data["V"], Kc):
            sh = shared_memory.SharedMemory(create=True, size=arr.nbytes)
            np.ndarray(arr.shape, dtype=arr.dtype, buffer=sh.buf)[...] = arr
            self.shms.append(sh)
            names.append(sh.name)
            shapes.append(arr.shape)
            dtypes.append(arr.dtype)
        self.workers = workers or max(1, min(os.cpu_count() or 1, 32))
        self.pool = mp.get_context("spawn").Pool(
            self.workers, initializer=_oracle_worker_init,
            initargs=(names, (shapes, dtypes), p, w.Hq // w.Hkv))
        self.rng = np.random.default_rng(0)
        self.pool.map(_oracle_rows, [[0]] * self.workers)  # workers up and warm

    def run(self, seconds):
        """Rows processed in about `seconds` of wall time, and that time."""
        batch = 4
        t0 = time.perf_counter()
        pending, rows = [], 0
        while time.perf_counter() - t0 < seconds:
            while len(pending) < 2 * self.workers:
                ts = [int(x) for x in self.rng.integers(0, self.w.T, batch)]
                pending.append(self.pool.apply_async(_oracle_rows, (ts,)))
            done = [r for r in pending if r.ready()]
            for r in done:
                rows += r.get()
                pending.remove(r)
            if not done:
                time.sleep(0.005)
        for r in pending:
            rows += r.get()
        return rows, time.perf_counter() - t0

    def close(self):
        self.pool.terminate()
        self.pool.join()
        for sh in self.shms:
            sh.close()
            sh.unlink()


def cpu_oracle_sample(w, seconds=15.0):
    """The oracle on the host cores for about `seconds`; tokens/s (a token =
    its Hkv query groups) extrapolated to the whole workload."""
    base = OracleBaseline(w)
    try:
        rows, el = base.run(seconds)
    finally:
        base.close()
    rate = rows / el
    total_s = base.t_cmp + w.T * w.B / rate
    return dict(value=w.T * w.B / total_s, unit="tokens/s", cores=base.workers, kind="oracle",
                sample=f"{rows} random query tokens x {w.Hkv} kv groups of {w.name} (selection + "
                       f"attention, fp64 numpy) on {base.workers} worker processes, one thread "
                       f"each, in {el:.1f} s, plus the full compressed keys ({base.t_cmp:.1f} s); "
                       f"extrapolated to all {w.T} tokens")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the 32k and decode extras")
    ap.add_argument("--baseline-seconds", type=float, default=15.0)
    ap.add_argument("--profile-case", metavar="WORKLOAD",
                    help="run the path a few times on one workload for a profiler, then exit")
    ap.add_argument("--iters", type=int, default=2, help="--profile-case: passes of the path")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="--profile-case: decode steps instead of prefill")
    ap.add_argument("--decode-len", type=int, default=131072,
                    help="--profile-case: cached tokens per sequence for the decode steps")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.profile_case:
        from trainable_block_sparse_compressed_b200 import infllmv2 as api
        from trainable_block_sparse_compressed_b200 import workloads as wl
        api.load()
        profile_case(api, wl, args.profile_case, args.iters, args.decode_steps, args.decode_len)
        return

    from trainable_block_sparse_compressed_b200 import workloads as wl
    w = wl.WORKLOADS[MAIN]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        t0 = time.perf_counter()
        # every step: the oracle on a bounded sample of the workload's query
        # tokens (all kv groups each), on the host cores
        base = OracleBaseline(w)
        per_step = max(2.0, args.baseline_seconds / 4)
        try:
            for _ in range(args.warmup):
                base.run(per_step)
            runs = [base.run(per_step) for _ in range(args.steps)]
        finally:
            base.close()
        rows = sum(r for r, _ in runs)
        el = sum(e for _, e in runs)
        value = rows / el
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 0,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": main_config(w, int(os.environ.get("WORLD_SIZE", "1"))),
                "cpu_baseline": {
                    "value": value, "unit": "tokens/s", "cores": base.workers, "kind": "oracle",
                    "sample": f"each step: random query tokens of {w.name} (selection + "
                              f"attention of every kv group, fp64 numpy) for {per_step:.1f} s on "
                              f"{base.workers} worker processes, one thread each; "
                              f"{rows} tokens over {args.steps} steps"},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": time.perf_counter() - t0}
        print(json.dumps(line), flush=True)
        return

    import torch
    from trainable_block_sparse_compressed_b200 import infllmv2 as api
    dist = Dist(args.gpus)
    torch.cuda.set_device(dist.local)
    api.load()
    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def flush():
        flush_buf.zero_()

    clocks = ClockSampler(dist.local)
    main_r = run_prefill(api, wl, w, args.steps, args.warmup, dist, flush, True, clocks,
                         chunk_len=0 if args.no_extras else 8192, measure_gather=True)
    ms = dist.max(main_r["ms"])
    e2e_ms = dist.max(main_r["e2e_ms"])
    value = whole_job_rate(main_r["tokens"], dist.world, ms)

    extras = {}
    if "chunk" in main_r:
        c = main_r["chunk"]
        cms = dist.max(c["ms"])
        extras["prefill_chunk_T131072_last8192"] = {
            "tokens_per_s": whole_job_rate(w.B * c["q_len"], dist.world, cms), "ms_per_chunk": cms,
            "q_offset": c["q_offset"], "q_len": c["q_len"],
            "timing": "queries of tokens 122880..131071 over the full caches; L2 flushed"}
    if not args.no_extras:
        side = run_prefill(api, wl, wl.WORKLOADS[SIDE], args.steps, args.warmup, dist, flush,
                           False, None)
        sms = dist.max(side["ms"])
        extras["prefill_T32768"] = {
            "tokens_per_s": whole_job_rate(side["tokens"], dist.world, sms), "ms_per_step": sms,
            "useful_tflops": (side["useful_attn_flops"] + side["useful_score_flops"]) / (sms / 1e3) / 1e12,
            "kernels_ms": side["kernels"]}
        small = run_prefill(api, wl, wl.WORKLOADS[SMALL], args.steps, args.warmup, dist, flush,
                            False, None)
        s1 = dist.max(small["ms"])
        a1 = small["kernels"]["sparse_attn"]
        extras["prefill_T2048_Hq8_Hkv2"] = {
            "tokens_per_s": whole_job_rate(small["tokens"], dist.world, s1), "ms_per_step": s1,
            "useful_tflops": (small["useful_attn_flops"] + small["useful_score_flops"]) / (s1 / 1e3) / 1e12,
            "attn_tensor_frac_of_burst": small["useful_attn_flops"] / (a1 / 1e3) / 1e12 / peaks["bf16_tflops"],
            "kernels_ms": small["kernels"], "switch_threshold": 0}
        dn = run_dense(api, wl, wl.WORKLOADS[DENSE], args.steps, args.warmup, flush)
        d1 = dist.max(dn["ms"])
        extras["dense_switch_B2_T4096"] = {
            "path": "dense", "tokens_per_s": whole_job_rate(dn["tokens"], dist.world, d1),
            "ms_per_step": d1, "tflops": dn["flops"] / (d1 / 1e3) / 1e12,
            "tensor_frac_of_burst": dn["flops"] / (d1 / 1e3) / 1e12 / peaks["bf16_tflops"],
            "flops_per_step": dn["flops"]}
        bw = run_backward(api, wl, wl.WORKLOADS[SIDE], args.steps, args.warmup, flush)
        b1 = dist.max(bw["ms"])
        extras["backward_T32768"] = {
            "tokens_per_s": whole_job_rate(bw["tokens"], dist.world, b1), "ms_per_step": b1,
            "useful_tflops": bw["flops"] / (b1 / 1e3) / 1e12,
            "tensor_frac_of_burst": bw["flops"] / (b1 / 1e3) / 1e12 / peaks["bf16_tflops"],
            "timing": "dQ, dK, dV with the forward's selection fixed (delta, dQ, index, dK/dV, "
                      "reduce); L2 flushed"}
        cm = run_compressed(api, wl, w, args.steps, args.warmup, flush)
        c1 = dist.max(cm["ms"])
        extras["compressed_branch_T131072"] = {
            "tokens_per_s": whole_job_rate(cm["tokens"], dist.world, c1), "ms_per_step": c1,
            "attn_ms": cm["attn_ms"], "tflops": cm["flops"] / (cm["attn_ms"] / 1e3) / 1e12,
            "tensor_frac_of_burst": cm["flops"] / (cm["attn_ms"] / 1e3) / 1e12 / peaks["bf16_tflops"],
            "flops_per_step": cm["flops"],
            "timing": "compress V + attention over the visible window means; L2 flushed"}
        wd = wl.WORKLOADS[DECODE]
        dec = run_decode(api, wl, wd, 256, 8, flush)
        dms = dist.max(dec["ms_per_step"])
        extras["decode_B16_L131072"] = {
            "tokens_per_s": whole_job_rate(wd.B, dist.world, dms), "ms_per_step": dms,
            "hbm_gbs": dec["bytes_per_step"] / (dms / 1e3) / 1e9,
            "hbm_frac_of_measured": dec["bytes_per_step"] / (dms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "hbm_frac_of_nominal_8tbs": dec["bytes_per_step"] / (dms / 1e3) / 1e9 / 8000.0,
            "algorithmic_bytes_per_step": dec["bytes_per_step"],
            "not_counted_lo_plane_bytes_per_step": dec["lo_plane_bytes_per_step"],
            "steps": 256,
            "timing": "256 steps in one CUDA graph, L2 flushed before the replay"}

    # roofline of the dominant kernel (the block-sparse attention)
    kern = main_r["kernels"]
    dom = max(kern, key=kern.get)
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    if dom == "sparse_attn":
        achieved = main_r["useful_attn_flops"] / (kern[dom] / 1e3) / 1e12
        # G >= 4 runs the query-tile kernel over the union of the tile's blocks
        kfile = "tile_attn.cu" if w.Hq // w.Hkv >= 4 else "sparse_attn.cu"
    else:
        achieved = main_r["useful_score_flops"] / (kern[dom] / 1e3) / 1e12
        kfile = "score.cu"
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": sustained,
                "unit": "TFLOP/s", "frac": achieved / sustained,
                "peak_source": f"{peak_src} bf16 sustained",
                "traffic": profiled_traffic(kfile, MAIN)}
    if main_r["gather"] and dom == "sparse_attn":
        roofline["gather_frac"] = main_r["gather"]["frac"]
    useful = main_r["useful_attn_flops"] + main_r["useful_score_flops"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": main_config(w, dist.world),
        "useful_tflops": whole_job_rate(useful, dist.world, ms) / 1e12,
        "executed_tflops": whole_job_rate(
            main_r["executed_attn_flops"] + main_r["executed_score_flops"], dist.world, ms) / 1e12,
        "kernels_ms": kern,
        "roofline": roofline,
        "gather_roofline": main_r["gather"],
        "e2e": {"value": whole_job_rate(main_r["tokens"], dist.world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": main_r["h2d"], "d2h_bytes_per_step": main_r["d2h"]},
        "gpu_launches": main_r["launches_per_step"] * args.steps,
        "clocks": main_r["clocks"],
    }
    line.update(extras)
    if dist.rank == 0:
        line["cpu_baseline"] = cpu_oracle_sample(w, args.baseline_seconds)
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
