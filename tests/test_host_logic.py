"""Host-side logic without a GPU: the ctypes mirror of the C parameter block,
the constants the binding shares with the header, the seeded workload
generators and bench.py's bookkeeping helpers."""
import ctypes
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest

from trainable_block_sparse_compressed_b200 import infllmv2 as api
from trainable_block_sparse_compressed_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "infllmv2.h")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_params_struct_layout_matches_the_header(tmp_path):
    """sizeof and every field offset of infllmv2_params, as a C compiler lays
    the header out, equal the ctypes mirror the binding passes."""
    names = [f[0] for f in api.Params._fields_]
    src = tmp_path / "layout.c"
    body = "\n".join(f'  printf("{n} %zu\\n", offsetof(infllmv2_params, {n}));' for n in names)
    src.write_text(f'#include <stddef.h>\n#include <stdio.h>\n#include "{HEADER}"\n'
                   f'int main(void) {{\n  printf("sizeof %zu\\n", sizeof(infllmv2_params));\n'
                   f'{body}\n  return 0;\n}}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-o", str(exe), str(src)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], check=True, capture_output=True,
                                                       text=True).stdout.splitlines())
    assert int(out["sizeof"]) == ctypes.sizeof(api.Params)
    for n in names:
        assert int(out[n]) == getattr(api.Params, n).offset, n


def test_binding_constants_match_the_header():
    text = open(HEADER).read()
    defs = dict(re.findall(r"#define\s+(INFLLMV2_\w+)\s+\(?(-?\w+)", text))
    assert int(defs["INFLLMV2_OK"]) == api.OK
    assert int(defs["INFLLMV2_ERR_INVALID_ARG"]) == api.ERR_INVALID_ARG
    assert int(defs["INFLLMV2_ERR_UNSUPPORTED"]) == api.ERR_UNSUPPORTED
    assert int(defs["INFLLMV2_ERR_WORKSPACE"]) == api.ERR_WORKSPACE
    for op in ("SELECT", "FORWARD", "DECODE", "ATTN"):
        assert int(defs[f"INFLLMV2_OP_{op}"]) == getattr(api, f"OP_{op}")
    assert int(defs["INFLLMV2_PATH_DENSE"]) == api.PATH_DENSE
    assert int(defs["INFLLMV2_PATH_SPARSE"]) == api.PATH_SPARSE


def test_workloads_are_seeded_and_bf16():
    w = wl.small_workload(B=1, T=300, Hq=8, Hkv=2, needles=1, seed=3)
    a, b = wl.make_prefill(w), wl.make_prefill(w)
    for k in "QKV":
        assert a[k].dtype == np.uint16 and np.array_equal(a[k], b[k])
    c = wl.make_prefill(wl.small_workload(B=1, T=300, Hq=8, Hkv=2, needles=1, seed=4))
    assert not np.array_equal(a["Q"], c["Q"])
    # bf16 rounding is round-to-nearest-even on the fp32 bits
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5], dtype=np.float32)
    assert np.array_equal(wl.bf16_to_f64(wl.f32_to_bf16_bits(x)), [1.0, 1.0, 1.0 + 2.0 ** -6, -2.5])


def test_planted_needles_follow_the_recipe():
    """Every key of a needle block is 3 sqrt(d) times the unit mean query
    direction of the group over the query range that follows the block."""
    w = wl.small_workload(B=1, T=1000, Hq=8, Hkv=2, needles=3, seed=9)
    d = wl.make_prefill(w)
    K, Q = wl.bf16_to_f64(d["K"]), wl.bf16_to_f64(d["Q"])
    assert len(d["needles"]) == 3
    G = w.Hq // w.Hkv
    nb = (w.T + 63) // 64
    for nd in d["needles"]:
        assert 1 <= nd.block <= nb - 3 and nd.block + 2 <= nd.query_block < nb
        rows = K[nd.batch, nd.block * 64:(nd.block + 1) * 64]    # [64, Hkv, d]
        t0, t1 = nd.query_block * 64, min(nd.query_block * 64 + 64, w.T)
        for g in range(w.Hkv):
            kg = rows[:, g]
            assert np.array_equal(kg, np.broadcast_to(kg[0], kg.shape))  # one planted key
            assert abs(np.linalg.norm(kg[0]) - 3 * np.sqrt(128)) < 0.1    # bf16 rounding only
            mq = Q[nd.batch, t0:t1, g * G:(g + 1) * G].reshape(-1, 128).mean(axis=0)
            cos = kg[0] @ mq / (np.linalg.norm(kg[0]) * np.linalg.norm(mq))
            assert cos > 0.999


def test_bench_traffic_lookup_requires_the_current_kernel_source(monkeypatch, tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(
        '{"k.cu": {"wl": {"source_sha": "abc", "dram_bytes_per_launch": 123}}}')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda name: "abc")
    assert bench.profiled_traffic("k.cu", "wl") == 123
    monkeypatch.setattr(bench, "kernel_source_hash", lambda name: "changed")
    assert bench.profiled_traffic("k.cu", "wl") is None
    assert bench.profiled_traffic("other.cu", "wl") is None


def test_both_bench_arms_report_the_same_config():
    sys.path.insert(0, ROOT)
    import bench
    w = wl.WORKLOADS[bench.MAIN]
    c = bench.main_config(w, 1)
    assert c["workload"] == bench.MAIN and c["T"] == 131072 and c["Hq"] == 32 and c["Hkv"] == 2
    assert c["topk"] == 64 and c["n_init"] == 1 and c["n_local"] == 2
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert src.count("\"config\": main_config(w,") == 2  # the reference arm and ours


def test_kernel_code_hash_ignores_comments_but_not_code(monkeypatch, tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    d = tmp_path / "trainable_block_sparse_compressed_b200" / "csrc"
    d.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (d / "k.cu").write_text("// a kernel\nint f(int x) {  return x + 1; }  /* note */\n")
    h0 = bench.kernel_source_hash("k.cu")
    (d / "k.cu").write_text("// the kernel, described anew\n/* more\n text */\nint f(int x) { return x + 1; }\n")
    assert bench.kernel_source_hash("k.cu") == h0
    (d / "k.cu").write_text("int f(int x) { return x + 2; }\n")
    assert bench.kernel_source_hash("k.cu") != h0
