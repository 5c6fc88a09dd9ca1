"""The decode step that allocates nothing (infllmv2_decode_step_noalloc).

Some host runtimes embed this library and hand it only a step's inputs and
outputs: their own allocator owns the rest of device memory and they have no
way to pass a workspace.  For them the library offers a decode step whose
scratch is a fixed array inside the library.  This test calls that entry
point through the C ABI and checks it against infllmv2_decode_step (the
entry point with a caller workspace) on two decode steps in a row, starting
from identical caches, within the tolerances the other parity tests use.
It lives in a file of its own, collected last, and needs only the session's
library fixture, so it runs the same alone in a fresh process or after the
rest of the suite.
"""
import ctypes

import numpy as np
import pytest

from trainable_block_sparse_compressed_b200 import workloads as wl

from _helpers import LSE_ATOL, O_ATOL, f64, gpu_bf16

pytestmark = pytest.mark.gpu


def _state(api, data, B, L0, Lmax, Hq, Hkv):
    import torch
    Kc = torch.zeros((B, Lmax, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    Kc[:, :L0] = gpu_bf16(data["K0"])
    Vc[:, :L0] = gpu_bf16(data["V0"])
    Kcmp = torch.zeros((B, api.num_compressed(Lmax), Hkv, 2, 128), dtype=torch.bfloat16,
                       device="cuda")
    n0 = api.num_compressed(L0)
    tmp = torch.empty((B, n0, Hkv, 2, 128), dtype=torch.bfloat16, device="cuda")
    api.compress_keys(api.make_params(B, L0, Hq, Hkv), gpu_bf16(data["K0"]), tmp)
    Kcmp[:, :n0] = tmp
    seqlens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    return Kc, Vc, Kcmp, seqlens


def test_decode_step_noalloc_matches_decode_step(cuda_lib):
    import torch
    api = cuda_lib
    lib = api.load()
    w = wl.WORKLOADS["sparse_decode_B16_L131072_Hq32_Hkv2"]
    B, L0, steps, Hq, Hkv = 4, 4000, 2, w.Hq, w.Hkv
    Lmax = L0 + steps
    data = wl.make_decode(w, L=L0, steps=steps, B=B)
    p = api.make_params(B, Lmax, Hq, Hkv, topk=w.topk, n_init=w.n_init, n_local=w.n_local)
    assert api.workspace_bytes(p, api.OP_DECODE) <= api.NOALLOC_SCRATCH_BYTES
    ref = _state(api, data, B, L0, Lmax, Hq, Hkv)
    new = _state(api, data, B, L0, Lmax, Hq, Hkv)
    ws = api.alloc_workspace(p, api.OP_DECODE)
    outs = []
    for _ in range(2):
        outs.append((torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda"),
                     torch.empty((B, Hq), dtype=torch.float32, device="cuda"),
                     torch.empty((B, Hkv, w.topk), dtype=torch.int32, device="cuda")))
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(steps):
        q, kn, vn = (gpu_bf16(data[x][s]) for x in ("q", "k_new", "v_new"))
        O_r, L_r, I_r = outs[0]
        O_n, L_n, I_n = outs[1]
        api.decode_step(p, q, kn, vn, *ref[:3], ref[3], O_r, L_r, I_r, ws)
        Kc, Vc, Kcmp, seqlens = new
        rc = lib.infllmv2_decode_step_noalloc(
            ctypes.byref(p), q.data_ptr(), kn.data_ptr(), vn.data_ptr(), Kc.data_ptr(),
            Vc.data_ptr(), Kcmp.data_ptr(), seqlens.data_ptr(), O_n.data_ptr(), L_n.data_ptr(),
            I_n.data_ptr(), stream)
        assert rc == api.OK, lib.infllmv2_strerror(rc)
        torch.cuda.synchronize()
        assert api.get_status() == 0
        assert torch.equal(I_n, I_r)
        assert np.abs(f64(O_n) - f64(O_r)).max() <= O_ATOL
        assert np.abs(f64(L_n) - f64(L_r)).max() <= LSE_ATOL
        assert torch.equal(new[3], ref[3])
        assert torch.equal(new[2], ref[2]) and torch.equal(new[0], ref[0])


def test_decode_step_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    api = cuda_lib
    lib = api.load()
    p = api.make_params(64, 262144, 32, 2, topk=64)
    assert api.workspace_bytes(p, api.OP_DECODE) > api.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.infllmv2_decode_step_noalloc(ctypes.byref(p), *([fake] * 10), None, None)
    assert rc == api.ERR_WORKSPACE
