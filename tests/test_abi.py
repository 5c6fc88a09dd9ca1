"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from trainable_block_sparse_compressed_b200 import infllmv2 as api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "infllmv2.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(api._LIB_PATH):
        from trainable_block_sparse_compressed_b200 import build
        build.build()
    return api.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(infllmv2_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(api.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    nm = os.popen(f"nm -D --defined-only {api._LIB_PATH}").read()
    for name in declared_symbols():
        assert re.search(rf"\bT {name}\b", nm), name


def test_checked_build_exports_every_declared_symbol():
    """libinfllmv2_checks.so (device index checks) offers the same ABI."""
    from trainable_block_sparse_compressed_b200 import build
    path = build.build(checks=True)
    nm = os.popen(f"nm -D --defined-only {path}").read()
    for name in declared_symbols():
        assert re.search(rf"\bT {name}\b", nm), name


def test_host_helpers(lib):
    assert lib.infllmv2_version() == 100
    assert api.num_compressed(31) == 0
    assert api.num_compressed(32) == 1
    assert api.num_compressed(131072) == 8191
    for code in [0, -1, -2, -3, -4, -5, -6]:
        assert lib.infllmv2_strerror(code)


def _union_bytes(B, Tq, Hkv, G, topk, T=None):
    """Workspace of the query-tile schedule: per tile of 128/G query tokens,
    room for every token's topk (block, token mask) entries of 8 bytes, then
    one count per tile (each part 256-byte aligned), then K and V of all T
    keys repacked into 16 KB block tiles."""
    T = Tq if T is None else T
    tpt = 128 // G
    tiles = B * Hkv * (-(-Tq // tpt))
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    return up(tiles * tpt * topk * 8) + up(tiles * 4) + _packed_bytes(B, T, Hkv)


def _packed_bytes(B, T, Hkv):
    return 2 * B * Hkv * (-(-T // 64)) * 16384


def test_workspace_sizes(lib):
    p = api.make_params(1, 131072, 32, 2, topk=64)
    # causally packed block scores: sum_t (t//64 + 1) floats per (b, kv head)
    T = 131072
    per = sum((t // 64 + 1) for t in range(0, T, 64)) * 64
    assert api.workspace_bytes(p, api.OP_SELECT) == 2 * per * 4
    # groups of 16 heads: the query-tile schedule's union lists
    assert api.workspace_bytes(p, api.OP_ATTN) == _union_bytes(1, T, 2, 16, 64)
    assert api.workspace_bytes(p, api.OP_ATTN_PER_TOKEN) == _packed_bytes(1, T, 2)
    # groups of 4 heads: 32-token query tiles
    p4 = api.make_params(1, 2048, 8, 2, topk=8)
    assert api.workspace_bytes(p4, api.OP_ATTN) == _union_bytes(1, 2048, 2, 4, 8)
    # smaller groups: the per-token schedule's packed K/V tiles
    p2 = api.make_params(1, 2048, 4, 2, topk=8)
    assert api.workspace_bytes(p2, api.OP_ATTN) == _packed_bytes(1, 2048, 2)
    p8 = api.make_params(1, 2000, 16, 2, topk=8)
    assert api.workspace_bytes(p8, api.OP_ATTN) == _union_bytes(1, 2000, 2, 8, 8)
    # the dense forward needs no workspace
    dense = api.make_params(2, 4096, 32, 2, switch_threshold=8192)
    assert api.workspace_bytes(dense, api.OP_FORWARD) == 0
    # sparse forward: block scores (256-byte aligned) then the attention's
    assert api.workspace_bytes(p, api.OP_FORWARD) == \
        (-(-api.workspace_bytes(p, api.OP_SELECT) // 256) * 256) + api.workspace_bytes(p, api.OP_ATTN)
    assert api.workspace_bytes(api.make_params(16, 131328, 32, 2), api.OP_DECODE) > 0
    bad = api.make_params(1, 100, 32, 2, head_dim=64)
    with pytest.raises(api.InfLLMV2Error):
        api.workspace_bytes(bad, api.OP_SELECT)
    # sizes beyond the selection / decode limits are refused before any launch
    with pytest.raises(api.InfLLMV2Error):
        api.workspace_bytes(api.make_params(1, 262144 + 64, 32, 2), api.OP_SELECT)
    with pytest.raises(api.InfLLMV2Error):
        api.workspace_bytes(api.make_params(1, 524288 + 64, 32, 2), api.OP_DECODE)


def test_size_limits_rejected_before_any_launch(lib):
    big = api.make_params(1, 262144 + 64, 32, 2, topk=64, switch_threshold=0)
    P = ctypes.byref(big)
    assert lib.infllmv2_select_blocks(P, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == api.ERR_UNSUPPORTED
    assert lib.infllmv2_forward(P, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                                None) == api.ERR_UNSUPPORTED
    dec = api.make_params(1, 524288 + 64, 32, 2, topk=64)
    assert lib.infllmv2_decode_step(ctypes.byref(dec), *([FAKE] * 11), 1 << 40, None) == \
        api.ERR_UNSUPPORTED


FAKE = 0x10000  # never dereferenced: validation fails first


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), api.ERR_UNSUPPORTED),
    (dict(block_size=32), api.ERR_UNSUPPORTED),
    (dict(cmp_kernel=16), api.ERR_UNSUPPORTED),
    (dict(cmp_stride=32), api.ERR_UNSUPPORTED),
    (dict(Hq=24), api.ERR_UNSUPPORTED),        # G = 12
    (dict(Hq=33), api.ERR_INVALID_ARG),        # Hq % Hkv != 0
    (dict(topk=2), api.ERR_INVALID_ARG),       # < n_init + n_local
    (dict(topk=257), api.ERR_INVALID_ARG),
    (dict(n_local=-1), api.ERR_INVALID_ARG),
    (dict(scale=-1.0), api.ERR_INVALID_ARG),
])
def test_bad_params_rejected_on_host(lib, kw, code):
    base = dict(B=1, T=256, Hq=32, Hkv=2, topk=8)
    base.update(kw)
    p = api.make_params(**base)
    P = ctypes.byref(p)
    assert lib.infllmv2_select_blocks(P, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == code
    assert lib.infllmv2_sparse_attn(P, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None) == code


def test_null_and_misaligned_pointers(lib):
    p = api.make_params(1, 256, 32, 2, topk=8)
    P = ctypes.byref(p)
    assert lib.infllmv2_compress_keys(P, None, FAKE, None) == api.ERR_INVALID_ARG
    assert lib.infllmv2_compress_keys(P, FAKE + 2, FAKE, None) == api.ERR_UNSUPPORTED
    assert lib.infllmv2_dense_attn(P, FAKE, FAKE, FAKE, None, FAKE, None, 0, None) == api.ERR_INVALID_ARG
    assert lib.infllmv2_select_blocks(P, FAKE, FAKE, FAKE, FAKE, 16, None) == api.ERR_WORKSPACE
    assert lib.infllmv2_get_status(None, None) == api.ERR_INVALID_ARG


def test_empty_problems_are_noops(lib):
    p = api.make_params(0, 256, 32, 2, topk=8)
    assert lib.infllmv2_compress_keys(ctypes.byref(p), None, None, None) == api.OK
    p = api.make_params(1, 0, 32, 2, topk=8)
    assert lib.infllmv2_sparse_attn(ctypes.byref(p), None, None, None, None, None, None, None, 0,
                                    None) == api.OK


def test_prefill_chunk_rejected_on_host(lib):
    p = api.make_params(1, 1000, 32, 2, topk=8, switch_threshold=0)
    P = ctypes.byref(p)
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None)
    # the chunk must end at p->T
    assert lib.infllmv2_prefill_chunk(P, 400, 500, *args) == api.ERR_INVALID_ARG
    assert lib.infllmv2_prefill_chunk(P, -1, 1001, *args) == api.ERR_INVALID_ARG
    assert lib.infllmv2_prefill_chunk(P, 400, 600, FAKE + 8, *args[1:]) == api.ERR_UNSUPPORTED
    assert lib.infllmv2_prefill_chunk(P, 1000, 0, *args) == api.OK  # no queries
    with pytest.raises(api.InfLLMV2Error):
        api.prefill_chunk_workspace_bytes(p, 10, 10)


def test_prefill_chunk_workspace_sizes(lib):
    p = api.make_params(1, 131072, 32, 2, topk=64, switch_threshold=8192)
    # the whole sequence as one chunk needs what forward needs
    assert api.prefill_chunk_workspace_bytes(p, 0, 131072) == api.workspace_bytes(p, api.OP_FORWARD)
    # a tail chunk: the block scores of its rows only, then the union lists of
    # its tiles and the packed K/V of every key
    q0, n = 131072 - 4096, 4096
    rows = sum(t // 64 + 1 for t in range(q0, q0 + n))
    sel = 2 * rows * 4
    assert api.prefill_chunk_workspace_bytes(p, q0, n) == \
        (-(-sel // 256) * 256) + _union_bytes(1, n, 2, 16, 64, T=131072)
    d = api.make_params(1, 4096, 32, 2, switch_threshold=8192)
    assert api.prefill_chunk_workspace_bytes(d, 1000, 3096) == 0


def test_prefill_varlen_rejected_on_host(lib):
    p = api.make_params(1, 1, 32, 2, topk=8, switch_threshold=0)
    # a sequence with more queries than keys
    with pytest.raises(api.InfLLMV2Error):
        api.prefill_varlen_workspace_bytes(p, [0, 10, 30], [0, 10, 20])
    # offsets must start at 0 and ascend
    with pytest.raises(api.InfLLMV2Error):
        api.prefill_varlen_workspace_bytes(p, [5, 10], [0, 10])
    # no sequences: nothing to do
    assert api.prefill_varlen_workspace_bytes(p, [0], [0]) == 0
    # the workspace is the largest any one sequence needs (they share it)
    w1 = api.prefill_chunk_workspace_bytes(api.make_params(1, 3000, 32, 2, topk=8,
                                                           switch_threshold=0), 0, 3000)
    w2 = api.prefill_chunk_workspace_bytes(api.make_params(1, 2000, 32, 2, topk=8,
                                                           switch_threshold=0), 1000, 1000)
    assert api.prefill_varlen_workspace_bytes(p, [0, 3000, 4000], [0, 3000, 5000]) == max(w1, w2)
