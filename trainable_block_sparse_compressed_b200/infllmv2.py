"""ctypes binding of libinfllmv2.so (declared in include/infllmv2.h).

Argument marshalling only: every computation runs in the CUDA library.
Functions take torch CUDA tensors (the caller owns all memory), pass their
device pointers and torch's current CUDA stream, and raise
:class:`InfLLMV2Error` on a non-zero return code.  There is no CPU fallback:
if the shared library is missing, :func:`load` raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libinfllmv2.so")
_lib = None

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_TIMEOUT = -4
ERR_WORKSPACE = -5
ERR_DEVICE_CHECK = -6
STATUS_TIMEOUT = 0x1
STATUS_SEQ_FULL = 0x2
OP_SELECT, OP_FORWARD, OP_DECODE, OP_ATTN, OP_ATTN_PER_TOKEN, OP_FORWARD_FP32 = 1, 2, 3, 4, 5, 6
OP_BACKWARD = 7
PATH_DENSE, PATH_SPARSE = 1, 2

# every symbol include/infllmv2.h declares
EXPORTS = (
    "infllmv2_compress_keys", "infllmv2_select_blocks", "infllmv2_sparse_attn",
    "infllmv2_dense_attn", "infllmv2_forward", "infllmv2_decode_step",
    "infllmv2_workspace_bytes", "infllmv2_num_compressed", "infllmv2_get_status",
    "infllmv2_set_wait_limit", "infllmv2_selftest_timeout", "infllmv2_strerror",
    "infllmv2_version", "infllmv2_decode_step_noalloc", "infllmv2_prefill_chunk",
    "infllmv2_prefill_chunk_workspace_bytes", "infllmv2_gather_peak",
    "infllmv2_sparse_attn_per_token", "infllmv2_compressed_attn", "infllmv2_forward_fp32",
    "infllmv2_prefill_varlen", "infllmv2_prefill_varlen_workspace_bytes",
    "infllmv2_sparse_attn_backward",
)
NOALLOC_SCRATCH_BYTES = 32 << 20


class InfLLMV2Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = _lib.infllmv2_strerror(code).decode() if _lib is not None else str(code)
        super().__init__(f"{fn} failed: {msg} ({code})")
        self.code = code


class Params(ctypes.Structure):
    """Mirror of ``infllmv2_params``."""
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("cmp_kernel", ctypes.c_int32), ("cmp_stride", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("n_init", ctypes.c_int32), ("n_local", ctypes.c_int32),
        ("switch_threshold", ctypes.c_int32), ("scale", ctypes.c_float),
        ("causal", ctypes.c_int32),
    ]


def make_params(B, T, Hq, Hkv, head_dim=128, topk=64, n_init=1, n_local=2,
                switch_threshold=8192, scale=0.0, block_size=64, cmp_kernel=32,
                cmp_stride=16) -> Params:
    return Params(B, T, Hq, Hkv, head_dim, block_size, cmp_kernel, cmp_stride, topk, n_init,
                  n_local, switch_threshold, scale, 1)


def load(path: Optional[str] = None):
    """Loads the shared library once; raises if it is missing.  The
    environment variable INFLLMV2_LIB may name another build of it (the
    bounds-checked libinfllmv2_checks.so)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or os.environ.get("INFLLMV2_LIB") or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"CUDA library not built: {p} (run __graft_entry__.build())")
    lib = ctypes.CDLL(p)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    P = ctypes.POINTER(Params)
    sig = {
        "infllmv2_compress_keys": (ctypes.c_int, [P, vp, vp, vp]),
        "infllmv2_select_blocks": (ctypes.c_int, [P, vp, vp, vp, vp, sz, vp]),
        "infllmv2_sparse_attn": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_sparse_attn_per_token": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_dense_attn": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_compressed_attn": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp]),
        "infllmv2_sparse_attn_backward": (ctypes.c_int, [P] + [vp] * 11 + [sz, vp]),
        "infllmv2_forward": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_forward_fp32": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_decode_step": (ctypes.c_int,
                                 [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "infllmv2_decode_step_noalloc": (ctypes.c_int,
                                         [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "infllmv2_workspace_bytes": (sz, [P, i32]),
        "infllmv2_prefill_chunk": (ctypes.c_int, [P, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                                  vp, vp, sz, vp]),
        "infllmv2_prefill_chunk_workspace_bytes": (sz, [P, i32, i32]),
        "infllmv2_prefill_varlen": (ctypes.c_int, [P, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                   vp, vp, sz, vp]),
        "infllmv2_prefill_varlen_workspace_bytes": (sz, [P, i32, vp, vp]),
        "infllmv2_num_compressed": (i32, [i32]),
        "infllmv2_get_status": (ctypes.c_int, [vp, ctypes.POINTER(i32)]),
        "infllmv2_set_wait_limit": (None, [ctypes.c_int64]),
        "infllmv2_selftest_timeout": (ctypes.c_int, [vp]),
        "infllmv2_strerror": (ctypes.c_char_p, [ctypes.c_int]),
        "infllmv2_version": (ctypes.c_int, []),
        "infllmv2_gather_peak": (ctypes.c_int, [vp, sz, i32, ctypes.POINTER(i32), vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn: str, code: int):
    if code != OK:
        raise InfLLMV2Error(fn, code)


def num_compressed(T: int) -> int:
    return int(load().infllmv2_num_compressed(T))


def workspace_bytes(p: Params, op: int) -> int:
    n = load().infllmv2_workspace_bytes(ctypes.byref(p), op)
    if n == ctypes.c_size_t(-1).value:
        raise InfLLMV2Error("infllmv2_workspace_bytes", ERR_INVALID_ARG)
    return int(n)


def get_status(stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("infllmv2_get_status", load().infllmv2_get_status(_stream(stream), ctypes.byref(out)))
    return int(out.value)


def set_wait_limit(ns: int):
    load().infllmv2_set_wait_limit(int(ns))


def selftest_timeout(stream=None):
    _check("infllmv2_selftest_timeout", load().infllmv2_selftest_timeout(_stream(stream)))


def gather_peak(src, rounds: int, stream=None) -> int:
    """Enqueues the L2 -> shared-memory gather measurement over the device
    buffer ``src``; returns the bytes it moves (the caller times it)."""
    ctas = ctypes.c_int32(0)
    _check("infllmv2_gather_peak",
           load().infllmv2_gather_peak(_ptr(src), src.numel() * src.element_size(), int(rounds),
                                       ctypes.byref(ctas), _stream(stream)))
    return int(ctas.value) * int(rounds) * 3 * 65536


# --------------------------------------------------------------------------
# the five operations and the switch
# --------------------------------------------------------------------------
def compress_keys(p: Params, K, Kc, stream=None):
    """Kc[b, j] = mean(K[b, 16j : 16j+32]) (bf16 tensors on the GPU)."""
    _check("infllmv2_compress_keys",
           load().infllmv2_compress_keys(ctypes.byref(p), _ptr(K), _ptr(Kc), _stream(stream)))


def select_blocks(p: Params, Q, Kc, idx, ws, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("infllmv2_select_blocks",
           load().infllmv2_select_blocks(ctypes.byref(p), _ptr(Q), _ptr(Kc), _ptr(idx), _ptr(ws),
                                         nbytes, _stream(stream)))


def _nbytes(ws) -> int:
    return ws.numel() * ws.element_size() if ws is not None else 0


def sparse_attn(p: Params, Q, K, V, idx, O, lse, ws=None, stream=None):
    """Block-sparse attention; ws (OP_ATTN bytes) enables the query-tile
    schedule (groups of 4, 8 or 16 heads) or the packed K/V gather."""
    _check("infllmv2_sparse_attn",
           load().infllmv2_sparse_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                       _ptr(O), _ptr(lse), _ptr(ws), _nbytes(ws),
                                       _stream(stream)))


def sparse_attn_per_token(p: Params, Q, K, V, idx, O, lse, ws=None, stream=None):
    """Block-sparse attention, one work item per query token; ws
    (OP_ATTN_PER_TOKEN bytes) enables the packed K/V gather."""
    _check("infllmv2_sparse_attn_per_token",
           load().infllmv2_sparse_attn_per_token(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V),
                                                 _ptr(idx), _ptr(O), _ptr(lse), _ptr(ws),
                                                 _nbytes(ws), _stream(stream)))


def sparse_attn_backward(p: Params, Q, K, V, idx, O, lse, dO, dQ, dK, dV, ws, stream=None):
    """Gradients (fp32 dQ, dK, dV) of sparse_attn with the selection idx fixed."""
    _check("infllmv2_sparse_attn_backward",
           load().infllmv2_sparse_attn_backward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V),
                                                _ptr(idx), _ptr(O), _ptr(lse), _ptr(dO), _ptr(dQ),
                                                _ptr(dK), _ptr(dV), _ptr(ws), _nbytes(ws),
                                                _stream(stream)))


def compressed_attn(p: Params, Q, Kc, Vc, O, lse, stream=None):
    """Attention over the compressed windows (Kc, Vc from compress_keys of K, V)."""
    _check("infllmv2_compressed_attn",
           load().infllmv2_compressed_attn(ctypes.byref(p), _ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(O),
                                           _ptr(lse), _stream(stream)))


def dense_attn(p: Params, Q, K, V, O, lse, ws=None, stream=None):
    _check("infllmv2_dense_attn",
           load().infllmv2_dense_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                      _ptr(lse), _ptr(ws), _nbytes(ws), _stream(stream)))


def forward(p: Params, Q, K, V, O, lse, Kc_ws=None, idx_ws=None, ws=None, stream=None) -> int:
    """The switchable attention; returns PATH_DENSE or PATH_SPARSE."""
    path = ctypes.c_int32(0)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("infllmv2_forward",
           load().infllmv2_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                   _ptr(Kc_ws), _ptr(idx_ws), ctypes.byref(path), _ptr(ws), nbytes,
                                   _stream(stream)))
    return int(path.value)


def forward_fp32(p: Params, Q, K, V, O, lse, Kc32_ws=None, idx_ws=None, ws=None,
                 stream=None) -> int:
    """The fp32 validation build of forward (O fp32); returns the path taken."""
    path = ctypes.c_int32(0)
    _check("infllmv2_forward_fp32",
           load().infllmv2_forward_fp32(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                        _ptr(lse), _ptr(Kc32_ws), _ptr(idx_ws), ctypes.byref(path),
                                        _ptr(ws), _nbytes(ws), _stream(stream)))
    return int(path.value)


def prefill_chunk_workspace_bytes(p: Params, q_offset: int, q_len: int) -> int:
    n = load().infllmv2_prefill_chunk_workspace_bytes(ctypes.byref(p), q_offset, q_len)
    if n == ctypes.c_size_t(-1).value:
        raise InfLLMV2Error("infllmv2_prefill_chunk_workspace_bytes", ERR_INVALID_ARG)
    return int(n)


def prefill_chunk(p: Params, q_offset: int, q_len: int, Q, K, V, Kc, O, lse, idx=None, ws=None,
                  stream=None) -> int:
    """Queries for tokens q_offset .. q_offset+q_len-1 over caches of p.T tokens;
    returns PATH_DENSE or PATH_SPARSE."""
    path = ctypes.c_int32(0)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("infllmv2_prefill_chunk",
           load().infllmv2_prefill_chunk(ctypes.byref(p), q_offset, q_len, _ptr(Q), _ptr(K),
                                         _ptr(V), _ptr(Kc), _ptr(O), _ptr(lse), _ptr(idx),
                                         ctypes.byref(path), _ptr(ws), nbytes, _stream(stream)))
    return int(path.value)


def _i32_array(xs):
    arr = (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])
    return arr


def prefill_varlen_workspace_bytes(p: Params, cu_q, cu_k) -> int:
    n = len(cu_q) - 1
    n_bytes = load().infllmv2_prefill_varlen_workspace_bytes(
        ctypes.byref(p), n, ctypes.cast(_i32_array(cu_q), ctypes.c_void_p),
        ctypes.cast(_i32_array(cu_k), ctypes.c_void_p))
    if n_bytes == ctypes.c_size_t(-1).value:
        raise InfLLMV2Error("infllmv2_prefill_varlen_workspace_bytes", ERR_INVALID_ARG)
    return int(n_bytes)


def prefill_varlen(p: Params, cu_q, cu_k, Q, K, V, Kc, O, lse, idx=None, ws=None,
                   stream=None):
    """A packed batch of ragged sequences (host offset lists cu_q, cu_k);
    returns the path taken per sequence."""
    n = len(cu_q) - 1
    aq, ak = _i32_array(cu_q), _i32_array(cu_k)
    paths = (ctypes.c_int32 * max(n, 1))()
    _check("infllmv2_prefill_varlen",
           load().infllmv2_prefill_varlen(ctypes.byref(p), n, ctypes.cast(aq, ctypes.c_void_p),
                                          ctypes.cast(ak, ctypes.c_void_p), _ptr(Q), _ptr(K),
                                          _ptr(V), _ptr(Kc), _ptr(O), _ptr(lse), _ptr(idx),
                                          ctypes.cast(paths, ctypes.c_void_p), _ptr(ws),
                                          _nbytes(ws), _stream(stream)))
    return [int(paths[i]) for i in range(n)]


def decode_step(p: Params, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse,
                idx_out=None, ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("infllmv2_decode_step",
           load().infllmv2_decode_step(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new),
                                       _ptr(K_cache), _ptr(V_cache), _ptr(Kc_cache),
                                       _ptr(seqlens), _ptr(O), _ptr(lse), _ptr(idx_out), _ptr(ws),
                                       nbytes, _stream(stream)))


def decode_step_noalloc(p: Params, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O,
                        lse, idx_out=None, stream=None):
    """decode_step with the library's fixed scratch array instead of a
    workspace (for callers that cannot allocate device memory)."""
    _check("infllmv2_decode_step_noalloc",
           load().infllmv2_decode_step_noalloc(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new),
                                               _ptr(K_cache), _ptr(V_cache), _ptr(Kc_cache),
                                               _ptr(seqlens), _ptr(O), _ptr(lse), _ptr(idx_out),
                                               _stream(stream)))


# --------------------------------------------------------------------------
# allocation conveniences (torch is used for device memory only)
# --------------------------------------------------------------------------
def alloc_workspace(p: Params, op: int, device="cuda"):
    import torch
    n = workspace_bytes(p, op)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def prefill(Q, K, V, topk=64, n_init=1, n_local=2, threshold=8192, scale=0.0, stream=None):
    """Allocates outputs and runs :func:`forward`.  Q [B,T,Hq,128], K/V [B,T,Hkv,128] bf16.

    Returns (O, lse, path, idx or None).
    """
    import torch
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    p = make_params(B, T, Hq, Hkv, d, topk, n_init, n_local, threshold, scale)
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    if T <= threshold:
        ws = alloc_workspace(p, OP_FORWARD, Q.device)
        path = forward(p, Q, K, V, O, lse, ws=ws, stream=stream)
        return O, lse, path, None
    Kc = torch.empty((B, num_compressed(T), Hkv, 2, d), dtype=Q.dtype, device=Q.device)
    idx = torch.empty((B, Hkv, T, topk), dtype=torch.int32, device=Q.device)
    ws = alloc_workspace(p, OP_FORWARD, Q.device)
    path = forward(p, Q, K, V, O, lse, Kc, idx, ws, stream=stream)
    return O, lse, path, idx
