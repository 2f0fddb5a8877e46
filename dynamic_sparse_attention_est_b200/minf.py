"""Python binding of libminf.so: argument marshalling only.

Every function here takes torch CUDA tensors, checks their dtype/layout,
allocates the outputs and the workspace with torch (PyTorch is the allocator
and stream provider), and calls the C entry point of the same name.  There is
no fallback: if ``libminf.so`` is missing or a call fails, an exception is
raised.  See ``include/minf.h`` for the semantics of each call.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libminf.so")

MINF_OK = 0
MINF_ERR_INVALID = -1
MINF_ERR_UNSUPPORTED = -2
MINF_ERR_CUDA = -3
MINF_ERR_TIMEOUT = -4
MINF_ERR_WORKSPACE = -5
MINF_MAX_HEADS = 256
MINF_STATUS_BYTES = 256

OP_VS_ESTIMATE = 1
OP_VS_ATTENTION = 2
OP_BLOCK_ESTIMATE = 3
OP_BLOCK_ATTENTION = 4
OP_ASHAPE_ATTENTION = 5
OP_DENSE_ATTENTION = 6
OP_MIXED_LAYER = 7
OP_TRISHAPE_ATTENTION = 8

PATTERN_CODES = {"dense": 0, "vs": 1, "block": 2, "ashape": 3, "trishape": 4}

_P, _I, _F, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64

_SIGS = {
    "minf_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "minf_vs_estimate": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_vs_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_vs_estimate_topp": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _F, _P, _I, _P, _P, _P, _P, _P, _SZ,
                                   _P]),
    "minf_vs_attention_tiles": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_block_estimate": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_block_scores": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "minf_block_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_ashape_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "minf_trishape_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "minf_dense_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P, _SZ, _P]),
    "minf_mixed_layer": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "minf_vs_estimate_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P]),
    "minf_vs_estimate_noalloc_status": (_I, [_I, _P]),
    "minf_vs_estimate_noalloc_check_timeout": (_I, [_I, _U64, _P]),
    "minf_status": (_I, [_P, _P]),
    "minf_stats": (_I, [_P, _P, ctypes.POINTER(_U64), ctypes.POINTER(_U64)]),
    "minf_stats_detail": (_I, [_P, _P, ctypes.POINTER(_U64), _I]),
    "minf_set_wait_limit_ns": (None, [_U64]),
    "minf_set_vs_diag_ratio": (None, [ctypes.c_float]),
    "minf_profile_enable": (None, [_I]),
    "minf_profile_read": (_I, [ctypes.c_char_p, _SZ]),
    "minf_check_wait_timeout": (_I, [_P, _SZ, _U64, _P]),
    "minf_selftest_exp2": (_I, [_P, _P, _P, _I, _P]),
    "minf_version": (ctypes.c_char_p, []),
    "minf_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libminf.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not built: run python -m dynamic_sparse_attention_est_b200.build_lib")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class MinfError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib().minf_last_error().decode(errors="replace")
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


def _check(code: int, where: str):
    if code != MINF_OK:
        raise MinfError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _qkv(q, k, v=None):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 3 and t.shape[-1] == 128):
            raise ValueError(f"{name} must be a CUDA bf16 tensor [heads, n, 128]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    hq, n, d = q.shape
    hkv = k.shape[0]
    if k.shape[1] != n or (v is not None and tuple(v.shape) != tuple(k.shape)):
        raise ValueError("q, k, v sequence lengths / kv shapes disagree")
    return hq, hkv, n, d


def _heads(hq: int, head_ids: Optional[Sequence[int]]):
    if head_ids is None:
        return None, hq
    arr = (ctypes.c_int32 * len(head_ids))(*[int(h) for h in head_ids])
    return arr, len(head_ids)


def _scale(scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(128) if scale is None else float(scale)


def workspace_bytes(op: int, hq: int, hkv: int, n: int, n_heads: int = 0, p1: int = 0, p2: int = 0,
                    p3: int = 0) -> int:
    return int(lib().minf_workspace_bytes(op, hq, hkv, n, n_heads, p1, p2, p3))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device byte buffer for `ws` (torch allocations are 512-byte aligned)."""
    return torch.zeros(max(int(nbytes), MINF_STATUS_BYTES), dtype=torch.uint8, device=device)


def _ws_for(ws, need, device):
    if ws is None:
        return workspace(need, device)
    if ws.numel() < need:
        raise ValueError(f"workspace of {ws.numel()} bytes, need {need}")
    return ws


def minf_vs_estimate(q, k, last_q: int = 64, n_vertical: int = 1000, n_slash: int = 6096,
                     scale: Optional[float] = None, head_ids=None, ws=None) -> Tuple[torch.Tensor, torch.Tensor]:
    hq, hkv, n, d = _qkv(q, k)
    ids, nh = _heads(hq, head_ids)
    need = workspace_bytes(OP_VS_ESTIMATE, hq, hkv, n, nh)
    ws = _ws_for(ws, need, q.device)
    v_idx = torch.empty(nh, n_vertical, dtype=torch.int32, device=q.device)
    s_idx = torch.empty(nh, n_slash, dtype=torch.int32, device=q.device)
    _check(lib().minf_vs_estimate(_ptr(q), _ptr(k), hq, hkv, n, d, last_q, n_vertical, n_slash, _scale(scale),
                                  ids, nh, _ptr(v_idx), _ptr(s_idx), _ptr(ws), ws.numel(), _stream(q.device)),
           "minf_vs_estimate")
    return v_idx, s_idx


def minf_vs_estimate_topp(q, k, last_q: int = 64, n_vertical: int = 1000, n_slash: int = 6096,
                          p_vertical: float = 0.9, p_slash: float = 0.9, scale: Optional[float] = None,
                          head_ids=None, ws=None):
    """Top-p budgets (the budgets are caps); returns (v_idx, s_idx, v_cnt, s_cnt)."""
    hq, hkv, n, d = _qkv(q, k)
    ids, nh = _heads(hq, head_ids)
    need = workspace_bytes(OP_VS_ESTIMATE, hq, hkv, n, nh)
    ws = _ws_for(ws, need, q.device)
    v_idx = torch.empty(nh, n_vertical, dtype=torch.int32, device=q.device)
    s_idx = torch.empty(nh, n_slash, dtype=torch.int32, device=q.device)
    v_cnt = torch.empty(nh, dtype=torch.int32, device=q.device)
    s_cnt = torch.empty(nh, dtype=torch.int32, device=q.device)
    _check(lib().minf_vs_estimate_topp(_ptr(q), _ptr(k), hq, hkv, n, d, last_q, n_vertical, n_slash,
                                       float(p_vertical), float(p_slash), _scale(scale), ids, nh, _ptr(v_idx),
                                       _ptr(s_idx), _ptr(v_cnt), _ptr(s_cnt), _ptr(ws), ws.numel(),
                                       _stream(q.device)),
           "minf_vs_estimate_topp")
    return v_idx, s_idx, v_cnt, s_cnt


def minf_vs_estimate_noalloc(q, k, last_q: int = 64, n_vertical: int = 1000, n_slash: int = 6096,
                             scale: Optional[float] = None, head_ids=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """minf_vs_estimate with the library's built-in scratch instead of a workspace.

    For callers that cannot allocate device memory for scratch; only the two
    index outputs are allocated here (by torch, on behalf of this binding).
    """
    hq, hkv, n, d = _qkv(q, k)
    ids, nh = _heads(hq, head_ids)
    v_idx = torch.empty(nh, n_vertical, dtype=torch.int32, device=q.device)
    s_idx = torch.empty(nh, n_slash, dtype=torch.int32, device=q.device)
    _check(lib().minf_vs_estimate_noalloc(_ptr(q), _ptr(k), hq, hkv, n, d, last_q, n_vertical, n_slash,
                                          _scale(scale), ids, nh, _ptr(v_idx), _ptr(s_idx), _stream(q.device)),
           "minf_vs_estimate_noalloc")
    return v_idx, s_idx


def minf_vs_estimate_noalloc_status(device=None) -> int:
    """Status code of the last allocation-free estimate on `device` (read and cleared)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(lib().minf_vs_estimate_noalloc_status(dev.index or 0, _stream(dev)))


def minf_vs_estimate_noalloc_check_timeout(limit_ns: int, device=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(lib().minf_vs_estimate_noalloc_check_timeout(dev.index or 0, int(limit_ns), _stream(dev)),
           "minf_vs_estimate_noalloc_check_timeout")


def _vs_attention(fn_name, q, k, v, v_idx, s_idx, scale, head_ids, out, want_lse, ws):
    hq, hkv, n, d = _qkv(q, k, v)
    ids, nh = _heads(hq, head_ids)
    v_idx = v_idx.to(torch.int32).contiguous()
    s_idx = s_idx.to(torch.int32).contiguous()
    need = workspace_bytes(OP_VS_ATTENTION, hq, hkv, n, nh, v_idx.shape[-1], s_idx.shape[-1])
    ws = _ws_for(ws, need, q.device)
    out = torch.empty(nh, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(nh, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(getattr(lib(), fn_name)(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), ids, nh, _ptr(v_idx),
                                   v_idx.shape[-1], _ptr(s_idx), s_idx.shape[-1], _ptr(out), _ptr(lse), _ptr(ws),
                                   ws.numel(), _stream(q.device)),
           fn_name)
    return out, lse


def minf_vs_attention(q, k, v, v_idx, s_idx, scale: Optional[float] = None, head_ids=None, out=None,
                      want_lse: bool = True, ws=None):
    return _vs_attention("minf_vs_attention", q, k, v, v_idx, s_idx, scale, head_ids, out, want_lse, ws)


def minf_vs_attention_tiles(q, k, v, v_idx, s_idx, scale: Optional[float] = None, head_ids=None, out=None,
                            want_lse: bool = True, ws=None):
    """Vertical-Slash attention with every computed slash range attended whole."""
    return _vs_attention("minf_vs_attention_tiles", q, k, v, v_idx, s_idx, scale, head_ids, out, want_lse, ws)


def minf_block_estimate(q, k, topk: int = 100, block: int = 64, head_ids=None, ws=None):
    hq, hkv, n, d = _qkv(q, k)
    ids, nh = _heads(hq, head_ids)
    need = workspace_bytes(OP_BLOCK_ESTIMATE, hq, hkv, n, nh, topk)
    ws = _ws_for(ws, need, q.device)
    nb = n // 64
    blk_idx = torch.empty(nh, nb, topk, dtype=torch.int32, device=q.device)
    blk_cnt = torch.empty(nh, nb, dtype=torch.int32, device=q.device)
    _check(lib().minf_block_estimate(_ptr(q), _ptr(k), hq, hkv, n, d, block, topk, ids, nh, _ptr(blk_idx),
                                     _ptr(blk_cnt), _ptr(ws), ws.numel(), _stream(q.device)),
           "minf_block_estimate")
    return blk_idx, blk_cnt


def minf_block_scores(q, k, block: int = 64, head_ids=None, ws=None):
    """Pooled block scores [n_heads][n/64][n/64] (fp32); entries j > i unspecified."""
    hq, hkv, n, d = _qkv(q, k)
    ids, nh = _heads(hq, head_ids)
    need = workspace_bytes(OP_BLOCK_ESTIMATE, hq, hkv, n, nh, 1)
    ws = _ws_for(ws, need, q.device)
    nb = n // 64
    scores = torch.empty(nh, nb, nb, dtype=torch.float32, device=q.device)
    _check(lib().minf_block_scores(_ptr(q), _ptr(k), hq, hkv, n, d, block, ids, nh, _ptr(scores), _ptr(ws),
                                   ws.numel(), _stream(q.device)),
           "minf_block_scores")
    return scores


def minf_block_attention(q, k, v, blk_idx, blk_cnt, scale: Optional[float] = None, head_ids=None, out=None,
                         want_lse: bool = True, ws=None):
    hq, hkv, n, d = _qkv(q, k, v)
    ids, nh = _heads(hq, head_ids)
    blk_idx = blk_idx.to(torch.int32).contiguous()
    blk_cnt = blk_cnt.to(torch.int32).contiguous()
    topk = blk_idx.shape[-1]
    need = workspace_bytes(OP_BLOCK_ATTENTION, hq, hkv, n, nh, topk)
    ws = _ws_for(ws, need, q.device)
    out = torch.empty(nh, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(nh, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().minf_block_attention(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), ids, nh,
                                      _ptr(blk_idx), _ptr(blk_cnt), topk, _ptr(out), _ptr(lse), _ptr(ws),
                                      ws.numel(), _stream(q.device)),
           "minf_block_attention")
    return out, lse


def minf_ashape_attention(q, k, v, n_sink: int = 128, window: int = 4096, scale: Optional[float] = None,
                          head_ids=None, out=None, want_lse: bool = True, ws=None):
    hq, hkv, n, d = _qkv(q, k, v)
    ids, nh = _heads(hq, head_ids)
    ws = _ws_for(ws, MINF_STATUS_BYTES, q.device)
    out = torch.empty(nh, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(nh, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().minf_ashape_attention(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), ids, nh, n_sink,
                                       window, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)),
           "minf_ashape_attention")
    return out, lse


def minf_trishape_attention(q, k, v, n_sink: int = 128, window: int = 4096, n_last: int = 64,
                            scale: Optional[float] = None, head_ids=None, out=None, want_lse: bool = True, ws=None):
    hq, hkv, n, d = _qkv(q, k, v)
    ids, nh = _heads(hq, head_ids)
    ws = _ws_for(ws, MINF_STATUS_BYTES, q.device)
    out = torch.empty(nh, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(nh, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().minf_trishape_attention(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), ids, nh, n_sink,
                                         window, n_last, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(q.device)),
           "minf_trishape_attention")
    return out, lse


def minf_dense_attention(q, k, v, scale: Optional[float] = None, head_ids=None, out=None, want_lse: bool = True,
                         ws=None):
    hq, hkv, n, d = _qkv(q, k, v)
    ids, nh = _heads(hq, head_ids)
    ws = _ws_for(ws, MINF_STATUS_BYTES, q.device)
    out = torch.empty(nh, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(nh, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().minf_dense_attention(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), ids, nh, _ptr(out),
                                      _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)),
           "minf_dense_attention")
    return out, lse


def minf_mixed_layer(q, k, v, head_patterns: Sequence[str], last_q: int = 64, n_vertical: int = 1000,
                     n_slash: int = 6096, topk: int = 100, n_sink: int = 128, window: int = 4096,
                     scale: Optional[float] = None, out=None, want_lse: bool = True, ws=None):
    hq, hkv, n, d = _qkv(q, k, v)
    if len(head_patterns) != hq:
        raise ValueError("one pattern per q-head")
    codes = (ctypes.c_int8 * hq)(*[PATTERN_CODES[p] for p in head_patterns])
    need = workspace_bytes(OP_MIXED_LAYER, hq, hkv, n, hq, n_vertical, n_slash, topk)
    ws = _ws_for(ws, need, q.device)
    out = torch.empty(hq, n, d, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(hq, n, dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().minf_mixed_layer(_ptr(q), _ptr(k), _ptr(v), hq, hkv, n, d, _scale(scale), codes, last_q,
                                  n_vertical, n_slash, topk, n_sink, window, _ptr(out), _ptr(lse), _ptr(ws),
                                  ws.numel(), _stream(q.device)),
           "minf_mixed_layer")
    return out, lse


def minf_status(ws: torch.Tensor) -> int:
    return int(lib().minf_status(_ptr(ws), _stream(ws.device)))


def minf_stats(ws: torch.Tensor) -> Tuple[int, int]:
    t, p = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(lib().minf_stats(_ptr(ws), _stream(ws.device), ctypes.byref(t), ctypes.byref(p)), "minf_stats")
    return int(t.value), int(p.value)


def minf_stats_detail(ws: torch.Tensor) -> Dict[str, int]:
    """Counters of the last attention call on ws, split by kernel."""
    arr = (_U64 * 7)()
    n = lib().minf_stats_detail(_ptr(ws), _stream(ws.device), arr, 7)
    if n < 0:
        _check(n, "minf_stats_detail")
    keys = ["tiles", "pairs", "tiles_dense", "tiles_vs", "tiles_block", "tiles_ashape", "diag_pairs"]
    return {k: int(arr[i]) for i, k in enumerate(keys[:n])}


def minf_set_wait_limit_ns(ns: int) -> None:
    lib().minf_set_wait_limit_ns(int(ns))


def minf_set_vs_diag_ratio(ratio: float) -> None:
    """Sparse slash groups of m offsets over H half-tiles go to the CUDA-core pass when m < ratio * H."""
    lib().minf_set_vs_diag_ratio(float(ratio))


def minf_profile_enable(on: bool = True) -> None:
    lib().minf_profile_enable(1 if on else 0)


def minf_profile_read() -> Dict[str, Tuple[int, float]]:
    """{kernel name: (launches, total ms)} of the launches timed since the last read."""
    n = int(lib().minf_profile_read(None, 0))
    buf = ctypes.create_string_buffer(n + 1)
    lib().minf_profile_read(buf, n + 1)
    out = {}
    for line in buf.value.decode().splitlines():
        name, cnt, ms = line.split("\t")
        out[name] = (int(cnt), float(ms))
    return out


def minf_check_wait_timeout(ws: torch.Tensor, limit_ns: int) -> None:
    _check(lib().minf_check_wait_timeout(_ptr(ws), ws.numel(), int(limit_ns), _stream(ws.device)),
           "minf_check_wait_timeout")


def minf_selftest_exp2(x: torch.Tensor):
    """(polynomial 2^x, hardware 2^x) as the attention kernels compute them."""
    x = x.to(torch.float32).contiguous()
    y_poly, y_hw = torch.empty_like(x), torch.empty_like(x)
    _check(lib().minf_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_hw), x.numel(), _stream(x.device)),
           "minf_selftest_exp2")
    return y_poly, y_hw


def minf_version() -> str:
    return lib().minf_version().decode()
