"""fp64 CPU oracle for dynamic sparse prefill attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``libminf.so`` and its Python binding) never imports it; the two share no
code.  The arithmetic lives in ``minf_oracle.c`` (plain C, fp64, OpenMP); this
module compiles it with gcc and marshals numpy arrays.

Inputs are the bf16 tensors both sides receive, widened exactly to float32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "minf_oracle.c")


def lib_path(mutant: int = 0, out_dir: Optional[str] = None) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mut{mutant}.so"
    return os.path.join(out_dir or _HERE, name)


def build(mutant: int = 0, out_dir: Optional[str] = None, force: bool = False) -> str:
    """Compiles the oracle (optionally with one planted mistake) and returns the .so path."""
    out = lib_path(mutant, out_dir)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    tmp = f"{out}.{os.getpid()}.tmp"  # concurrent builders (spawned ranks) never share a temp file
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", f"-DORC_MUTANT={mutant}",
           _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double

_SIGS = {
    "orc_vs_estimate": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _D, _P, _I, _P, _P, _P, _P],
    "orc_vs_estimate_topp": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _D, _D, _D, _P, _I, _P, _P, _P, _P, _P, _P],
    "orc_block_estimate": [_P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P],
    "orc_dense_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _P, _I, _P, _P],
    "orc_ashape_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _I, _I, _P, _I, _P, _P],
    "orc_trishape_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _I, _I, _I, _P, _I, _P, _P],
    "orc_block_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _I, _P, _P, _I, _P, _I, _P, _P],
    "orc_vs_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _P, _I, _P, _I, _P, _I, _P, _P],
    "orc_vs_tiles_attention": [_P, _P, _P, _I, _I, _I, _I, _D, _P, _I, _P, _I, _P, _I, _I, _P, _I, _P, _P],
    "orc_threads": [],
    "orc_mutant": [],
}


class Oracle:
    """ctypes view of one build of the oracle library."""

    def __init__(self, mutant: int = 0, out_dir: Optional[str] = None):
        self.path = build(mutant, out_dir)
        self.lib = ctypes.CDLL(self.path)
        for name, argtypes in _SIGS.items():
            fn = getattr(self.lib, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_int

    # -- helpers ---------------------------------------------------------------
    @staticmethod
    def _f32(x) -> np.ndarray:
        if hasattr(x, "detach"):  # torch tensor (bf16 or fp32) -> exact fp32 widening
            x = x.detach().to("cpu").float().numpy()
        return np.ascontiguousarray(x, dtype=np.float32)

    @staticmethod
    def _i32(x) -> Optional[np.ndarray]:
        if x is None:
            return None
        if hasattr(x, "detach"):
            x = x.detach().to("cpu").numpy()
        return np.ascontiguousarray(x, dtype=np.int32)

    @staticmethod
    def _ptr(a: Optional[np.ndarray]):
        return None if a is None else a.ctypes.data

    def _heads(self, hq: int, head_ids: Optional[Sequence[int]]):
        ids = None if head_ids is None else np.ascontiguousarray(head_ids, dtype=np.int32)
        return ids, (hq if ids is None else len(ids))

    @staticmethod
    def _check(rc: int, what: str):
        if rc != 0:
            raise RuntimeError(f"oracle {what} failed with status {rc}")

    # -- 1. Vertical-Slash estimation -------------------------------------------
    def vs_estimate(self, q, k, last_q: int, n_vertical: int, n_slash: int, scale: float,
                    head_ids=None, return_scores: bool = False):
        q, k = self._f32(q), self._f32(k)
        hq, n, d = q.shape
        hkv = k.shape[0]
        ids, nh = self._heads(hq, head_ids)
        v_idx = np.empty((nh, n_vertical), np.int32)
        s_idx = np.empty((nh, n_slash), np.int32)
        vert = np.empty((nh, n), np.float64) if return_scores else None
        slash = np.empty((nh, n), np.float64) if return_scores else None
        rc = self.lib.orc_vs_estimate(self._ptr(q), self._ptr(k), hq, hkv, n, d, last_q,
                                      n_vertical, n_slash, scale, self._ptr(ids), nh,
                                      self._ptr(v_idx), self._ptr(s_idx), self._ptr(vert),
                                      self._ptr(slash))
        self._check(rc, "vs_estimate")
        if return_scores:
            return v_idx, s_idx, vert, slash
        return v_idx, s_idx

    def vs_estimate_topp(self, q, k, last_q: int, n_vertical: int, n_slash: int, p_vertical: float,
                         p_slash: float, scale: float, head_ids=None, return_scores: bool = False):
        """Top-p budgets: returns (v_idx, s_idx, v_cnt, s_cnt[, vert, slash])."""
        q, k = self._f32(q), self._f32(k)
        hq, n, d = q.shape
        hkv = k.shape[0]
        ids, nh = self._heads(hq, head_ids)
        v_idx = np.empty((nh, n_vertical), np.int32)
        s_idx = np.empty((nh, n_slash), np.int32)
        v_cnt = np.empty(nh, np.int32)
        s_cnt = np.empty(nh, np.int32)
        vert = np.empty((nh, n), np.float64) if return_scores else None
        slash = np.empty((nh, n), np.float64) if return_scores else None
        rc = self.lib.orc_vs_estimate_topp(self._ptr(q), self._ptr(k), hq, hkv, n, d, last_q, n_vertical,
                                           n_slash, p_vertical, p_slash, scale, self._ptr(ids), nh,
                                           self._ptr(v_idx), self._ptr(s_idx), self._ptr(v_cnt),
                                           self._ptr(s_cnt), self._ptr(vert), self._ptr(slash))
        self._check(rc, "vs_estimate_topp")
        if return_scores:
            return v_idx, s_idx, v_cnt, s_cnt, vert, slash
        return v_idx, s_idx, v_cnt, s_cnt

    # -- 2. Block-Sparse estimation ---------------------------------------------
    def block_estimate(self, q, k, block: int, topk: int, head_ids=None,
                       return_scores: bool = False):
        q, k = self._f32(q), self._f32(k)
        hq, n, d = q.shape
        hkv = k.shape[0]
        ids, nh = self._heads(hq, head_ids)
        nb = n // block
        blk_idx = np.empty((nh, nb, topk), np.int32)
        blk_cnt = np.empty((nh, nb), np.int32)
        pq = np.empty((nh, nb, d), np.float64) if return_scores else None
        pk = np.empty((nh, nb, d), np.float64) if return_scores else None
        sc = np.empty((nh, nb, nb), np.float64) if return_scores else None
        rc = self.lib.orc_block_estimate(self._ptr(q), self._ptr(k), hq, hkv, n, d, block, topk,
                                         self._ptr(ids), nh, self._ptr(blk_idx),
                                         self._ptr(blk_cnt), self._ptr(pq), self._ptr(pk),
                                         self._ptr(sc))
        self._check(rc, "block_estimate")
        if return_scores:
            return blk_idx, blk_cnt, pq, pk, sc
        return blk_idx, blk_cnt

    # -- 4. attention ---------------------------------------------------------------
    def _attn_common(self, q, k, v, head_ids, rows):
        q, k, v = self._f32(q), self._f32(k), self._f32(v)
        hq, n, d = q.shape
        hkv = k.shape[0]
        ids, nh = self._heads(hq, head_ids)
        r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
        nr = n if r is None else len(r)
        out = np.empty((nh, nr, d), np.float64)
        lse = np.empty((nh, nr), np.float64)
        return q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse

    def dense_attention(self, q, k, v, scale: float, head_ids=None, rows=None):
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        rc = self.lib.orc_dense_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n, d,
                                          scale, self._ptr(ids), nh, self._ptr(r), nr,
                                          self._ptr(out), self._ptr(lse))
        self._check(rc, "dense_attention")
        return out, lse

    def ashape_attention(self, q, k, v, scale: float, n_sink: int, window: int, head_ids=None,
                         rows=None):
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        rc = self.lib.orc_ashape_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n,
                                           d, scale, self._ptr(ids), nh, n_sink, window,
                                           self._ptr(r), nr, self._ptr(out), self._ptr(lse))
        self._check(rc, "ashape_attention")
        return out, lse

    def trishape_attention(self, q, k, v, scale: float, n_sink: int, window: int, n_last: int,
                           head_ids=None, rows=None):
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        rc = self.lib.orc_trishape_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n,
                                             d, scale, self._ptr(ids), nh, n_sink, window, n_last,
                                             self._ptr(r), nr, self._ptr(out), self._ptr(lse))
        self._check(rc, "trishape_attention")
        return out, lse

    def block_attention(self, q, k, v, scale: float, block: int, blk_idx, blk_cnt,
                        head_ids=None, rows=None):
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        bi, bc = self._i32(blk_idx), self._i32(blk_cnt)
        rc = self.lib.orc_block_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n, d,
                                          scale, self._ptr(ids), nh, block, self._ptr(bi),
                                          self._ptr(bc), bi.shape[-1], self._ptr(r), nr,
                                          self._ptr(out), self._ptr(lse))
        self._check(rc, "block_attention")
        return out, lse

    def vs_attention(self, q, k, v, scale: float, v_idx, s_idx, head_ids=None, rows=None):
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        vi, si = self._i32(v_idx), self._i32(s_idx)
        rc = self.lib.orc_vs_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n, d,
                                       scale, self._ptr(ids), nh, self._ptr(vi), vi.shape[-1],
                                       self._ptr(si), si.shape[-1], self._ptr(r), nr,
                                       self._ptr(out), self._ptr(lse))
        self._check(rc, "vs_attention")
        return out, lse

    def vs_tiles_attention(self, q, k, v, scale: float, v_idx, s_idx, tile_rows: int = 128,
                           head_ids=None, rows=None):
        """Vertical-Slash with whole slash tiles of ``tile_rows`` query rows."""
        q, k, v, hq, hkv, n, d, ids, nh, r, nr, out, lse = self._attn_common(q, k, v, head_ids, rows)
        vi, si = self._i32(v_idx), self._i32(s_idx)
        rc = self.lib.orc_vs_tiles_attention(self._ptr(q), self._ptr(k), self._ptr(v), hq, hkv, n, d,
                                             scale, self._ptr(ids), nh, self._ptr(vi), vi.shape[-1],
                                             self._ptr(si), si.shape[-1], tile_rows, self._ptr(r), nr,
                                             self._ptr(out), self._ptr(lse))
        self._check(rc, "vs_tiles_attention")
        return out, lse

    def threads(self) -> int:
        return int(self.lib.orc_threads())


_DEFAULT: Optional[Oracle] = None


def get() -> Oracle:
    """The default (unmutated) oracle build, compiled on first use."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle(0)
    return _DEFAULT
