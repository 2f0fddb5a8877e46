"""The C ABI without a GPU: the library loads, exports every declared symbol,
sizes workspaces, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from dynamic_sparse_attention_est_b200 import minf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "minf.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(minf_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol(minf_lib):
    L = ctypes.CDLL(minf_lib)
    names = declared_symbols()
    assert len(names) >= 14
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_binding_covers_every_symbol(minf_lib):
    for name in declared_symbols():
        assert name in minf._SIGS, name


def test_version_string(minf_lib):
    assert "sm_100a" in minf.minf_version()


def test_workspace_sizes(minf_lib):
    ws = minf.workspace_bytes
    assert ws(minf.OP_DENSE_ATTENTION, 32, 8, 32768) == minf.MINF_STATUS_BYTES
    assert ws(minf.OP_ASHAPE_ATTENTION, 32, 8, 32768) == minf.MINF_STATUS_BYTES
    a = ws(minf.OP_VS_ATTENTION, 32, 8, 32768, 32, 1000, 6096)
    b = ws(minf.OP_VS_ATTENTION, 32, 8, 65536, 32, 1000, 6096)
    assert 0 < a < b
    assert ws(minf.OP_VS_ESTIMATE, 32, 8, 32768, 32) > 32 * 32768 * 8  # vertical + slash scores
    assert ws(minf.OP_BLOCK_ESTIMATE, 32, 8, 131072, 32, 100) > 0
    assert ws(minf.OP_BLOCK_ATTENTION, 32, 8, 131072, 32, 100) > 0
    m = ws(minf.OP_MIXED_LAYER, 32, 8, 32768, 32, 1000, 6096, 100)
    assert m >= ws(minf.OP_VS_ATTENTION, 32, 8, 32768, 32, 1000, 6096)
    # rejected shapes size to 0
    assert ws(minf.OP_VS_ATTENTION, 32, 8, 100, 32, 1000, 6096) == 0
    assert ws(minf.OP_VS_ATTENTION, 32, 7, 1024, 32, 1000, 6096) == 0
    assert ws(minf.OP_VS_ATTENTION, 32, 8, 1024, 32, 0, 6096) == 0


FAKE = 1 << 20  # a 256-byte aligned non-null address; never dereferenced


def _dense(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, hq=4, hkv=2, n=1024, d=128, scale=0.088, ids=None, nh=4, out=FAKE, lse=None,
             ws=FAKE, wsb=256, st=None)
    a.update(kw)
    return minf.lib().minf_dense_attention(a["q"], a["k"], a["v"], a["hq"], a["hkv"], a["n"], a["d"], a["scale"],
                                           a["ids"], a["nh"], a["out"], a["lse"], a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), minf.MINF_ERR_INVALID),
    (dict(hkv=3), minf.MINF_ERR_INVALID),
    (dict(d=64), minf.MINF_ERR_UNSUPPORTED),
    (dict(n=1000), minf.MINF_ERR_UNSUPPORTED),
    (dict(n=0), minf.MINF_ERR_UNSUPPORTED),
    (dict(scale=0.0), minf.MINF_ERR_INVALID),
    (dict(scale=float("nan")), minf.MINF_ERR_INVALID),
    (dict(q=FAKE + 8), minf.MINF_ERR_INVALID),
    (dict(ws=None), minf.MINF_ERR_INVALID),
    (dict(wsb=16), minf.MINF_ERR_WORKSPACE),
    (dict(out=None), minf.MINF_ERR_INVALID),
])
def test_dense_argument_checks(minf_lib, kw, code):
    assert _dense(**kw) == code


def test_head_id_checks(minf_lib):
    bad = (ctypes.c_int32 * 2)(0, 9)
    assert _dense(ids=bad, nh=2) == minf.MINF_ERR_INVALID
    assert _dense(ids=(ctypes.c_int32 * 1)(0), nh=0) == minf.MINF_ERR_INVALID


def test_estimate_argument_checks(minf_lib):
    L = minf.lib()
    vi = si = FAKE
    # last_q above 64, budgets below 1, block size other than 64
    assert L.minf_vs_estimate(FAKE, FAKE, 4, 2, 1024, 128, 65, 10, 10, 0.1, None, 4, vi, si, FAKE, 1 << 30,
                              None) == minf.MINF_ERR_UNSUPPORTED
    assert L.minf_vs_estimate(FAKE, FAKE, 4, 2, 1024, 128, 64, 0, 10, 0.1, None, 4, vi, si, FAKE, 1 << 30,
                              None) == minf.MINF_ERR_INVALID
    assert L.minf_block_estimate(FAKE, FAKE, 4, 2, 1024, 128, 32, 10, None, 4, FAKE, FAKE, FAKE, 1 << 30,
                                 None) == minf.MINF_ERR_UNSUPPORTED
    assert L.minf_block_estimate(FAKE, FAKE, 4, 2, 1024, 128, 64, 0, None, 4, FAKE, FAKE, FAKE, 1 << 30,
                                 None) == minf.MINF_ERR_INVALID
    assert L.minf_block_scores(FAKE, FAKE, 4, 2, 1024, 128, 32, None, 4, FAKE, FAKE, 1 << 30,
                               None) == minf.MINF_ERR_UNSUPPORTED
    assert L.minf_block_scores(FAKE, FAKE, 4, 2, 1024, 128, 64, None, 4, None, FAKE, 1 << 30,
                               None) == minf.MINF_ERR_INVALID
    assert L.minf_ashape_attention(FAKE, FAKE, FAKE, 4, 2, 1024, 128, 0.1, None, 4, -1, 10, FAKE, None, FAKE,
                                   256, None) == minf.MINF_ERR_INVALID
    codes = (ctypes.c_int8 * 4)(1, 2, 3, 7)
    assert L.minf_mixed_layer(FAKE, FAKE, FAKE, 4, 2, 1024, 128, 0.1, codes, 64, 10, 10, 4, 16, 64, FAKE, None,
                              FAKE, 1 << 30, None) == minf.MINF_ERR_INVALID
    assert "pattern" in minf.lib().minf_last_error().decode()
