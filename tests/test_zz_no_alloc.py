"""The allocation-free Vertical-Slash estimate against the workspace version.

Some callers cannot hand the library a workspace: code running inside a
runtime that owns every device allocation, or at a point where calling
cudaMalloc is not allowed.  minf_vs_estimate_noalloc serves them by taking its
scratch from an array built into the library.  Its index sets must equal those
of minf_vs_estimate on the same inputs -- integer outputs of the same kernels,
so equality is exact -- on consecutive calls that reuse the shared array.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import math

import pytest
import torch

from dynamic_sparse_attention_est_b200 import minf, synth

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
LIMIT = 32 << 20  # bytes of the built-in scratch array


def _inputs(seed, hq=4, hkv=2, n=4096, device="cpu"):
    w = synth.Workload("noalloc", "vs", hq, hkv, n, "vertical", n_heavy=16)
    x = synth.generate(w, seed=seed, device=device)
    return x["q"].cuda(), x["k"].cuda()


def test_noalloc_estimate_matches_workspace_estimate():
    for seed in (0, 1):  # two calls in a row, the second on different inputs
        q, k = _inputs(seed)
        ref_v, ref_s = minf.minf_vs_estimate(q, k, 64, 256, 512, SCALE)
        got_v, got_s = minf.minf_vs_estimate_noalloc(q, k, 64, 256, 512, SCALE)
        torch.cuda.synchronize()
        assert torch.equal(got_v, ref_v), f"vertical indices differ (call {seed})"
        assert torch.equal(got_s, ref_s), f"slash indices differ (call {seed})"
        assert minf.minf_vs_estimate_noalloc_status(q.device) == minf.MINF_OK


def _largest_n_that_fits(hq, hkv):
    """The longest sequence (a multiple of 64) whose estimate scratch fits the array."""
    need = lambda n: minf.workspace_bytes(minf.OP_VS_ESTIMATE, hq, hkv, n, hq)
    lo, hi = 64, 1 << 22
    assert need(lo) <= LIMIT < need(hi)
    while hi - lo > 64:
        mid = (lo + hi) // 2 // 64 * 64
        lo, hi = (mid, hi) if need(mid) <= LIMIT else (lo, mid)
    return lo


def test_noalloc_estimate_at_the_size_limit():
    """The largest request the array holds succeeds and matches the workspace version;
    64 more tokens are rejected."""
    hq, hkv = 16, 4
    n = _largest_n_that_fits(hq, hkv)
    assert minf.workspace_bytes(minf.OP_VS_ESTIMATE, hq, hkv, n + 64, hq) > LIMIT
    q, k = _inputs(5, hq, hkv, n, device="cuda")
    ref_v, ref_s = minf.minf_vs_estimate(q, k, 64, 1000, 2000, SCALE)
    got_v, got_s = minf.minf_vs_estimate_noalloc(q, k, 64, 1000, 2000, SCALE)
    torch.cuda.synchronize()
    assert minf.minf_vs_estimate_noalloc_status(q.device) == minf.MINF_OK
    assert torch.equal(got_v, ref_v) and torch.equal(got_s, ref_s)
    del q, k
    q, k = _inputs(6, hq, hkv, n + 64, device="cuda")
    with pytest.raises(minf.MinfError) as err:
        minf.minf_vs_estimate_noalloc(q, k, 64, 1000, 2000, SCALE)
    assert err.value.code == minf.MINF_ERR_WORKSPACE


def test_noalloc_estimate_rejects_oversized_requests():
    q, k = _inputs(0)
    # 16 heads x 256K tokens: the vertical and slash score rows alone fill the
    # 32 MiB (16 x 262144 x 4 B x 2); the status block and the other buffers
    # push the request past it
    big = torch.empty(16, 1 << 18, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(minf.MinfError) as err:
        minf.minf_vs_estimate_noalloc(big, big[:4], 64, 256, 512, SCALE)
    assert err.value.code == minf.MINF_ERR_WORKSPACE
    # the library still works after the rejection
    v, s = minf.minf_vs_estimate_noalloc(q, k, 64, 256, 512, SCALE)
    torch.cuda.synchronize()
    assert int(v.min()) >= 0 and int(s.min()) >= 0


def test_noalloc_status_reports_a_timeout():
    """A bounded wait that runs out in the built-in array's status block is reported
    once by the status call, then cleared; the next estimate reports OK."""
    dev = torch.device("cuda", torch.cuda.current_device())
    minf.minf_vs_estimate_noalloc_check_timeout(2_000_000, dev)  # 2 ms
    assert minf.minf_vs_estimate_noalloc_status(dev) == minf.MINF_ERR_TIMEOUT
    assert minf.minf_vs_estimate_noalloc_status(dev) == minf.MINF_OK
    q, k = _inputs(2)
    ref_v, ref_s = minf.minf_vs_estimate(q, k, 64, 256, 512, SCALE)
    got_v, got_s = minf.minf_vs_estimate_noalloc(q, k, 64, 256, 512, SCALE)
    assert minf.minf_vs_estimate_noalloc_status(dev) == minf.MINF_OK
    assert torch.equal(got_v, ref_v) and torch.equal(got_s, ref_s)
