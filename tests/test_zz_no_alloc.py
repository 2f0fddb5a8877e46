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


def _inputs(seed):
    w = synth.Workload("noalloc", "vs", 4, 2, 4096, "vertical", n_heavy=16)
    x = synth.generate(w, seed=seed)
    return x["q"].cuda(), x["k"].cuda()


def test_noalloc_estimate_matches_workspace_estimate():
    for seed in (0, 1):  # two calls in a row, the second on different inputs
        q, k = _inputs(seed)
        ref_v, ref_s = minf.minf_vs_estimate(q, k, 64, 256, 512, SCALE)
        got_v, got_s = minf.minf_vs_estimate_noalloc(q, k, 64, 256, 512, SCALE)
        torch.cuda.synchronize()
        assert torch.equal(got_v, ref_v), f"vertical indices differ (call {seed})"
        assert torch.equal(got_s, ref_s), f"slash indices differ (call {seed})"


def test_noalloc_estimate_rejects_oversized_requests():
    q, k = _inputs(0)
    # 16 heads x 256K tokens: the vertical and slash scores alone need 32 MiB + 1
    big = torch.empty(16, 1 << 18, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(minf.MinfError) as err:
        minf.minf_vs_estimate_noalloc(big, big[:4], 64, 256, 512, SCALE)
    assert err.value.code == minf.MINF_ERR_WORKSPACE
    # the library still works after the rejection
    v, s = minf.minf_vs_estimate_noalloc(q, k, 64, 256, 512, SCALE)
    torch.cuda.synchronize()
    assert int(v.min()) >= 0 and int(s.min()) >= 0
