"""bench.py's host-side helpers on the CPU (argument parsing, work and byte counts).

The timed path needs a GPU; these catch slips in the code around it that would
otherwise only show on a GPU machine.
"""
import math
import sys

import pytest

import bench
from dynamic_sparse_attention_est_b200 import synth


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_estimate_bytes_per_workload(name):
    w = synth.WORKLOADS[name]
    b = bench.estimate_bytes(w)
    if w.pattern in ("vs", "block"):
        assert b > w.hkv * w.n * 256  # at least one read of K
    else:
        assert b == 0.0


def test_parse_defaults_and_options(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse()
    assert (a.gpus, a.workload, a.impl, a.vs_mode, a.shard, a.topp) == (1, "mixed-gqa-1m", "minf", "exact", "layers", None)
    assert a.steps == 5 and a.cpu_mode == "auto"
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "vs-gqa-32k"])
    assert bench.parse().steps == 20
    monkeypatch.setattr(sys, "argv", ["bench.py", "--vs-mode", "tiles", "--topp", "0.9", "--shard", "heads"])
    a = bench.parse()
    assert (a.vs_mode, a.topp, a.shard) == ("tiles", 0.9, "heads")


def test_traffic_only_for_the_captured_source():
    assert bench.kernel_traffic("attn_kernel<VS>", None) is None
    assert bench.kernel_traffic("attn_kernel<VS>", "no-such-workload") is None
    assert bench.kernel_traffic("vs_diag_kernel", "mixed-gqa-1m") is None  # not captured there
    for kernel, workload in (("attn_kernel<VS>", "vs-gqa-32k"), ("vs_diag_kernel", "vs-1h-1m")):
        v = bench.kernel_traffic(kernel, workload)
        assert v is None or v > 0  # None once the kernel's source differs from the captured one



def test_tile_flops():
    assert bench.TILE_FLOPS == 4 * 128 ** 3 and math.isclose(bench.TILE_FLOPS / 1e6, 8.388608)


def test_clock_lines_parse():
    lines = ["1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "1830, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "garbage"]
    r = bench.ClockSampler.parse(lines)
    assert r == {"sm_mhz": 1897.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert bench.ClockSampler.parse([])["samples"] == 0


def test_bf16_peak_choice():
    peaks = {"bf16_tflops": 1661.7, "bf16_tflops_sustained": 1406.6, "sm_max_mhz": 1965.0,
             "clocks_under_load": {"sm_mhz_median": 1350.0}}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    capped = {"sm_mhz": 1387.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.pick_bf16_peak(peaks, 200.0, full) == (1661.7, "bf16_tflops")
    assert bench.pick_bf16_peak(peaks, 9000.0, capped) == (1406.6, "bf16_tflops_sustained")
    # no clock record: the duration and the throttle reasons decide
    assert bench.pick_bf16_peak(peaks, 200.0, {"sm_mhz": None, "reasons": []}) == (1661.7, "bf16_tflops")
    assert bench.pick_bf16_peak(peaks, 200.0, {"sm_mhz": None, "reasons": ["sw_power_cap"]})[1] == "bf16_tflops_sustained"
    assert bench.pick_bf16_peak(peaks, 9000.0, None)[1] == "bf16_tflops_sustained"
    assert bench.pick_bf16_peak({"bf16_tflops": 1590.0}, 9000.0, capped) == (1590.0, "bf16_tflops")


def test_cpu_sample_projects_every_pattern_of_a_mixed_layer(orc):
    """The bounded CPU sample of a mixed layer times each pattern present and says it
    is a projection; at a small size the full layer is timed instead."""
    import dataclasses

    w = dataclasses.replace(synth.WORKLOADS["mixed-gqa-1m"], n=4096, hq=8, hkv=2, n_vertical=64, n_slash=128,
                            topk=8, window=512)
    pats = synth.mixed_head_patterns(w, seed=0)
    x = synth.generate(w, seed=0, device="cpu", hq=1, hkv=1)
    r = bench.cpu_sample(w, x, orc, 0.5, pats=pats)
    assert r["projected"] and r["value"] > 0 and r["cores"] >= 1
    for p in set(pats):
        assert f"{p} x{pats.count(p)}" in r["sample"]
    wv = dataclasses.replace(synth.WORKLOADS["vs-gqa-32k"], n=1024, hq=2, hkv=1, n_vertical=32, n_slash=64)
    xf = synth.generate(wv, seed=1, device="cpu")
    rf = bench.cpu_sample(wv, xf, orc, 0.5, full=True)
    assert not rf["projected"] and rf["value"] > 0 and "timed" in rf["sample"]
