"""Benchmark: dynamic sparse prefill attention (estimate + attention) per layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl minf|reference]

A step is one pass of the whole path over one layer of synthetic input:
  vs-gqa-32k       minf_vs_estimate + minf_vs_attention (32 q-heads / 8 kv-heads, 32K tokens)
  block-gqa-128k   minf_block_estimate + minf_block_attention (128K tokens)
  ashape-gqa-128k  minf_ashape_attention (128K tokens)
  trishape-gqa-128k minf_trishape_attention (A-shape + dense last 64 rows, 128K tokens)
  mixed-gqa-1m     minf_mixed_layer, per-head patterns drawn from the seed (1M tokens)
The default is mixed-gqa-1m, the layer the 1M-token targets are stated on.
Inputs stay resident in HBM and are larger than L2,
so no flush is needed between steps.  The line also carries the roofline of the
attention kernel (computed-tile FLOPs / its CUDA-event time), the same metric
end to end from pinned host buffers, the dense causal kernel on the same
inputs, and the fp64 CPU oracle timed on a bounded sample.

With --gpus N (under torchrun), every rank runs its own layer (weak scaling,
no collective on the data path); value = max-over-ranks time / layers run.
``--impl reference`` times the fp64 oracle (the reference arm) on the host.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse prefill attention ms/layer"
_T0 = time.time()


def log(msg: str) -> None:
    """Progress on stderr (the JSON line alone goes to stdout)."""
    print(f"[bench {time.time() - _T0:7.1f}s] {msg}", file=sys.stderr, flush=True)
UNIT = "ms/layer"
TILE_FLOPS = 4 * 128 * 128 * 128  # QK^T and PV of one 128x128 tile, d = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 20; 5 at 1M tokens)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="mixed-gqa-1m")
    ap.add_argument("--impl", default="minf", choices=["minf", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--shard", default="layers", choices=["layers", "heads"],
                    help="N > 1: one layer per rank (weak scaling), or the heads of one layer split over the "
                         "ranks in whole GQA groups with an all-gather of the output (strong scaling)")
    ap.add_argument("--topp", type=float, default=None,
                    help="Vertical-Slash top-p budgets (p for verticals and slashes; the budgets become caps)")
    ap.add_argument("--vs-mode", default="exact", choices=["exact", "tiles"],
                    help="Vertical-Slash key set: token-exact, or every computed slash range attended whole")
    ap.add_argument("--vs-diag-ratio", type=float, default=None,
                    help="Vertical-Slash routing: slash groups of m offsets over H half-tiles run on the CUDA "
                         "cores when m < ratio * H (0: tensor cores only; default: the library's)")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-kernel comparison")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle attention rows to sample")
    ap.add_argument("--cpu-mode", default="auto", choices=["auto", "full", "sample"],
                    help="CPU baseline: the whole layer (auto up to 32K tokens) or a bounded sample, projected")
    a = ap.parse_args()
    if a.steps is None:
        from dynamic_sparse_attention_est_b200 import synth

        a.steps = 5 if synth.WORKLOADS[a.workload].n > 131072 else 20
    return a


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a
# kernel on a workload, from the ncu captures summarised in profiles/ (taken on
# that workload's own bench command), valid only for the source it was taken
# on (sha1 of the kernel's file).
TRAFFIC = {
    ("attn_kernel<VS>", "vs-gqa-32k"): ("attention.cu", "3f22d096b5042b08e8f74f0b3b6f3dc29b4de356",
                                        3.393959e9 + 0.241058e9),
    ("vs_diag_kernel", "vs-1h-1m"): ("diag.cu", "1c46171e2aa10929f6a120b36237fe141ac0255b",
                                     197.478696e9 + 0.548004e9),
}


def kernel_traffic(kernel: str, workload: str):
    import hashlib

    entry = TRAFFIC.get((kernel, workload)) if workload else None
    if entry is None:
        return None
    src = os.path.join(ROOT, "dynamic_sparse_attention_est_b200", "csrc", entry[0])
    with open(src, "rb") as f:
        sha = hashlib.sha1(f.read()).hexdigest()
    return entry[2] if sha == entry[1] else None


def pick_bf16_peak(peaks, elapsed_ms, clk):
    """The bf16 denominator of the attention roofline and its key in the peaks file.

    The burst figure (cuBLAS timed alone at full clocks) fits a timed region
    whose median SM clock stayed near the maximum; the sustained figure (a
    seconds-long loop under the 1 kW cap, at the lower clock recorded with it)
    fits a region whose clock fell below the midpoint of the two.  Without a
    clock record, a region of a second or more, or one that saw sw_power_cap,
    takes the sustained figure."""
    clk = clk or {}
    mhz = clk.get("sm_mhz")
    low = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
    high = peaks.get("sm_max_mhz") or clk.get("sm_max_mhz")
    if mhz and low and high:
        sustained = mhz < 0.5 * (low + high)
    else:
        sustained = elapsed_ms >= 1000.0 or "sw_power_cap" in (clk.get("reasons") or [])
    key = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    return peaks.get(key), key


# Peak fp32 FMA rate of the CUDA cores, from the unit counts: 148 SMs x 4
# sub-partitions x 32 FMA lanes, 2 FLOP per FMA, at the SM clock.
def alu_peak_tflops(sm_mhz: float) -> float:
    return 148 * 4 * 32 * 2 * sm_mhz * 1e6 / 1e12


def kernel_rooflines(kernels, detail, peaks, src, peak, peak_key, elapsed, clk, traffic_key):
    """(roofline of the kernel with the largest share of the timed region, roofline of
    the attention tile kernel with the largest share) from the live per-kernel times.

    attn_kernel<P>: computed-tile FLOPs (4 x 128^3 per 128x128 tile, tiles of that
    kernel from the counters) per launch over its average launch time, against the
    bf16 tensor peak.  vs_diag_kernel: useful FLOPs (2 x 128 multiply-adds per
    (query, key) pair, QK^T and PV) per launch over its launch time, against the
    fp32 FMA peak of the CUDA cores at the maximum SM clock."""
    pat_key = {"attn_kernel<DENSE>": "tiles_dense", "attn_kernel<VS>": "tiles_vs",
               "attn_kernel<BLOCK>": "tiles_block", "attn_kernel<ASHAPE>": "tiles_ashape"}

    def one(name):
        k = kernels[name]
        sec = k["ms_per_launch"] * 1e-3
        if name in pat_key:
            flops = detail.get(pat_key[name], 0) * TILE_FLOPS
            ach = flops / sec / 1e12
            return {"kernel": name, "bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                    "frac": round(ach / peak, 4), "flops_per_launch": flops,
                    "traffic": kernel_traffic(name, traffic_key),
                    "ms_per_launch": k["ms_per_launch"],
                    "peak_source": f"{src} {peak_key} (timed region {elapsed:.0f} ms, median SM clock "
                                   f"{clk.get('sm_mhz')} MHz)"}
        if name == "vs_diag_kernel":
            flops = 4 * 128 * detail.get("diag_pairs", 0)
            ach = flops / sec / 1e12
            pk = alu_peak_tflops(peaks.get("sm_max_mhz") or 1965.0)
            return {"kernel": name, "bound": "alu", "achieved": round(ach, 2), "peak": round(pk, 1),
                    "unit": "TFLOP/s", "frac": round(ach / pk, 4), "flops_per_launch": flops,
                    "traffic": kernel_traffic(name, traffic_key),
                    "ms_per_launch": k["ms_per_launch"],
                    "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 FLOP x max SM clock"}
        return {"kernel": name, "bound": None, "achieved": None, "peak": None, "unit": None, "frac": None,
                "traffic": None, "ms_per_launch": k["ms_per_launch"]}

    if not kernels:
        return None, None
    top = max(kernels, key=lambda n: kernels[n]["ms_total"])
    attn = [n for n in kernels if n in pat_key]
    top_attn = max(attn, key=lambda n: kernels[n]["ms_total"]) if attn else None
    return one(top), (one(top_attn) if top_attn else None)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region.

    start() launches the sampler and waits for its first line, so that a slow
    first NVML start does not leave the timed region without samples; mark()
    and stop() bracket the timed region, and only samples that arrive between
    them are kept (if the region is shorter than one interval, the first sample
    after it stands in, and `samples` says how many were used)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []  # (arrival time, text)
        self.t_mark = None

    def start(self, wait_s: float = 10.0):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.INTERVAL_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
            return
        t0 = time.monotonic()
        while not self.lines and time.monotonic() - t0 < wait_s and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self):
        self.t_mark = time.monotonic()

    @staticmethod
    def parse(lines):
        """Median SM clock, max clock and the active throttle reasons of the sample lines."""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        t_end = time.monotonic()
        # one more interval, so that a region shorter than the interval still gets the next sample
        time.sleep(2 * self.INTERVAL_MS / 1000)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0 = self.t_mark if self.t_mark is not None else 0.0
        inside = [ln for t, ln in self.lines if t0 <= t <= t_end]
        if not inside:
            inside = [ln for t, ln in self.lines if t > t_end][:1]
        return self.parse(inside)


# ----------------------------------------------------------------------------- workload
def make_step(w, x, torch, minf, synth, seed, vs_mode="exact", topp=None, pats=None):
    """Returns (step(ws) -> out, attention-only call for timing, label of the attention call)."""
    q, k, v = x["q"], x["k"], x["v"]
    hq, hkv, n = w.hq, w.hkv, w.n
    dev = q.device
    scale = 1.0 / math.sqrt(128)
    if w.pattern == "vs":
        ws_est = minf.workspace(minf.workspace_bytes(minf.OP_VS_ESTIMATE, hq, hkv, n, hq), dev)
        ws = minf.workspace(minf.workspace_bytes(minf.OP_VS_ATTENTION, hq, hkv, n, hq, w.n_vertical, w.n_slash),
                            dev)
        out = torch.empty_like(q)
        state = {}

        def estimate():
            if topp is None:
                state["idx"] = minf.minf_vs_estimate(q, k, w.last_q, w.n_vertical, w.n_slash, scale, ws=ws_est)
            else:
                vi, si, _, _ = minf.minf_vs_estimate_topp(q, k, w.last_q, w.n_vertical, w.n_slash, topp, topp,
                                                          scale, ws=ws_est)
                state["idx"] = (vi, si)

        vs_attention = minf.minf_vs_attention_tiles if vs_mode == "tiles" else minf.minf_vs_attention

        def attend():
            vi, si = state["idx"]
            vs_attention(q, k, v, vi, si, scale, out=out, want_lse=False, ws=ws)

        # launches: 4 estimate kernels, top-k of both row sets (one kernel up to 48K keys,
        # else 12 per row set), top-p counts (one kernel up to 48K keys, else 11 per row set)
        topk_launches = 1 if n <= 48 * 1024 else 24
        topp_launches = (1 if n <= 48 * 1024 else 22) if topp is not None else 0
        return estimate, attend, ws, out, 4 + topk_launches + topp_launches, 4
    if w.pattern == "block":
        ws_est = minf.workspace(minf.workspace_bytes(minf.OP_BLOCK_ESTIMATE, hq, hkv, n, hq, w.topk), dev)
        ws = minf.workspace(minf.workspace_bytes(minf.OP_BLOCK_ATTENTION, hq, hkv, n, hq, w.topk), dev)
        out = torch.empty_like(q)
        state = {}

        def estimate():
            state["idx"] = minf.minf_block_estimate(q, k, w.topk, ws=ws_est)

        def attend():
            bi, bc = state["idx"]
            minf.minf_block_attention(q, k, v, bi, bc, scale, out=out, want_lse=False, ws=ws)

        nbatch = math.ceil(hq / max(1, min(hq, (1 << 30) // ((n // 64) ** 2 * 4))))
        return estimate, attend, ws, out, 2 + 2 * nbatch, 2
    if w.pattern == "ashape":
        ws = minf.workspace(256, dev)
        out = torch.empty_like(q)

        def attend():
            minf.minf_ashape_attention(q, k, v, w.n_sink, w.window, scale, out=out, want_lse=False, ws=ws)

        return (lambda: None), attend, ws, out, 0, 1
    if w.pattern == "trishape":
        ws = minf.workspace(256, dev)
        out = torch.empty_like(q)

        def attend():
            minf.minf_trishape_attention(q, k, v, w.n_sink, w.window, w.last_q, scale, out=out, want_lse=False,
                                         ws=ws)

        return (lambda: None), attend, ws, out, 0, 1
    if w.pattern == "mixed":
        pats = pats if pats is not None else synth.mixed_head_patterns(w, seed)
        ws = minf.workspace(minf.workspace_bytes(minf.OP_MIXED_LAYER, hq, hkv, n, hq, w.n_vertical, w.n_slash,
                                                 w.topk), dev)
        out = torch.empty_like(q)

        def attend():
            minf.minf_mixed_layer(q, k, v, pats, w.last_q, w.n_vertical, w.n_slash, w.topk, w.n_sink, w.window,
                                  scale, out=out, want_lse=False, ws=ws)

        # launches per layer, by the pattern groups present
        n_vs, n_bs = pats.count("vs"), pats.count("block")
        topk_launches = 1 if n <= 48 * 1024 else 24
        per_batch = max(1, min(n_bs, (1 << 30) // ((n // 64) ** 2 * 4))) if n_bs else 1
        launches = (4 + topk_launches + 4) if n_vs else 0                            # estimate, top-k, plan, attention
        launches += (2 + 2 * math.ceil(n_bs / per_batch) + 2) if n_bs else 0        # pool, scores + top-k, plan, attention
        launches += sum(1 for p in ("ashape", "trishape", "dense") if p in pats)
        return (lambda: None), attend, ws, out, 0, launches
    raise ValueError(w.pattern)


def estimate_bytes(w) -> float:
    """Algorithmic HBM bytes of one layer's index estimation (+ top-k), by pattern.

    Vertical-Slash: both passes stream K once per pair of q-heads sharing a
    kv-head (256 B per key), the vertical and slash score rows are written once
    and read by five radix passes, the 191-offset diagonal partials are written
    and read once.  Block-Sparse: Q and K are read once for pooling, the pooled
    rows written as three bf16 parts (768 B per block), and the lower triangle
    of pooled scores written once and read once by the per-row selection.
    """
    n, hq, hkv = w.n, w.hq, w.hkv
    if w.pattern == "vs":
        pairs = hkv * math.ceil((hq // hkv) / 2)
        k_stream = 2 * pairs * n * 256
        scores = 2 * hq * n * 4 * (1 + 5)
        diag = 2 * hq * math.ceil(n / 128) * 191 * 4
        return float(k_stream + scores + diag + hq * 64 * 256)
    if w.pattern == "block":
        nb = n // 64
        pool = (hq + hkv) * n * 256 + (hq + hkv) * nb * 768
        tri = hq * nb * (nb + 1) / 2 * 4
        return float(pool + 2 * tri)
    return 0.0


def _time_rows(w, pattern, orc, q1, k1, v1, scale, idx, budget_s, vs_mode):
    """Seconds per attention row of one head, over rows spread across the sequence,
    grown until about half of `budget_s` is spent (the oracle spreads rows over
    its threads, so a layer's rows scale linearly)."""
    import numpy as np

    n = w.n
    nrows, spent = 64, 0.0
    while True:
        rows = np.linspace(0, n - 1, nrows).astype(np.int32)
        t1 = time.perf_counter()
        if pattern == "vs" and vs_mode == "tiles":
            orc.vs_tiles_attention(q1, k1, v1, scale, idx[0], idx[1], 128, rows=rows)
        elif pattern == "vs":
            orc.vs_attention(q1, k1, v1, scale, idx[0], idx[1], rows=rows)
        elif pattern == "block":
            orc.block_attention(q1, k1, v1, scale, 64, idx[0], idx[1], rows=rows)
        elif pattern == "trishape":
            orc.trishape_attention(q1, k1, v1, scale, w.n_sink, w.window, w.last_q, rows=rows)
        elif pattern == "ashape":
            orc.ashape_attention(q1, k1, v1, scale, w.n_sink, w.window, rows=rows)
        else:
            orc.dense_attention(q1, k1, v1, scale, rows=rows)
        dt = time.perf_counter() - t1
        spent += dt
        if spent > budget_s * 0.5 or nrows >= n:
            return dt / nrows, nrows
        nrows = min(n, int(nrows * max(2.0, (budget_s * 0.5) / max(dt, 1e-3))))


def cpu_estimates(w, pattern, orc, q1, k1, scale):
    """One head's index estimate for `pattern`: (seconds, indices for the row timing, note).

    Block-Sparse estimates beyond 4,096 blocks (their pooled-score triangle grows
    with the square of the block count) are timed on the first 2,048 blocks and
    scaled by (blocks / 2,048)^2; the row timing then uses the first topk blocks
    of each row, which has the same number of keys as any top-k list."""
    import numpy as np

    t0 = time.perf_counter()
    if pattern == "vs":
        vi, si = orc.vs_estimate(q1, k1, w.last_q, w.n_vertical, w.n_slash, scale)
        return time.perf_counter() - t0, (vi, si), "estimate of 1 head timed"
    if pattern == "block":
        nb = w.n // 64
        if nb <= 4096:
            bi, bc = orc.block_estimate(q1, k1, 64, w.topk)
            return time.perf_counter() - t0, (bi, bc), "estimate of 1 head timed"
        m = 2048 * 64
        orc.block_estimate(q1[:, :m], k1[:, :m], 64, w.topk)
        dt = (time.perf_counter() - t0) * (nb / 2048) ** 2
        bi = np.tile(np.arange(w.topk, dtype=np.int32), (1, nb, 1))
        bc = np.full((1, nb), w.topk, np.int32)
        return dt, (bi, bc), f"estimate of 1 head timed on 2,048 blocks, scaled by ({nb}/2048)^2"
    return 0.0, None, ""


def cpu_sample(w, x, orc, budget_s, vs_mode="exact", pats=None, full=False, cache=None):
    """The fp64 oracle on the host cores, as the CPU baseline of one layer.

    full: every head's estimate and every row's attention are run (feasible up
    to 32K tokens); x then holds the whole layer.  Otherwise x holds one q-head
    and its kv-head, and the layer is projected from a bounded sample, per
    pattern present: one head's estimate (the oracle runs one head per thread,
    so the layer's estimates of c heads take ceil(c / threads) of it) plus
    attention rows spread over the sequence, scaled to c x n rows.  `cache`
    keeps the estimates between calls (the reference arm re-times rows only).
    """
    import numpy as np

    scale = 1.0 / math.sqrt(128)
    threads = orc.threads()
    t_start = time.perf_counter()
    if full:
        q, k, v = (x[key].float().cpu().numpy() for key in ("q", "k", "v"))
        t0 = time.perf_counter()
        if w.pattern == "vs":
            vi, si = orc.vs_estimate(q, k, w.last_q, w.n_vertical, w.n_slash, scale)
            est = time.perf_counter() - t0
            if vs_mode == "tiles":
                orc.vs_tiles_attention(q, k, v, scale, vi, si, 128)
            else:
                orc.vs_attention(q, k, v, scale, vi, si)
        elif w.pattern == "block":
            bi, bc = orc.block_estimate(q, k, 64, w.topk)
            est = time.perf_counter() - t0
            orc.block_attention(q, k, v, scale, 64, bi, bc)
        else:
            raise ValueError("full CPU timing covers the Vertical-Slash and Block-Sparse layers")
        total = time.perf_counter() - t0
        return {"value": total * 1000.0, "unit": UNIT, "cores": threads, "kind": "oracle", "projected": False,
                "sample": f"whole layer ({w.hq} heads x {w.n} rows): estimate {est:.2f} s + attention "
                          f"{total - est:.2f} s, timed", "seconds": round(time.perf_counter() - t_start, 2)}
    q1, k1, v1 = (x[key][0:1].float().cpu().numpy() for key in ("q", "k", "v"))
    counts = {}
    for p in (pats if pats is not None else [w.pattern] * w.hq):
        counts[p] = counts.get(p, 0) + 1
    cache = {} if cache is None else cache
    layer_s, notes = 0.0, []
    share = budget_s / max(1, len(counts))
    for p, c in sorted(counts.items()):
        if p not in cache:
            cache[p] = cpu_estimates(w, p, orc, q1, k1, scale)
        est_s, idx, note = cache[p]
        t_row, nrows = _time_rows(w, p, orc, q1, k1, v1, scale, idx, share, vs_mode)
        layer_s += math.ceil(c / threads) * est_s + c * w.n * t_row
        notes.append(f"{p} x{c}: " + (f"{note} ({est_s:.2f} s), x ceil({c}/{threads}); " if note else "") +
                     f"attention of {nrows} rows of 1 head ({t_row * 1e3:.3f} ms/row), x {c} x {w.n} rows")
    return {"value": layer_s * 1000.0, "unit": UNIT, "cores": threads, "kind": "oracle", "projected": True,
            "sample": "projected from a sample -- " + "; ".join(notes),
            "seconds": round(time.perf_counter() - t_start, 2)}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from dynamic_sparse_attention_est_b200 import synth

    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle
        import torch

        orc = oracle.get()
        pats = synth.mixed_head_patterns(w, args.seed) if w.pattern == "mixed" else None
        full = args.cpu_mode == "full" or (args.cpu_mode == "auto" and w.n <= 32768 and w.pattern in ("vs", "block"))
        # a sample needs q-head 0 and its kv-head only; the full layer needs every head
        x = synth.generate(w, seed=args.seed, device="cpu") if full else \
            synth.generate(w, seed=args.seed, device="cpu", hq=1, hkv=1)
        per = max(2.0, 60.0 / max(1, args.steps + args.warmup))
        vals, step_s, cache = [], [], {}
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            r = cpu_sample(w, x, orc, per, args.vs_mode, pats, full, cache)
            if i >= args.warmup:
                vals.append(r["value"])
                step_s.append(time.perf_counter() - t0)
        val = statistics.median(vals)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                # wall time of one step of this arm: the timed sample (or the whole layer when not projected)
                "ms_per_step": round(1000.0 * statistics.mean(step_s), 1), "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "projected": r["projected"],
                "config": {"workload": w.name, "hq": w.hq, "hkv": w.hkv, "n": w.n,
                           **({"vs_mode": args.vs_mode} if w.pattern == "vs" else {})},
                "cpu_baseline": {"value": val, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                                 "projected": r["projected"], "sample": r["sample"]},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist

    from dynamic_sparse_attention_est_b200 import minf

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.vs_diag_ratio is not None:
        minf.minf_set_vs_diag_ratio(args.vs_diag_ratio)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    from dynamic_sparse_attention_est_b200 import shard

    sharded = args.shard == "heads" and world > 1
    parts, pats_local, w_run = None, None, w
    if sharded:
        # one layer, the same on every rank; this rank runs its whole GQA groups as a smaller layer
        import dataclasses

        if world > w.hkv:
            raise SystemExit(f"--shard heads needs at most {w.hkv} ranks (one kv-head each)")
        seed = args.seed
        pats_all = synth.mixed_head_patterns(w, seed) if w.pattern == "mixed" else [w.pattern] * w.hq
        parts = shard.partition_heads(pats_all, w.hkv, world, w.n, n_vertical=w.n_vertical, n_slash=w.n_slash,
                                      topk=w.topk, n_sink=w.n_sink, window=w.window, n_last=w.last_q)
        mine = parts[rank]
        grp = w.hq // w.hkv
        kvs = sorted({h // grp for h in mine})
        log(f"generating {w.name} on {dev}; this rank: q-heads {mine}")
        xf = synth.generate(w, seed=seed, device=dev)
        x = {"q": xf["q"][mine].contiguous(), "k": xf["k"][kvs].contiguous(), "v": xf["v"][kvs].contiguous()}
        del xf
        w_run = dataclasses.replace(w, hq=len(mine), hkv=len(kvs))
        pats_local = [pats_all[h] for h in mine] if w.pattern == "mixed" else None
        args.no_dense = True
    else:
        seed = shard.rank_seed(args.seed, rank)
        log(f"generating {w.name} on {dev}")
        x = synth.generate(w, seed=seed, device=dev)
    torch.cuda.synchronize()
    log("inputs ready")
    estimate, attend_local, ws, out, n_est_k, n_att_k = make_step(w_run, x, torch, minf, synth, seed, args.vs_mode,
                                                                  args.topp, pats_local)
    stream = torch.cuda.current_stream(dev)

    if sharded:
        def attend():
            attend_local()
            shard.gather_heads(out, parts, w.hq)  # the whole layer's output on every rank
    else:
        attend = attend_local

    for i in range(max(3, args.warmup)):
        estimate()
        torch.cuda.synchronize()
        log(f"warm-up {i}: estimate done")
        attend()
        torch.cuda.synchronize()
        log(f"warm-up {i}: attention done")
    tiles, pairs = minf.minf_stats(ws)
    detail = minf.minf_stats_detail(ws)
    if minf.minf_status(ws) != minf.MINF_OK:
        raise RuntimeError("device status not OK after warm-up")
    minf.minf_profile_read()  # drop anything recorded before the timed region

    # ---- timed region: K steps, events around the whole and around each attention call
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    clocks.mark()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    minf.minf_profile_enable(True)  # an event pair around each of the library's launches, on its stream
    t_start.record(stream)
    for i in range(args.steps):
        estimate()
        ev[i][0].record(stream)
        attend()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    minf.minf_profile_enable(False)
    kernel_ms = minf.minf_profile_read()
    clk = clocks.stop()
    elapsed = t_start.elapsed_time(t_end)
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    if world > 1:
        elapsed = shard.max_over_ranks(elapsed, device=dev)
        dist.barrier()
    layers_per_step = 1 if sharded else world  # whole-job layers finished per step
    ms_per_layer = elapsed / (args.steps * layers_per_step)
    ms_per_step = elapsed / args.steps

    log(f"timed region done: {ms_per_layer:.3f} ms/layer")
    # ---- end to end through the public API from pinned host buffers.  Every step
    # copies its inputs host -> device and its output device -> host; three streams
    # and two device buffer sets let step s+1's upload and step s-1's download
    # overlap step s's compute (the timing is device events on the upload stream).
    e2e = None
    if rank == 0 or world > 1:
        host_in = {key: x[key].cpu().pin_memory() for key in ("q", "k", "v")}
        x2 = {key: torch.empty_like(x[key]) for key in ("q", "k", "v")}
        sets = [(x, estimate, attend, out)]
        e2, a2, _, o2, _, _ = make_step(w_run, x2, torch, minf, synth, seed, args.vs_mode, args.topp, pats_local)
        sets.append((x2, e2, a2, o2))
        host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        up_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        e2e_steps = max(3, min(args.steps, 20 if w.n <= 131072 else 3))
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s_up)
        for i in range(e2e_steps):
            bi = i % 2
            xb, est_b, att_b, out_b = sets[bi]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(comp_done[bi])  # step i-2 no longer reads these inputs
                for key in ("q", "k", "v"):
                    xb[key].copy_(host_in[key], non_blocking=True)
                up_done[bi].record(s_up)
            stream.wait_event(up_done[bi])
            if i >= 2:
                stream.wait_event(down_done[bi])  # step i-2's output has been read back
            est_b()
            att_b()
            comp_done[bi].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[bi])
                host_out[bi].copy_(out_b, non_blocking=True)
                down_done[bi].record(s_down)
        s_up.wait_event(down_done[(e2e_steps - 1) % 2])
        s_up.wait_event(down_done[(e2e_steps - 2) % 2])
        b.record(s_up)
        torch.cuda.synchronize()
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            e2e_ms = shard.max_over_ranks(e2e_ms, device=dev)
        # whole-job figure, like `value`: every rank ran e2e_steps layers
        e2e = {"value": e2e_ms / (e2e_steps * layers_per_step), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": host_out[0].numel() * host_out[0].element_size(),
               "steps": e2e_steps, "overlap": "upload, compute and download on separate streams"}
        del sets, x2

    log("end-to-end timing done")
    # ---- dense kernel on the same inputs (context for the sparse speedup)
    dense = None
    if not args.no_dense:
        # at 1M tokens a dense layer takes seconds: time a few heads and scale by the head count
        heads = None if w.n <= 131072 else list(range(min(4, w.hq)))
        nh = w.hq if heads is None else len(heads)
        wsd = minf.workspace(256, dev)
        outd = torch.empty((nh,) + tuple(x["q"].shape[1:]), dtype=x["q"].dtype, device=dev)
        minf.minf_dense_attention(x["q"], x["k"], x["v"], head_ids=heads, out=outd, want_lse=False, ws=wsd)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        reps = 3 if heads is None else 1
        a.record(stream)
        for _ in range(reps):
            minf.minf_dense_attention(x["q"], x["k"], x["v"], head_ids=heads, out=outd, want_lse=False, ws=wsd)
        b.record(stream)
        torch.cuda.synchronize()
        dtiles, _ = minf.minf_stats(wsd)
        dms_timed = a.elapsed_time(b) / reps
        dms = dms_timed * w.hq / nh
        dense = {"ms_per_layer": dms, "tflops_computed": dtiles * TILE_FLOPS / (dms_timed * 1e-3) / 1e12,
                 "sparse_speedup": dms / ms_per_layer * world, "heads_timed": nh,
                 "scaled_from_heads": heads is not None}
        del outd

    peaks, src = measured_peaks()
    peak, peak_key = pick_bf16_peak(peaks, elapsed, clk)
    kernels = {name: {"launches": c, "ms_total": round(ms, 3), "ms_per_launch": round(ms / max(c, 1), 4),
                      "share": round(ms / elapsed, 4)} for name, (c, ms) in kernel_ms.items()}
    roofline, tensor_roofline = kernel_rooflines(kernels, detail, peaks, src, peak, peak_key, elapsed, clk,
                                                 w.name if args.vs_mode == "exact" else None)

    log("dense comparison done")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle

        full = args.cpu_mode == "full" or (args.cpu_mode == "auto" and w.n <= 32768 and w.pattern in ("vs", "block"))
        pats = synth.mixed_head_patterns(w, seed) if w.pattern == "mixed" else None
        xs = x if full else {"q": x["q"][:1].cpu(), "k": x["k"][:1].cpu(), "v": x["v"][:1].cpu()}
        log("CPU baseline: " + ("whole layer" if full else "bounded sample"))
        cpu = cpu_sample(w, xs, oracle.get(), args.cpu_budget, args.vs_mode, pats, full)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(ms_per_layer, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": False,
            "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; RoPE'd N(0,1) with planted structure)",
            "config": {"workload": w.name, "pattern": w.pattern, "hq": w.hq, "hkv": w.hkv, "n": w.n,
                       "last_q": w.last_q, "n_vertical": w.n_vertical, "n_slash": w.n_slash, "topk": w.topk,
                       "n_sink": w.n_sink, "window": w.window,
                       **({"vs_mode": args.vs_mode} if w.pattern == "vs" else {}),
                       **({"budgets": f"top-p {args.topp} (n_vertical, n_slash as caps)"}
                          if w.pattern == "vs" and args.topp is not None else {}),
                       "l2": "inputs larger than L2 (no flush)",
                       "parallelism": (f"heads of one layer over {world} ranks in whole GQA groups, "
                                       f"output all-gathered (shards {[len(p) for p in parts]})") if sharded
                       else f"one layer per rank x{world}"},
            "roofline": roofline,
            "tensor_roofline": tensor_roofline,
            "kernels": kernels,
            "counters": detail,
            "attention_ms": round(attn_ms, 4),
            "estimate_ms": round(ms_per_step - attn_ms, 4),
            "estimate_roofline": ({"bound": "hbm", "bytes": estimate_bytes(w_run),
                                   "achieved": round(estimate_bytes(w_run) / ((ms_per_step - attn_ms) * 1e-3) / 1e9, 1),
                                   "peak": peaks.get("hbm_gbs"), "unit": "GB/s",
                                   "frac": round(estimate_bytes(w_run) / ((ms_per_step - attn_ms) * 1e-3) / 1e9
                                                 / peaks.get("hbm_gbs"), 4)}
                                  if w.pattern in ("vs", "block") and ms_per_step > attn_ms else None),
            "computed_tiles": tiles, "mask_pairs": pairs,
            "useful_tflops": round(4 * 128 * pairs / (attn_ms * 1e-3) / 1e12, 1),
            "dense": dense,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": (n_est_k + n_att_k) * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
