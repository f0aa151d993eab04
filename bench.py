"""Benchmark: one attention layer of the 3.8B-style model, prefill + batched decode.

One step = one pass of the whole hot path over one batch of synthetic input:
  prefill phase  (B=8, T=2048, Hq=24, Hkv=8, D=128, QK-RMSNorm, RoPE base 1e4)
      gqa_rope_append (q in place; rotated k and v into the cache) + gqa_prefill
  decode step    (B=64, Hq=24, Hkv=8, D=128, cached lengths U[256, 2048], QK-norm)
      gqa_rope_append (new token at position lens[b]) + gqa_decode over lens[b] + 1
value = tokens processed per second (8*2048 prompt + 64 generated tokens per step,
times the number of GPUs), timed on the device with CUDA events; the inputs of a
step (about 0.9 GB) exceed the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch under torch.distributed.run: every rank runs its own replica of
the workload (the path has no exchange step), the timed region is bracketed by
a barrier and a device synchronise, and the slowest rank's time is used.
"""
from __future__ import annotations

import argparse
import hashlib
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from rope_gqa_kv_b200 import inputs  # noqa: E402

METRIC = "GQA prefill TFLOP/s & KV-cache decode GB/s, tokens/s (frac of B200 peak)"
PREFILL = inputs.BY_NAME["prefill_3p8b"]
DECODE = inputs.BY_NAME["batched_decode"]
WORKLOAD = ("3.8B-style attention layer: prefill B=8 T=2048 Hq=24 Hkv=8 D=128 QK-norm, "
            "then one decode step B=64 Hq=24 Hkv=8 D=128 with cached lengths U[256,2048]")
# kernels of libgqa launched per step: rope/append + prefill, rope/append + decode split + merge
LAUNCHES_PER_STEP = 5
DATA = "synthetic (seeded N(0,1) bf16 tensors shaped like the pages' 3.8B model)"


def bench_config(world: int) -> dict:
    """The `config` object of both arms' lines."""
    return {"workload": WORKLOAD, "prefill_batch": PREFILL.B, "seq_len": PREFILL.T,
            "decode_batch": DECODE.B, "heads": "24q/8kv", "head_dim": 128,
            "l2": "inputs exceed L2 (~0.9 GB touched per step); no flush",
            "parallelism": "replicas" if world > 1 else "single"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# work accounting (algorithmic, not what the kernels happen to move)
# ---------------------------------------------------------------------------
def prefill_flops(w=PREFILL) -> float:
    """4*D flops per (query, visible key, query head): QK^T and PV, causal pairs only."""
    return 4.0 * w.D * (w.T * (w.T + 1) / 2) * w.B * w.Hq


def chunk_flops(pos0, w) -> float:
    """Causal FLOPs of a continuation chunk: 4*D per (query, visible key, query
    head), query t of sequence b seeing pos0[b] + t + 1 keys."""
    T = w.T
    per_b = [T * int(p) + T * (T + 1) / 2.0 for p in pos0]
    return 4.0 * w.D * w.Hq * sum(per_b)


def decode_bytes(lens_new, w=DECODE) -> float:
    """K and V of every visible slot, once per KV head, plus q in and o out."""
    kv = float(np.sum(lens_new)) * w.Hkv * w.D * 2 * 2
    return kv + 2 * w.B * w.Hq * w.D * 2


def append_bytes(w=PREFILL) -> float:
    """Prefill-sized rope+append: q read and written in place, k and v read and
    written into the cache, all bf16."""
    return 2.0 * w.B * w.T * (w.Hq + 2 * w.Hkv) * w.D * 2


def tokens_per_step() -> int:
    return PREFILL.B * PREFILL.T + DECODE.B


# ---------------------------------------------------------------------------
# peaks, clocks, profile summary
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed loops run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, util, reasons = [], [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                s, m, u = float(parts[1]), float(parts[2]), float(parts[4])
            except ValueError:
                continue
            sm.append(s)
            smax.append(m)
            util.append(u)
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s, u in zip(sm, util) if u > 0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def kernel_source_hash() -> str:
    """Hash of the prefill kernel's code (its sources with // comments and
    blank lines dropped, so that a comment edit keeps a profile valid)."""
    h = hashlib.sha256()
    for f in ("prefill.cu", "ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "rope_gqa_kv_b200", "csrc", f), encoding="utf-8") as fh:
            for ln in fh:
                code = ln.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per prefill launch from the committed ncu summary, if it still
    describes the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "prefill_3p8b_ncu.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for ln in f:
            if ":" in ln:
                k, v = ln.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Layer:
    """Device-resident buffers of one replica of the workload."""

    def __init__(self, dev):
        import rope_gqa_kv_b200 as gqa
        self.gqa = gqa
        gqa.load()
        self.dev = dev
        xp = inputs.make_inputs(PREFILL)
        xd = inputs.make_inputs(DECODE)
        self.host_p = {k: xp[k] for k in ("q", "k", "v")}
        q1, k1, v1 = xd["steps"][0]
        self.host_d = {"q": q1, "k": k1, "v": v1, "lens": xd["lens"]}
        d = lambda t: t.to(dev)  # noqa: E731
        self.pq, self.pk, self.pv = d(xp["q"]), d(xp["k"]), d(xp["v"])
        self.pkc, self.pvc = d(xp["k_cache"]), d(xp["v_cache"])
        self.pout = torch.empty_like(self.pq)
        self.dq, self.dk, self.dv = d(q1), d(k1), d(v1)
        self.dkc, self.dvc = d(xd["k_cache"]), d(xd["v_cache"])
        self.pos = d(xd["lens"])
        self.lens_new = torch.empty_like(self.pos)
        self.max_len = int(xd["lens"].max()) + 1
        self.dout = torch.empty_like(self.dq)
        self.ws = gqa.decode_workspace(DECODE.B, DECODE.Hq, DECODE.D, self.max_len, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.lens_new_host = (xd["lens"] + 1).numpy()
        # pinned host copies for the end-to-end leg
        self.pin = {k: v.pin_memory() for k, v in
                    (("pq", xp["q"]), ("pk", xp["k"]), ("pv", xp["v"]), ("dq", q1), ("dk", k1),
                     ("dv", v1), ("pos", xd["lens"]))}
        self.pin_out_p = torch.empty(self.pout.shape, dtype=torch.bfloat16).pin_memory()
        self.pin_out_d = torch.empty(self.dout.shape, dtype=torch.bfloat16).pin_memory()

    def io_set(self, other=False):
        """The step's inputs and outputs on the device: the layer's own tensors,
        or (other=True) a second set of the same shapes for the pipelined
        end-to-end leg."""
        names = ("pq", "pk", "pv", "dq", "dk", "dv", "pos", "pout", "dout")
        if not other:
            return {k: getattr(self, k) for k in names}
        return {k: torch.empty_like(getattr(self, k)) for k in names}

    def step(self, ev=None, io=None):
        """The device-resident step.  ev: optional list of 5 events recorded
        around the four phases (prefill append, prefill, decode append, decode);
        io: the input / output tensors (default: the layer's own)."""
        g = self.gqa
        x = io if io is not None else self.io_set()
        if ev is not None:
            ev[0].record()
        g.gqa_rope_append(x["pq"], x["pk"], x["pv"], self.pkc, self.pvc, qk_norm=True,
                          max_pos0=0, status=self.status)
        if ev is not None:
            ev[1].record()
        g.gqa_prefill(x["pq"], self.pkc, self.pvc, out=x["pout"], status=self.status)
        if ev is not None:
            ev[2].record()
        g.gqa_rope_append(x["dq"], x["dk"], x["dv"], self.dkc, self.dvc, pos0=x["pos"],
                          max_pos0=self.max_len - 1, new_len=self.lens_new, qk_norm=True,
                          status=self.status)
        if ev is not None:
            ev[3].record()
        g.gqa_decode(x["dq"], self.dkc, self.dvc, self.lens_new, self.max_len, out=x["dout"],
                     workspace=self.ws, status=self.status)
        if ev is not None:
            ev[4].record()

    def run_e2e(self, steps):
        """`steps` steps from pinned host buffers: every step copies its inputs
        host -> device and reads both outputs back device -> host.  Pipelined
        over two device input / output sets and three streams: the upload of
        step i + 1 and the download of step i - 1 run while step i computes
        (and the two copy directions share the PCIe link's two halves).  The
        kernels still run one step after another on the compute stream, which
        is the stream the returned events are recorded on."""
        if not hasattr(self, "_sets"):
            self._sets = [self.io_set(), self.io_set(other=True)]
            self._h2d = torch.cuda.Stream(device=self.dev)
            self._d2h = torch.cuda.Stream(device=self.dev)
        comp = torch.cuda.current_stream(self.dev)
        mk = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        ev_in, ev_comp, ev_out = [mk(), mk()], [mk(), mk()], [mk(), mk()]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(comp)
        self._h2d.wait_event(start)
        self._d2h.wait_event(start)
        for i in range(steps):
            s = i & 1
            io = self._sets[s]
            with torch.cuda.stream(self._h2d):
                if i >= 2:
                    self._h2d.wait_event(ev_comp[s])     # step i - 2 is done with set s
                for k in ("pq", "pk", "pv", "dq", "dk", "dv", "pos"):
                    io[k].copy_(self.pin[k], non_blocking=True)
                ev_in[s].record(self._h2d)
            comp.wait_event(ev_in[s])
            if i >= 2:
                comp.wait_event(ev_out[s])               # step i - 2's outputs are read
            self.step(io=io)
            ev_comp[s].record(comp)
            with torch.cuda.stream(self._d2h):
                self._d2h.wait_event(ev_comp[s])
                self.pin_out_p.copy_(io["pout"], non_blocking=True)
                self.pin_out_d.copy_(io["dout"], non_blocking=True)
                ev_out[s].record(self._d2h)
        for s in range(min(steps, 2)):
            comp.wait_event(ev_out[s])
        stop.record(comp)
        return start, stop

    def e2e_bytes(self):
        h2d = sum(t.numel() * t.element_size() for t in self.pin.values())
        d2h = self.pin_out_p.numel() * 2 + self.pin_out_d.numel() * 2
        return h2d, d2h


def _barrier_sync(dist_on):
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def _max_over_ranks(x: float, dist_on: bool, dev) -> float:
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_ours(args, rank, world, dev, dist_on):
    layer = Layer(dev)
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    # The warm-up steps run after the sampler's start-up pause, right before the
    # timed steps, so that those begin on a busy GPU rather than on clocks
    # ramping up from an idle wait.
    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()

    # -- device-resident timed region (per-kernel events on the launching stream) --
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    _barrier_sync(dist_on)
    start.record()
    for i in range(args.steps):
        layer.step(evs[i])
    stop.record()
    _barrier_sync(dist_on)
    ms_total = start.elapsed_time(stop)
    t_append_p = t_prefill = t_append_d = t_decode = 0.0
    for i in range(args.steps):
        e = evs[i]
        t_append_p += e[0].elapsed_time(e[1])
        t_prefill += e[1].elapsed_time(e[2])
        t_append_d += e[2].elapsed_time(e[3])
        t_decode += e[3].elapsed_time(e[4])
    ms_total = _max_over_ranks(ms_total, dist_on, dev)

    # -- end-to-end region: host buffers in, results out, every step --
    layer.run_e2e(min(args.warmup, 3))
    _barrier_sync(dist_on)
    s2, e2 = layer.run_e2e(args.steps)
    _barrier_sync(dist_on)
    ms_e2e = _max_over_ranks(s2.elapsed_time(e2), dist_on, dev)
    clocks = sampler.stop() if sampler else None
    status = int(layer.status.item())
    if rank != 0:
        return None

    K = args.steps
    ms_step = ms_total / K
    tok = tokens_per_step() * world
    pf_ms = t_prefill / K
    dec_ms = t_decode / K
    pf_tflops = prefill_flops() / (pf_ms * 1e-3) / 1e12
    dec_gbs = decode_bytes(layer.lens_new_host) / (dec_ms * 1e-3) / 1e9
    long_run = ms_total > 1000.0
    tpeak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    hpeak = peaks["hbm_gbs"]
    tag = "of " + peak_src
    traffic = profiled_traffic()
    h2d, d2h = layer.e2e_bytes()
    line = {
        "metric": METRIC,
        "value": round(tok / (ms_step * 1e-3), 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": DATA,
        "config": bench_config(world),
        "roofline": {"bound": "tensor", "kernel": "gqa_prefill",
                     "achieved": round(pf_tflops, 1), "peak": tpeak, "unit": "TFLOP/s",
                     "frac": round(pf_tflops / tpeak, 4),
                     "peak_kind": ("bf16 sustained " if long_run else "bf16 burst ") + tag,
                     "traffic": traffic,
                     "algorithmic_per_launch": prefill_flops()},
        "decode_roofline": {"bound": "hbm", "kernel": "gqa_decode",
                            "achieved": round(dec_gbs, 1), "peak": hpeak, "unit": "GB/s",
                            "frac": round(dec_gbs / hpeak, 4), "peak_kind": "hbm copy " + tag,
                            "algorithmic_per_launch": decode_bytes(layer.lens_new_host),
                            "us_per_launch": round(dec_ms * 1e3, 2)},
        "phases_ms": {"prefill_append": round(t_append_p / K, 4),
                      "prefill_kernel": round(pf_ms, 4),
                      "decode_append": round(t_append_d / K, 4),
                      "decode_kernels": round(dec_ms, 4)},
        "append_roofline": {"bound": "hbm", "kernel": "gqa_rope_append (prefill-sized)",
                            "achieved": round(append_bytes() / (t_append_p / K * 1e-3) / 1e9, 1),
                            "peak": hpeak, "unit": "GB/s",
                            "frac": round(append_bytes() / (t_append_p / K * 1e-3) / 1e9 / hpeak, 4),
                            "algorithmic_per_launch": append_bytes()},
        "e2e": {"value": round(tok / (ms_e2e / K * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e / K, 4),
                "pipelined": "two device input/output sets; step i+1's upload and step "
                             "i-1's download overlap step i's kernels"},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks,
        "device_status": status,
    }
    line["next_rows"] = {"chunked_prefill": with_clocks(measure_chunk, dev, peaks, tag),
                         "rope_scaling": with_clocks(measure_scaled_append, layer, peaks, tag),
                         "doc_masked_prefill": with_clocks(measure_docs, layer, peaks, tag),
                         "attention_backward": with_clocks(measure_backward, layer, peaks, tag)}
    step = {"C4": {"workload": "B=8 T=2048 24q/8kv D=128, QK-norm (the timed step's prefill)",
                   "prefill_append_us": round(t_append_p / K * 1e3, 2),
                   "prefill_kernel_us": round(pf_ms * 1e3, 2),
                   "prefill_phase_us": round((t_append_p / K + pf_ms) * 1e3, 2),
                   "prefill_tokens_per_s": round(PREFILL.B * PREFILL.T /
                                                 ((t_append_p / K + pf_ms) * 1e-3), 1),
                   "prefill_tflops": round(pf_tflops, 2), "prefill_frac": round(pf_tflops / tpeak, 4),
                   "peak": tpeak, "bound": "tensor"},
            "C5": {"workload": "B=64 24q/8kv D=128, lens U[256,2048] (the timed step's decode)",
                   "decode_append_us": round(t_append_d / K * 1e3, 2),
                   "decode_kernels_us": round(dec_ms * 1e3, 2),
                   "decode_gbs": round(dec_gbs, 1), "decode_frac": round(dec_gbs / hpeak, 4),
                   "decode_tokens_per_s": round(DECODE.B / ((t_append_d / K + dec_ms) * 1e-3), 1),
                   "peak": hpeak, "bound": "hbm"}}
    line["configs"] = measure_configs(dev, peaks, tag, step)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    return line


def with_clocks(measure, *args):
    """One kernel timed alone, with its own clock record: the sampler starts, the
    GPU idles through the sampler's start-up pause, then the measurement runs
    (its warm-up launches included) while the clocks are sampled."""
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    try:
        row = measure(*args)
    finally:
        clocks = sampler.stop()
    row["clocks"] = clocks
    return row


def measure_scaled_append(layer, peaks, tag, reps: int = 30):
    """The prefill-sized fused QK-norm + RoPE + append with YaRN (s = 4 over a
    2048-token trained length), outside the timed step: the same HBM-bound
    kernel as plain RoPE with a different frequency table and a scale."""
    import rope_gqa_kv_b200 as gqa
    sc = gqa.RopeScaling("yarn", 4.0, original_max_pos=2048)
    args = (layer.pq, layer.pk, layer.pv, layer.pkc, layer.pvc)
    for _ in range(3):
        gqa.gqa_rope_append(*args, qk_norm=True, max_pos0=0, status=layer.status, scaling=sc)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        ev[i][0].record()
        gqa.gqa_rope_append(*args, qk_norm=True, max_pos0=0, status=layer.status, scaling=sc)
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)[reps // 2]
    gbs = append_bytes() / (ms * 1e-3) / 1e9
    return {"workload": "prefill-sized append, YaRN s=4 over 2048 trained positions",
            "kernel": "gqa_rope_append", "bound": "hbm", "us_median": round(ms * 1e3, 2),
            "achieved": round(gbs, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": "hbm copy " + tag,
            "algorithmic_per_launch": append_bytes(),
            "l2": "inputs (335 MB moved per launch) exceed L2"}


def measure_backward(layer, peaks, tag, reps: int = 20):
    """Attention backward (gqa_attention_backward: rowsum(dO * O), dK/dV, dQ), outside
    the timed step, on the 3.8B-style prompt (8 x 2048, 24/8 heads, D = 128) with a
    seeded N(0,1) output gradient.  Work is counted the usual way for attention
    backwards, 2.5 x the forward's causal FLOPs (five products per (query, key,
    head) instead of two); the kernels recompute S and dP once more for dQ, so
    they execute 3.5 x.  Each launch follows an L2-evicting write."""
    import rope_gqa_kv_b200 as gqa
    g = torch.Generator().manual_seed(4242)
    dout = torch.randn(tuple(layer.pq.shape), generator=g).to(torch.bfloat16).to(layer.dev)
    out, lse = gqa.gqa_prefill_lse(layer.pq, layer.pkc, layer.pvc, status=layer.status)
    dq = torch.empty_like(layer.pq)
    dk = torch.empty_like(layer.pkc)
    dv = torch.empty_like(layer.pvc)
    ws = torch.empty(gqa.gqa_backward_workspace_bytes(PREFILL.B, PREFILL.T, PREFILL.Hq),
                     dtype=torch.uint8, device=layer.dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=layer.dev)
    call = lambda: gqa.gqa_attention_backward(layer.pq, layer.pkc, layer.pvc, out, dout, lse,  # noqa: E731
                                              dq=dq, dk=dk, dv=dv, workspace=ws,
                                              status=layer.status)
    for _ in range(3):
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        flush.fill_(i & 255)
        ev[i][0].record()
        call()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)[reps // 2]
    fl = 2.5 * prefill_flops()
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "backward of the 8 x 2048 causal prompt, 24q/8kv, D=128",
            "kernel": "gqa_attention_backward (3 launches)", "bound": "tensor",
            "us_median": round(ms * 1e3, 2), "achieved": round(tf, 1), "unit": "TFLOP/s",
            "peak": peaks["bf16_tflops"], "frac": round(tf / peaks["bf16_tflops"], 4),
            "peak_kind": "bf16 burst " + tag, "algorithmic_per_launch": fl,
            "l2": "flushed (256 MB write) before each launch"}


def measure_docs(layer, peaks, tag, reps: int = 30):
    """Document-masked prefill (gqa_prefill_docs), outside the timed step: the
    3.8B-style prompt (8 x 2048, 24/8 heads, D = 128) holding packed documents of
    mean length 512 (lengths 1 + exponential).  Useful work counts each query's
    keys inside its own document only; each launch follows an L2-evicting write."""
    import rope_gqa_kv_b200 as gqa
    ids = inputs.packed_doc_ids(PREFILL.B, PREFILL.T, 512.0, seed=2048)
    starts = gqa.gqa_doc_start(ids.to(layer.dev))
    st_host = starts.cpu().numpy().astype(np.float64)
    t_idx = np.arange(PREFILL.T, dtype=np.float64)[None, :]
    fl = 4.0 * PREFILL.D * PREFILL.Hq * float((t_idx - st_host + 1.0).sum())
    out = torch.empty_like(layer.pq)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=layer.dev)
    for _ in range(3):
        gqa.gqa_prefill_docs(layer.pq, layer.pkc, layer.pvc, starts, out=out, status=layer.status)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        flush.fill_(i & 255)
        ev[i][0].record()
        gqa.gqa_prefill_docs(layer.pq, layer.pkc, layer.pvc, starts, out=out, status=layer.status)
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)[reps // 2]
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "8 x 2048 packed documents (mean 512 tokens), 24q/8kv, D=128, QK-norm",
            "kernel": "gqa_prefill_docs", "bound": "tensor", "us_median": round(ms * 1e3, 2),
            "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": peaks["bf16_tflops"],
            "frac": round(tf / peaks["bf16_tflops"], 4), "peak_kind": "bf16 burst " + tag,
            "algorithmic_per_launch": fl,
            "causal_fraction_kept": round(fl / prefill_flops(), 4),
            "l2": "flushed (256 MB write) before each launch"}


def measure_decode_loop(dev, name: str):
    """A workload's generation loop (its prompt, then its decode steps), per
    generated token: eager (the append and the decode's two kernels launched
    from the host each token) and replayed from CUDA graphs (DecodeGraph).
    Device time of the whole loop between two CUDA events, so the gaps the
    host's launches leave count."""
    import rope_gqa_kv_b200 as gqa
    w = inputs.BY_NAME[name]
    steps = w.decode_steps
    x = inputs.make_inputs(w, decode_steps=1)
    d = lambda t: t.to(dev)  # noqa: E731
    q0, k0, v0 = (d(t) for t in x["steps"][0])
    per_token = {}
    for mode in ("eager", "graph"):
        kc, vc = d(x["k_cache"]), d(x["v_cache"])
        gqa.gqa_rope_append(d(x["q"]), d(x["k"]), d(x["v"]), kc, vc, qk_norm=w.qk_norm)
        pos = torch.full((w.B,), w.T, dtype=torch.int32, device=dev)
        if mode == "graph":
            dg = gqa.DecodeGraph(kc, vc, pos, w.Hq, qk_norm=w.qk_norm)
            dg.q.copy_(q0)
            dg.k.copy_(k0)
            dg.v.copy_(v0)
            run = dg.step
        else:
            ws = gqa.decode_workspace(w.B, w.Hq, w.D, w.Lmax, dev)
            out = torch.empty_like(q0)
            lens = [pos.clone(), pos.clone()]
            cur = [0]

            def run():
                a, b = cur[0], cur[0] ^ 1
                gqa.gqa_rope_append(q0, k0, v0, kc, vc, pos0=lens[a], new_len=lens[b],
                                    qk_norm=w.qk_norm)
                gqa.gqa_decode(q0, kc, vc, lens[b], w.Lmax, out=out, workspace=ws)
                cur[0] = b
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        per_token[mode] = e0.elapsed_time(e1) * 1e3 / steps
    return {"workload": "B=%d %dq/%dkv D=%d: %d-token prompt, then %d generated tokens"
            % (w.B, w.Hq, w.Hkv, w.D, w.T, steps),
            "kernels_per_token": 3, "eager_us_per_token": round(per_token["eager"], 2),
            "graph_us_per_token": round(per_token["graph"], 2),
            "graph_tokens_per_s": round(w.B * 1e6 / per_token["graph"], 1),
            "frac": "n/m (latency-bound)"}


def measure_prefill_phase(dev, name, peaks, tag, reps: int = 50):
    """A workload's prompt prefill phase (fused QK-norm/RoPE/append, then the
    tcgen05 prefill), each launch timed with CUDA events after a 256 MB
    L2-evicting write; median over the repetitions."""
    import rope_gqa_kv_b200 as gqa
    w = inputs.BY_NAME[name]
    x = inputs.make_inputs(w, decode_steps=0)
    d = lambda t: t.to(dev)  # noqa: E731
    q, k, v, kc, vc = d(x["q"]), d(x["k"]), d(x["v"]), d(x["k_cache"]), d(x["v_cache"])
    out = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def once(ev=None):
        if ev:
            ev[0].record()
        gqa.gqa_rope_append(q, k, v, kc, vc, qk_norm=w.qk_norm, max_pos0=0)
        if ev:
            ev[1].record()
        gqa.gqa_prefill(q, kc, vc, out=out)
        if ev:
            ev[2].record()
    for _ in range(5):
        once()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for i in range(reps):
        flush.fill_(i & 255)
        once(ev[i])
    torch.cuda.synchronize()
    med = lambda xs: sorted(xs)[len(xs) // 2]  # noqa: E731
    app = med([e[0].elapsed_time(e[1]) for e in ev])
    pf = med([e[1].elapsed_time(e[2]) for e in ev])
    phase = med([e[0].elapsed_time(e[2]) for e in ev])
    fl = prefill_flops(w)
    tf = fl / (pf * 1e-3) / 1e12
    return {"workload": "B=%d T=%d %dq/%dkv D=%d%s" % (w.B, w.T, w.Hq, w.Hkv, w.D,
                                                      ", QK-norm" if w.qk_norm else ""),
            "prefill_append_us": round(app * 1e3, 2), "prefill_kernel_us": round(pf * 1e3, 2),
            "prefill_phase_us": round(phase * 1e3, 2),
            "prefill_tokens_per_s": round(w.B * w.T / (phase * 1e-3), 1),
            "prefill_tflops": round(tf, 2), "algorithmic_flops": fl,
            "l2": "flushed (256 MB write) before each repetition"}, tf


def measure_configs(dev, peaks, tag, step):
    """Every workload: a time, a rate and a fraction of the roofline, or
    "n/m (latency-bound)" where the launch is too small to load the GPU."""
    tpeak = peaks["bf16_tflops"]
    res = {}
    c1, _ = measure_prefill_phase(dev, "tiny_gqa", peaks, tag)
    c1["prefill_frac"] = "n/m (latency-bound)"
    c1["decode_loop"] = measure_decode_loop(dev, "tiny_gqa")
    res["C1_tiny_gqa"] = c1
    c2, tf2 = measure_prefill_phase(dev, "mha_prefill", peaks, tag)
    c2.update({"prefill_frac": round(tf2 / tpeak, 4), "peak": tpeak,
               "peak_kind": "bf16 burst " + tag, "bound": "tensor"})
    res["C2_mha_prefill"] = c2
    c3, _ = measure_prefill_phase(dev, "generation", peaks, tag)
    c3["prefill_frac"] = "n/m (latency-bound)"
    c3["decode_loop"] = measure_decode_loop(dev, "generation")
    res["C3_generation"] = c3
    res["C4_prefill_3p8b"] = step["C4"]
    res["C5_batched_decode"] = step["C5"]
    return res


def measure_chunk(dev, peaks, tag, reps: int = 30):
    """Continuation chunk (gqa_prefill_chunk), outside the timed step: 8 sequences
    with cached prefixes U[512, 1536] and 1024 new tokens each, 24/8 heads,
    D = 128.  Each launch is timed alone with CUDA events after a 256 MB write
    that evicts the L2."""
    import rope_gqa_kv_b200 as gqa
    w = inputs.BY_NAME["chunked_prefill_3p8b"]
    x = inputs.make_inputs(w)
    d = lambda t: t.to(dev)  # noqa: E731
    q, k, v, kc, vc = d(x["q"]), d(x["k"]), d(x["v"]), d(x["k_cache"]), d(x["v_cache"])
    pos0 = d(x["lens"])
    max_pos0 = int(x["lens"].max())
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.gqa_rope_append(q, k, v, kc, vc, pos0=pos0, max_pos0=max_pos0, qk_norm=True,
                        status=status)
    out = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        gqa.gqa_prefill_chunk(q, kc, vc, pos0, max_pos0, out=out, status=status)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        flush.fill_(i & 255)
        ev[i][0].record()
        gqa.gqa_prefill_chunk(q, kc, vc, pos0, max_pos0, out=out, status=status)
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)[reps // 2]
    fl = chunk_flops(x["lens"].tolist(), w)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "8 x (prefix U[512,1536] + 1024 new tokens), 24q/8kv, D=128, QK-norm",
            "kernel": "gqa_prefill_chunk", "bound": "tensor", "us_median": round(ms * 1e3, 2),
            "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": peaks["bf16_tflops"],
            "frac": round(tf / peaks["bf16_tflops"], 4), "peak_kind": "bf16 burst " + tag,
            "algorithmic_per_launch": fl, "l2": "flushed (256 MB write) before each launch",
            "device_status": int(status.item())}


# ---------------------------------------------------------------------------
# the oracle on the host cores (reported baseline / reference arm)
# ---------------------------------------------------------------------------
_CPU_BASELINE_INPUTS = []


def _baseline_inputs():
    if not _CPU_BASELINE_INPUTS:
        _CPU_BASELINE_INPUTS.append((inputs.make_inputs(PREFILL), inputs.make_inputs(DECODE)))
    return _CPU_BASELINE_INPUTS[0]


def oracle_step(nthreads: int = 0) -> float:
    """One whole step of the workload through the float64 oracle, as it stands:
    QK-norm + RoPE of every prompt token and the causal attention of every
    prompt row (8 x 2048 x 24 heads), then the decode step of all 64 sequences
    (norm + RoPE of the new token, attention over lens + 1 keys).  Returns the
    seconds it took."""
    import oracle
    xp, xd = _baseline_inputs()
    b = inputs.bits
    q, k, v = xd["steps"][0]
    t0 = time.perf_counter()
    oracle.prefill(b(xp["q"]), b(xp["k"]), b(xp["v"]), True, nthreads=nthreads)
    oracle.decode_step(b(q), b(k), b(v), b(xd["k_cache"]), b(xd["v_cache"]), xd["lens"].numpy(),
                       True, nthreads=nthreads)
    return time.perf_counter() - t0


def oracle_step_sampled(budget_s: float, nthreads: int = 0) -> float:
    """A bounded stand-in for oracle_step when whole steps would not fit the
    run: the prompt rows of a random sample of (b, t, h), the decode of 8 of the
    64 sequences, each scaled by its share of the key visits.  Returns the
    estimated seconds of one whole step."""
    import oracle
    xp, xd = _baseline_inputs()
    rng = np.random.default_rng(0)
    B, T, Hq = PREFILL.B, PREFILL.T, PREFILL.Hq
    t0 = time.perf_counter()
    pos = oracle.positions(0, 1, T)
    q1 = oracle.prep(inputs.bits(xp["q"][:1]), pos, True)
    k1 = oracle.prep(inputs.bits(xp["k"][:1]), pos, True)
    v1 = oracle.bf16_to_f64(inputs.bits(xp["v"][:1]))
    t_prep = (time.perf_counter() - t0) * B
    n_rows = max(64, int(budget_s * 2000))
    rows = rng.integers(0, T * Hq, size=n_rows)
    t0 = time.perf_counter()
    oracle.attention(q1, k1, v1, pos, rows=rows, nthreads=nthreads)
    t_rows = time.perf_counter() - t0
    t_pf = t_rows * (B * Hq * T * (T + 1) / 2.0) / float(np.sum(rows // Hq + 1))
    lens = xd["lens"].numpy()
    q, k, v = xd["steps"][0]
    sel = np.arange(0, DECODE.B, 8)
    t0 = time.perf_counter()
    oracle.decode_step(inputs.bits(q[sel]), inputs.bits(k[sel]), inputs.bits(v[sel]),
                       inputs.bits(xd["k_cache"][sel]), inputs.bits(xd["v_cache"][sel]),
                       lens[sel], True, nthreads=nthreads)
    t_dec = (time.perf_counter() - t0) * float(np.sum(lens + 1)) / float(np.sum(lens[sel] + 1))
    return t_prep + t_pf + t_dec


def oracle_small_configs():
    """The float64 oracle on the three small workloads, with one host core and
    with all: the prompt prefill phase (norm + RoPE + causal attention) and,
    where the workload generates tokens, its whole decode loop (each step
    against the oracle's own cache)."""
    import oracle
    res = {}
    b = inputs.bits
    for name in ("tiny_gqa", "mha_prefill", "generation"):
        w = inputs.BY_NAME[name]
        x = inputs.make_inputs(w)
        r = {}
        for label, nt in (("1core", 1), ("all_cores", 0)):
            t0 = time.perf_counter()
            _, k_rot, v = oracle.prefill(b(x["q"]), b(x["k"]), b(x["v"]), w.qk_norm, nthreads=nt)
            r["prefill_s_" + label] = round(time.perf_counter() - t0, 4)
            if x["steps"]:
                B, T = w.B, w.T
                kc = np.zeros((B, w.Hkv, w.Lmax, w.D))
                vc = np.zeros_like(kc)
                kc[:, :, :T] = k_rot.transpose(0, 2, 1, 3)
                vc[:, :, :T] = v.transpose(0, 2, 1, 3)
                lens = np.full(B, T)
                t0 = time.perf_counter()
                for s, (q, k, vv) in enumerate(x["steps"]):
                    _, knew = oracle.decode_step(b(q), b(k), b(vv), kc, vc, lens, w.qk_norm,
                                                 nthreads=nt)
                    kc[:, :, T + s] = knew
                    vc[:, :, T + s] = oracle.bf16_to_f64(b(vv))
                    lens = lens + 1
                r["decode_loop_s_" + label] = round(time.perf_counter() - t0, 4)
                r["decode_steps"] = len(x["steps"])
        res[name] = r
    return res


def cpu_baseline():
    """The float64 oracle, as it stands, on this host's cores: one whole step
    of the workload (no sampling, no extrapolation), plus the three small
    workloads on one core and on all."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    _baseline_inputs()
    step_s = oracle_step()
    return {"value": round(tokens_per_step() / step_s, 2), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": ("one whole step of the workload through the float64 oracle on %d host "
                       "threads: QK-norm + RoPE and causal attention of all 8 x 2048 x 24 prompt "
                       "rows, then the decode step of all 64 sequences (%.2f s)" % (cores, step_s)),
            "seconds_per_step": round(step_s, 3),
            "small_configs": oracle_small_configs()}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle, as it stands, on the host cores,
    one whole step of the workload per timed step (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    _baseline_inputs()
    # a bounded sample first estimates a whole step: whole steps when the run
    # fits the budget, else the same bounded samples throughout
    est = oracle_step_sampled(min(args.cpu_seconds, 10.0))
    whole = est * (args.steps + args.warmup) <= args.reference_budget
    times = []
    for i in range(args.warmup + args.steps):
        t = oracle_step() if whole else oracle_step_sampled(min(args.cpu_seconds, 10.0))
        if i >= args.warmup:
            times.append(t)
    step_s = statistics.median(times)
    value = round(tokens_per_step() / step_s, 2)
    sample = ("every step one whole step of the workload through the float64 oracle on %d "
              "host threads" % cores if whole else
              "every step a bounded sample of the workload (random prompt rows, 8 of 64 decode "
              "sequences) scaled by key visits: whole steps (about %.1f s each) would not fit "
              "the run" % est)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_s * 1e3, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": DATA, "config": bench_config(1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the CPU-baseline sample (oracle)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-budget", type=float, default=420.0,
                    help="seconds the reference arm may take with whole oracle steps; beyond "
                         "it every step is a bounded sample")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.stderr.write("note: --gpus %d but WORLD_SIZE=%d; using WORLD_SIZE\n"
                         % (args.gpus, world))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        line = run_ours(args, rank, world, dev, dist_on)
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
