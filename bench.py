#!/usr/bin/env python
"""Benchmark of the causal attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one call of the library on one batch of the workload (default: the
BitNet-3B-shaped causal MHA prefill, B=1, H=32, T=2048, d=80, bf16).  The
line also carries the GQA prefill (B=8, H=16/8, T=4096, d=128, bf16), the MQA
chunked prefill against a cache (B=32, H=8/1, 512 new tokens at 3584 over 4096
keys, d=128, fp16), the cached-decode half of the metric (GQA decode, B=64,
H=32/8, S=8192, d=128, bf16), the same decode over a paged cache (64-token
pages), the GQA prefill with a 2048-key local window (B=2, T=8192), the
KV-cache append with RoPE on K of the GQA prefill's keys and values (B=8,
Hkv=8, 4096 tokens, d=128, bf16), and the backward pass of the GQA prefill
(dQ, dK, dV from the forward's O and row statistic), each measured the same
way with its own roofline and its own bounded oracle baseline.

Timing: W untimed steps, then exactly K timed steps bracketed by a barrier and
torch.cuda.synchronize() on both sides.  Before every timed call L2 is flushed
by writing 256 MiB (> 126 MB L2); each call is bracketed by CUDA events on the
launching stream, and the per-step time is the mean event duration, max over
ranks.  Multi-GPU runs are weak scaling: every rank runs the whole workload on
its own GPU (the path shards by sequence and head with no exchange).

--impl reference times the fp64 CPU oracle (the only other implementation of
this operation here) on the host cores, on bounded row samples of the same
workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "prefill TFLOP/s & cached-decode HBM GB/s, causal GQA attn, % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # the four 16-bit workloads; the default is the BitNet-3B-shaped prefill
    "bitnet3b_mha_prefill_bf16": dict(kind="prefill", dtype="bf16", B=1, H=32, Hkv=32, T=2048,
                                      d=80),
    "gqa16x8_prefill_bf16": dict(kind="prefill", dtype="bf16", B=8, H=16, Hkv=8, T=4096, d=128),
    # local attention: the GQA shape over 8192 tokens with a 2048-key window
    "gqa_prefill_swa_bf16": dict(kind="prefill", dtype="bf16", B=2, H=32, Hkv=8, T=8192, d=128,
                                 window=2048),
    "gqa_decode_bf16": dict(kind="cached", dtype="bf16", B=64, H=32, Hkv=8, Tnew=1, start=8191,
                            S=8192, d=128),
    "mqa_chunked_prefill_f16": dict(kind="cached", dtype="f16", B=32, H=8, Hkv=1, Tnew=512,
                                    start=3584, S=4096, d=128),
    # the GQA decode over a paged cache: 64-token pages in a seeded physical order
    "gqa_decode_paged_bf16": dict(kind="paged", dtype="bf16", B=64, H=32, Hkv=8, Tnew=1,
                                  start=8191, S=8192, d=128, page=64),
    # the backward pass of the GQA prefill (its forward runs untimed during setup)
    "gqa16x8_backward_bf16": dict(kind="backward", dtype="bf16", B=8, H=16, Hkv=8, T=4096,
                                  d=128),
    # the step before attention: the GQA prefill's 4096 new keys (RoPE) and values
    # written into an empty cache
    "kv_append_rope_gqa16x8_bf16": dict(kind="append", dtype="bf16", B=8, H=16, Hkv=8,
                                        Tnew=4096, start=0, S=4096, d=128, base=10000.0),
}
DEFAULT_WORKLOAD = "bitnet3b_mha_prefill_bf16"
GQA_PREFILL_WORKLOAD = "gqa16x8_prefill_bf16"
MQA_CHUNKED_WORKLOAD = "mqa_chunked_prefill_f16"
# seconds of oracle work behind each leg's cpu_baseline (the line's own: 10 s)
LEG_BASELINE_S = 3.0
DECODE_WORKLOAD = "gqa_decode_bf16"
APPEND_WORKLOAD = "kv_append_rope_gqa16x8_bf16"
WINDOW_WORKLOAD = "gqa_prefill_swa_bf16"
PAGED_WORKLOAD = "gqa_decode_paged_bf16"
BACKWARD_WORKLOAD = "gqa16x8_backward_bf16"
TORCH_DTYPE = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}
KERNEL_SOURCES = {"tcgen05": "prefill_tcgen05.cuh", "splitkv": "decode_mma.cuh",
                  "paged": "decode_mma.cuh",
                  "simt": "simt_attn.cuh", "append": "kv_append.cuh",
                  "backward": "prefill_backward.cuh"}


# ------------------------------------------------------------------ workload algebra

def full_sequence(w):
    return w["kind"] in ("prefill", "backward")


def q_len(w):
    return w["T"] if full_sequence(w) else w["Tnew"]


def kv_len(w):
    return w["T"] if full_sequence(w) else w["S"]


def start_pos(w):
    return 0 if full_sequence(w) else w["start"]


def visible_pairs(w):
    """Visible (query, key) pairs per query head: sum over rows of (p_i + 1),
    or of min(p_i + 1, window) with a local window."""
    Tq, s0 = q_len(w), start_pos(w)
    win = w.get("window", 0)
    if win:
        return sum(min(s0 + i + 1, win) for i in range(Tq))
    return Tq * s0 + Tq * (Tq + 1) // 2


def flops_per_pair(w):
    """Forward: 4*d per visible (query, key) pair per query head (2*d for Q.K,
    2*d for P.V).  Backward: 10*d (the five products S, dP, dV, dK, dQ); the
    second recomputation of S and dP in the dQ kernel is not credited."""
    return (10 if w["kind"] == "backward" else 4) * w["d"]


def algorithmic_flops(w):
    """FLOPs of the visible pairs; masked pairs, exponentials and maxima are
    not counted."""
    return flops_per_pair(w) * w["B"] * w["H"] * visible_pairs(w)


def esize(w):
    return 2 if w["dtype"] in ("bf16", "f16") else 4


def algorithmic_bytes(w):
    """Attention: Q read + the visible K/V rows read once per K/V head + O
    written.  Append: the new K and V rows read once and written once."""
    esz = esize(w)
    if w["kind"] == "append":
        return 4 * w["B"] * w["Hkv"] * w["Tnew"] * w["d"] * esz
    kv_vis = min(kv_len(w), start_pos(w) + q_len(w))
    q_o = 2 * w["B"] * w["H"] * q_len(w) * w["d"] * esz
    return q_o + 2 * w["B"] * w["Hkv"] * kv_vis * w["d"] * esz


def bound(w):
    if w["kind"] in ("append", "paged"):
        return "hbm"
    return "hbm" if w["kind"] == "cached" and q_len(w) * w["H"] // w["Hkv"] <= 16 else "tensor"


def config_of(name, w, world):
    cfg = {"workload": name, "B": w["B"], "H": w["H"], "Hkv": w["Hkv"], "d": w["d"],
           "dtype": w["dtype"], "causal": True, "scale": f"1/sqrt({w['d']})"}
    if full_sequence(w):
        cfg["T"] = w["T"]
        if w["kind"] == "backward":
            cfg["pass"] = "backward: dq, dk, dv from q, k, v, o, lse, dout"
        if w.get("window"):
            cfg["window"] = w["window"]
    elif w["kind"] == "paged":
        cfg.update(Tnew=w["Tnew"], kv_len=w["S"], page_size=w["page"],
                   pages="seeded random physical order")
    elif w["kind"] == "append":
        cfg = {"workload": name, "B": w["B"], "Hkv": w["Hkv"], "d": w["d"], "dtype": w["dtype"],
               "Tnew": w["Tnew"], "start_pos": w["start"], "S_cap": w["S"],
               "rope": f"NeoX, base {w['base']:g}"}
    else:
        cfg.update(Tnew=w["Tnew"], start_pos=w["start"], S=w["S"])
    cfg["l2"] = "flushed by a 256 MiB write before every timed call"
    cfg["global_batch"] = w["B"] * world
    cfg["parallelism"] = f"replicas x{world} (weak scaling, no data-path collective)"
    return cfg


# ------------------------------------------------------------------ peaks, clocks, profiles

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            peaks = json.load(fh)
        return peaks, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(device_index)
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nvml = None

    def _sample(self):
        n = self._nvml
        try:
            mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
            reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:  # noqa: BLE001
            return
        self.samples.append((mhz, reasons))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = set()
        for _, mask in self.samples:
            for bit, name in REASON_BITS.items():
                if mask & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples)}


def clocks_rejected(cl):
    if cl["sm_mhz"] is None:
        return False
    if BAD_REASONS & set(cl["reasons"]):
        return True
    # stuck well below max with no reason at all: a leftover clock lock
    return (cl["sm_max_mhz"] and cl["sm_mhz"] < 0.6 * cl["sm_max_mhz"] and
            not (set(cl["reasons"]) - {"gpu_idle"}))


def kernel_source_sha(kernel: str) -> str:
    path = os.path.join(ROOT, "transformer_attention_causal_b200", "csrc", KERNEL_SOURCES[kernel])
    with open(path, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


PROFILED_KEYS = ("dram_bytes_per_launch", "tensor_pipe_active_pct", "dram_throughput_pct")


def profiled(kernel: str, workload: str):
    """Figures of the committed ncu summary of this kernel and workload
    (profiles/<kernel>_<workload>.md): DRAM bytes per launch and, where
    captured, the tensor-pipe active and DRAM throughput percentages.  Empty
    when there is no summary or the kernel source changed since it was taken."""
    rel = os.path.join("profiles", f"{kernel}_{workload}.md")
    try:
        text = open(os.path.join(ROOT, rel)).read()
    except OSError:
        return {}
    m_sha = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_sha or m_sha.group(1) != kernel_source_sha(kernel):
        return {}
    out = {}
    for key in PROFILED_KEYS:
        m = re.search(key + r":\s*([0-9.eE+]+)", text)
        if m:
            out[key] = float(m.group(1))
    if out:
        out["source"] = rel
    return out



# ------------------------------------------------------------------ our implementation

class Case:
    """Device buffers and the library call for one workload."""

    def __init__(self, name, w, device, seed=0):
        import transformer_attention_causal_b200 as attn
        from transformer_attention_causal_b200 import inputs

        self.attn, self.name, self.w = attn, name, w
        dt = TORCH_DTYPE[w["dtype"]]
        self.dtype = dt
        Tq, S = q_len(w), kv_len(w)
        if w["kind"] == "append":
            k_new = inputs.normal((w["B"], w["Hkv"], Tq, w["d"]), seed, 1, dt)
            v_new = inputs.normal((w["B"], w["Hkv"], Tq, w["d"]), seed, 2, dt)
            self.host = [t.pin_memory() for t in (k_new, v_new)]
            self.dev_in = [t.to(device, non_blocking=True) for t in self.host]
            self.dev_out = [torch.zeros((w["B"], w["Hkv"], S, w["d"]), dtype=dt, device=device)
                            for _ in range(2)]
            self.host_out = [torch.empty(t.shape, dtype=dt).pin_memory() for t in self.dev_out]
            self.kernel, self.launches, self.device = "append", 1, device
            return
        q, k, v = inputs.qkv(w["B"], w["H"], w["Hkv"], Tq, S, w["d"], dt, seed=seed)
        if w["kind"] == "backward":
            self.scale = 1.0 / math.sqrt(w["d"])
            dout = inputs.upstream(w["B"], w["H"], Tq, w["d"], dt, seed=seed)
            qd, kd, vd = (t.to(device) for t in (q, k, v))
            lse = torch.empty((w["B"], w["H"], Tq), dtype=torch.float32, device=device)
            o = attn.prefill(qd, kd, vd, scale=self.scale, causal=True, lse=lse)
            self.host = [t.pin_memory() for t in (q, k, v, o.cpu(), lse.cpu(), dout)]
            self.dev_in = [qd, kd, vd, o, lse, dout.to(device)]
            self.dev_out = [torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)]
            self.host_out = [torch.empty(t.shape, dtype=dt).pin_memory() for t in self.dev_out]
            need = attn.prefill_backward_workspace_size(dt, w["B"], w["H"], w["Hkv"], Tq, w["d"])
            self.ws = torch.empty(need, dtype=torch.uint8, device=device)
            self.kernel, self.launches, self.device = "backward", 3, device
            return
        if w["kind"] == "paged":
            # pages [B * S / P, Hkv, P, d] in a seeded physical order, and the table
            P, n = w["page"], S // w["page"]
            perm = torch.randperm(w["B"] * n, generator=torch.Generator().manual_seed(seed))
            def to_pages(t):
                blocks = t.reshape(w["B"], w["Hkv"], n, P, w["d"]).permute(0, 2, 1, 3, 4)
                pages = torch.empty((w["B"] * n, w["Hkv"], P, w["d"]), dtype=dt)
                pages[perm] = blocks.reshape(w["B"] * n, w["Hkv"], P, w["d"])
                return pages
            k, v = to_pages(k), to_pages(v)
            self.table = perm.reshape(w["B"], n).to(torch.int32).to(device)
            self.lens = torch.full((w["B"],), S, dtype=torch.int32, device=device)
        self.host = [t.pin_memory() for t in (q, k, v)]
        self.q, self.k, self.v = (t.to(device, non_blocking=True) for t in self.host)
        self.out = torch.empty_like(self.q)
        self.dev_in, self.dev_out = [self.q, self.k, self.v], [self.out]
        self.host_out = [torch.empty(self.out.shape, dtype=dt).pin_memory()]
        self.device = device
        self.scale = 1.0 / math.sqrt(w["d"])
        if w["kind"] == "prefill":
            self.kernel = attn.prefill_plan(dt, w["B"], w["H"], w["Hkv"], Tq, w["d"])
            self.ws = None
        elif w["kind"] == "paged":
            self.kernel = "splitkv"
            need = attn.cached_paged_workspace_size(dt, w["B"], w["H"], w["Hkv"], Tq, w["d"], S)
            self.ws = torch.empty(need, dtype=torch.uint8, device=device) if need else None
        else:
            self.kernel = attn.cached_plan(dt, w["B"], w["H"], w["Hkv"], Tq, S, S, w["d"],
                                           w["start"])
            need = attn.cached_workspace_size(dt, w["B"], w["H"], w["Hkv"], Tq, S, w["d"],
                                              w["start"])
            self.ws = torch.empty(need, dtype=torch.uint8, device=device) if need else None
        # launches of this library's kernels per call: a workspace means a
        # second kernel merges partial results (the split-KV decode's splits,
        # or the pieces of a chunked prefill's last pass of units)
        self.launches = 1
        if self.kernel in ("splitkv", "tcgen05") and self.ws is not None:
            self.launches = 2

    def call(self, bufs=None, stream=None):
        """One library call on (inputs, outputs) = bufs (default: the case's
        own device buffers), enqueued on `stream` (default: the current one)."""
        w = self.w
        dev_in, dev_out = bufs if bufs is not None else (self.dev_in, self.dev_out)
        if w["kind"] == "append":
            self.attn.kv_append_rope(*dev_in, *dev_out, start_pos=w["start"], rope_base=w["base"],
                                     stream=stream)
        elif w["kind"] == "backward":
            dq, dk, dv = dev_out
            self.attn.prefill_backward(*dev_in, scale=self.scale, causal=True, dq=dq, dk=dk, dv=dv,
                                       workspace=self.ws, stream=stream)
        elif w["kind"] == "prefill":
            q, k, v = dev_in
            self.attn.prefill(q, k, v, scale=self.scale, causal=True, out=dev_out[0],
                              window=w.get("window", 0), stream=stream)
        elif w["kind"] == "paged":
            q, k, v = dev_in
            self.attn.cached_paged(q, k, v, self.table, self.lens, max_kv_len=w["S"],
                                   scale=self.scale, out=dev_out[0], workspace=self.ws,
                                   stream=stream)
        else:
            q, k, v = dev_in
            self.attn.cached(q, k, v, start_pos=w["start"], scale=self.scale, out=dev_out[0],
                             workspace=self.ws, stream=stream)


# per-call device times (ms) of the latest time_device() call on this rank
_LAST_CALL_MS: list = []


def spread(times_ms):
    """Median and 10th / 90th percentiles (nearest rank) of per-call times."""
    t = sorted(times_ms)
    if not t:
        return None

    def pick(q):
        return t[min(len(t) - 1, max(0, math.ceil(q * len(t)) - 1))]

    return {"median_ms": round(statistics.median(t), 5), "p10_ms": round(pick(0.10), 5),
            "p90_ms": round(pick(0.90), 5)}


def time_device(case, steps, warmup, dist_ctx):
    """Mean per-call device time (ms) over `steps` timed calls, L2 flushed
    before each; returns (kernel_ms, bracket_ms).  The per-call times are
    left in _LAST_CALL_MS."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=case.device)
    for _ in range(warmup):
        flush.zero_()
        case.call()
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    b0.record()
    for i in range(steps):
        flush.zero_()
        ev_s[i].record()
        case.call()
        ev_e[i].record()
    b1.record()
    torch.cuda.synchronize()
    dist_ctx.barrier()
    times = [ev_s[i].elapsed_time(ev_e[i]) for i in range(steps)]
    _LAST_CALL_MS[:] = times
    kernel_ms = sum(times) / steps
    return kernel_ms, b0.elapsed_time(b1)


def time_graph(case, calls=20, replays=10):
    """Device time per call of `calls` back-to-back library calls captured in
    one CUDA graph (launch overhead amortised), L2 flushed before each replay;
    the median over `replays`."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=case.device)
    stream = torch.cuda.Stream(device=case.device)
    stream.wait_stream(torch.cuda.current_stream(case.device))
    with torch.cuda.stream(stream):
        for _ in range(3):
            case.call(stream=stream)        # first calls set kernel attributes
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(calls):
            case.call(stream=stream)
    times = []
    for _ in range(replays):
        flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        graph.replay()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) / calls)
    del graph
    return statistics.median(times)


def time_e2e(case, steps, warmup, dist_ctx):
    """Per-step time (ms) with the inputs copied host -> device from pinned
    memory and the output copied back, every step, through the public API.

    Steps are pipelined over two device buffer sets and three streams, the way
    a serving loop would run them: step k's host -> device copy overlaps step
    k-1's call and step k-2's device -> host copy.  Every step still moves all
    of its bytes; events order each buffer's reuse."""
    sets = [(case.dev_in, case.dev_out),
            ([torch.empty_like(t) for t in case.dev_in], [torch.empty_like(t) for t in case.dev_out])]
    s_h2d, s_call, s_d2h = (torch.cuda.Stream(device=case.device) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, call_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(k):
        slot = k & 1
        dev_in, dev_out = sets[slot]
        with torch.cuda.stream(s_h2d):
            if used[slot]:
                s_h2d.wait_event(call_done[slot])     # the call of step k-2 has read dev_in
            for dev, host in zip(dev_in, case.host):
                dev.copy_(host, non_blocking=True)
            h2d_done[slot].record(s_h2d)
        s_call.wait_event(h2d_done[slot])
        if used[slot]:
            s_call.wait_event(d2h_done[slot])         # step k-2's result has left dev_out
        case.call((dev_in, dev_out), stream=s_call)
        call_done[slot].record(s_call)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(call_done[slot])
            for host, dev in zip(case.host_out, dev_out):
                host.copy_(dev, non_blocking=True)
            d2h_done[slot].record(s_d2h)
        used[slot] = True

    for k in range(warmup):
        step(k)
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    b0.record(s_h2d)
    s_call.wait_stream(s_h2d)
    s_d2h.wait_stream(s_h2d)
    for k in range(warmup, warmup + steps):
        step(k)
    s_d2h.wait_stream(s_call)
    s_d2h.wait_stream(s_h2d)
    b1.record(s_d2h)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    h2d = sum(t.numel() * t.element_size() for t in case.host)
    d2h = sum(t.numel() * t.element_size() for t in case.host_out)
    return b0.elapsed_time(b1) / steps, h2d, d2h


class DistCtx:
    """One process per GPU (torchrun env).  NCCL carries only the barrier and
    the max-over-ranks of the timings; the data path has no collective.
    ``backend="gloo"`` runs the same host logic on CPU (tests)."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            kwargs = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
                kwargs["device_id"] = torch.device("cuda", self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kwargs)
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def roofline(w, kernel_ms, kernel, name, peaks, peak_src):
    if bound(w) == "hbm":
        achieved = algorithmic_bytes(w) / (kernel_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    else:
        achieved = algorithmic_flops(w) / (kernel_ms * 1e-3) / 1e12
        # a kernel timed alone: the burst GEMM figure
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    prof = profiled(kernel, name)
    line = {"bound": bound(w), "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} (MEASURED_PEAKS.json)"
            if peak_src == "measured" else "fallback",
            "traffic": prof.get("dram_bytes_per_launch"), "kernel": kernel}
    if prof:
        # from the committed ncu summary (same kernel source): percentages of
        # the capture's elapsed cycles / of peak DRAM throughput
        line["ncu"] = {k: v for k, v in prof.items() if k != "dram_bytes_per_launch"}
    return line


class OracleSample:
    """The fp64 oracle, as it stands, on seeded random samples of a workload:
    query rows for attention, (batch, token) rows for the append.  Work is
    counted in the workload's own unit: the FLOPs of the sampled rows, or
    their share of the algorithmic bytes."""

    def __init__(self, w, seed=0):
        from transformer_attention_causal_b200 import inputs

        self.w = w
        dt = TORCH_DTYPE[w["dtype"]]
        self.unit = "GB/s" if bound(w) == "hbm" else "TFLOP/s"
        if w["kind"] == "append":
            shape = (w["B"], w["Hkv"], w["Tnew"], w["d"])
            self.k_new = inputs.normal(shape, seed, 1, dt)
            self.v_new = inputs.normal(shape, seed, 2, dt)
            self.total = w["B"] * w["Tnew"]
            self.what = "(batch, token) rows of"
        elif w["kind"] == "paged":
            self.q, self.k, self.v = inputs.qkv(w["B"], w["H"], w["Hkv"], q_len(w), kv_len(w),
                                                w["d"], dt, seed=seed)
            self.total = w["B"]
            self.what = "sequences (paged, all heads) of"
        elif w["kind"] == "backward":
            self.q, self.k, self.v = inputs.qkv(w["B"], w["H"], w["Hkv"], q_len(w), kv_len(w),
                                                w["d"], dt, seed=seed)
            self.dout = inputs.upstream(w["B"], w["H"], q_len(w), w["d"], dt, seed=seed)
            self.total = w["B"] * w["H"]
            self.what = "(batch, head) slices (full backward of one head) of"
        else:
            self.q, self.k, self.v = inputs.qkv(w["B"], w["H"], w["Hkv"], q_len(w), kv_len(w),
                                                w["d"], dt, seed=seed)
            self.total = w["B"] * w["H"] * q_len(w)
            self.what = "query rows of"
        whole = algorithmic_bytes(w) / 1e9 if self.unit == "GB/s" else algorithmic_flops(w) / 1e12
        self.per_unit = whole / self.total

    def run(self, n, rng):
        """Oracle time (s), work and count of one sample of n rows."""
        import numpy as np

        from oracle import attention as oracle_attention
        from oracle import rope_append

        w = self.w
        n = int(min(n, self.total))
        if w["kind"] == "append":
            T = w["Tnew"]
            jobs, left = [], n
            while left > 0:
                m = min(left, T)
                b, t0 = int(rng.integers(w["B"])), int(rng.integers(T - m + 1))
                jobs.append((self.k_new[b:b + 1, :, t0:t0 + m].contiguous(),
                             self.v_new[b:b + 1, :, t0:t0 + m].contiguous(), w["start"] + t0))
                left -= m
            t0 = time.perf_counter()
            for kn, vn, pos in jobs:
                rope_append(kn, vn, start_pos=pos, base=w["base"])
            return time.perf_counter() - t0, n * self.per_unit, n
        if w["kind"] == "backward":
            from oracle import attention_backward

            G = w["H"] // w["Hkv"]
            secs = 0.0
            for idx in rng.choice(self.total, size=n, replace=False):
                b, h = divmod(int(idx), w["H"])
                kvh = h // G
                t0 = time.perf_counter()
                attention_backward(self.q[b:b + 1, h:h + 1], self.k[b:b + 1, kvh:kvh + 1],
                                   self.v[b:b + 1, kvh:kvh + 1], self.dout[b:b + 1, h:h + 1],
                                   scale=1 / math.sqrt(w["d"]))
                secs += time.perf_counter() - t0
            return secs, n * self.per_unit, n
        if w["kind"] == "paged":
            from oracle import paged_attention

            P, S = w["page"], kv_len(w)
            secs = 0.0
            for b in rng.choice(self.total, size=n, replace=False):
                perm = torch.as_tensor(rng.permutation(S // P))
                def pages(t):
                    blocks = t[b].reshape(w["Hkv"], S // P, P, w["d"]).permute(1, 0, 2, 3)
                    out = torch.empty_like(blocks)
                    out[perm] = blocks
                    return out
                kp, vp = pages(self.k), pages(self.v)
                t0 = time.perf_counter()
                paged_attention(self.q[b:b + 1], kp, vp, perm.reshape(1, -1), [S],
                                scale=1 / math.sqrt(w["d"]))
                secs += time.perf_counter() - t0
            return secs, n * self.per_unit, n
        rows = np.sort(rng.choice(self.total, size=n, replace=False))
        t0 = time.perf_counter()
        oracle_attention(self.q, self.k, self.v, scale=1 / math.sqrt(w["d"]), causal=True,
                         start_pos=start_pos(w), rows=rows, window=w.get("window", 0))
        secs = time.perf_counter() - t0
        if self.unit == "GB/s":
            return secs, n * self.per_unit, n
        vis = start_pos(w) + rows % q_len(w) + 1
        if w.get("window"):
            vis = np.minimum(vis, w["window"])
        return secs, float(np.sum(4 * w["d"] * vis)) / 1e12, n

    def sized(self, target_s, rng):
        """Rows that take the oracle about target_s seconds, from a pilot run."""
        from oracle import num_cores

        secs, work, _ = self.run(1 if self.w["kind"] == "backward" else 4 * num_cores(), rng)
        return int(min(self.total, max(16, target_s * (work / max(secs, 1e-6)) / self.per_unit)))


def cpu_baseline(w, name, target_s=10.0):
    """The oracle on a bounded sample of the workload, on every host core."""
    import numpy as np

    from oracle import num_cores

    rng = np.random.default_rng(0)
    sample = OracleSample(w)
    n = sample.sized(target_s, rng)
    secs, work, nrows = sample.run(n, rng)
    return {"value": work / secs, "unit": sample.unit, "cores": num_cores(), "kind": "oracle",
            "sample": f"{nrows} seeded random {sample.what} {sample.total} ({secs:.1f} s, fp64)"}


def whole_job_value(world: int, work_per_step: float, slowest_ms: float) -> float:
    """Weak scaling: every rank does `work_per_step`; the job is as fast as
    its slowest rank."""
    return world * work_per_step / (slowest_ms * 1e-3)


def workload(name: str, batch: int | None = None):
    w = dict(WORKLOADS[name])
    if batch:
        w["B"] = int(batch)
    return w


def run_ours(args, dist_ctx):
    name = args.workload
    w = workload(name, args.batch)
    device = torch.device("cuda", dist_ctx.local_rank)
    torch.cuda.set_device(device)
    from transformer_attention_causal_b200.build import build

    if dist_ctx.rank == 0:
        build()
    dist_ctx.barrier()
    peaks, peak_src = load_peaks()
    case = Case(name, w, device)
    torch.cuda.synchronize()

    def measure():
        with ClockSampler(device.index) as cs:
            k_ms, br_ms = time_device(case, args.steps, args.warmup, dist_ctx)
            call_spread = spread(_LAST_CALL_MS)
            e_ms, h2d, d2h = time_e2e(case, args.steps, args.warmup, dist_ctx)
        return k_ms, br_ms, e_ms, h2d, d2h, cs.summary(), call_spread

    k_ms, br_ms, e_ms, h2d, d2h, clocks, call_spread = measure()
    if clocks_rejected(clocks):
        k_ms, br_ms, e_ms, h2d, d2h, clocks, call_spread = measure()
        clocks["remeasured"] = True
    k_ms, br_ms, e_ms = dist_ctx.max(k_ms), dist_ctx.max(br_ms), dist_ctx.max(e_ms)
    # a prefill workload also as 20 back-to-back calls in one CUDA graph
    g_ms = dist_ctx.max(time_graph(case)) if w["kind"] == "prefill" else None
    from transformer_attention_causal_b200 import device_status

    status = device_status()
    N = dist_ctx.world
    unit = "GB/s" if bound(w) == "hbm" else "TFLOP/s"
    work = algorithmic_bytes(w) / 1e9 if unit == "GB/s" else algorithmic_flops(w) / 1e12
    line = {
        "metric": METRIC,
        "value": round(whole_job_value(N, work, k_ms), 3),
        "unit": unit,
        "n_gpus": N,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(k_ms, 5),
        "bracket_ms": round(br_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w["dtype"],
        "data": "synthetic: i.i.d. N(0,1) from seed 0, rounded to the dtype",
        "config": config_of(name, w, N),
        "e2e": {"value": round(whole_job_value(N, work, e_ms), 3), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": roofline(w, k_ms, case.kernel, name, peaks, peak_src),
        # this rank's per-call device times (value and ms_per_step use the mean)
        "spread": call_spread,
        "gpu_launches": args.steps * case.launches,
        "clocks": clocks,
        "device_status": status,
    }
    if g_ms is not None:
        gwork = algorithmic_flops(w) / 1e12
        line["graph"] = {"calls": 20, "ms_per_call": round(g_ms, 5),
                         "value": round(whole_job_value(N, gwork, g_ms), 3), "unit": "TFLOP/s",
                         "note": "20 calls captured in one CUDA graph, L2 flushed before each replay; "
                                 "not counted in gpu_launches"}
    legs = [] if args.no_decode else [("gqa_prefill", GQA_PREFILL_WORKLOAD),
                                      ("mqa_chunked_prefill", MQA_CHUNKED_WORKLOAD),
                                      ("decode", DECODE_WORKLOAD), ("paged", PAGED_WORKLOAD),
                                      ("window", WINDOW_WORKLOAD), ("append", APPEND_WORKLOAD),
                                      ("backward", BACKWARD_WORKLOAD)]
    baselines = dist_ctx.rank == 0 and N == 1 and not args.no_cpu_baseline
    del case
    for key, leg in legs:
        if leg == name:
            continue
        torch.cuda.empty_cache()
        wl = WORKLOADS[leg]
        lcase = Case(leg, wl, device)
        lsteps = max(args.steps, 5)
        l_ms, _ = time_device(lcase, lsteps, max(args.warmup, 3), dist_ctx)
        l_spread = spread(_LAST_CALL_MS)
        l_ms = dist_ctx.max(l_ms)
        hbm = bound(wl) == "hbm"
        work = algorithmic_bytes(wl) / 1e9 if hbm else algorithmic_flops(wl) / 1e12
        line[key] = {
            "workload": leg,
            "value": round(N * work / (l_ms * 1e-3), 2),
            "unit": "GB/s" if hbm else "TFLOP/s", "ms_per_step": round(l_ms, 5), "steps": lsteps,
            "spread": l_spread,
            "gpu_launches": lsteps * lcase.launches,
            "roofline": roofline(wl, l_ms, lcase.kernel, leg, peaks, peak_src),
        }
        del lcase
        if baselines:
            line[key]["cpu_baseline"] = cpu_baseline(wl, leg, target_s=LEG_BASELINE_S)
    if baselines:
        line["cpu_baseline"] = cpu_baseline(w, name)
    if dist_ctx.rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, dist_ctx):
    """The oracle as the reference arm: each step a bounded row sample."""
    if dist_ctx.rank != 0:
        return
    import numpy as np

    from oracle import num_cores

    name = args.workload
    w = workload(name, args.batch)
    per_step_s = min(5.0, 150.0 / max(1, args.steps + args.warmup))
    rng = np.random.default_rng(1)
    sample = OracleSample(w)
    n = sample.sized(per_step_s, rng)
    for _ in range(args.warmup):
        sample.run(n, rng)
    tot_s, tot_w = 0.0, 0.0
    for _ in range(args.steps):
        s_, w_, _ = sample.run(n, rng)
        tot_s, tot_w = tot_s + s_, tot_w + w_
    value = tot_w / tot_s
    unit = sample.unit
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: i.i.d. N(0,1) from seed 0, rounded to the dtype",
        "config": config_of(name, w, 1),
        "cpu_baseline": {"value": value, "unit": unit, "cores": num_cores(), "kind": "oracle",
                         "sample": f"{n} seeded random {sample.what} {sample.total} per step"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode and append legs of the line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # no process group: under torchrun the other ranks simply exit
        run_reference(args, _NoDist())
        return
    dist_ctx = DistCtx()
    try:
        run_ours(args, dist_ctx)
    finally:
        dist_ctx.close()


class _NoDist:
    def __init__(self):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    def barrier(self):
        pass


if __name__ == "__main__":
    main()
