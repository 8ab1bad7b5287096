#!/usr/bin/env python
"""Benchmark of the gated delta-rule library on B200.

`python bench.py --gpus N --steps K --warmup W` prints ONE JSON line.

Headline (`value`): GDN-2 chunkwise forward + backward tokens/s on the workload
B=8, T=4096, H=16, dk=dv=128, bf16 inputs, fp32 state, chunk 64 (whole job over all ranks; one
step = one gdn_chunk_fwd + one gdn_chunk_bwd over the batch).  The same run also measures the
decode step (256 sequences x 1024 tokens, H=16, d=128; "decode"), the forward alone, the
scalar-gate Gated DeltaNet forward and the GQA layer core ("parts"), each with its roofline.

Timing: CUDA events on the launching stream, W untimed warm-up steps, K timed steps bracketed
by a barrier and a device synchronisation, max over ranks.  Every workload's inputs are larger
than the 126 MB L2, so no flush is needed between steps.  Multi-GPU runs (torchrun) shard
nothing: every rank runs the full per-GPU workload (weak scaling, no collective on the data
path).

`--impl reference` times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (the reference arm).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN-2 chunkwise fwd+bwd tokens/s and decode tokens/s on 1 B200; % roofline"
HEADLINE = "gdn2_fwd_bwd_bf16"
DECODE = "gdn2_decode_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------------------------
# algorithmic work per token (all heads of one token), from the recurrence's definition
# --------------------------------------------------------------------------------------------
def _es(dt):
    return 4 if dt == "f32" else 2


def fwd_bytes_per_token(wl, T=None, with_h0=None, gate=False):
    """API-level bytes of one forward token: inputs read + output written (+ states amortised)."""
    T = T or wl.T
    es, gs = _es(wl.dtype), _es(wl.gate_dtype)
    b = wl.Hk * 2 * wl.dk * es                                     # q, k
    b += wl.Hv * wl.dv * es * 2                                    # v, o
    b += wl.Hv * (wl.dk if wl.alpha_per_channel else 1) * gs       # alpha
    b += wl.Hv * ((wl.dk + wl.dv) if wl.gates_per_channel else 1) * gs  # b, w or beta
    if gate:
        b += wl.Hv * wl.dv * es                                    # z
    nstates = 1 + (1 if (wl.has_h0 if with_h0 is None else with_h0) else 0)
    b += nstates * wl.Hv * wl.dk * wl.dv * 4 / T
    return b


def bwd_bytes_per_token(wl, T=None):
    """API-level bytes of one backward token: q, k, v, alpha, b, w and dO read; the gradients of
    q, k, v, alpha, b, w written in their inputs' dtypes (+ h0 read, dh0 written in fp32)."""
    T = T or wl.T
    es, gs = _es(wl.dtype), _es(wl.gate_dtype)
    ges, ggs = es, gs
    n_qk = wl.Hk * 2 * wl.dk
    n_v = wl.Hv * wl.dv
    n_a = wl.Hv * (wl.dk if wl.alpha_per_channel else 1)
    n_g = wl.Hv * ((wl.dk + wl.dv) if wl.gates_per_channel else 1)
    b = (n_qk + n_v) * es + (n_a + n_g) * gs + n_v * es           # inputs and dO read
    b += (n_qk + n_v) * ges + (n_a + n_g) * ggs                    # gradients written
    b += (2 if wl.has_h0 else 1) * wl.Hv * wl.dk * wl.dv * 4 / T   # h0 read, dh0 written
    return b


def fwd_flops_per_token(wl, C=64):
    d = wl.dk
    return wl.Hv * (5 * 2 * C * d + 3 * 2 * d * d)


def bwd_flops_per_token(wl, C=64):
    return 2 * fwd_flops_per_token(wl, C) + wl.Hv * 4 * C * C


def decode_bytes_per_token(wl):
    es, gs = _es(wl.dtype), _es(wl.gate_dtype)
    b = wl.Hv * 2 * wl.dk * wl.dv * 4                              # state read + write
    b += wl.Hk * 2 * wl.dk * es + wl.Hv * 2 * wl.dv * es           # q, k, v, o
    b += wl.Hv * ((wl.dk if wl.alpha_per_channel else 1) + ((wl.dk + wl.dv) if wl.gates_per_channel else 1)) * gs
    return b


def decode_flops_per_token(wl):
    return wl.Hv * 7 * wl.dk * wl.dv


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (read + write) of one gdn_chunk_bwd call on the headline workload, summed over its two
# kernels (reverse scan 341,024,768 B, gradients 811,200,512 B) from ncu's dram__bytes_read.sum +
# dram__bytes_write.sum on B=8 T=1024 (the same 128 (sequence, head) pairs, a quarter of the
# chunks; the traffic is per chunk, so x4).  To be reset to None whenever those kernels change.
BWD_CALL_TRAFFIC_BYTES = (341024768 + 811200512) * 4


def roofline(bytes_per_launch, flops_per_launch, seconds, peaks, peak_kind, scope, sustained=False,
             traffic=None):
    t_mem = bytes_per_launch / (peaks["hbm_gbs"] * 1e9)
    fpk = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_flop = flops_per_launch / (fpk * 1e12)
    if t_mem >= t_flop:
        achieved = bytes_per_launch / seconds / 1e9
        out = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "frac": round(achieved / peaks["hbm_gbs"], 4)}
    else:
        achieved = flops_per_launch / seconds / 1e12
        out = {"bound": "tensor", "achieved": round(achieved, 2), "peak": fpk, "unit": "TFLOP/s",
               "frac": round(achieved / fpk, 4)}
    out.update({"traffic": None if traffic is None else int(traffic), "peak_source": peak_kind, "scope": scope,
                "algorithmic_bytes": int(bytes_per_launch), "algorithmic_flops": int(flops_per_launch)})
    return out


# --------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["index", "pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, bus_id=None, index=None):
        self.bus_id, self.index = bus_id, index
        self.proc = None
        self.out = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.out.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        rows = []
        for line in self.out:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            if self.bus_id and parts[1].lower()[-12:] != self.bus_id.lower()[-12:]:
                continue
            if self.bus_id is None and self.index is not None and parts[0] != str(self.index):
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[2]) for r in rows]
        smax = max(float(r[3]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        power = [float(r[4]) for r in rows if r[4] not in ("[N/A]", "")]
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


# --------------------------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------------------------
class Dist:
    """One process per GPU: NCCL for the timing reduction (gloo on CPU, for the host-logic tests).
    Every rank takes the same collective steps: one barrier on each side of a timed region and one
    max-reduction of its elapsed time."""

    def __init__(self, ngpus, backend=None):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cuda"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = backend or "nccl"
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            else:
                self.device = "cpu"
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600), **kw)
            self.pg = dist
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def timed(fn, steps, warmup, dist, stream):
    """Device time per step (ms) of fn(), CUDA events on `stream`, max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    ms = a.elapsed_time(b) / steps
    return dist.max(ms)


# --------------------------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------------------------
def chunk_inputs(name, device, with_dout):
    import torch
    from gated_delta_rule_76_b200.inputs import workload_inputs
    x = workload_inputs(name, with_dout=with_dout)
    return x, {k: v.to(device) for k, v in x.items() if torch.is_tensor(v)}


def gates(g):
    return dict(beta=g["beta"]) if "beta" in g else dict(b=g["b"], w=g["w"])


def bench_headline(args, dist, peaks, peak_kind, stream, device):
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS
    wl = WORKLOADS[HEADLINE]
    x, g = chunk_inputs(HEADLINE, device, with_dout=True)
    B, T = wl.B, wl.T
    o = torch.empty_like(g["v"])
    ht = torch.empty((B, wl.Hv, wl.dk, wl.dv), dtype=torch.float32, device=device)
    import ctypes
    lib = gdn.load()
    # the forward keeps what the backward needs (chunk states, V') in a cache: training's forward +
    # backward, without recomputing the forward inside the backward
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], **gates(g)),
                        dtype=torch.uint8, device=device)
    fa, _ = gdn.fwd_args(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], o=o, ht=ht, bwd_cache=cache, **gates(g))
    ws_f = torch.empty(lib.gdn_chunk_fwd_workspace_size(ctypes.byref(fa)), dtype=torch.uint8, device=device)
    # gradients in the inputs' dtype (bf16; fp32 accumulation inside), dh0 in fp32
    grads = {"dq": torch.empty_like(g["q"]), "dk": torch.empty_like(g["k"]), "dv": torch.empty_like(g["v"]),
             "dalpha": torch.empty_like(g["alpha"]), "db": torch.empty_like(g["b"]), "dw": torch.empty_like(g["w"]),
             "dh0": torch.empty_like(g["h0"])}
    ba, _ = gdn.bwd_args(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], grads=grads,
                         fwd_cache=cache, grads_in_dtype=True, **gates(g))
    ws_b = torch.empty(lib.gdn_chunk_bwd_workspace_size(ctypes.byref(ba)), dtype=torch.uint8, device=device)
    sptr = ctypes.c_void_p(stream.cuda_stream)

    def fwd():
        gdn.check(lib.gdn_chunk_fwd(ctypes.byref(fa), ctypes.c_void_p(ws_f.data_ptr()), ws_f.numel(), sptr), "fwd")

    def bwd():
        gdn.check(lib.gdn_chunk_bwd(ctypes.byref(ba), ctypes.c_void_p(ws_b.data_ptr()), ws_b.numel(), sptr), "bwd")

    # per-call device times inside the timed step (for the dominant call's roofline)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    per_call = {"fwd": [], "bwd": []}

    def step_timed():
        ev[0].record(stream)
        fwd()
        ev[1].record(stream)
        bwd()
        ev[2].record(stream)

    launches0 = gdn.kernel_launches()
    with torch.cuda.stream(stream):
        ms = timed(lambda: (fwd(), bwd()), args.steps, args.warmup, dist, stream)
    launches = gdn.kernel_launches() - launches0
    launches_per_step = launches // (args.steps + args.warmup)
    # separate pass for the per-call split (not part of the headline number)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.steps // 2)):
            step_timed()
            torch.cuda.synchronize()
            per_call["fwd"].append(ev[0].elapsed_time(ev[1]))
            per_call["bwd"].append(ev[1].elapsed_time(ev[2]))
    fwd_ms = float(np.mean(per_call["fwd"]))
    bwd_ms = float(np.mean(per_call["bwd"]))
    tokens = B * T
    bytes_f = fwd_bytes_per_token(wl) * tokens
    bytes_b = bwd_bytes_per_token(wl) * tokens
    flops_f = fwd_flops_per_token(wl) * tokens
    flops_b = bwd_flops_per_token(wl) * tokens
    dominant = "bwd" if bwd_ms >= fwd_ms else "fwd"
    dom = {"fwd": (bytes_f, flops_f, fwd_ms), "bwd": (bytes_b, flops_b, bwd_ms)}[dominant]
    roof = roofline(dom[0], dom[1], dom[2] * 1e-3, peaks, peak_kind,
                    f"gdn_chunk_{dominant} call (dominant call of the step; its kernels back to back)",
                    traffic=BWD_CALL_TRAFFIC_BYTES if dominant == "bwd" else None)
    step_roof = roofline(bytes_f + bytes_b, flops_f + flops_b, ms * 1e-3, peaks, peak_kind,
                         "whole fwd+bwd step")
    return {"ms": ms, "tokens": tokens, "launches_per_step": launches_per_step, "fwd_ms": fwd_ms,
            "bwd_ms": bwd_ms, "roofline": roof, "step_roofline": step_roof,
            "fwd_roofline": roofline(bytes_f, flops_f, fwd_ms * 1e-3, peaks, peak_kind, "gdn_chunk_fwd call")}, (x, g, o, ht, grads)


def bench_headline_e2e(args, dist, x, stream, device, slices=8):
    """Same metric through the public API with host buffers: H2D of the step's inputs from pinned
    memory, forward + backward, D2H of every result, all inside the timed region.  The batch's
    sequences are independent, so the step runs as `slices` slices of the batch on three streams
    (copy in, compute, copy out): the copies of one slice overlap the compute and the
    other-direction copies of the others, and the PCIe link carries both directions at once.
    The device inputs are double-buffered across steps, so that a step's copies in overlap the
    previous step's copies out; a set is overwritten only after the compute that read it two
    steps before."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    names_in = ["q", "k", "v", "alpha", "b", "w", "h0", "dout"]
    host = {n: x[n].pin_memory() for n in names_in}
    dev = {n: torch.empty_like(host[n], device=device) for n in names_in}
    dev_sets = [dev, {n: torch.empty_like(host[n], device=device) for n in names_in}]
    set_free = [None, None]  # per set: an event on `stream` after the last compute that read it
    n_steps = [0]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    B = host["q"].shape[0]
    ns = slices if B % slices == 0 else 1
    sb = B // ns
    cut = lambda t, i: t[i * sb:(i + 1) * sb]
    caches = [torch.empty(gdn.gdn_chunk_fwd_cache_size(cut(dev["q"], i), cut(dev["k"], i), cut(dev["v"], i),
                                                       cut(dev["alpha"], i), b=cut(dev["b"], i), w=cut(dev["w"], i),
                                                       h0=cut(dev["h0"], i)), dtype=torch.uint8, device=device)
              for i in range(ns)]
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    out_host = {}

    def step():
        cur = n_steps[0] & 1
        n_steps[0] += 1
        dset = dev_sets[cur]
        if set_free[cur] is not None:
            s_in.wait_event(set_free[cur])
        ev_in = []
        with torch.cuda.stream(s_in):
            for i in range(ns):
                for n in names_in:
                    cut(dset[n], i).copy_(cut(host[n], i), non_blocking=True)
                ev_in.append(torch.cuda.Event())
                ev_in[-1].record(s_in)
        res, ev_c = [], []
        for i in range(ns):
            stream.wait_event(ev_in[i])
            d = {n: cut(dset[n], i) for n in names_in}
            o, ht = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], b=d["b"], w=d["w"], h0=d["h0"],
                                      bwd_cache=caches[i], stream=stream)
            gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], b=d["b"], w=d["w"], h0=d["h0"],
                                   grad_o=d["dout"], fwd_cache=caches[i], grads_in_dtype=True, stream=stream)
            res.append({"o": o, "ht": ht, **gr})
            ev_c.append(torch.cuda.Event())
            ev_c[-1].record(stream)
        set_free[cur] = ev_c[-1]
        with torch.cuda.stream(s_out):
            for i in range(ns):
                s_out.wait_event(ev_c[i])
                for n, t in res[i].items():
                    if n not in out_host:
                        out_host[n] = torch.empty((B,) + tuple(t.shape[1:]), dtype=t.dtype, pin_memory=True)
                    cut(out_host[n], i).copy_(t, non_blocking=True)
        # the timing stream ends after the last copy; the slices' device outputs are released
        # only after that point in stream order
        stream.wait_stream(s_out)

    with torch.cuda.stream(stream):
        ms = timed(step, max(2, args.steps // 4), 1, dist, stream)
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    return ms, h2d, d2h


def bench_decode(args, dist, peaks, peak_kind, stream, device):
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS, decode_initial_state, decode_inputs
    wl = WORKLOADS[DECODE]
    steps = wl.decode_steps
    xs = decode_inputs(DECODE, steps, threads=min(16, os.cpu_count() or 4))
    g = {k: v.to(device) for k, v in xs.items()}
    state = decode_initial_state(DECODE).to(device)
    o = torch.empty((steps, wl.B, wl.Hv, wl.dv), dtype=torch.bfloat16, device=device)

    def run_all():
        for s in range(steps):
            gdn.gdn_decode_step(state, g["q"][s], g["k"][s], g["v"][s], g["alpha"][s], b=g["b"][s],
                                w=g["w"][s], o=o[s], stream=stream)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        run_all()  # warm up (sets kernel attributes) before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            run_all()
        launches0 = gdn.kernel_launches()
        ms = timed(graph.replay, max(2, args.steps // 4), max(1, args.warmup // 2), dist, stream)
    tokens = wl.B * steps
    per_step_s = ms * 1e-3 / steps
    roof = roofline(decode_bytes_per_token(wl) * wl.B, decode_flops_per_token(wl) * wl.B, per_step_s, peaks,
                    peak_kind, "decode_step_kernel (one launch = one token for 256 sequences x 16 heads)")

    # e2e: per step, H2D of that step's inputs (pinned) and D2H of its output.
    host = {k: v.pin_memory() for k, v in xs.items()}
    dev = {k: torch.empty_like(v[0], device=device) for k, v in xs.items()}
    oh = torch.empty((steps,) + tuple(o.shape[1:]), dtype=o.dtype, pin_memory=True)
    e2e_steps = 256

    def e2e():
        for s in range(e2e_steps):
            for k in dev:
                dev[k].copy_(host[k][s], non_blocking=True)
            gdn.gdn_decode_step(state, dev["q"], dev["k"], dev["v"], dev["alpha"], b=dev["b"], w=dev["w"],
                                o=o[s], stream=stream)
            oh[s].copy_(o[s], non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_ms = timed(e2e, 2, 1, dist, stream)
    h2d = sum(v[0].numel() * v.element_size() for v in host.values())
    d2h = o[0].numel() * o.element_size()
    return {"workload": DECODE, "value": tokens / (ms * 1e-3) * dist.world, "unit": "tokens/s",
            "ms_per_1024_tokens": round(ms, 4), "us_per_token_step": round(per_step_s * 1e6, 2),
            "graph": True, "roofline": roof,
            "e2e": {"value": e2e_steps * wl.B / (e2e_ms * 1e-3) * dist.world, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
            "config": {"N": wl.B, "H": wl.Hv, "dk": wl.dk, "dv": wl.dv, "steps": steps,
                       "state_bytes": wl.B * wl.Hv * wl.dk * wl.dv * 4, "l2": "state (268 MB) larger than L2"}}


def bench_part_fwd(name, args, dist, peaks, peak_kind, stream, device):
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS
    wl = WORKLOADS[name]
    x, g = chunk_inputs(name, device, with_dout=False)
    o = torch.empty_like(g["v"])
    ws = None
    with torch.cuda.stream(stream):
        if wl.conv:
            def fn():
                gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], y=o,
                                       want_ht=True, stream=stream, **gates(g))
        else:
            def fn():
                gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g.get("h0"), o=o, stream=stream,
                                  **gates(g))
        ms = timed(fn, max(2, args.steps // 2), args.warmup, dist, stream)
    tokens = wl.B * wl.T
    by = fwd_bytes_per_token(wl, gate=wl.swish_gate) * tokens
    if wl.conv:
        by += (2 * wl.Hk * wl.dk + wl.Hv * wl.dv) * 4 * _es(wl.dtype) / wl.T * wl.B * 0  # weights: negligible
    fl = fwd_flops_per_token(wl) * tokens
    del x, g
    return {"workload": name, "value": tokens / (ms * 1e-3) * dist.world, "unit": "tokens/s",
            "ms_per_step": round(ms, 4),
            "roofline": roofline(by, fl, ms * 1e-3, peaks, peak_kind,
                                 "gdn_layer_core_fwd call" if wl.conv else "gdn_chunk_fwd call"),
            "config": {"B": wl.B, "T": wl.T, "Hk": wl.Hk, "Hv": wl.Hv, "dk": wl.dk, "dv": wl.dv,
                       "alpha": "channel" if wl.alpha_per_channel else "scalar",
                       "gates": "channel" if wl.gates_per_channel else "scalar beta"}}


def bench_part_layer_train(args, dist, peaks, peak_kind, stream, device):
    """The GQA layer core's training step: gdn_layer_core_fwd keeping its cache, then
    gdn_layer_core_bwd reading it (the recurrence's backward on the tensor cores, once per bf16
    half of do), inputs resident, gradients of every input."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS
    name = "gqa_layer_core_bf16"
    wl = WORKLOADS[name]
    x, g = chunk_inputs(name, device, with_dout=True)
    y = torch.empty_like(g["v"])
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, **gates(g)), dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        def fn():
            gdn.gdn_layer_core_fwd(*lin, y=y, want_ht=False, bwd_cache=cache, stream=stream, **gates(g))
            gdn.gdn_layer_core_bwd(*lin, g["dout"], fwd_cache=cache, stream=stream, **gates(g))
        ms = timed(fn, max(2, args.steps // 4), args.warmup, dist, stream)
    tokens = wl.B * wl.T
    by = (fwd_bytes_per_token(wl, gate=True) + bwd_bytes_per_token(wl)
          + wl.Hv * wl.dv * 2 * _es(wl.dtype)) * tokens                 # + z read, dz written
    fl = (fwd_flops_per_token(wl) + bwd_flops_per_token(wl)) * tokens
    del x, g
    return {"workload": name + " (training step: layer forward + backward)",
            "value": tokens / (ms * 1e-3) * dist.world, "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "roofline": roofline(by, fl, ms * 1e-3, peaks, peak_kind,
                                 "gdn_layer_core_fwd + gdn_layer_core_bwd calls"),
            "config": {"B": wl.B, "T": wl.T, "Hk": wl.Hk, "Hv": wl.Hv, "dk": wl.dk, "dv": wl.dv,
                       "backward": "from the forward's cache (conv results as bf16 hi/lo pairs, o, states, V'); "
                                   "recurrence on the tensor-core backward kernels, once per bf16 half of do"}}


# --------------------------------------------------------------------------------------------
# CPU oracle timings (baseline and reference arm)
# --------------------------------------------------------------------------------------------
def oracle_sample_run(x, nb, threads):
    """Oracle forward + backward over the first nb sequences of the headline batch."""
    from oracle import oracle
    sl = {k: v[:nb] for k, v in x.items()}
    t0 = time.perf_counter()
    oracle.fwd(sl["q"], sl["k"], sl["v"], sl["alpha"], b=sl["b"], w=sl["w"], h0=sl["h0"], nthreads=threads)
    oracle.bwd(sl["q"], sl["k"], sl["v"], sl["alpha"], b=sl["b"], w=sl["w"], h0=sl["h0"],
               dout=sl["dout"], nthreads=threads)
    return time.perf_counter() - t0


def cpu_threads():
    from oracle import oracle
    return oracle.threads()


def cpu_baseline(x, wl):
    threads = cpu_threads()
    nb = 1
    secs = oracle_sample_run(x, nb, threads)
    tokens = nb * wl.T
    return {"value": round(tokens / secs, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle forward+backward of {nb} of {wl.B} sequences ({nb * wl.Hv} (batch, head) "
                      f"pairs x {wl.T} tokens, all heads of a token counted once), {secs:.1f} s wall"}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle, as it stands, on the headline workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_76_b200.inputs import WORKLOADS, workload_inputs
    wl = WORKLOADS[HEADLINE]
    x = workload_inputs(HEADLINE, with_dout=True, B=1)
    threads = cpu_threads()
    for _ in range(args.warmup):
        oracle_sample_run(x, 1, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_run(x, 1, threads)
    secs = (time.perf_counter() - t0) / args.steps
    value = wl.T / secs
    line = {"metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": HEADLINE, "B": wl.B, "T": wl.T, "H": wl.Hv,
                                            "dk": wl.dk, "dv": wl.dv, "chunk": 64},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"one of {wl.B} sequences per step (16 (batch, head) pairs x {wl.T} "
                                       f"tokens), forward + backward, fp64 sequential recurrence"},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
def _profile_train_b2_t2048():
    """GDN-2 training step on B=2 T=2048 H=16 d=128 bf16 (seed 21), twice: the forward keeping the
    backward cache, then the backward from it (gradients in bf16, as the benchmark takes them)."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import draw
    x = draw(2, 2048, 16, 16, 128, 128, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=21, has_h0=True, with_dout=True)
    g = {k: v.cuda() for k, v in x.items()}
    kw = dict(b=g["b"], w=g["w"], h0=g["h0"])
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw),
                        dtype=torch.uint8, device="cuda")
    for _ in range(2):
        gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], bwd_cache=cache, **kw)
        grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], fwd_cache=cache,
                                  grads_in_dtype=True, **kw)
    torch.cuda.synchronize()
    print("ok", float(grads["dq"].float().abs().mean()))
    return 0


def _profile_train_b8_t1024():
    """GDN-2 training step on B=8 T=1024 H=16 d=128 bf16 (seed 21): the headline's 128 (sequence, head)
    pairs, a quarter of its tokens; twice: the forward keeping the cache, then the backward from it
    (gradients in bf16, as the benchmark takes them)."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import draw
    x = draw(8, 1024, 16, 16, 128, 128, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=21, has_h0=True, with_dout=True)
    g = {k: v.cuda() for k, v in x.items()}
    kw = dict(b=g["b"], w=g["w"], h0=g["h0"])
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw),
                        dtype=torch.uint8, device="cuda")
    for _ in range(2):
        gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], bwd_cache=cache, **kw)
        grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], fwd_cache=cache,
                                  grads_in_dtype=True, **kw)
    torch.cuda.synchronize()
    print("ok", float(grads["dq"].float().abs().mean()))
    return 0


def _profile_fwd_b8_t1024():
    """GDN-2 forward on B=8 T=1024 H=16 d=128 bf16 (seed 21), twice, without a cache."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import draw
    x = draw(8, 1024, 16, 16, 128, 128, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=21, has_h0=True)
    g = {k: v.cuda() for k, v in x.items()}
    for _ in range(2):
        o, _ = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"])
    torch.cuda.synchronize()
    print("ok", float(o.float().abs().mean()))
    return 0


def _profile_layer_b2_t16384():
    """GQA layer core (conv k=4 + SiLU + L2, chunk forward, swish gate) on its full workload
    (B=2 T=16384, 16 key / 128 value heads, d=128 bf16, seed of the workload), twice."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import workload_inputs
    x = workload_inputs("gqa_layer_core_bf16")
    g = {k: v.cuda() for k, v in x.items()}
    for _ in range(2):
        y, _, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], beta=g["beta"])
    torch.cuda.synchronize()
    print("ok", float(y.float().abs().mean()))
    return 0


def _profile_train_b8_t4096():
    """The headline training step (gdn_chunk_fwd keeping the cache, gdn_chunk_bwd from it, gradients
    in bf16) on its full workload, three times."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    x, g = chunk_inputs(HEADLINE, torch.device("cuda"), with_dout=True)
    kw = dict(b=g["b"], w=g["w"], h0=g["h0"])
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw),
                        dtype=torch.uint8, device="cuda")
    for _ in range(3):
        gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], bwd_cache=cache, **kw)
        grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], fwd_cache=cache,
                                  grads_in_dtype=True, **kw)
    torch.cuda.synchronize()
    print("ok", float(grads["dq"].float().abs().mean()))
    return 0


def _profile_layer_train_b2_t16384():
    """GQA layer core's training step (gdn_layer_core_fwd, then gdn_layer_core_bwd) on its full
    workload, once."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import workload_inputs
    x = workload_inputs("gqa_layer_core_bf16", with_dout=True)
    g = {k: v.cuda() for k, v in x.items()}
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, beta=g["beta"]), dtype=torch.uint8, device="cuda")
    y, _, _ = gdn.gdn_layer_core_fwd(*lin, beta=g["beta"], bwd_cache=cache)
    grads = gdn.gdn_layer_core_bwd(*lin, g["dout"], beta=g["beta"], fwd_cache=cache)
    torch.cuda.synchronize()
    print("ok", float(y.float().abs().mean()), float(grads["dxq"].abs().mean()))
    return 0


def _profile_decode_b256():
    """GDN-2 decode on its full workload shape (256 sequences, 16 heads, d=128, fp32 state of
    268 MB), 8 consecutive steps."""
    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS, decode_initial_state, decode_inputs
    wl = WORKLOADS[DECODE]
    xs = decode_inputs(DECODE, 8)
    g = {k: v.cuda() for k, v in xs.items()}
    state = decode_initial_state(DECODE).cuda()
    for s in range(8):
        o = gdn.gdn_decode_step(state, g["q"][s], g["k"][s], g["v"][s], g["alpha"][s], b=g["b"][s], w=g["w"][s])
    torch.cuda.synchronize()
    print("ok", float(o.float().abs().mean()), wl.B)
    return 0


PROFILE_CASES = {"decode_b256": _profile_decode_b256, "train_b2_t2048": _profile_train_b2_t2048,
                 "train_b8_t1024": _profile_train_b8_t1024, "fwd_b8_t1024": _profile_fwd_b8_t1024,
                 "layer_b2_t16384": _profile_layer_b2_t16384, "train_b8_t4096": _profile_train_b8_t4096,
                 "layer_train_b2_t16384": _profile_layer_train_b2_t16384}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parts", default="all", help="all | headline | comma list of: decode,fwd,gdn,layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None, choices=sorted(PROFILE_CASES),
                    help="run one small untimed case for an ncu capture (prints 'ok') and exit")
    args = ap.parse_args()
    if args.profile_case:
        return PROFILE_CASES[args.profile_case]()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    from gated_delta_rule_76_b200 import gdn
    from gated_delta_rule_76_b200.inputs import WORKLOADS
    gdn.load()  # fail loudly if the CUDA library is missing
    dist = Dist(args.gpus)
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream(device=device)
    peaks, peak_kind = load_peaks()
    props = torch.cuda.get_device_properties(device)
    bus = getattr(props, "pci_bus_id", None)
    if isinstance(bus, int):
        bus = None
    parts = {"decode", "fwd", "gdn", "layer"} if args.parts == "all" else (
        set() if args.parts == "headline" else set(args.parts.split(",")))
    if dist.world > 1 and args.parts == "all":
        parts = {"decode"}

    clocks = ClockSampler(bus_id=bus, index=dist.local)
    clocks.start()
    head, keep = bench_headline(args, dist, peaks, peak_kind, stream, device)
    x = keep[0]
    del keep
    torch.cuda.empty_cache()
    e2e_ms, h2d, d2h = bench_headline_e2e(args, dist, x, stream, device)
    torch.cuda.empty_cache()
    extra = {}
    if "decode" in parts:
        extra["decode"] = bench_decode(args, dist, peaks, peak_kind, stream, device)
        torch.cuda.empty_cache()
    sub = {}
    if "fwd" in parts:
        # the forward alone (inference: no backward cache), then the training step's forward
        sub["gdn2_fwd"] = bench_part_fwd(HEADLINE, args, dist, peaks, peak_kind, stream, device)
        torch.cuda.empty_cache()
        sub["gdn2_fwd_keeping_cache"] = {"workload": HEADLINE,
                                         "value": head["tokens"] / (head["fwd_ms"] * 1e-3) * dist.world,
                                         "unit": "tokens/s", "ms_per_step": round(head["fwd_ms"], 4),
                                         "roofline": head["fwd_roofline"]}
    if "gdn" in parts:
        sub["gdn_fwd_scalar"] = bench_part_fwd("gdn_fwd_scalar_bf16", args, dist, peaks, peak_kind, stream, device)
        torch.cuda.empty_cache()
    if "layer" in parts:
        sub["gqa_layer_core"] = bench_part_fwd("gqa_layer_core_bf16", args, dist, peaks, peak_kind, stream, device)
        torch.cuda.empty_cache()
        sub["gqa_layer_train"] = bench_part_layer_train(args, dist, peaks, peak_kind, stream, device)
        torch.cuda.empty_cache()
    clk = clocks.stop()

    wl = WORKLOADS[HEADLINE]
    value = head["tokens"] * dist.world / (head["ms"] * 1e-3)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(head["ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy draws, recipe in gated_delta_rule_76_b200/inputs.py)",
        "config": {"workload": HEADLINE, "B": wl.B, "T": wl.T, "H": wl.Hv, "dk": wl.dk, "dv": wl.dv,
                   "chunk": 64, "state": "fp32", "gates": "channel alpha, b, w (bf16)",
                   "parallelism": f"dp{dist.world} (independent replicas of the workload)",
                   "l2": "inputs larger than L2 (~0.9 GB read per step); no flush needed",
                   "step": "gdn_chunk_fwd (keeping the backward cache) + gdn_chunk_bwd (from the cache)"},
        "roofline": head["roofline"],
        "step_roofline": head["step_roofline"],
        "fwd_ms": round(head["fwd_ms"], 4), "bwd_ms": round(head["bwd_ms"], 4),
        "e2e": {"value": round(head["tokens"] * dist.world / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(head["launches_per_step"] * args.steps),
        "clocks": clk,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x, wl)
    # the other workloads last: a reader that keeps only the line's tail still sees them, and
    # the line ends with a compact summary of every workload's rate and roofline fraction
    line.update(extra)
    if sub:
        line["parts"] = sub
    summary = {"step_frac": head["step_roofline"]["frac"], "bwd_frac": head["roofline"]["frac"],
               "fwd_keeping_cache_frac": head["fwd_roofline"]["frac"]}
    if "decode" in extra:
        summary["decode_tokens_s"] = round(extra["decode"]["value"], 1)
        summary["decode_frac"] = extra["decode"]["roofline"]["frac"]
    for key, part in sub.items():
        summary[key + "_tokens_s"] = round(part["value"], 1)
        summary[key + "_frac"] = part["roofline"]["frac"]
    line["summary"] = summary
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
