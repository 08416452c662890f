"""Benchmark: routed-expert decode (and prefill) on B200 through the C ABI.

Headline (N=1 and every rank at N>1): IQ2_KS routed-expert decode, one token
per call, 256 experts, top-6, gate/up [2048 x 4096], down [4096 x 2048]
(seeded synthetic streams, bf16 N(0,1) activations, softmax routing weights).
A step is one decode call; consecutive calls take their experts from a chain
of random permutations, so no expert repeats within 42 calls and the 41 MB a
call reads are never resident in the 126 MB L2. Steps are captured once into
CUDA graphs and replayed; device time comes from CUDA events on the launching
stream, max over ranks.

Printed: one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import iqk_synth as S  # noqa: E402

METRIC = "MoE decode µs/token & weight GB/s vs HBM floor; prefill bf16 TFLOP/s"
RING = 420  # calls per captured graph (10 permutation cycles of 42 calls)


# DRAM bytes (read + write) of the two tile kernels of one headline decode
# call (IQ2_KS, 256 experts, top-6, one token), from one ncu capture of
# `bench.py --profile decode --experts 24` (its summary is kept under
# profiles/); per call, not per resident expert.
DECODE_CALL_TRAFFIC = 42_272_768  # 27,812,864 (gate/up) + 14,459,904 (down), all reads


def env_int(k, d):
    try:
        return int(os.environ.get(k, d))
    except ValueError:
        return d


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with nvidia-smi (50 ms period)
    over a window of back-to-back replays that contains the timed region;
    only this GPU's lines (by PCI bus id) count."""

    REASONS = {
        0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x10: "sync_boost",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, props):
        # nvidia-smi prints e.g. 00000000:1B:00.0; match on bus:device.function
        try:
            self.bus = f"{int(props.pci_bus_id):02x}:{int(props.pci_device_id):02x}.0"
        except Exception:
            self.bus = ""
        self.samples, self.max_mhz, self.reasons = [], None, set()
        self.proc = None

    def __enter__(self):
        import subprocess
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=pci.bus_id,clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 4 or (self.bus and not f[0].lower().endswith(self.bus)):
                continue
            try:
                self.samples.append(float(f[1]))
                self.max_mhz = float(f[2])
                r = int(f[3], 16)
            except ValueError:
                continue
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- helpers

def cuda_time(torch, stream, fn):
    """Device seconds of fn's work: fn runs with `stream` current (graph
    replays launch on the current stream) between two events on it. A short
    device-side delay (about 0.5 ms of spinning) goes ahead of the first
    event, so that the host has enqueued fn's launches by the time that event
    fires: the interval is device time only, not host launch latency."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(1_000_000)
        a.record(stream)
        fn()
        b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) * 1e-3  # seconds


def job_time(torch, dist, t_local, steps, world, device):
    """Max over ranks of the timed region (one all-reduce), and the whole-job
    µs per token: every rank runs `steps` single-token calls of its own."""
    t = float(t_local)
    if dist is not None:
        tt = torch.tensor([t], dtype=torch.float64, device=device)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t = float(tt.item())
    return t, t / (steps * world) * 1e6


def log(msg):
    print(f"[bench {time.strftime('%H:%M:%S')}] {msg}", file=sys.stderr, flush=True)


def capture(torch, stream, fn, mode="global"):
    """Capture fn's launches into a CUDA graph. Every C-ABI path captured here
    has run once eagerly first, so no attribute/occupancy query happens
    inside the capture (mode "relaxed" for calls that query pointer types)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream, capture_error_mode=mode):
            fn()
    return g


def run_steps(graphs, K):
    """Replay graphs so that exactly K steps run (full rings, then a remainder)."""
    full, rem_graphs = graphs
    for _ in range(K // RING):
        full.replay()
    r = K % RING
    if r:
        rem_graphs[r].replay()


class DecodeBench:
    """One routed-expert decode workload (format, token count) resident on the GPU."""

    def __init__(self, torch, B, weights, values, T, seed, device, stream, remainders=()):
        self.torch, self.B, self.T, self.stream = torch, B, T, stream
        gate, up, down = weights
        E = gate.experts
        self.dw = [B.Weights.from_host(w, device) for w in weights]
        self.host_w = weights
        rng = S.rng_for(seed)
        ids = np.empty((RING, T, S.TOPK), np.int32)
        p = np.empty((RING, T, S.TOPK), np.float32)
        if T == 1:
            ids, p = S.routing_ring(rng, RING, E, S.TOPK)
        else:
            for c in range(RING):
                ids[c], p[c] = S.routing(rng, T, E, S.TOPK)
        x = S.random_bf16(rng, (RING, T, S.HIDDEN))
        self.ids_h, self.p_h, self.x_h = ids, p, x
        self.ids = torch.from_numpy(ids).to(device)
        self.p = torch.from_numpy(p).to(device)
        self.x = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        self.y = torch.empty((RING, T, S.HIDDEN), dtype=torch.bfloat16, device=device)
        ws_bytes = B.iqk_moe_workspace_bytes(0, T, S.TOPK, E, S.HIDDEN, S.INTER)
        self.ws = B.workspace(ws_bytes, device)
        self.distinct = np.array([len(np.unique(ids[c])) for c in range(RING)])
        self.bytes_per_expert = sum(w.nbytes() // w.experts for w in weights)
        self.values = values
        self.remainders = remainders

    def call(self, c):
        B = self.B
        g, u, d = self.dw
        B.iqk_moe_decode(g, u, d, self.values, self.x[c], self.ids[c], self.p[c], y=self.y[c], ws=self.ws,
                         stream=self.stream)

    def graphs(self):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            self.call(0)
        torch.cuda.synchronize()
        full = capture(torch, self.stream, lambda: [self.call(c) for c in range(RING)])
        rem = {r: capture(torch, self.stream, lambda r=r: [self.call(c) for c in range(r)]) for r in self.remainders}
        return full, rem

    def weight_bytes(self, calls):
        return float(sum(self.distinct[c % RING] for c in range(calls))) * self.bytes_per_expert


def e2e_graph(torch, bench, stream, n):
    """n steps, each one iqk_moe_decode_host call on that step's inputs (x,
    ids, p) in page-locked host memory, writing y to page-locked host memory:
    the call's kernels read the inputs over the host link and write y back."""
    T = bench.T
    hx = torch.stack([bench.x[c].cpu() for c in range(n)]).pin_memory()
    hids = torch.stack([bench.ids[c].cpu() for c in range(n)]).pin_memory()
    hp = torch.stack([bench.p[c].cpu() for c in range(n)]).pin_memory()
    hy = torch.empty((n, T, S.HIDDEN), dtype=torch.bfloat16, pin_memory=True)
    g, u, d = bench.dw

    with torch.cuda.stream(stream):
        bench.B.iqk_moe_decode_host(g, u, d, bench.values, hx[0], hids[0], hp[0], y=hy[0], ws=bench.ws, stream=stream)
    torch.cuda.synchronize()

    def body():
        for c in range(n):
            bench.B.iqk_moe_decode_host(g, u, d, bench.values, hx[c], hids[c], hp[c], y=hy[c], ws=bench.ws,
                                        stream=stream)

    graph = capture(torch, stream, body, mode="relaxed")
    h2d = hx[0].numel() * 2 + hids[0].numel() * 4 + hp[0].numel() * 4
    return graph, h2d, T * S.HIDDEN * 2, (hx, hids, hp, hy)


def floor_graph(torch, bench, stream, n):
    """The deleted-decode address floor over the same experts, n calls."""
    B = bench.B
    g, u, d = bench.dw
    lists = [torch.from_numpy(np.unique(bench.ids_h[c]).astype(np.int32)).to(bench.x.device) for c in range(n)]
    outs = [(torch.empty((len(l), g.rows), dtype=torch.int32, device=bench.x.device),
             torch.empty((len(l), d.rows), dtype=torch.int32, device=bench.x.device)) for l in lists]

    with torch.cuda.stream(stream):
        B.iqk_floor(g, lists[0], out=outs[0][0], stream=stream)
        B.iqk_floor(d, lists[0], out=outs[0][1], stream=stream)
    torch.cuda.synchronize()

    def body():
        for c in range(n):
            B.iqk_floor(g, lists[c], out=outs[c][0], stream=stream)
            B.iqk_floor(u, lists[c], out=outs[c][0], stream=stream)
            B.iqk_floor(d, lists[c], out=outs[c][1], stream=stream)

    return capture(torch, stream, body)


def prefill_leg(torch, B, weights, values, device, stream, peaks, calls=4, reps=3):
    """The prefill workload: 2048 tokens routed top-6 over 256 experts, one call =
    route + grouped gate/up GEMM + SwiGLU + grouped down GEMM + combine."""
    T = 2048
    rng = S.rng_for(4)
    ids, p = S.routing(rng, T, weights[0].experts, S.TOPK)
    x = S.random_bf16(rng, (T, S.HIDDEN))
    dw = [B.Weights.from_host(w, device) for w in weights]
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    idsd = torch.from_numpy(ids).to(device)
    pd = torch.from_numpy(p).to(device)
    y = torch.empty((T, S.HIDDEN), dtype=torch.bfloat16, device=device)
    ws = B.workspace(B.iqk_moe_workspace_bytes(1, T, S.TOPK, weights[0].experts, S.HIDDEN, S.INTER), device)

    def call():
        B.iqk_moe_prefill(dw[0], dw[1], dw[2], values, xd, idsd, pd, y=y, ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    g = capture(torch, stream, lambda: [call() for _ in range(calls)])
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    t = cuda_time(torch, stream, lambda: [g.replay() for _ in range(reps)])
    per_call = t / (calls * reps)
    flops = 2.0 * T * S.TOPK * 3 * S.INTER * S.HIDDEN
    tf = flops / per_call / 1e12
    status = B.iqk_moe_status(ws)
    del g, dw
    return {"workload": "routed-expert prefill, IQ2_KS, 2048 tokens, 256 experts top-6",
            "us_per_call": per_call * 1e6, "tflops": tf, "flop_per_call": flops,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16"], "frac_of_sustained": tf / peaks["bf16_sustained"],
                         "peak_source": peaks["source"] + " bf16_tflops (cuBLAS burst)"},
            "weight_gbs": sum(w.nbytes() for w in weights) / per_call / 1e9, "status": status}


def gemv_leg(torch, B, case, device, stream, calls=200, cold_copies=128):
    """A single-matrix workload: one matrix, one activation row. Warm: the
    same matrix every call (L2-resident). Cold: calls rotate over
    ``cold_copies`` distinct matrices of the same shape and distribution
    (more bytes than the 126 MB L2 for the 2048 x 4096 case), so each call's
    weights come from HBM."""
    w, x, values = S.matrix_case(case)
    dw = B.Weights.from_host(w)
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((xd.shape[0], w.rows), dtype=torch.float32, device=device)
    ws = B.workspace(B.iqk_gemv_workspace_bytes(xd.shape[0], w.rows, w.cols), device)
    with torch.cuda.stream(stream):
        B.iqk_gemv(dw, 0, values, xd, y=y, ws=ws, stream=stream)
    torch.cuda.synchronize()
    g = capture(torch, stream, lambda: [B.iqk_gemv(dw, 0, values, xd, y=y, ws=ws, stream=stream)
                                        for _ in range(calls)])
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    t = cuda_time(torch, stream, lambda: g.replay()) / calls
    nb = w.nbytes()
    out = {"us_per_call": t * 1e6, "weight_bytes": nb, "weight_gbs_l2_warm": nb / t / 1e9}
    if nb * cold_copies > 2 * 126e6:
        rng = S.rng_for(S.seed_of(case) + 50)
        stack = S.random_streams(rng, w.fmt, cold_copies, w.rows, w.cols)
        dstack = B.Weights.from_host(stack, device)
        with torch.cuda.stream(stream):
            B.iqk_gemv(dstack, 0, values, xd, y=y, ws=ws, stream=stream)
        torch.cuda.synchronize()
        gc = capture(torch, stream, lambda: [B.iqk_gemv(dstack, c % cold_copies, values, xd, y=y, ws=ws,
                                                        stream=stream) for c in range(calls)])
        with torch.cuda.stream(stream):
            gc.replay()
        torch.cuda.synchronize()
        tc = cuda_time(torch, stream, lambda: gc.replay()) / calls
        out.update({"us_per_call_l2_cold": tc * 1e6, "weight_gbs_l2_cold": nb / tc / 1e9,
                    "hbm_frac_l2_cold": nb / tc / 1e9 / measured_peaks()["hbm_gbs"],
                    "cold": f"{calls} calls rotating over {cold_copies} distinct matrices "
                            f"({nb * cold_copies / 1e6:.0f} MB)"})
        del gc, dstack
    del g
    return out


# ------------------------------------------------------------- pricing
# Every kernel priced against its own deleted-decode address floor (the page's
# "Pricing" section): identical loads, decode removed, an integer signature
# reaching the output. Per member and projection: the routed projection
# decode (iqk_switch_linear on the decode kernel, one token, top-6) against
# iqk_floor over the same experts, and the dequantizer (iqk_dequant) against
# iqk_dequant_floor (same loads and same stores). Arms alternate inside a
# cell. Declared gates:
PRICE_BAR = {"decode": 2.5, "dequant": 1.10}  # kernel time / own floor time, at most
FLOOR_BAND = (0.6, 1.05)  # a floor arm streams at this fraction of the measured HBM copy rate
PRICE_MIN_RATIO = 0.95  # a kernel clearly faster than its own floor skips loads the floor makes


class PriceCell:
    """One (member, projection) cell: the four arms captured as graphs over a
    ring of single-token routings (no expert repeats within experts/6 calls)."""

    def __init__(self, torch, B, w, values, device, stream, seed, calls=168):
        self.torch, self.B, self.stream = torch, B, stream
        self.w, self.values = w, values
        self.dw = B.Weights.from_host(w, device)
        rng = S.rng_for(seed)
        self.ids_h, _ = S.routing_ring(rng, calls, w.experts, S.TOPK)
        self.x_h = S.random_bf16(rng, (calls, 1, w.cols))
        self.ids = torch.from_numpy(self.ids_h).to(device)
        self.x = torch.from_numpy(self.x_h.view(np.int16)).to(device).view(torch.bfloat16)
        self.y = torch.empty((calls, 1, S.TOPK, w.rows), dtype=torch.float32, device=device)
        self.ws = B.workspace(B.iqk_switch_linear_workspace_bytes(1, 1, S.TOPK, w.experts, w.rows, w.cols), device)
        self.elist = [torch.from_numpy(np.unique(self.ids_h[c]).astype(np.int32)).to(device) for c in range(calls)]
        self.fout = torch.empty((calls, S.TOPK, w.rows), dtype=torch.int32, device=device)
        self.deq_e = [int(self.ids_h[c, 0, 0]) for c in range(calls)]
        # four output buffers in turn (134 MB for a 2048x4096 expert, more than
        # the 126 MB L2), so that each call's stores reach HBM
        self.dq = [torch.empty((w.rows, w.cols), dtype=torch.float32, device=device) for _ in range(4)]
        self.dqf = [torch.empty((w.rows, w.cols), dtype=torch.int32, device=device) for _ in range(4)]
        self.calls = calls
        row_b = B.iqk_row_bytes(w.fmt, w.cols)
        self.decode_bytes = float(np.mean([len(l) for l in self.elist])) * w.rows * row_b
        self.dequant_bytes = w.rows * row_b + w.rows * w.cols * 4  # streams read + float32 written

    def decode(self, c):
        self.B.iqk_switch_linear(self.dw, self.values, self.x[c], self.ids[c], mode=1, y=self.y[c], ws=self.ws,
                                 stream=self.stream)

    def floor(self, c):
        l = self.elist[c]
        self.B.iqk_floor(self.dw, l, out=self.fout[c, :l.numel()], stream=self.stream)

    def dequant(self, c):
        self.B.iqk_dequant(self.dw, self.deq_e[c], self.values, out=self.dq[c % 4], stream=self.stream)

    def dequant_floor(self, c):
        self.B.iqk_dequant_floor(self.dw, self.deq_e[c], out=self.dqf[c % 4], stream=self.stream)

    def graph(self, arm, n):
        torch = self.torch
        fn = getattr(self, arm)
        with torch.cuda.stream(self.stream):
            fn(0)
        torch.cuda.synchronize()
        return capture(torch, self.stream, lambda: [fn(c) for c in range(n)])

    def time(self, reps=5, dequant_calls=42):
        """Median µs per call of each arm, the arms of a pair alternating."""
        torch = self.torch
        pairs = (("decode", "floor", self.calls), ("dequant", "dequant_floor", dequant_calls))
        out = {}
        for a, b, n in pairs:
            ga, gb = self.graph(a, n), self.graph(b, n)
            for g in (ga, gb):
                with torch.cuda.stream(self.stream):
                    g.replay()
            torch.cuda.synchronize()
            ta, tb = [], []
            for _ in range(reps):
                ta.append(cuda_time(torch, self.stream, ga.replay) / n)
                tb.append(cuda_time(torch, self.stream, gb.replay) / n)
            out[a], out[b] = statistics.median(ta) * 1e6, statistics.median(tb) * 1e6
            del ga, gb
        return out


def price_gates(cells, hbm_gbs):
    """Apply the declared gates to timed cells; returns the failures (empty = pass)."""
    fails = []
    lo, hi = FLOOR_BAND[0] * hbm_gbs, FLOOR_BAND[1] * hbm_gbs
    for c in cells:
        tag = f"{c['member']} {c['projection']}"
        for k in ("decode", "dequant"):
            r = c[f"{k}_over_floor"]
            if r > PRICE_BAR[k]:
                fails.append(f"{tag}: {k} {r:.3f}x its floor, above the declared bar {PRICE_BAR[k]}")
            if r < PRICE_MIN_RATIO:
                fails.append(f"{tag}: {k} {r:.3f}x its floor: faster than its own loads (deleted-load signature)")
        for k in ("floor_gbs", "dequant_floor_gbs"):
            if not lo <= c[k] <= hi:
                fails.append(f"{tag}: {k} {c[k]:.0f} GB/s outside the floor band [{lo:.0f}, {hi:.0f}]")
    return fails


def pricing_leg(torch, B, members, device, stream, peaks, reps=5):
    """The pricing table: members = {name: (gate streams, down streams, values)}."""
    cells = []
    for mi, (member, (wg, wd, values)) in enumerate(members.items()):
        for pj, (proj, w) in enumerate((("gate/up", wg), ("down", wd))):
            cell = PriceCell(torch, B, w, values, device, stream, seed=500 + 10 * mi + pj)
            t = cell.time(reps)
            cells.append({"member": member, "projection": proj,
                          "decode_us": t["decode"], "floor_us": t["floor"],
                          "decode_over_floor": t["decode"] / t["floor"],
                          "dequant_us": t["dequant"], "dequant_floor_us": t["dequant_floor"],
                          "dequant_over_floor": t["dequant"] / t["dequant_floor"],
                          "floor_gbs": cell.decode_bytes / (t["floor"] * 1e-6) / 1e9,
                          "dequant_floor_gbs": cell.dequant_bytes / (t["dequant_floor"] * 1e-6) / 1e9})
            del cell
            torch.cuda.empty_cache()
    fails = price_gates(cells, peaks["hbm_gbs"])
    return {"cells": cells,
            "gates": {"ratio_bar": PRICE_BAR, "floor_band_of_hbm": FLOOR_BAND, "min_ratio": PRICE_MIN_RATIO,
                      "hbm_gbs": peaks["hbm_gbs"], "pass": not fails, "failures": fails},
            "arms": "decode = iqk_switch_linear (decode kernel, 1 token, top-6) vs iqk_floor on the same experts; "
                    "dequant = iqk_dequant (float32) vs iqk_dequant_floor; medians of "
                    f"{reps} alternating repeats"}


# ------------------------------------------------------------ cpu oracle

def oracle_decode_seconds(weights, values, budget_s, seed=99):
    """Time the CPU oracle (as it stands) on whole single-token decode calls of
    the same workload until ``budget_s`` of CPU work has run."""
    from oracle import oracle as O
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:
        limiter = None
    gate, up, down = weights
    rng = S.rng_for(seed)
    tokens, t0 = 0, time.perf_counter()
    while True:
        x = S.random_bf16(rng, (1, S.HIDDEN))
        ids, p = S.routing(rng, 1, S.EXPERTS, S.TOPK)
        O.moe(gate, up, down, values, x, ids, p)
        tokens += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    if limiter is not None:
        limiter.unregister() if hasattr(limiter, "unregister") else None
    return el / tokens, tokens


def _oracle_worker(args):
    """One host core's share of the all-core oracle timing: whole
    single-token decode calls at the headline geometry on its own seeded
    experts (eight resident; a call touches six), for ``budget_s`` seconds."""
    seed, budget_s = args
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    from oracle import oracle as O
    rng = S.rng_for(seed)
    gate, up, down = S.moe_weights(rng, "iq2_ks", 8, S.HIDDEN, S.INTER)
    values = S.value_table("int", 2)
    tokens, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        x = S.random_bf16(rng, (1, S.HIDDEN))
        ids, p = S.routing(rng, 1, 8, S.TOPK)
        O.moe(gate, up, down, values, x, ids, p)
        tokens += 1
    return tokens, time.perf_counter() - t0


def oracle_all_cores(budget_s, max_workers=16):
    """Whole-job oracle throughput on the host cores: independent workers
    (spawned processes, one thread each) run whole decode calls side by side;
    µs per token = wall time / tokens of all workers."""
    import multiprocessing as mp
    n = max(1, min(os.cpu_count() or 1, max_workers))
    ctx = mp.get_context("spawn")
    t0 = time.perf_counter()
    with ctx.Pool(n) as pool:
        res = pool.map(_oracle_worker, [(7000 + i, budget_s) for i in range(n)])
    wall = time.perf_counter() - t0
    tokens = sum(r[0] for r in res)
    busy = max(r[1] for r in res)
    return {"value": busy / max(tokens, 1) * 1e6, "unit": "us/token", "cores": n, "nproc": os.cpu_count(),
            "kind": "oracle", "sample": f"{n} spawned single-thread workers, {tokens} whole single-token decode "
                                        f"calls in {busy:.1f} s (each worker on its own 8 seeded experts at the "
                                        f"headline geometry); wall {wall:.1f} s including start-up"}


def oracle_pair_sample_seconds(weights, values, rows_per_matrix, seed):
    """One bounded sample of the decode work: dequantize and multiply
    ``rows_per_matrix`` rows of the gate, up and down matrices of one routed
    expert (the oracle's own functions). Returns (seconds, weights processed)."""
    from oracle import oracle as O
    gate, up, down = weights
    rng = S.rng_for(seed)
    e = int(rng.integers(0, S.EXPERTS))
    t0 = time.perf_counter()
    n = 0
    for w in (gate, up, down):
        r0 = int(rng.integers(0, w.rows - rows_per_matrix + 1))
        sl = slice(r0, r0 + rows_per_matrix)
        dq = O.dequant(w.fmt, rows_per_matrix, w.cols, w.qs[e, sl], w.scl[e, sl],
                       None if w.sch is None else w.sch[e, sl], w.sex[e, sl], w.dv[e, sl], values)
        x = S.random_bf16(rng, (1, w.cols))
        O.gemv(dq, x)
        n += rows_per_matrix * w.cols
    return time.perf_counter() - t0, n


def decode_weights_per_token():
    return S.TOPK * (2 * S.INTER * S.HIDDEN + S.HIDDEN * S.INTER)


def config_block(extra=None):
    c = {"workload": "routed-expert decode, IQ2_KS, 1 token/call, 256 experts top-6, gate/up 2048x4096, "
                     "down 4096x2048",
         "global_batch": 1, "experts": S.EXPERTS, "topk": S.TOPK, "hidden": S.HIDDEN, "inter": S.INTER,
         "format": "iq2_ks", "parallelism": "replicas",
         "l2": "inputs larger than L2: consecutive calls' experts come from a chain of random "
               "permutations (no expert reused within 42 calls; 1.77 GB resident, 41 MB per call)"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ main

def run_reference(args):
    """The CPU oracle as the reference arm (rank 0 only). A step is one whole
    single-token decode call when K + W calls fit in about two minutes of
    host time (about 1.1 s each on one core); otherwise a bounded sample of
    the call (rows of one routed expert's three matrices), scaled to a token."""
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    rng = S.rng_for(2)
    weights = S.moe_weights(rng, "iq2_ks", S.EXPERTS, S.HIDDEN, S.INTER)
    values = S.value_table("int", 2)
    per_token = decode_weights_per_token()
    whole = (args.steps + args.warmup) * 1.2 <= 150.0
    if whole:
        from oracle import oracle as O
        try:
            from threadpoolctl import threadpool_limits
            threadpool_limits(limits=1)
        except Exception:
            pass
        gate, up, down = weights
        calls = []
        for k in range(args.warmup + args.steps):
            r = S.rng_for(2000 + k)
            x = S.random_bf16(r, (1, S.HIDDEN))
            ids, p = S.routing(r, 1, S.EXPERTS, S.TOPK)
            calls.append((x, ids, p))
        for x, ids, p in calls[:args.warmup]:
            O.moe(gate, up, down, values, x, ids, p)
        t0 = time.perf_counter()
        for x, ids, p in calls[args.warmup:]:
            O.moe(gate, up, down, values, x, ids, p)
        tot_s = time.perf_counter() - t0
        us_per_token = tot_s / max(args.steps, 1) * 1e6
        sample = f"each step is one whole single-token headline decode call (fresh routing), one thread"
    else:
        rows = max(16, int(64 * 150.0 / ((args.steps + args.warmup) * 1.2)))
        rows = min(rows, 64)
        for w in range(args.warmup):
            oracle_pair_sample_seconds(weights, values, rows, 1000 + w)
        tot_s, tot_n = 0.0, 0
        for k in range(args.steps):
            sec, n = oracle_pair_sample_seconds(weights, values, rows, 2000 + k)
            tot_s += sec
            tot_n += n
        us_per_token = tot_s / tot_n * per_token * 1e6
        sample = (f"each step dequantizes and multiplies {rows} rows of each of the gate, up and down matrices of "
                  f"one routed expert ({tot_n // max(args.steps, 1)} weights); us/token = time per weight x "
                  f"{per_token} weights per token")
    line = {"impl": "reference", "metric": METRIC, "value": us_per_token, "unit": "us/token",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_s / max(args.steps, 1) * 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_block(),
            "cpu_baseline": {"value": us_per_token, "unit": "us/token", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": us_per_token, "unit": "us/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=250 * RING)
    ap.add_argument("--warmup", type=int, default=RING)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-details", action="store_true")
    ap.add_argument("--no-price", action="store_true", help="skip the pricing table (kernels vs own floors)")
    ap.add_argument("--profile", choices=["decode", "prefill", "dequant", "gemv"], default=None,
                    help="plain launches without graphs or reporting (for ncu captures)")
    ap.add_argument("--experts", type=int, default=S.EXPERTS,
                    help="experts resident in --profile mode (fewer keeps ncu captures small)")
    ap.add_argument("--tokens", type=int, default=256, help="tokens per call in --profile prefill mode")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    from gemm_iq2_ks_b200 import binding as B
    B.lib()
    peaks = measured_peaks()
    stream = torch.cuda.Stream(device)

    if args.profile == "decode":
        rng = S.rng_for(2)
        w_ks = S.moe_weights(rng, "iq2_ks", args.experts, S.HIDDEN, S.INTER)
        dec = DecodeBench(torch, B, w_ks, S.value_table("int", 2), 1, 20, device, stream)
        with torch.cuda.stream(stream):
            for c in range(args.warmup + args.steps):
                dec.call(c % RING)
        torch.cuda.synchronize()
        return 0
    if args.profile == "dequant":  # iqk_dequant of one 2048x4096 IQ2_KS expert per call, float32 out
        rng = S.rng_for(2)
        w = S.random_streams(rng, "iq2_ks", args.experts, S.INTER, S.HIDDEN)
        dw = B.Weights.from_host(w, device)
        out = torch.empty((S.INTER, S.HIDDEN), dtype=torch.float32, device=device)
        with torch.cuda.stream(stream):
            for c in range(args.warmup + args.steps):
                B.iqk_dequant(dw, c % args.experts, S.value_table("int", 2), out=out, stream=stream)
        torch.cuda.synchronize()
        return 0
    if args.profile == "gemv":  # iqk_gemv of one 2048x4096 IQ2_K matrix per call, rotating over --experts copies
        w, x, values = S.matrix_case("gemv_iq2_k_2048x4096")
        stack = S.random_streams(S.rng_for(S.seed_of("gemv_iq2_k_2048x4096") + 50), w.fmt, args.experts, w.rows, w.cols)
        dw = B.Weights.from_host(stack, device)
        xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        y = torch.empty((xd.shape[0], w.rows), dtype=torch.float32, device=device)
        ws = B.workspace(B.iqk_gemv_workspace_bytes(xd.shape[0], w.rows, w.cols), device)
        with torch.cuda.stream(stream):
            for c in range(args.warmup + args.steps):
                B.iqk_gemv(dw, c % args.experts, values, xd, y=y, ws=ws, stream=stream)
        torch.cuda.synchronize()
        return 0
    if args.profile == "prefill":
        rng = S.rng_for(4)
        w_ks = S.moe_weights(rng, "iq2_ks", args.experts, S.HIDDEN, S.INTER)
        T = args.tokens
        ids, p = S.routing(rng, T, args.experts, S.TOPK)
        x = S.random_bf16(rng, (T, S.HIDDEN))
        dw = [B.Weights.from_host(w, device) for w in w_ks]
        xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        idsd, pd = torch.from_numpy(ids).to(device), torch.from_numpy(p).to(device)
        ws = B.workspace(B.iqk_moe_workspace_bytes(1, T, S.TOPK, args.experts, S.HIDDEN, S.INTER), device)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup + args.steps):
                B.iqk_moe_prefill(dw[0], dw[1], dw[2], S.value_table("int", 4), xd, idsd, pd, ws=ws, stream=stream)
        torch.cuda.synchronize()
        return 0

    # ---------------- headline: IQ2_KS routed decode, one token per call
    log("generating the headline decode weights")
    rng = S.rng_for(2 + 1000 * rank)
    w_ks = S.moe_weights(rng, "iq2_ks", S.EXPERTS, S.HIDDEN, S.INTER)
    values = S.value_table("int", 2)
    K, W = args.steps, args.warmup
    rems = sorted({K % RING, W % RING} - {0})
    dec = DecodeBench(torch, B, w_ks, values, 1, 20 + rank, device, stream, remainders=rems)
    log("capturing decode graphs")
    graphs = dec.graphs()
    torch.cuda.synchronize()
    log("warmup")
    with torch.cuda.stream(stream):
        run_steps(graphs, W)
    torch.cuda.synchronize()
    # The clock sampler runs over a window of back-to-back replays (about
    # 0.3 s before and after) that contains the timed region, which at small
    # K is far shorter than the sampling period.
    ring_s = cuda_time(torch, stream, lambda: graphs[0].replay())
    rolls = max(1, int(math.ceil(0.3 / max(ring_s, 1e-6))))

    def roll():
        with torch.cuda.stream(stream):
            for _ in range(rolls):
                graphs[0].replay()
            if K % RING:  # the timed remainder graph's first launch (its upload) stays out of the timed region
                graphs[1][K % RING].replay()

    with ClockSampler(torch.cuda.get_device_properties(device)) as clk:
        roll()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t = cuda_time(torch, stream, lambda: run_steps(graphs, K))
        torch.cuda.synchronize()
        roll()
        torch.cuda.synchronize()
    t, us_per_token = job_time(torch, dist, t, K, world, device)
    if dist:
        dist.barrier()
    bytes_per_call = dec.weight_bytes(K) / K
    gbs = bytes_per_call * K / t / 1e9  # one GPU's weight stream (each rank reads its own)

    log(f"decode timed: {t / K * 1e6:.2f} us/call")
    # e2e through the C ABI with host buffers: iqk_moe_decode_host, whose kernels read the
    # inputs and write y over the host link inside the timed region
    ng = min(RING, K)
    eg, h2d, d2h, e2e_bufs = e2e_graph(torch, dec, stream, ng)  # the pinned buffers live as long as the graph
    with torch.cuda.stream(stream):
        eg.replay()
    torch.cuda.synchronize()
    reps = max(1, K // ng)
    te = cuda_time(torch, stream, lambda: [eg.replay() for _ in range(reps)])
    e2e_us = te / (reps * ng) * 1e6

    log(f"e2e: {e2e_us:.2f} us/token")
    # floor arm on the same experts (identical loads, decode removed)
    fg = floor_graph(torch, dec, stream, ng)
    with torch.cuda.stream(stream):
        fg.replay()
    torch.cuda.synchronize()
    tf = cuda_time(torch, stream, lambda: [fg.replay() for _ in range(reps)])
    floor_us = tf / (reps * ng) * 1e6
    floor_status = B.iqk_floor_status(stream)  # a floor whose waits ran out would read too short

    log(f"floor: {floor_us:.2f} us/call")
    details = {}
    if not args.no_details and rank == 0:
        # IQ2_K routed decode at T = 1, 4, 16
        rng3 = S.rng_for(3)
        w_k = S.moe_weights(rng3, "iq2_k", S.EXPERTS, S.HIDDEN, S.INTER)
        for T in (1, 4, 16):
            db = DecodeBench(torch, B, w_k, S.value_table("f16", 3), T, 30 + T, device, stream)
            gr = db.graphs()
            with torch.cuda.stream(stream):
                run_steps(gr, RING)
            torch.cuda.synchronize()
            tt3 = cuda_time(torch, stream, lambda: run_steps(gr, 2 * RING))
            per_call = tt3 / (2 * RING)
            by = db.weight_bytes(2 * RING) / (2 * RING)
            details[f"decode_iq2_k_T{T}"] = {"us_per_call": per_call * 1e6, "us_per_token": per_call / T * 1e6,
                                             "weight_gbs": by / per_call / 1e9,
                                             "hbm_frac": by / per_call / 1e9 / peaks["hbm_gbs"],
                                             "mean_distinct_experts": float(db.distinct.mean())}
            del db, gr
        if not args.no_price:
            log("pricing against own floors")
            details["pricing"] = pricing_leg(torch, B, {"IQ2_KS": (w_ks[0], w_ks[2], values),
                                                        "IQ2_K": (w_k[0], w_k[2], S.value_table("f16", 3))},
                                             device, stream, peaks)
        del w_k
        torch.cuda.empty_cache()
        log("prefill")
        details["prefill_iq2_ks_2048"] = prefill_leg(torch, B, w_ks, values, device, stream, peaks)
        torch.cuda.empty_cache()
        for case in S.MATRIX_CASES:
            details[case] = gemv_leg(torch, B, case, device, stream)

    launches = 3 * K  # per call: the prep kernel (run counters), the gate/up kernel and the down kernel
    line = {
        "metric": METRIC, "value": us_per_token, "unit": "us/token", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": t / K * 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": config_block({"format": "iq2_ks", "global_batch": world}),
        "weight_gbs": gbs * world, "hbm_frac": gbs / peaks["hbm_gbs"],
        "floor": {"us_per_token": floor_us, "decode_over_floor": us_per_token / floor_us if world == 1 else
                  (t / K * 1e6) / floor_us, "status_ok": floor_status == B.IQK_OK},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": DECODE_CALL_TRAFFIC,
                     "kernel": "one decode call (prep, gate/up+SwiGLU, down+combine, PDL-chained)",
                     "peak_source": peaks["source"] + " hbm_gbs (copy)"},
        "e2e": {"value": e2e_us, "unit": "us/token", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": dict(clk.summary(), window="nvidia-smi every 50 ms over back-to-back replays of the decode "
                                               "ring for about 0.3 s before and after the timed region"),
        "details": details,
    }
    if rank == 0 and world >= 1:
        log("cpu baseline (oracle)")
        sec, ntok = oracle_decode_seconds(w_ks, values, args.cpu_budget)
        line["cpu_baseline"] = {"value": sec * 1e6, "unit": "us/token", "cores": 1, "kind": "oracle",
                                "sample": f"{ntok} whole single-token headline decode calls "
                                          f"(fresh routing each), one thread",
                                "nproc": os.cpu_count()}
        log("cpu baseline on all cores (oracle)")
        try:
            line["cpu_baseline"]["all_cores"] = oracle_all_cores(args.cpu_budget)
        except Exception as e:  # the single-thread figure above stands on its own
            line["cpu_baseline"]["all_cores"] = {"error": repr(e)[:200]}
    if dist:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
