#!/usr/bin/env python
"""Throughput of the POET layer hot path on B200: forward + backward (dX and
packed-skew gradients, Cayley-Neumann for every primitive) over a LLaMA-shaped
layer set, in tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl poet|reference]
                    [--workload llama1.3b|llama60m|llama350m|llama3b]

One step = Cayley-Neumann of every primitive, then the forward of every
linear of every layer, then the backward of every linear in reverse order;
for the default workload both variants (fully stochastic and block-stochastic
b=256 at LLaMA-1.3B shapes) run back to back, each over its own T tokens.
Merge-then-reinitialize (every 400 steps in the pages' setup) is timed
separately and reported amortized.  Under torchrun each rank trains its own
replica on its own tokens (data parallel, weak scaling) and the packed-skew
gradients are all-reduced over NCCL once per step.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD_SETS = {
    "llama1.3b": ["llama1.3b_fs", "llama1.3b_bs256"],
    "llama60m": ["llama60m_fs"],
    "llama350m": ["llama350m_bs256"],
    "llama3b": ["llama3b_fs"],
}
METRIC = "POET layer fwd+bwd tokens/s at LLaMA-1.3B shapes; % of TC/HBM roofline"
PLANS = {"auto": 0, "token": 1, "weight": 2}


def row_stride(d):
    """Row stride of the bench's activations: the width rounded up to 8 elements (16-byte aligned bf16 rows)."""
    return (d + 7) // 8 * 8
PLAN_NAMES = {1: "token", 2: "weight"}

# DRAM traffic / algorithmic bytes of one launch, from an ncu capture, with the
# engine revisions (as named in poet_version()) that run that launch unchanged:
# the counters were taken on r22; r25 changes only the plan of grouped launches
# whose problems are at most 256 columns wide, which these launches are not;
# r26 keeps the epilogue's problem fields in registers (instructions, not bytes);
# r27 returns the grouped launches of r25 to single CTAs.
_T_SIZED = ("gemm_tc r22;", "gemm_tc r25;", "gemm_tc r26;", "gemm_tc r27;")
NCU_TRAFFIC_RATIO = {"w0_fwd": (0.999, _T_SIZED), "w0_bwd": (1.025, _T_SIZED), "w_grad": (1.273, _T_SIZED)}
NCU_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of the grouped launch of one LLaMA-1.3B "
                      "layer at 16384 tokens (profiles/w0_gemm_llama1.3b_layer_T16384.md), as a ratio to the "
                      "algorithmic bytes of that launch, scaled to this run's launches")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["poet", "reference"], default="poet")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_SETS), default="llama1.3b")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-merge", action="store_true")
    ap.add_argument("--plan", choices=sorted(PLANS), default="auto",
                    help="where the primitives act: auto (cost model), token (activations) or weight (W0)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches instead of replaying each variant's step as a CUDA graph")
    ap.add_argument("--no-token-plan", action="store_true",
                    help="skip the second timed pass that runs every layer on the token plan")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (small profiling cases)")
    ap.add_argument("--tokens", type=int, default=0, help="override the token count (small profiling cases)")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip timing the other LLaMA layer sets after the headline")
    ap.add_argument("--probe", default="",
                    help="measure only this one of the other layer sets or small-block probes and print its line "
                         "(profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="poet_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        busy = [s for s in sm if smax and s > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- CUDA path

class Variant:
    """All POET linears of one workload, resident on the device."""

    def __init__(self, wl, rank, device, w0_cache, act_cache, saved_pool, plan=0):
        import torch

        from orthogonal_reparameterized_poet_b200 import inputs as I
        from orthogonal_reparameterized_poet_b200 import poet

        self.wl = wl
        self.T = wl.tokens
        tdt = poet.torch_dtype(wl.dtype)
        shapes = wl.linear_shapes()
        self.layers = []
        nth = []
        for layer in range(wl.layers):
            for t, (m, n) in enumerate(shapes):
                key = (wl.seed, layer, t, m, n, wl.dtype)
                if key not in w0_cache:
                    w0_cache[key] = torch.from_numpy(I.w0(wl.seed, layer, t, m, n, wl.dtype)).to(device=device,
                                                                                              dtype=tdt)
                    W0 = w0_cache[key]
                else:  # another variant of the same model: its own copy (merge updates W0 in place)
                    W0 = w0_cache[key].clone()
                nR, sR = poet.side_geometry(m, wl.mode, wl.b)
                nP, sP = poet.side_geometry(n, wl.mode, wl.b)
                thR = torch.from_numpy(I.theta(wl.seed, layer, t, 0, nR * sR * (sR - 1) // 2, wl.sigma)).to(device)
                thP = torch.from_numpy(I.theta(wl.seed, layer, t, 1, nP * sP * (sP - 1) // 2, wl.sigma)).to(device)
                L = poet.PoetLayer(W0, thR, thP, mode=wl.mode, b=wl.b, k=wl.k, seed=wl.seed,
                                   layer_id=layer * len(shapes) + t, plan=plan)
                L.prepare()
                self.layers.append((layer, t, m, n, L))
                nth.append((thR.numel(), thP.numel()))
        # one flat gradient buffer (one all-reduce per step under data parallelism)
        total = sum(a + b for a, b in nth)
        self.dtheta = torch.zeros(max(total, 1), dtype=torch.float32, device=device)
        self.dslices = []
        off = 0
        for a, b in nth:
            self.dslices.append((self.dtheta[off:off + a], self.dtheta[off + a:off + a + b]))
            off += a + b
        # per-shape activations (each rank draws its own tokens), in rows whose
        # stride is the width rounded up to 8 elements (16-byte aligned rows)
        self.x, self.dy, self.y, self.dx = {}, {}, {}, {}

        def rows(d):
            return torch.zeros(self.T, row_stride(d), dtype=tdt, device=device)[:, :d]

        def act(d, grad):
            key = (wl.seed + 7919 * rank, d, self.T, wl.dtype, grad)
            if key not in act_cache:  # the variants of one model see the same tokens
                t = rows(d)
                t.copy_(torch.from_numpy(I.activations(wl.seed + 7919 * rank, d, self.T, d, wl.dtype, grad=grad)))
                act_cache[key] = t
            return act_cache[key]

        for (m, n) in set(shapes):
            if n not in self.x:
                self.x[n] = act(n, False)
                self.dx[n] = rows(n)
            if m not in self.dy:
                self.dy[m] = act(m, True)
                self.y[m] = rows(m)
        # saved activations: one buffer per linear position, shared by the variants (they run one after the other)
        self.saved = []
        for i, (_, _, _, _, L) in enumerate(self.layers):
            need = poet.poet_saved_bytes(L.struct, self.T)
            if i >= len(saved_pool) or saved_pool[i].numel() < need:
                buf = torch.empty(need, dtype=torch.uint8, device=device)
                if i < len(saved_pool):
                    saved_pool[i] = buf
                else:
                    saved_pool.append(buf)
            self.saved.append(saved_pool[i])
        self.per_call = len(shapes)  # the grouped calls take one block's linears at a time
        self.ws_need = self._ws_need()
        self.ws = None
        self.input_bytes = sum(v.numel() * v.element_size() for v in list(self.x.values()) + list(self.dy.values()))

    def _ws_need(self):
        from orthogonal_reparameterized_poet_b200 import poet

        pl = [L for (_, _, _, _, L) in self.layers]
        need = max(L.workspace_bytes(0) for L in pl)  # merge
        for c0 in range(0, len(pl), self.per_call):
            chunk = self.layers[c0:c0 + self.per_call]
            need = max(need, poet.many_workspace_bytes([c[4] for c in chunk], self.T,
                                                       [self.dy[c[2]] for c in chunk]))
        return need

    def use_plan(self, plan, saved_pool, device):
        """Run every layer on `plan` from now on; grow the shared saved buffers to fit."""
        import torch

        from orthogonal_reparameterized_poet_b200 import poet

        for i, (_, _, _, _, L) in enumerate(self.layers):
            L.struct.plan = plan
            need = poet.poet_saved_bytes(L.struct, self.T)
            if saved_pool[i].numel() < need:
                saved_pool[i] = None
                saved_pool[i] = torch.empty(need, dtype=torch.uint8, device=device)
            self.saved[i] = saved_pool[i]
        self.ws_need = self._ws_need()

    def plan_names(self):
        return "+".join(sorted({PLAN_NAMES[L.plan_for(self.T)] for (_, _, _, _, L) in self.layers}))

    def alloc_grads(self, device, chunk):
        """Per-primitive gradient buffers of every side (one flat buffer) and the
        workspace of the grouped Cayley-Neumann backward over `chunk` layers."""
        import torch

        from orthogonal_reparameterized_poet_b200 import poet

        sizes = []
        for (_, _, _, _, L) in self.layers:
            sizes.append((poet.poet_block_grad_bytes(L.struct.R) // 4, poet.poet_block_grad_bytes(L.struct.P) // 4))
        total = sum(a + b for a, b in sizes)
        self.gflat = torch.empty(max(total, 4), dtype=torch.float32, device=device)
        self.G = []
        off = 0
        for a, b in sizes:
            self.G.append((self.gflat[off:off + a], self.gflat[off + a:off + a + b]))
            off += a + b
        self.chunk = chunk
        pl = [L for (_, _, _, _, L) in self.layers]
        return max(poet.cayley_neumann_grad_many_workspace_bytes(pl[i:i + chunk]) for i in range(0, len(pl), chunk))

    def step(self, world=1):
        from orthogonal_reparameterized_poet_b200 import poet

        pl = [L for (_, _, _, _, L) in self.layers]
        poet.cayley_neumann_many(pl)  # a1 for every primitive of every layer
        k = self.per_call
        for c0 in range(0, len(pl), k):  # a2..a4, one block's linears per grouped call
            ch = self.layers[c0:c0 + k]
            poet.forward_many([c[4] for c in ch], [self.x[c[3]] for c in ch], [self.y[c[2]] for c in ch],
                              self.saved[c0:c0 + k], self.ws)
        for c0 in reversed(range(0, len(pl), k)):  # a5..a7, blocks in reverse order
            ch = self.layers[c0:c0 + k]
            poet.backward_blocks_many([c[4] for c in ch], [self.x[c[3]] for c in ch], self.saved[c0:c0 + k],
                                      [self.dy[c[2]] for c in ch], [self.dx[c[3]] for c in ch],
                                      self.G[c0:c0 + k], self.ws)
        for c0 in range(0, len(pl), self.chunk):  # a8 for every layer, in grouped launches
            poet.cayley_neumann_grad_many(pl[c0:c0 + self.chunk], self.G[c0:c0 + self.chunk],
                                          self.dslices[c0:c0 + self.chunk], self.gws)
        if world > 1:  # data parallel: the one exchange of the step
            from orthogonal_reparameterized_poet_b200 import dp

            dp.allreduce_gradients_(self.dtheta)

    def merge_flop(self):
        """Algorithmic flops of one merge of every linear: the R blocks on W0's
        rows and the P blocks on its columns, 2 (c_R n s_R + m c_P s_P)."""
        from orthogonal_reparameterized_poet_b200 import poet

        total = 0.0
        for (_, _, m, n, L) in self.layers:
            nR, sR = poet.side_geometry(m, self.wl.mode, self.wl.b)
            nP, sP = poet.side_geometry(n, self.wl.mode, self.wl.b)
            total += 2.0 * (nR * sR * n * sR + m * nP * sP * sP)
        return total

    def merge_all(self):
        for (_, _, _, _, L) in self.layers:
            L.merge(ws=self.ws)
            L.resample()


def trace_on(poet):
    """Start the library's per-kind event trace, with the ridge of the measured
    peaks splitting launches into tensor- and HBM-bound ones."""
    peaks = load_peaks()
    poet.poet_trace_set_ridge(peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9))
    poet.poet_trace_enable(True)


def kernel_table(rows, steps):
    """Per trace kind: launches, ms per step, share, achieved TFLOP/s and GB/s,
    and the fraction of its roofline.  Every launch is held to its own bound:
    the library sums the flops of the launches whose flop/byte is at or above
    the ridge of the measured peaks (flop_tc) and the bytes of the others
    (bytes_hbm), so the roofline time is flop_tc / tensor peak + bytes_hbm /
    copy peak and frac = that time over the measured one.  `bound` names the
    larger of the two terms."""
    peaks = load_peaks()
    pt, ph = peaks["bf16_tflops_sustained"] * 1e12, peaks["hbm_gbs"] * 1e9
    total = sum(x["ms"] for x in rows.values()) or 1.0
    out = {}
    for k, r in sorted(rows.items(), key=lambda kv: -kv[1]["ms"]):
        sec = r["ms"] / 1e3
        tf = r["flop"] / sec / 1e12 if sec and r["flop"] else None
        gb = r["bytes"] / sec / 1e9 if sec else None
        t_tc, t_hbm = r.get("flop_tc", 0.0) / pt, r.get("bytes_hbm", 0.0) / ph
        frac = (t_tc + t_hbm) / sec if sec and (t_tc or t_hbm) else None
        out[k] = {"launches": r["launches"], "ms_per_step": round(r["ms"] / steps, 3), "share": round(r["ms"] / total, 4),
                  "tflops": round(tf, 1) if tf else None, "gbs": round(gb, 1) if gb else None,
                  "bound": "tensor" if t_tc >= t_hbm else "hbm", "frac": round(frac, 4) if frac is not None else None}
    return out


def roofline_of(rows, version):
    """Roofline of the dominant kind of a trace: achieved = its algorithmic flops
    (or bytes) over its CUDA-event time, against the measured sustained bf16
    peak (or the copy bandwidth) that its flop/byte ratio selects."""
    peaks = load_peaks()
    if not rows:
        return None
    dominant = max(rows, key=lambda k: rows[k]["ms"])
    r = rows[dominant]
    intensity = r["flop"] / r["bytes"] if r["bytes"] else float("inf")
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    avg_ms = r["ms"] / r["launches"]
    if intensity >= ridge:
        achieved = r["flop"] / (r["ms"] / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "unit": "TFLOP/s", "peak_kind": "bf16 sustained, " + peaks["source"]}
    else:
        achieved = r["bytes"] / (r["ms"] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s", "peak_kind": "copy, " + peaks["source"]}
    traffic = None
    ratio = NCU_TRAFFIC_RATIO.get(dominant)
    if ratio and any(r in version for r in ratio[1]):  # counters valid for this kernel revision
        traffic = round(ratio[0] * r["bytes"] / r["launches"])
    roof.update({"kernel": dominant, "achieved": round(achieved, 1), "peak": peak,
                 "frac": round(achieved / peak, 4), "traffic": traffic, "avg_launch_ms": round(avg_ms, 4),
                 "launches": r["launches"], "algorithmic_per_launch": {
                     "flop": r["flop"] / r["launches"], "bytes": r["bytes"] / r["launches"]},
                 "traffic_source": NCU_TRAFFIC_SOURCE})
    return roof


# The other layer sets of the pages' LLaMA family, measured after the headline
# in the same run (each built, timed and freed in turn).
OTHER_WORKLOADS = ["single256_fp32_bs32", "llama60m_fs", "llama350m_bs256", "llama3b_fs"]


# Small primitives (size 32) at a token count whose block passes exceed L2: the
# small-block kernels against the copy bandwidth (token plan).
SMALLB_PROBES = {"smallb_fp32_b32_T262144": ("single256_fp32_bs32", {"tokens": 262144}),
                 "smallb_bf16_b32_T262144": ("single256_fp32_bs32", {"tokens": 262144, "dtype": 1, "k": 4,
                                                                    "sigma": 0.02})}


def measure_workload(name, args, device, rank, plan, overrides=None):
    """tokens/s of one workload's step (CUDA-graph replay, inputs resident), its
    per-kind trace and dominant-kernel roofline, and its merge time."""
    import dataclasses

    import torch

    from orthogonal_reparameterized_poet_b200 import inputs as I
    from orthogonal_reparameterized_poet_b200 import poet

    wl = I.WORKLOADS[name]
    if overrides:
        wl = dataclasses.replace(wl, **overrides)
    v = Variant(wl, rank, device, {}, {}, [], plan)
    v.ws = torch.empty(max(v.ws_need, 1), dtype=torch.uint8, device=device)
    gws_need = v.alloc_grads(device, chunk=4 * len(wl.linear_shapes()))
    v.gws = torch.empty(max(gws_need, 1), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 1)):
        v.step()
    poet.poet_sync_status()
    trace_on(poet)
    for _ in range(args.steps):
        v.step()
    trace = poet.poet_trace_read()
    poet.poet_trace_enable(False)
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    gph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gph, stream=cap):
        v.step()
    stream.wait_stream(cap)
    gph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        gph.replay()
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / args.steps
    poet.poet_sync_status()
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    m0.record(stream)
    v.merge_all()
    m1.record(stream)
    m1.synchronize()
    poet.poet_sync_status()
    rows = {k: dict(r) for k, r in trace.items()}
    roof = roofline_of(rows, poet.poet_version())
    out = {"tok_s": round(v.T / (ms / 1e3), 1), "ms": round(ms, 3), "tokens": v.T, "layers": wl.layers,
           "mode": "FS" if wl.mode == I.FS else f"BS{wl.b}", "dtype": "f32" if wl.dtype == I.F32 else "bf16",
           "plan": v.plan_names(), "merge_ms": round(m0.elapsed_time(m1), 3),
           "merge_tflops": round(v.merge_flop() / (m0.elapsed_time(m1) / 1e3) / 1e12, 1),
           "kernel": roof["kernel"] if roof else None, "bound": roof["bound"] if roof else None,
           "frac": roof["frac"] if roof else None,
           "per_kind_ms": {k: round(r["ms"] / args.steps, 3) for k, r in
                           sorted(rows.items(), key=lambda kv: -kv[1]["ms"])[:6]}}
    if overrides:  # probes: every kind's bandwidth and fraction of its roofline
        out["kinds"] = {k: [r["gbs"], r["frac"], r["bound"]] for k, r in kernel_table(rows, args.steps).items()}
    del gph, v
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# One LLaMA block around seven POET linears (forward, backward and the grouped
# a8 of its fourteen sides) at LLaMA-1.3B shapes: hidden 2048, FFN 5461, 32
# heads of 64, 16 sequences of 2048 tokens.
BLOCK_WORKLOADS = {"llama1.3b_block_fs": ("llama1.3b_fs", 32, 64, 2048),
                   "llama1.3b_block_bs256": ("llama1.3b_bs256", 32, 64, 2048)}


def measure_block(name, args, device):
    import torch

    from orthogonal_reparameterized_poet_b200 import inputs as I
    from orthogonal_reparameterized_poet_b200 import poet

    base, heads, head_dim, seq = BLOCK_WORKLOADS[name]
    wl = I.WORKLOADS[base]
    T = wl.tokens
    layers = []
    for t, (m, n) in enumerate(wl.linear_shapes()):
        nR, sR = poet.side_geometry(m, wl.mode, wl.b)
        nP, sP = poet.side_geometry(n, wl.mode, wl.b)
        W0 = torch.from_numpy(I.w0(wl.seed, 0, t, m, n, wl.dtype)).to(device=device, dtype=torch.bfloat16)
        thR = torch.from_numpy(I.theta(wl.seed, 0, t, 0, nR * sR * (sR - 1) // 2, wl.sigma)).to(device)
        thP = torch.from_numpy(I.theta(wl.seed, 0, t, 1, nP * sP * (sP - 1) // 2, wl.sigma)).to(device)
        L = poet.PoetLayer(W0, thR, thP, mode=wl.mode, b=wl.b, k=wl.k, seed=wl.seed, layer_id=t)
        L.prepare()
        layers.append(L)
    blk = poet.PoetBlock(layers, seq, heads, head_dim)
    h = torch.from_numpy(I.activations(wl.seed, wl.hidden, T, wl.hidden, wl.dtype)).to(device, torch.bfloat16)
    dout = torch.from_numpy(I.activations(wl.seed, wl.hidden, T, wl.hidden, wl.dtype, grad=True)).to(device,
                                                                                                     torch.bfloat16)
    out = torch.empty_like(h)
    dh = torch.empty_like(h)
    saved = torch.empty(blk.saved_bytes(T), dtype=torch.uint8, device=device)
    G = [L.block_grad_buffers() for L in layers]
    dth = [(torch.empty_like(L.theta_R), torch.empty_like(L.theta_P)) for L in layers]
    gws = torch.empty(max(poet.cayley_neumann_grad_many_workspace_bytes(layers), 1), dtype=torch.uint8,
                      device=device)
    blk.workspace(T)

    def step():
        poet.cayley_neumann_many(layers)
        blk.forward(h, out=out, saved=saved)
        blk.backward(saved, dout, dh=dh, G=G)
        poet.cayley_neumann_grad_many(layers, G, dth, gws)

    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 1)):
        step()
    poet.poet_sync_status()
    trace_on(poet)
    for _ in range(args.steps):
        step()
    rows = poet.poet_trace_read()
    poet.poet_trace_enable(False)
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    gph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gph, stream=cap):
        step()
    stream.wait_stream(cap)
    gph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        gph.replay()
    b.record(stream)
    b.synchronize()
    poet.poet_sync_status()
    ms = a.elapsed_time(b) / args.steps
    roof = roofline_of({k: dict(r) for k, r in rows.items()}, poet.poet_version())
    res = {"tok_s": round(T / (ms / 1e3), 1), "ms": round(ms, 3), "tokens": T, "seq_len": seq, "heads": heads,
           "head_dim": head_dim, "mode": "FS" if wl.mode == I.FS else f"BS{wl.b}", "plan": "auto",
           "kernel": roof["kernel"] if roof else None, "frac": roof["frac"] if roof else None,
           "per_kind_ms": {k: round(r["ms"] / args.steps, 3) for k, r in
                           sorted(rows.items(), key=lambda kv: -kv[1]["ms"])[:8]}}
    del gph, blk, layers, saved, G, dth, gws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_poet(args):
    import torch

    from orthogonal_reparameterized_poet_b200 import inputs as I
    from orthogonal_reparameterized_poet_b200 import poet

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    poet.lib()

    wls = [I.WORKLOADS[name] for name in WORKLOAD_SETS[args.workload]]
    if args.layers or args.tokens:
        import dataclasses

        wls = [dataclasses.replace(w, layers=args.layers or w.layers, tokens=args.tokens or w.tokens) for w in wls]
    w0_cache, act_cache, saved_pool = {}, {}, []
    variants = [Variant(wl, rank, device, w0_cache, act_cache, saved_pool, PLANS[args.plan]) for wl in wls]
    del w0_cache
    ws = torch.empty(max(v.ws_need for v in variants), dtype=torch.uint8, device=device)  # one shared workspace
    gws_need = max(v.alloc_grads(device, chunk=4 * len(v.wl.linear_shapes())) for v in variants)
    gws = torch.empty(max(gws_need, 1), dtype=torch.uint8, device=device)
    for v in variants:
        v.ws = ws
        v.gws = gws
    torch.cuda.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()

    def step():
        for v in variants:
            v.step(world)

    for _ in range(args.warmup):
        step()
    poet.poet_sync_status()

    # ---- timed region
    stream = torch.cuda.current_stream()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = vis.split(",")[local] if vis else str(local)

    def timed(steps, clocks=None):
        """K steps of every variant back to back, the kernel trace read per variant.
        Returns (elapsed ms, per-variant ms, merged trace, per-variant traces, launches)."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in variants]
        barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.start()
        trace_on(poet)
        launches0 = poet.poet_launch_count()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        traces = []
        for i, v in enumerate(variants):
            ev[i][0].record(stream)
            for _ in range(steps):
                v.step(world)
            ev[i][1].record(stream)
            traces.append(poet.poet_trace_read())  # waits for this variant's recorded events
        t1.record(stream)
        torch.cuda.synchronize()
        per_variant_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(len(variants))]
        launches = poet.poet_launch_count() - launches0
        poet.poet_trace_enable(False)
        clk = clocks.stop() if clocks else None
        barrier()
        elapsed = t0.elapsed_time(t1)
        trace = {}
        for tr in traces:
            for k, r in tr.items():
                a = trace.setdefault(k, {"launches": 0, "ms": 0.0, "flop": 0.0, "bytes": 0.0, "flop_tc": 0.0,
                                         "bytes_hbm": 0.0})
                for f in a:
                    a[f] += r[f]
        poet.poet_sync_status()
        if dist is not None:
            from orthogonal_reparameterized_poet_b200 import dp

            mx = dp.max_over_ranks([elapsed] + per_variant_ms, device=device)
            elapsed, per_variant_ms = mx[0], mx[1:]
        return elapsed, per_variant_ms, trace, traces, launches, clk

    # The kernel trace (per-kind times for the roofline) comes from eager steps.
    # The headline time replays each variant's step captured as one CUDA graph
    # (one process per GPU; every buffer is resident, so a step launches the
    # same kernels on the same pointers every time).  Under data parallelism the
    # step holds an NCCL all-reduce and stays eager.
    use_graph = not args.no_graph and world == 1
    e_elapsed, e_per_variant_ms, trace, traces, launches, e_clk = timed(args.steps, None if use_graph else
                                                                        ClockSampler(smi_index))
    graphs = None
    if use_graph:
        graphs = []
        cap = torch.cuda.Stream()
        for v in variants:
            cap.wait_stream(torch.cuda.current_stream())
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=cap):
                v.step(world)
            torch.cuda.current_stream().wait_stream(cap)
            graphs.append(gph)
        for gph in graphs:  # warm replays
            gph.replay()
        torch.cuda.synchronize()
        poet.poet_sync_status()
        clocks = ClockSampler(smi_index)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in variants]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        clocks.start()
        t0.record(stream)
        for i, gph in enumerate(graphs):
            ev[i][0].record(stream)
            for _ in range(args.steps):
                gph.replay()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        poet.poet_sync_status()
        elapsed = t0.elapsed_time(t1)
        per_variant_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(len(variants))]
    else:
        elapsed, per_variant_ms, clk = e_elapsed, e_per_variant_ms, e_clk
    plans_run = [v.plan_names() for v in variants]

    tokens_per_step = sum(v.T for v in variants) * world
    ms_per_step = elapsed / args.steps
    value = tokens_per_step / (ms_per_step / 1e3)

    # ---- the same steps with every layer on the token plan (primitives on the
    # activations): the block contractions and permutations the cost model
    # replaced, measured against their own rooflines
    token = None
    if not args.no_token_plan and any(p != "token" for p in plans_run):
        for v in variants:
            v.use_plan(1, saved_pool, device)
        need = max(v.ws_need for v in variants)
        if ws.numel() < need:
            ws = None
            ws = torch.empty(need, dtype=torch.uint8, device=device)
        for v in variants:
            v.ws = ws
        for _ in range(max(1, min(args.warmup, 2))):
            step()
        t_el, t_pv, t_trace, t_traces, _, _ = timed(args.steps)
        token = {"ms_per_step": round(t_el / args.steps, 3),
                 "tokens_per_s": round(sum(v.T for v in variants) * world / (t_el / args.steps / 1e3), 1),
                 "variants": {v.wl.name: round(t_pv[i] / args.steps, 3) for i, v in enumerate(variants)},
                 "kernels": None}
        token["kernels"] = {v.wl.name: kernel_table(t_traces[i], args.steps) for i, v in enumerate(variants)}
        for v in variants:
            v.use_plan(PLANS[args.plan], saved_pool, device)

    # ---- merge-then-reinitialize (timed once, amortized over the merge period)
    merge = {}
    if not args.no_merge:
        for v in variants:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            v.merge_all()
            b.record(stream)
            b.synchronize()
            merge[v.wl.name] = a.elapsed_time(b)
        poet.poet_sync_status()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, variants, world)

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    rows = {k: dict(v) for k, v in trace.items()}
    roof = roofline_of(rows, poet.poet_version())
    kernels = kernel_table(rows, args.steps)

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline([v.wl for v in variants])

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wls[0].dtype == I.BF16 else "f32",
        "data": "synthetic (seeded N(0,1) tokens, normalized-Gaussian W0, random-init skew parameters)",
        "config": {"workload": args.workload + "_" + "+".join(w.name.split("_", 1)[1] for w in wls),
                   "hidden": wls[0].hidden, "ffn": wls[0].ffn, "layers": wls[0].layers,
                   "linears_per_layer": len(wls[0].linear_shapes()), "tokens_per_variant": wls[0].tokens,
                   "variants": [{"name": v.wl.name, "mode": "FS" if v.wl.mode == I.FS else "BS", "b": v.wl.b,
                                 "k": v.wl.k, "plan": plans_run[i]} for i, v in enumerate(variants)],
                   "plan_requested": args.plan,
                   "parallelism": f"dp{world}", "l2": "inputs larger than L2 (no flush needed)",
                   "activation_rows": "row stride = width rounded up to 8 elements (16-byte aligned rows)",
                   "linears_per_call": variants[0].per_call},
        "variants": {v.wl.name: {"ms_per_step": round(per_variant_ms[i] / args.steps, 3),
                                 "tokens_per_s": round(v.T * world / (per_variant_ms[i] / args.steps / 1e3), 1),
                                 "merge_ms": round(merge.get(v.wl.name, float("nan")), 3) if merge else None,
                                 "merge_tflops": (round(v.merge_flop() / (merge[v.wl.name] / 1e3) / 1e12, 1)
                                                  if merge else None),
                                 "kernels_ms_per_step": {k: round(r["ms"] / args.steps, 2) for k, r in
                                                         sorted(traces[i].items(), key=lambda kv: -kv[1]["ms"])}}
                     for i, v in enumerate(variants)},
        "value_merge_amortized": (round(tokens_per_step / ((ms_per_step + sum(merge.values()) / 400.0) / 1e3), 1)
                                  if merge else None),
        "timing": {"mode": "cuda_graph" if use_graph else "eager",
                   "eager_ms_per_step": round(e_elapsed / args.steps, 3)},
        "roofline": roof, "kernels": kernels, "gpu_launches": int(launches), "clocks": clk,
        "e2e": e2e, "cpu_baseline": cpu, "token_plan": token,
    }
    out["roofline"]["per_kind_ms_frac"] = {k: [r["ms_per_step"], r["frac"], r["bound"]] for k, r in kernels.items()}
    if not args.no_other_workloads and world == 1:
        # the other layer sets, one at a time, after the headline's buffers are freed
        del variants, ws, gws, saved_pool, act_cache, graphs, e2e, token
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        others = {}
        for name in OTHER_WORKLOADS:
            others[name] = measure_workload(name, args, device, rank, PLANS[args.plan])
            if not args.no_cpu_baseline:
                wl = I.WORKLOADS[name]
                full = wl.tokens * wl.layers <= 4096  # the small sets: every token of the layer set
                widest = max(max(m, n) for m, n in wl.linear_shapes())
                # one thread only where the widest primitive is <= 1024 (a 3456-wide Cayley-Neumann
                # gradient alone takes about a minute on one core)
                one_ok = wl.mode == I.BS or widest // 2 <= 1024
                one = cpu_baseline([wl], budget_s=6.0, threads=1, full=full) if one_ok else None
                allc = cpu_baseline([wl], budget_s=6.0, full=full)
                others[name].update({"cpu_1t_tok_s": one["value"] if one else None,
                                     "cpu_all_tok_s": allc["value"], "cpu_cores": allc["cores"], "cpu_full": full})
                if not one:
                    others[name]["cpu_1t_note"] = "not timed: primitives wider than 1024 (minutes on one core)"
        for name, (base, ov) in SMALLB_PROBES.items():
            others[name] = measure_workload(base, args, device, rank, PLANS["token"], ov)
        for name in BLOCK_WORKLOADS:
            others[name] = measure_block(name, args, device)
        out["workloads"] = others
    print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_e2e(args, variants, world):
    """The same steps through the public API with host buffers.  Every step
    copies its inputs (x and dy of every linear shape) from pinned host memory
    and reads its results (all dtheta, and y and dx of the first layer) back
    into pinned host memory.  The copies run on a second stream, double
    buffered: step i+1's inputs go up while step i computes, and step i's
    results come down (from a device-side snapshot) while step i+1 computes.
    The timed region spans the first upload to the last download."""
    import torch

    stream = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    def whole_rows(t):
        """The activation's padded rows (a dense view), so that copies of it are plain memory copies."""
        return t.as_strided((t.shape[0], t.stride(0)), (t.stride(0), 1)) if t.dim() == 2 else t

    # device inputs: set 0 = the tensors the variants hold, set 1 = copies (one per distinct tensor),
    # each in the same padded row layout
    uniq = {}
    for v in variants:
        for d in (v.x, v.dy):
            for t in d.values():
                uniq[id(t)] = t
    second = {k: torch.empty_like(whole_rows(t))[:, : t.shape[1]] for k, t in uniq.items()}
    sets = [{k: t for k, t in uniq.items()}, second]
    host_in = {k: whole_rows(t).cpu().pin_memory() for k, t in uniq.items()}
    base = [({n: t for n, t in v.x.items()}, {m: t for m, t in v.dy.items()}) for v in variants]

    def use_set(sidx):
        for v, (bx, bdy) in zip(variants, base):
            v.x = {n: sets[sidx][id(t)] for n, t in bx.items()}
            v.dy = {m: sets[sidx][id(t)] for m, t in bdy.items()}

    # results: per variant dtheta, y and dx of the first layer; a device snapshot and a host copy per set
    outs = []
    for v in variants:
        last_m, last_n = v.layers[0][2], v.layers[0][3]
        outs += [v.dtheta, whole_rows(v.y[last_m]), whole_rows(v.dx[last_n])]
    snap = [[torch.empty_like(t) for t in outs] for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs] for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in host_in.values())
    d2h = sum(h.numel() * h.element_size() for h in host_out[0])

    use_graph = not args.no_graph and world == 1
    graphs = None
    if use_graph:  # one graph per variant and input set (the sets differ in pointers)
        graphs = []
        for sidx in range(2):
            use_set(sidx)
            row = []
            for v in variants:
                copy.wait_stream(stream)
                gph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gph, stream=copy):
                    v.step(world)
                stream.wait_stream(copy)
                row.append(gph)
            graphs.append(row)
        torch.cuda.synchronize()

    ev_in = [torch.cuda.Event() for _ in range(2)]       # set s uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]     # compute on set s finished
    ev_snap = [torch.cuda.Event() for _ in range(2)]     # snapshot s written
    ev_down = [torch.cuda.Event() for _ in range(2)]     # snapshot s downloaded

    def upload(sidx, after_use):
        with torch.cuda.stream(copy):
            if after_use:
                copy.wait_event(ev_used[sidx])
            for k, h in host_in.items():
                whole_rows(sets[sidx][k]).copy_(h, non_blocking=True)
            ev_in[sidx].record(copy)

    def run(steps):
        upload(0, False)
        for i in range(steps):
            sidx = i % 2
            if i + 1 < steps:
                upload(1 - sidx, i >= 1)
            stream.wait_event(ev_in[sidx])
            use_set(sidx)
            if graphs is not None:
                for gph in graphs[sidx]:
                    gph.replay()
            else:
                for v in variants:
                    v.step(world)
            ev_used[sidx].record(stream)
            if i >= 2:
                stream.wait_event(ev_down[sidx])
            for src, dst in zip(outs, snap[sidx]):
                dst.copy_(src, non_blocking=True)
            ev_snap[sidx].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(ev_snap[sidx])
                for src, dst in zip(snap[sidx], host_out[sidx]):
                    dst.copy_(src, non_blocking=True)
                ev_down[sidx].record(copy)
        stream.wait_stream(copy)

    run(2)  # warm
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run(args.e2e_steps)
    b.record(stream)
    b.synchronize()
    use_set(0)
    ms = a.elapsed_time(b) / args.e2e_steps
    tokens = sum(v.T for v in variants) * world
    return {"value": round(tokens / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 3),
            "steps": args.e2e_steps, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "copies": "second stream, double-buffered", "mode": "cuda_graph" if use_graph else "eager"}


# ---------------------------------------------------------------------------- CPU oracle

def cpu_baseline(wls, budget_s=25.0, threads=None, full=False):
    """The float64 CPU oracle, as it stands, on a bounded sample of the same
    workload, extrapolated to the full step in tokens/s (full: every token of
    one layer set).  threads: BLAS threads to allow (None: as configured)."""
    import contextlib

    from threadpoolctl import threadpool_info, threadpool_limits

    ctx = threadpool_limits(limits=threads, user_api="blas") if threads else contextlib.nullcontext()
    with ctx:
        return _cpu_baseline(wls, budget_s, full)


def _cpu_baseline(wls, budget_s, full):
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import poet_oracle as O
    from orthogonal_reparameterized_poet_b200 import inputs as I

    cores = sum(p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas") or 1
    total_s, total_tokens = 0.0, 0
    sample_desc = []
    t_start = time.perf_counter()
    for wl in wls:
        shapes = wl.linear_shapes()
        Ts = wl.tokens if full else 64
        # token-independent part: Cayley-Neumann forward + backward, once per distinct primitive size
        cnp_s = {}
        for (m, n) in set(shapes):
            for d in (m, n):
                nprim, size = O.side_shape(d, wl.mode, wl.b)
                if size in cnp_s or nprim == 0:
                    continue
                th = I.theta(wl.seed, 0, 0, 0, O.n_skew(size), wl.sigma).astype(np.float64)
                G = np.random.default_rng(0).standard_normal((1, size, size))
                t = time.perf_counter()
                O.cayley_neumann(th, 1, size, wl.k)
                O.theta_grad(G, th, size, wl.k)
                cnp_s[size] = time.perf_counter() - t
        # token-dependent part: dense forward + backward on Ts tokens, once per distinct linear shape
        tok_s = {}
        for t_idx, (m, n) in enumerate(shapes):
            if (m, n) in tok_s:
                continue
            W0 = I.w0(wl.seed, 0, t_idx, m, n, wl.dtype).astype(np.float64)
            nR, sR = O.side_shape(m, wl.mode, wl.b)
            nP, sP = O.side_shape(n, wl.mode, wl.b)
            permR, permP = O.draw_perm(wl.seed, t_idx, 0, 0, m), O.draw_perm(wl.seed, t_idx, 1, 0, n)
            Rb = np.broadcast_to(np.eye(sR), (nR, sR, sR)) if nR else np.zeros((0, 0, 0))
            Pb = np.broadcast_to(np.eye(sP), (nP, sP, sP)) if nP else np.zeros((0, 0, 0))
            x = I.activations(wl.seed, n, Ts, n, wl.dtype).astype(np.float64)
            dy = I.activations(wl.seed, m, Ts, m, wl.dtype, grad=True).astype(np.float64)
            t = time.perf_counter()
            R = O.dense_side(permR, Rb, wl.mode, wl.b)
            P = O.dense_side(permP, Pb, wl.mode, wl.b)
            O.forward(W0, R, P, x)
            O.backward(W0, R, P, x, dy, permR, wl.mode, wl.b, permP, wl.mode, wl.b)
            tok_s[(m, n)] = time.perf_counter() - t
        per_layer = 0.0
        for (m, n) in shapes:
            for d in (m, n):
                nprim, size = O.side_shape(d, wl.mode, wl.b)
                if nprim:
                    per_layer += nprim * cnp_s[size]
            per_layer += tok_s[(m, n)] * wl.tokens / Ts
        total_s += per_layer * wl.layers
        total_tokens += wl.tokens
        sample_desc.append(f"{wl.name}: Cayley-Neumann fwd+bwd once per distinct primitive size "
                           f"{sorted(cnp_s)}, dense fwd+bwd of {Ts} tokens once per distinct linear shape"
                           + ("" if Ts < wl.tokens else " (all tokens)"))
        if time.perf_counter() - t_start > budget_s:
            break
    wall = time.perf_counter() - t_start
    return {"value": round(total_tokens / total_s, 3), "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": "; ".join(sample_desc) + f"; extrapolated linearly to all layers and tokens "
                      f"({wall:.1f} s of CPU work)", "sample_wall_s": round(wall, 2)}


def run_reference(args):
    """The oracle as the reference arm: rank 0 times it on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from orthogonal_reparameterized_poet_b200 import inputs as I

    wls = [I.WORKLOADS[name] for name in WORKLOAD_SETS[args.workload]]
    vals = []
    res = None
    for i in range(args.warmup + args.steps):
        res = cpu_baseline(wls, budget_s=8.0)
        if i >= args.warmup:
            vals.append(res["value"])
    value = statistics.median(vals) if vals else res["value"]
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sum(w.tokens for w in wls) / value * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload + "_" + "+".join(w.name.split("_", 1)[1] for w in wls),
                   "tokens_per_variant": wls[0].tokens, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": res["cores"], "kind": "oracle",
                         "sample": res["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_probe(args):
    import torch

    from orthogonal_reparameterized_poet_b200 import poet

    torch.cuda.set_device(0)
    poet.lib()
    if args.probe in SMALLB_PROBES:
        base, ov = SMALLB_PROBES[args.probe]
        res = measure_workload(base, args, torch.device("cuda", 0), 0, PLANS["token"], ov)
    elif args.probe in BLOCK_WORKLOADS:
        res = measure_block(args.probe, args, torch.device("cuda", 0))
    else:
        res = measure_workload(args.probe, args, torch.device("cuda", 0), 0, PLANS[args.plan])
    print(json.dumps({"probe": args.probe, **res}), flush=True)


def main():
    args = parse_args()
    if args.probe:
        run_probe(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_poet(args)


if __name__ == "__main__":
    main()
