"""Benchmark of the Sparse-BitLinear forward on B200.

Workload (one "step"): the seven Qwen2.5-0.5B-shaped projections of one layer
(q 896->896, k/v 896->128, o 896->896, gate/up 896->4864, down 4864->896) at
3:4 sparsity, each taken from latent fp32 weights through the whole path:
weight preparation (mask, scale, ternarise, pack), activation quantisation,
the prefill contraction at T = 2048 tokens and the decode contraction at
T = 1, with fp32 outputs.  Inputs are seeded synthetic draws (W ~ N(0, 0.02^2),
x ~ N(0, 1) in bf16), resident in HBM; L2 is flushed (a 256 MiB write)
between timed steps.  The metric is tokens per second: 2049 tokens per step
per GPU (the 2048-token prefill batch plus one decode token).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own copy of the step on its own GPU (the
forward has no cross-GPU exchange): weak scaling, timed as the max over ranks.
``--impl reference`` times the CPU oracle on full steps of the same workload.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_linear_layers_b200 import synthetic  # noqa: E402

METRIC = "Sparse-BitLinear tokens/s; decode HBM GB/s and prefill int8 TOPS vs B200 peak"
N, M = 3, 4
T_PREFILL, T_DECODE = 2048, 1
TOKENS_PER_STEP = T_PREFILL + T_DECODE
WORKLOAD = "qwen2.5-0.5b layer projections (q,k,v,o,gate,up,down), 3:4, prep + T=2048 prefill + T=1 decode"


# DRAM bytes (read + write) per prefill call of one input group (activation
# quantisation + tcgen05 GEMM), mean over the four groups at T = 2048, from one
# ncu capture of the step's eager pass (`bench.py --only step_once`,
# dram__bytes_read.sum + dram__bytes_write.sum; outputs still in L2 when a
# launch ends are not counted).
# Only valid for the kernel sources the counters were taken on; reported as null
# once those change.
PREFILL_TRAFFIC = {"sources_sha256": "475680e8ebc388db0be773f273cb4307d186640a9dc5a0486c0853f79df3123a", "bytes_per_call": 16770752}


def _kernel_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for f in ("sbl_common.cuh", "tc_util.cuh", "quant.cu", "prefill.cu", "prefill_pair.cu"):
        with open(os.path.join(ROOT, "sparse_linear_layers_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _config(extra=None):
    c = {"workload": WORKLOAD, "layers": [f"{nm} {k}->{o}" for nm, k, o in synthetic.QWEN05_LAYER],
         "sparsity": f"{N}:{M}", "tokens_prefill": T_PREFILL, "tokens_decode": T_DECODE,
         "output_dtype": "fp32", "l2": "flushed between timed steps (256 MiB write)", "seed": 0}
    if extra:
        c.update(extra)
    return c


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling during the timed region (SM clock, throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- our arm

class Layer:
    """Weights and outputs of one projection."""

    def __init__(self, name, K, O, dev, seed=0):
        import sparse_linear_layers_b200 as sbl
        self.name, self.K, self.O = name, K, O
        W = synthetic.latent_weights(O, K, seed=seed, tag=f"bench-{name}")
        self.W_host = torch.from_numpy(W).pin_memory()
        self.W = self.W_host.to(dev)
        self.w = sbl.PreparedWeights(torch.empty((O, K // 4), dtype=torch.uint8, device=dev),
                                     torch.empty((O,), dtype=torch.float32, device=dev), N, M, K)
        self.y = torch.empty((T_PREFILL, O), dtype=torch.float32, device=dev)
        self.y1 = torch.empty((T_DECODE, O), dtype=torch.float32, device=dev)
        self.y_host = torch.empty((T_PREFILL, O), dtype=torch.float32).pin_memory()
        self.y1_host = torch.empty((T_DECODE, O), dtype=torch.float32).pin_memory()

    def prefill_ops(self):
        return 2.0 * T_PREFILL * self.O * self.K

    def weight_bytes(self):
        return self.O * self.K / 4 + 4 * self.O


# One layer's projections in dependency order, grouped by the input they read:
# q, k and v read the same normalised hidden state, o follows attention, gate
# and up read the same normalised input, down follows.  Each group is one call
# (sbl_linear_grouped for q|k|v and gate|up: x quantised once, and at decode
# sizes one launch over the stacked weights).
INPUT_GROUPS = (("attn", ("q", "k", "v")), ("attn_out", ("o",)), ("ffn", ("gate", "up")), ("ffn_out", ("down",)))
PREP_BY_K = (("q", "k", "v", "o", "gate", "up"), ("down",))
SCHEDULE = ("weight preparation: one sbl_prepare_weights_grouped launch for the six K = 896 projections, down "
            "concurrently; prefill and decode on one stream: grouped {q,k,v} -> o -> grouped {gate,up} -> down "
            "(projections that share an input are one sbl_linear_grouped call)")


class InputGroup:
    """The activations one group of projections reads, and the group's call."""

    def __init__(self, name, members, dev, seed=0):
        import sparse_linear_layers_b200 as sbl
        self.name, self.members = name, members
        self.K = K = members[0].K
        xb, _ = synthetic.activations(T_PREFILL, K, seed=seed, tag=f"bench-x-{name}")
        x1, _ = synthetic.activations(T_DECODE, K, seed=seed, tag=f"bench-x1-{name}")
        self.x_host = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
        self.x1_host = torch.from_numpy(x1.view(np.int16)).view(torch.bfloat16).pin_memory()
        self.x = self.x_host.to(dev)
        self.x1 = self.x1_host.to(dev)
        O = sum(L.O for L in members)
        self.ws = sbl.workspace_for(T_PREFILL, K, O, N, M, dev)

    def run(self, sbl, decode=False):
        x = self.x1 if decode else self.x
        if len(self.members) == 1:
            L = self.members[0]
            sbl.sbl_linear(x, L.w, y=L.y1 if decode else L.y, workspace=self.ws)
        else:
            sbl.sbl_linear_grouped(x, [L.w for L in self.members],
                                   ys=[L.y1 if decode else L.y for L in self.members], workspace=self.ws)

    # algorithmic bytes of one call: the shared activations once, every
    # member's codes, scales and outputs
    def prefill_bytes(self):
        return 2 * T_PREFILL * self.K + sum(L.weight_bytes() + 4 * T_PREFILL * L.O for L in self.members)

    def decode_bytes(self):
        return 2 * T_DECODE * self.K + sum(L.weight_bytes() + 4 * T_DECODE * L.O for L in self.members)


def make_step(dev):
    layers = [Layer(nm, K, O, dev) for nm, K, O in synthetic.QWEN05_LAYER]
    by_name = {L.name: L for L in layers}
    groups = [InputGroup(g, [by_name[n] for n in names], dev) for g, names in INPUT_GROUPS]
    return layers, groups


def _prep_phase(sbl, layers, groups, streams):
    by_name = {L.name: L for L in layers}
    main, side = streams[0], streams[1]
    fork = torch.cuda.Event()
    fork.record(main)
    side.wait_event(fork)
    for st, names in zip((main, side), PREP_BY_K):
        with torch.cuda.stream(st):
            Ls = [by_name[n] for n in names]
            sbl.sbl_prepare_weights_grouped([L.W for L in Ls], N, M, outs=[L.w for L in Ls])
    join = torch.cuda.Event()
    join.record(side)
    main.wait_event(join)


def _prefill_phase(sbl, layers, groups, streams):
    with torch.cuda.stream(streams[0]):
        for g in groups:
            g.run(sbl)


def _decode_phase(sbl, layers, groups, streams):
    with torch.cuda.stream(streams[0]):
        for g in groups:
            g.run(sbl, decode=True)


PHASES = (("prep", _prep_phase), ("prefill", _prefill_phase), ("decode", _decode_phase))


class StepGraphs:
    """The step captured as one CUDA graph (the timed region: no host launch
    latency, and every kernel a programmatic dependent of the one before it,
    across the phases too) and, for the per-phase breakdown, as three graphs
    (weight prep, T=2048 prefill, T=1 decode) with events between their
    launches.  The events and the graph boundaries cost about 7 us per step,
    so the phase times add up to more than the timed step.  Inside a phase
    the projections follow the layer's dependency order (SCHEDULE)."""

    def __init__(self, sbl, layers, groups, stream):
        self.stream = stream
        self.side = [torch.cuda.Stream() for _ in range(6)]
        streams = [stream] + self.side
        self.graphs = []
        with torch.cuda.stream(stream):
            for _, fn in PHASES:       # one eager pass: sets kernel attributes before capture
                fn(sbl, layers, groups, streams)
        torch.cuda.synchronize()
        for _, fn in PHASES:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn(sbl, layers, groups, streams)
            self.graphs.append(g)
        self.step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.step, stream=stream):
            for _, fn in PHASES:
                fn(sbl, layers, groups, streams)

    def replay(self, ev=None):
        """One step as one graph; ev = (start, end) events around it."""
        with torch.cuda.stream(self.stream):
            if ev is not None:
                ev[0].record(self.stream)
            self.step.replay()
            if ev is not None:
                ev[1].record(self.stream)

    def replay_phases(self, ev):
        """One step as the three phase graphs, ev[0..3] recorded around them."""
        with torch.cuda.stream(self.stream):
            ev[0].record(self.stream)
            for i, g in enumerate(self.graphs):
                g.replay()
                ev[i + 1].record(self.stream)


class E2E:
    """The step from pinned host buffers: H2D of W and x, D2H of y, inside the
    timed region, every copy through the library's C ABI (sbl_copy_to_device,
    sbl_copy_to_host) like every kernel.  Three streams: host-to-device
    copies, the kernels, and device-to-host copies, so both directions of the
    host link and the kernels overlap across groups and steps.  Two sets of
    device buffers (inputs and outputs) alternate between steps, as a serving
    loop double-buffers: a step's inputs land while the previous step
    computes, and its outputs are written while the previous step's are still
    being copied back.  Events keep every buffer safe: a set's inputs are not
    overwritten before the kernels of two steps ago have read them, nor its
    outputs before they have been copied back."""

    NSETS = 2

    def __init__(self, groups):
        self.main = torch.cuda.Stream()
        self.h2d = torch.cuda.Stream()
        self.back = torch.cuda.Stream()
        self.k = 0
        self.consumed = {(g.name, s): None for g in groups for s in range(self.NSETS)}
        self.done = {(g.name, s): None for g in groups for s in range(self.NSETS)}
        # per group and set: the device buffers, and the (destination, source,
        # bytes) of every copy, checked once here so the timed loop only makes
        # the C ABI calls; set 0 is the step's own buffers
        from sparse_linear_layers_b200 import api
        pair = api._need_host_pair
        self.bufs, self.ins, self.outs = {}, {}, {}
        for g in groups:
            for st in range(self.NSETS):
                if st == 0:
                    b = dict(x=g.x, x1=g.x1, W=[L.W for L in g.members], y=[L.y for L in g.members],
                             y1=[L.y1 for L in g.members])
                else:
                    b = dict(x=torch.empty_like(g.x), x1=torch.empty_like(g.x1),
                             W=[torch.empty_like(L.W) for L in g.members], y=[torch.empty_like(L.y) for L in g.members],
                             y1=[torch.empty_like(L.y1) for L in g.members])
                ins = [(b["x"].data_ptr(), g.x_host.data_ptr(), pair(g.x_host, b["x"], "x_host", "x")),
                       (b["x1"].data_ptr(), g.x1_host.data_ptr(), pair(g.x1_host, b["x1"], "x1_host", "x1"))]
                ins += [(W.data_ptr(), L.W_host.data_ptr(), pair(L.W_host, W, "W_host", "W"))
                        for L, W in zip(g.members, b["W"])]
                outs = []
                for L, y, y1 in zip(g.members, b["y"], b["y1"]):
                    outs.append((L.y_host.data_ptr(), y.data_ptr(), pair(L.y_host, y, "y_host", "y")))
                    outs.append((L.y1_host.data_ptr(), y1.data_ptr(), pair(L.y1_host, y1, "y1_host", "y1")))
                self.bufs[(g.name, st)], self.ins[(g.name, st)], self.outs[(g.name, st)] = b, ins, outs

    def begin(self):
        """Order the copy streams after everything already on the main stream."""
        ev = torch.cuda.Event()
        ev.record(self.main)
        self.h2d.wait_event(ev)
        self.back.wait_event(ev)

    @staticmethod
    def _contract(sbl, g, x, ys):
        if len(g.members) == 1:
            sbl.sbl_linear(x, g.members[0].w, y=ys[0], workspace=g.ws)
        else:
            sbl.sbl_linear_grouped(x, [L.w for L in g.members], ys=ys, workspace=g.ws)

    def step(self, sbl, groups):
        from sparse_linear_layers_b200._lib import check, lib
        h2d = d2h = 0
        s_in, s_out = self.h2d.cuda_stream, self.back.cuda_stream
        st = self.k % self.NSETS
        self.k += 1
        for g in groups:
            key = (g.name, st)
            b = self.bufs[key]
            with torch.cuda.stream(self.h2d):
                if self.consumed[key] is not None:
                    self.h2d.wait_event(self.consumed[key])  # the kernels that last read this set are done
                for dst, src, nb in self.ins[key]:
                    check(lib.sbl_copy_to_device(dst, src, nb, s_in), "sbl_copy_to_device")
                    h2d += nb
                copied = torch.cuda.Event()
                copied.record(self.h2d)
            with torch.cuda.stream(self.main):
                self.main.wait_event(copied)
                if self.done[key] is not None:
                    self.main.wait_event(self.done[key])  # this set's outputs have been copied back
                sbl.sbl_prepare_weights_grouped(b["W"], N, M, outs=[L.w for L in g.members])
                self._contract(sbl, g, b["x"], b["y"])
                self._contract(sbl, g, b["x1"], b["y1"])
                computed = torch.cuda.Event()
                computed.record(self.main)
                self.consumed[key] = computed
            self.back.wait_event(computed)
            with torch.cuda.stream(self.back):
                for dst, src, nb in self.outs[key]:
                    check(lib.sbl_copy_to_host(dst, src, nb, s_out), "sbl_copy_to_host")
                    d2h += nb
                ev = torch.cuda.Event()
                ev.record(self.back)
                self.done[key] = ev
        return h2d, d2h

    def join(self):
        """Make the main stream wait for every copy (end of a timed region)."""
        self.main.wait_stream(self.h2d)
        self.main.wait_stream(self.back)


def _decode_roofline(sbl, dev, hbm_peak, K=2048, O=7168, T=1, reps=64, group=1):
    """T-token decode of a 2048 -> 7168 layer over a pool of distinct packed weights
    larger than 3x L2, replayed from a CUDA graph: per-call GB/s on algorithmic bytes.
    With group > 1 every call is one sbl_linear_grouped over `group` such layers
    sharing x (each with its own output)."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per = O * K // 4
    pool = max(8, int(3 * l2 // per) + 1)
    W = torch.from_numpy(synthetic.latent_weights(O, K, seed=11, tag="decode-pool")).to(dev)
    base = sbl.sbl_prepare_weights(W, 2, 4)
    del W
    packs = [base.packed.clone() for _ in range(pool)]
    x1 = torch.from_numpy(synthetic.activations(T, K, seed=11, tag="decode-x")[0].view(np.int16)).view(
        torch.bfloat16).to(dev)
    y1 = torch.empty((T, O), dtype=torch.float32, device=dev)
    ws = sbl.workspace_for(T, K, O, 2, 4, dev)
    ws_list = [sbl.PreparedWeights(p, base.row_scale, 2, 4, K) for p in packs]
    ys = [torch.empty((T, O), dtype=torch.float32, device=dev) for _ in range(group)]

    def call(i):
        if group == 1:
            sbl.sbl_linear(x1, ws_list[i % pool], y=y1, workspace=ws)
        else:
            sbl.sbl_linear_grouped(x1, [ws_list[(i * group + j) % pool] for j in range(group)], ys=ys,
                                   workspace=ws)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for i in range(4):
            call(i)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(reps):
            call(i)
    torch.cuda.synchronize()
    n_rep = 10
    batches = []
    with torch.cuda.stream(s):
        for _ in range(3):
            g.replay()
        for _ in range(5):  # median of five batches of n_rep graph replays
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(n_rep):
                g.replay()
            e1.record(s)
            e1.synchronize()
            batches.append(e0.elapsed_time(e1) / 1e3 / (n_rep * reps))
    torch.cuda.synchronize()
    per_call_s = statistics.median(batches)
    # isolated single call (cold weights)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    iso = []
    for i in range(20):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call(i)
        b.record()
        torch.cuda.synchronize()
        iso.append(a.elapsed_time(b) / 1e3)
    byts = group * (O * K / 4 + 4 * O + T * 4 * O) + T * 2 * K
    del g, packs, ws_list, flush
    ach = byts / per_call_s / 1e9
    return {"layer": f"{K}->{O} 2:4 T={T}" + (f", {group} layers per grouped call" if group > 1 else ""),
            "bytes_per_call": byts, "calls_in_graph": reps, "weight_pool": pool,
            "us_per_call": per_call_s * 1e6, "achieved_gbs": ach, "peak_gbs": hbm_peak, "frac": ach / hbm_peak,
            "isolated_call_us": statistics.median(iso) * 1e6}


def _prefill_case(sbl, dev, int8_peak_tops, hbm_peak, K, O, n, m, dtypes, T=32768, reps=10, tag="prefill-roof"):
    """One prefill sbl_linear call (activation quantisation + GEMM) at T tokens,
    graph-replayed with L2 flushed before each call; x carries 1% outliers x20."""
    W = torch.from_numpy(synthetic.latent_weights(O, K, seed=12, tag=tag)).to(dev)
    w = sbl.sbl_prepare_weights(W, n, m)
    del W
    xb, _ = synthetic.activations(T, K, seed=12, tag=tag, outlier_p=0.01)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
    ws = sbl.workspace_for(T, K, O, n, m, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ops = 2.0 * T * O * K
    path = sbl.sbl_linear_plan(T, K, O, n, m, ws.numel())
    # the sparse tensor cores run at twice the dense rate: their utilisation is
    # dense-equivalent TOPS over twice the dense peak
    path_peak = int8_peak_tops * (2.0 if path == "prefill_sparse" else 1.0)
    out = {"layer": f"{K}->{O} {n}:{m} T={T}", "ops_per_call": ops, "path": path}
    for name, dt, esz in dtypes:
        y = torch.empty((T, O), dtype=dt, device=dev)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            sbl.sbl_linear(x, w, y=y, workspace=ws)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            sbl.sbl_linear(x, w, y=y, workspace=ws)
        ts = []
        with torch.cuda.stream(s):
            for i in range(reps + 3):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s)
                g.replay()
                b.record(s)
                b.synchronize()
                if i >= 3:
                    ts.append(a.elapsed_time(b) / 1e3)
        t = statistics.median(ts)
        byts = T * K * 2 + T * K * 2 + O * K / 4 + T * O * esz  # x read, x_q written + read, codes, y
        out[name] = {"us_per_call": t * 1e6, "tops": ops / t / 1e12, "tensor_frac": ops / t / 1e12 / int8_peak_tops,
                     "tensor_frac_of_path_peak": ops / t / 1e12 / path_peak,
                     "algorithmic_bytes": byts, "hbm_gbs": byts / t / 1e9, "hbm_frac": byts / t / 1e9 / hbm_peak}
        del g, y
    del w, x, ws, flush
    return out


def _prefill_roofline(sbl, dev, int8_peak_tops, hbm_peak):
    """The 0.5B FFN shapes at T = 32768, 3:4 against 2:4 (2:4 with K >= 2048 runs on
    the structured-sparse tensor cores; tensor_frac counts the dense-equivalent
    2*T*O*K ops).  The gate at 3:4 also with fp32 output."""
    torch.cuda.nvtx.range_push("prefill_roofline")  # lets a profiler select these launches
    bf16 = ("bf16_out", torch.bfloat16, 2)
    out = {"peak_tops": int8_peak_tops, "peak_source": "int8 = 2 x measured bf16 burst (nominal dense ratio)",
           "gate_3:4": _prefill_case(sbl, dev, int8_peak_tops, hbm_peak, 896, 4864, 3, 4,
                                     (bf16, ("fp32_out", torch.float32, 4))),
           "gate_2:4": _prefill_case(sbl, dev, int8_peak_tops, hbm_peak, 896, 4864, 2, 4, (bf16,)),
           "down_3:4": _prefill_case(sbl, dev, int8_peak_tops, hbm_peak, 4864, 896, 3, 4, (bf16,)),
           "down_2:4": _prefill_case(sbl, dev, int8_peak_tops, hbm_peak, 4864, 896, 2, 4, (bf16,))}
    # the pages claim 2x for 2:4 on the sparse tensor cores: time(3:4) / time(2:4) per shape, bf16 output
    out["time_ratio_3to4_over_2to4"] = {
        shape: out[f"{shape}_3:4"]["bf16_out"]["us_per_call"] / out[f"{shape}_2:4"]["bf16_out"]["us_per_call"]
        for shape in ("gate", "down")}
    torch.cuda.nvtx.range_pop()
    return out


def _step_once(sbl, dev):
    """One eager pass of the step's three phases, no graphs and nothing else:
    a small process for profilers (launch order: prep, then per input group
    one quantisation and one GEMM, then one decode launch per group)."""
    layers, groups = make_step(dev)
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    for _, fn in PHASES:
        fn(sbl, layers, groups, streams)
    torch.cuda.synchronize()
    status = sbl.sbl_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    return {"phases": [name for name, _ in PHASES], "groups": [g.name for g in groups], "status": status}


def _int8_peak(dev, n=8192, reps=20):
    """Dense int8 tensor throughput of the library GEMM (cuBLASLt through
    torch._int_mm) on n x n x n, best of `reps` after warm-up: the measured
    counterpart of the nominal int8 = 2 x bf16 peak."""
    a = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=dev).t()
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    best = min(ts)
    return {"shape": f"{n}^3 int8 -> int32", "best_us": best * 1e6, "median_us": statistics.median(ts) * 1e6,
            "tops_best": 2.0 * n ** 3 / best / 1e12, "tops_median": 2.0 * n ** 3 / statistics.median(ts) / 1e12,
            "nominal_2x_bf16_measured": 2.0 * _peaks()[1]}


def _flushed_graph_us(fn, dev, reps=10):
    """Median device time of ``fn`` captured in a CUDA graph, L2 flushed (256 MiB
    write) before every timed replay, three untimed replays first."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fn()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    ts = []
    with torch.cuda.stream(s):
        for i in range(reps + 3):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            g.replay()
            b.record(s)
            b.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
    del g, flush
    return statistics.median(ts)


def _rmsnorm_front(sbl, dev, hbm_peak, T=32768):
    """The guide module's front end (RMSNorm, then per-token absmax int8) against
    the plain quantisation at the 0.5B FFN input widths, and the whole module
    forward against sbl_linear on the FFN gate (896 -> 4864, 3:4, bf16 output)."""
    out = {"tokens": T, "eps": sbl.RMSNORM_EPS_F32}
    for K in (896, 4864):
        xb, _ = synthetic.activations(T, K, seed=14, tag="rms", outlier_p=0.01)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        gw = torch.from_numpy(np.random.default_rng(14).uniform(0.5, 1.5, K).astype(np.float32)).to(dev)
        byts = T * K * 2 + T * K + 4 * T + 4 * K
        q_us = _flushed_graph_us(lambda: sbl.sbl_quant_act(x), dev)
        r_us = _flushed_graph_us(lambda: sbl.sbl_rmsnorm_quant_act(x, gw), dev)
        out[f"K{K}"] = {"algorithmic_bytes": byts, "quant_us": q_us, "rmsnorm_quant_us": r_us,
                        "rmsnorm_quant_gbs": byts / r_us / 1e3, "rmsnorm_quant_hbm_frac": byts / r_us / 1e3 / hbm_peak,
                        "quant_gbs": byts / q_us / 1e3}
        del x
    K, O = 896, 4864
    W = torch.from_numpy(synthetic.latent_weights(O, K, seed=14, tag="rms-gate")).to(dev)
    w = sbl.sbl_prepare_weights(W, 3, 4)
    del W
    xb, _ = synthetic.activations(T, K, seed=14, tag="rms-gate", outlier_p=0.01)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
    gw = torch.ones(K, dtype=torch.float32, device=dev)
    y = torch.empty((T, O), dtype=torch.bfloat16, device=dev)
    ws = sbl.workspace_for(T, K, O, 3, 4, dev)
    lin = _flushed_graph_us(lambda: sbl.sbl_linear(x, w, y=y, workspace=ws), dev)
    mod = _flushed_graph_us(lambda: sbl.sbl_linear_rmsnorm(x, w, gw, y=y, workspace=ws), dev)
    out["gate_896->4864_3:4_bf16"] = {"sbl_linear_us": lin, "sbl_linear_rmsnorm_us": mod, "ratio": mod / lin}
    del x, y, ws, w
    return out


def _mask_monitor_bench(sbl, dev, hbm_peak):
    """Mask change count and verification between two bitmaps: a large pair
    (32768 x 8192 weights, 2 x 32 MiB, HBM-bound) and one 2048 -> 7168
    projection (2 x 1.8 MB, latency-bound), graph-replayed with L2 flushed."""
    out = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(15)
    for name, (O, K) in (("32768x8192", (32768, 8192)), ("7168x2048", (7168, 2048))):
        a = torch.randint(0, 256, (O, K // 8), dtype=torch.uint8, device=dev, generator=gen)
        b = torch.randint(0, 256, (O, K // 8), dtype=torch.uint8, device=dev, generator=gen)
        totals = torch.empty(2, dtype=torch.int64, device=dev)
        from sparse_linear_layers_b200 import _lib
        fn = lambda: _lib.check(_lib.lib.sbl_mask_monitor(a.data_ptr(), b.data_ptr(), O, K, 2, 4, totals.data_ptr(),
                                                          None, torch.cuda.current_stream().cuda_stream),
                                "sbl_mask_monitor")
        us = _flushed_graph_us(fn, dev)
        byts = 2 * O * K // 8
        out[name] = {"bytes": byts, "us_per_call": us, "gbs": byts / us / 1e3, "hbm_frac": byts / us / 1e3 / hbm_peak}
        del a, b
    return out


# fp32 FMA peak of the CUDA cores: SMs x 128 fp32 lanes x 2 flops x clocks.max.sm (1965 MHz)
FP32_LANES_PER_SM = 128
SM_MAX_MHZ = 1965.0


def _ste_backward_bench(sbl, dev, T=4096):
    """The training path's straight-through gradients (dX = dY . W_hat,
    dW = dY^T . x_hat) of the hidden-2048 stack's projections at T tokens,
    each call graph-replayed with L2 flushed; flops 2 * T * O * K per
    gradient.  Two paths: the tcgen05 tensor cores (sbl_linear_backward_ws:
    operand passes + a bf16 GEMM over three bf16 parts of the fp32 factor, so
    3 * 2 * T * O * K bf16 flops executed, against the measured bf16 peak) and
    the CUDA cores (sbl_linear_backward, against the fp32 FMA peak)."""
    props = torch.cuda.get_device_properties(dev)
    peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12
    bf16_peak = _peaks()[1]
    out = {"tokens": T, "fp32_peak_tflops": peak,
           "peak_source": f"{props.multi_processor_count} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 x {SM_MAX_MHZ} MHz",
           "bf16_peak_tflops": bf16_peak}
    gen = torch.Generator(device=dev)
    gen.manual_seed(17)
    from sparse_linear_layers_b200 import _lib
    for name, K, O in (("q 2048->2048", 2048, 2048), ("gate 2048->7168", 2048, 7168), ("down 7168->2048", 7168, 2048)):
        W = torch.randn((O, K), device=dev, generator=gen) * 0.02
        w = sbl.sbl_prepare_weights(W, 2, 4)
        x = torch.randn((T, K), device=dev, generator=gen).to(torch.bfloat16)
        xq, st = sbl.sbl_quant_act(x)
        dY = torch.randn((T, O), device=dev, generator=gen)
        dX = torch.empty((T, K), device=dev)
        dW = torch.empty((O, K), device=dev)
        ws = torch.empty((sbl.sbl_linear_backward_workspace_bytes(T, O, K),), dtype=torch.uint8, device=dev)
        res = {}
        for g, (px, pw) in (("dX", (dX.data_ptr(), None)), ("dW", (None, dW.data_ptr()))):
            fn = lambda px=px, pw=pw: _lib.check(_lib.lib.sbl_linear_backward_ws(
                dY.data_ptr(), T, O, xq.data_ptr(), st.data_ptr(), K, w.packed.data_ptr(), w.row_scale.data_ptr(),
                px, pw, 0, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream),
                "sbl_linear_backward_ws")
            us = _flushed_graph_us(fn, dev)
            tf = 2.0 * T * O * K / us / 1e6
            res[g] = {"us": us, "tflops": tf, "bf16_tflops_executed": 3 * tf, "frac_of_bf16_peak": 3 * tf / bf16_peak}
            fn = lambda px=px, pw=pw: _lib.check(_lib.lib.sbl_linear_backward(
                dY.data_ptr(), T, O, xq.data_ptr(), st.data_ptr(), K, w.packed.data_ptr(), w.row_scale.data_ptr(),
                px, pw, 0, torch.cuda.current_stream().cuda_stream), "sbl_linear_backward")
            us = _flushed_graph_us(fn, dev)
            tf = 2.0 * T * O * K / us / 1e6
            res[g + "_cuda_cores"] = {"us": us, "tflops": tf, "frac": tf / peak}
        out[name] = res
        del W, w, x, xq, dY, dX, dW, ws
    return out


def _pool_call_us(sbl, x, w, y, ws, reps=5):
    """Per-call device time of sbl_linear in steady state: a CUDA graph of
    back-to-back calls that cycle through copies of the weights and
    activations whose total exceeds 3x L2, so every call reads cold inputs.
    Median over ``reps`` replays of the graph, divided by its call count."""
    l2 = torch.cuda.get_device_properties(x.device).L2_cache_size
    per = w.packed.numel() + x.numel() * 2
    pool = max(2, min(64, -(-3 * l2 // per), (4 << 30) // per))
    calls = max(pool, 16)
    ws_ = [sbl.PreparedWeights(w.packed.clone(), w.row_scale, w.n, w.m, w.K) for _ in range(pool)]
    xs = [x.clone() for _ in range(pool)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for i in range(2):
            sbl.sbl_linear(xs[i], ws_[i], y=y, workspace=ws)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(calls):
            sbl.sbl_linear(xs[i % pool], ws_[i % pool], y=y, workspace=ws)
    ts = []
    with torch.cuda.stream(s):
        g.replay()
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            g.replay()
            b.record(s)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / calls)
    del g, ws_, xs
    return statistics.median(ts)


def _configs_sweep(sbl, dev):
    """Tokens/s of the other workload configurations (fp32 output, seeded
    synthetic inputs, steady-state per-call times from _pool_call_us).  A
    stack's time is the sum of its projections' calls; projections of equal
    shape are timed once and counted for each."""
    cache, weights, acts = {}, {}, {}

    def call_us(K, O, n, m, T, tag):
        key = (K, O, n, m, T)
        if key in cache:
            return cache[key]
        if (K, O, n, m) not in weights:
            W = torch.from_numpy(synthetic.latent_weights(O, K, seed=13, tag=f"cfg-{tag}")).to(dev)
            weights[(K, O, n, m)] = sbl.sbl_prepare_weights(W, n, m)
            del W
        if (T, K) not in acts:
            xb, _ = synthetic.activations(T, K, seed=13, tag=f"cfg-x-{tag}", outlier_p=0.01 if T >= 4096 else 0.0)
            acts[(T, K)] = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        w, x = weights[(K, O, n, m)], acts[(T, K)]
        y = torch.empty((T, O), dtype=torch.float32, device=dev)
        ws = sbl.workspace_for(T, K, O, n, m, dev)
        us = _pool_call_us(sbl, x, w, y, ws)
        cache[key] = (us, sbl.sbl_linear_plan(T, K, O, n, m, ws.numel()))
        del y, ws
        return cache[key]

    out = {}
    us, path = call_us(256, 512, 2, 4, 16, "c1")
    out["config1_256->512_2:4_T16"] = {"us_per_call": us, "tokens_per_s": 16 / (us * 1e-6), "path": path}
    for n, m in ((3, 4), (2, 4)):
        g_us, g_path = call_us(896, 4864, n, m, 32768, "c3-gate")
        d_us, d_path = call_us(4864, 896, n, m, 32768, "c3-down")
        t = 2 * g_us + d_us
        out[f"config3_ffn_{n}:{m}_T32768"] = {"us_per_stack": t, "tokens_per_s": 32768 / (t * 1e-6),
                                               "paths": {"gate/up": g_path, "down": d_path}}
    qo_us, qo_path = call_us(2048, 2048, 2, 4, 4096, "c4-qo")
    gu_us, gu_path = call_us(2048, 7168, 2, 4, 4096, "c4-gu")
    dn_us, dn_path = call_us(7168, 2048, 2, 4, 4096, "c4-down")
    t = 2 * qo_us + 2 * gu_us + dn_us
    out["config4_h2048_2:4_T4096"] = {"us_per_stack": t, "tokens_per_s": 4096 / (t * 1e-6),
                                      "paths": {"q/o": qo_path, "gate/up": gu_path, "down": dn_path}}
    sweep = {}
    for T in (1, 8, 64, 512, 4096):
        for K, O in ((2048, 7168), (7168, 2048)):
            for n, m in ((2, 4), (3, 4), (6, 8)):
                us, path = call_us(K, O, n, m, T, f"c5-{K}-{O}")
                sweep.setdefault(f"{K}->{O}_{n}:{m}", {})[f"T{T}"] = {
                    "us_per_call": us, "tokens_per_s": T / (us * 1e-6), "path": path}
    out["config5_sweep"] = sweep
    weights.clear()
    acts.clear()
    return out


def run_ours(args, rank, world, dev):
    import sparse_linear_layers_b200 as sbl
    hbm_peak, bf16_peak, bf16_sus, peak_kind = _peaks()
    int8_peak_tops = 2.0 * bf16_peak  # nominal dense int8 : bf16 ratio of B200 (4.5 : 2.25 POPS)
    layers, groups = make_step(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    stream = torch.cuda.Stream()
    graphs = StepGraphs(sbl, layers, groups, stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            graphs.replay()
    torch.cuda.synchronize()
    status = sbl.sbl_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)  # let nvidia-smi start sampling before the timed region
        with torch.cuda.stream(stream):
            for i in range(K):
                flush.zero_()
                graphs.replay(ev[i])
        torch.cuda.synchronize()
    _barrier(world)
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    total_s = sum(step_ms) / 1e3
    total_s = _max_over_ranks(total_s, world, dev)
    clocks = clk.summary()
    # per-phase breakdown, outside the timed region: the same steps as three
    # graphs with events between them
    K_ph = min(K, 20)
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)] for _ in range(K_ph)]
    with torch.cuda.stream(stream):
        for i in range(K_ph):
            flush.zero_()
            graphs.replay_phases(evp[i])
    torch.cuda.synchronize()
    phase_ms = {name: sum(evp[i][j].elapsed_time(evp[i][j + 1]) for i in range(K_ph)) / K_ph
                for j, (name, _) in enumerate(PHASES)}

    # prefill contraction roofline (quantisation + tcgen05 GEMM, the dominant phase)
    pre_s_per_step = phase_ms["prefill"] / 1e3
    ops = sum(L.prefill_ops() for L in layers)
    byts = sum(g.prefill_bytes() for g in groups)
    t_tensor = ops / (int8_peak_tops * 1e12)
    t_hbm = byts / (hbm_peak * 1e9)
    if t_hbm >= t_tensor:
        ach = byts / pre_s_per_step / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak}
    else:
        ach = ops / pre_s_per_step / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": int8_peak_tops, "unit": "TOPS", "frac": ach / int8_peak_tops}
    n_calls = len(groups)
    traffic = PREFILL_TRAFFIC["bytes_per_call"] if _kernel_sources_digest() == PREFILL_TRAFFIC["sources_sha256"] else None
    roof.update({"traffic": traffic, "traffic_unit": "bytes per launch (DRAM read+write, ncu)",
                 "kernel": "prefill call per input group (one activation quantisation + the tcgen05 int8 GEMM of "
                           "each projection), mean over the 4 groups {q,k,v}, o, {gate,up}, down",
                 "launches_per_step": n_calls, "us_per_launch": pre_s_per_step * 1e6 / n_calls,
                 "algorithmic_bytes_per_launch": byts / n_calls, "algorithmic_ops_per_launch": ops / n_calls,
                 "peak_source": f"{peak_kind} (int8 = 2 x bf16 burst)" if roof["bound"] == "tensor"
                 else f"{peak_kind} hbm_gbs (burst copy)",
                 "tensor_tops": ops / pre_s_per_step / 1e12, "tensor_frac": ops / pre_s_per_step / 1e12 / int8_peak_tops})
    prep_bytes = sum(L.O * L.K * 4 + L.O * L.K / 4 + 4 * L.O for L in layers)
    phases = {name: {"us_per_step": 1e3 * v} for name, v in phase_ms.items()}
    phases["prep"]["gbs"] = prep_bytes / (phase_ms["prep"] / 1e3) / 1e9
    phases["decode"]["gbs"] = sum(g.decode_bytes() for g in groups) / (phase_ms["decode"] / 1e3) / 1e9
    phases["decode"]["frac_of_hbm"] = phases["decode"]["gbs"] / hbm_peak

    # end to end through host buffers
    e2e = E2E(groups)
    e2e.begin()
    for _ in range(2):
        e2e.step(sbl, groups)
    e2e.join()
    torch.cuda.synchronize()
    _barrier(world)
    K_e2e = min(K, 50)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(e2e.main)
    e2e.begin()
    for _ in range(K_e2e):
        h2d, d2h = e2e.step(sbl, groups)
    e2e.join()
    e1.record(e2e.main)
    torch.cuda.synchronize()
    e2e_s = _max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)

    decode = _decode_roofline(sbl, dev, hbm_peak) if rank == 0 else None
    if decode is not None:
        decode["T8"] = _decode_roofline(sbl, dev, hbm_peak, T=8)
        decode["grouped4"] = _decode_roofline(sbl, dev, hbm_peak, reps=16, group=4)
    prefill_big = _prefill_roofline(sbl, dev, int8_peak_tops, hbm_peak) if rank == 0 else None
    configs = _configs_sweep(sbl, dev) if rank == 0 and not args.no_configs else None
    rms_front = _rmsnorm_front(sbl, dev, hbm_peak) if rank == 0 and not args.no_configs else None
    mask_mon = _mask_monitor_bench(sbl, dev, hbm_peak) if rank == 0 and not args.no_configs else None
    ste_bwd = _ste_backward_bench(sbl, dev) if rank == 0 and not args.no_configs else None
    # prep: one launch per K; prefill: per group one quantisation and one tcgen05 GEMM launch
    # (a group's layers share it); decode: one launch per group (it quantises x itself)
    launches_per_step = len(PREP_BY_K) + 2 * len(groups) + len(groups)
    value = _throughput(world, K, total_s)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic (seeded N(0,0.02^2) fp32 weights, N(0,1) bf16 activations)",
        "config": _config({"parallelism": f"replicas x{world} (no collective on the data path)",
                           "schedule": SCHEDULE}),
        "roofline": roof,
        "decode_roofline": decode,
        "prefill_roofline": prefill_big,
        "configs": configs,
        "rmsnorm_front": rms_front,
        "mask_monitor": mask_mon,
        "ste_backward": ste_bwd,
        "phases": phases,
        "phases_note": ("phase times from a separate run of the same steps as three graphs with events between them "
                        "(the timed step is one graph); their sum exceeds ms_per_step by those boundaries"),
        "e2e": {"value": world * TOKENS_PER_STEP * K_e2e / e2e_s, "steps": K_e2e, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "calls": "C ABI only: sbl_copy_to_device (W, x), sbl_prepare_weights_grouped, sbl_linear_grouped / "
                         "sbl_linear, sbl_copy_to_host (y); pinned host buffers"},
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_sample()
    return out


# --------------------------------------------------------------------------- oracle arm

def _oracle_inputs():
    """The step's inputs for the oracle: the same seeded draws as the GPU step
    (one activation matrix per input group, shared by its projections)."""
    out = []
    K_of = {nm: K for nm, K, _ in synthetic.QWEN05_LAYER}
    O_of = {nm: O for nm, _, O in synthetic.QWEN05_LAYER}
    for g, names in INPUT_GROUPS:
        K = K_of[names[0]]
        _, xv = synthetic.activations(T_PREFILL, K, seed=0, tag=f"bench-x-{g}")
        _, x1 = synthetic.activations(T_DECODE, K, seed=0, tag=f"bench-x1-{g}")
        for nm in names:
            out.append((synthetic.latent_weights(O_of[nm], K, seed=0, tag=f"bench-{nm}"), xv, x1))
    return out


def oracle_step(inputs):
    """One full step of the CPU oracle, nothing sampled or extrapolated: the
    weight preparation of all seven projections, the 2048-token prefill
    forward and the one-token decode forward of each.  Returns
    (seconds, prep seconds, contraction seconds)."""
    import oracle
    t_prep = t_lin = 0.0
    for W, xv, x1 in inputs:
        a = time.perf_counter()
        _, scale, _, Wt = oracle.prepare_weights(W, N, M)
        b = time.perf_counter()
        oracle.linear(xv, Wt, scale)
        oracle.linear(x1, Wt, scale)
        c = time.perf_counter()
        t_prep += b - a
        t_lin += c - b
    return t_prep + t_lin, t_prep, t_lin


def cpu_baseline_sample(budget_s=None, sample_tokens=None):
    """The CPU oracle timed on full steps of the workload (2049 tokens, all seven
    projections from latent weights): once on every host core the BLAS uses
    and once on one thread, after one untimed step."""
    import threadpoolctl
    inputs = _oracle_inputs()
    oracle_step(inputs)  # untimed: first-touch and library warm-up
    all_s, prep_s, lin_s = oracle_step(inputs)
    cores = _cpu_threads()
    with threadpoolctl.threadpool_limits(limits=1):
        one_s, _, _ = oracle_step(inputs)
    ops = 2.0 * TOKENS_PER_STEP * sum(O * K for _, K, O in synthetic.QWEN05_LAYER)
    return {"value": TOKENS_PER_STEP / all_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "single_thread": {"value": TOKENS_PER_STEP / one_s, "unit": "tokens/s", "cores": 1},
            "contraction_gops": ops / lin_s / 1e9,
            "sample": f"one full step (7 weight preparations + 2048 prefill tokens + 1 decode token), measured, "
                      f"not extrapolated: {all_s:.2f} s on {cores} threads (prep {prep_s:.2f} s, contraction "
                      f"{lin_s:.2f} s), {one_s:.2f} s on 1 thread; host {os.cpu_count()} logical CPUs"}


def _cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    """The oracle arm: W untimed and K timed full oracle steps on the host's
    cores (rank 0 only; the other ranks exit without work)."""
    if rank != 0:
        return None
    inputs = _oracle_inputs()
    for _ in range(args.warmup):
        oracle_step(inputs)
    times = []
    for _ in range(args.steps):
        times.append(oracle_step(inputs)[0])
    total = sum(times)
    v = TOKENS_PER_STEP * args.steps / total
    cores = _cpu_threads()
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config({"parallelism": "CPU oracle, rank 0 only"}), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} full oracle steps (7 weight preparations + 2048 prefill "
                                       f"tokens + 1 decode token each), measured on {cores} threads"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": total}


# --------------------------------------------------------------------------- plumbing

def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _throughput(world, steps, total_s):
    """Whole-job tokens/s: every rank runs the step on its own GPU (weak scaling)."""
    return world * TOKENS_PER_STEP * steps / total_s


def _max_over_ranks(v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration sweep (profiling runs)")
    ap.add_argument("--only", choices=("rmsnorm_front", "mask_monitor", "ste_backward", "int8_peak", "step_once",
                                       "decode_roofline", "prefill_roofline"),
                    help="run only this auxiliary measurement on one GPU and print its JSON (profiling runs)")
    ap.add_argument("--tokens", type=int, default=32768, help="tokens of the --only rmsnorm_front measurement")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.only:
        import sparse_linear_layers_b200 as sbl
        hbm_peak = _peaks()[0]
        if args.only == "rmsnorm_front":
            res = _rmsnorm_front(sbl, dev, hbm_peak, T=args.tokens)
        elif args.only == "mask_monitor":
            res = _mask_monitor_bench(sbl, dev, hbm_peak)
        elif args.only == "int8_peak":
            res = _int8_peak(dev)
        elif args.only == "step_once":
            res = _step_once(sbl, dev)
        elif args.only == "decode_roofline":
            res = _decode_roofline(sbl, dev, hbm_peak)
        elif args.only == "prefill_roofline":
            res = _prefill_roofline(sbl, dev, 2.0 * _peaks()[1], hbm_peak)
        else:
            res = _ste_backward_bench(sbl, dev)
        print(json.dumps({"only": args.only, "result": res}), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        out = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
