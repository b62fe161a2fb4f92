#!/usr/bin/env python
"""Benchmark of the quantized MoE expert matmul on B200.

Metric: MoE-layer microseconds and achieved HBM GB/s (algorithmic bytes /
time) against tokens-per-expert M.  Headline workload: a DeepSeek-V2-Lite-
shaped decode MoE layer (H=2048, I=1408, 64 routed experts top-6 + 2 shared,
INT4 FC1/FC2, block 64) with M tokens that share router logits, so each of
the 8 selected experts receives exactly M tokens; the headline line is M=1.
A step is one MoE-layer forward (route -> gather -> FC1+SwiGLU -> FC2 ->
combine) through the C ABI.  8 copies of the layer's weights (2.4 GB) are
rotated step by step, so consecutive steps never hit the 126 MB L2.

Also reported: the M sweep 1..32 of the same layer and the single quantized
linear K=5120 -> N=17408 (group 128, INT2 and INT4) at M = 1..32.

`--impl reference` times the CPU fp64 oracle on the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from skinny_gemm_top_b200 import synth  # noqa: E402

CFG = synth.V2LITE
SEED = 1
ROTATE = 8
METRIC = "MoE-layer µs and HBM GB/s (% of B200 peak) vs tokens-per-expert M=1..32"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", default="1,2,4,8,16,32")
    ap.add_argument("--linear-sweep", default="1,2,3,4,5,8,10,16,32")
    ap.add_argument("--quick", action="store_true", help="skip the sweeps")
    ap.add_argument("--profile", action="store_true",
                    help="a few eager layer forwards and linears only (for an ncu launch list or capture)")
    ap.add_argument("--profile-prefill", action="store_true",
                    help="two eager forwards of the prefill layer (T = 4096, one row tile) only, for an ncu capture")
    ap.add_argument("--profile-ternary", action="store_true",
                    help="a few eager forwards of the ternary layer (128 experts, T = 1) only, for an ncu capture")
    ap.add_argument("--profile-chan", action="store_true",
                    help="a few eager forwards of the channel-selective layer (V2-Lite, T = 1, 18%%) only, for ncu")
    return ap.parse_args()


# ------------------------------------------------------------------ byte accounting

def expert_bytes(fmt: str, rows: int, K: int, block: int) -> int:
    code = rows * K * 13 // 64 if fmt == "ternary" else rows * K * {"int2": 2, "int4": 4}[fmt] // 8
    return code + rows * (K // block) * 2


FC1_BYTES = expert_bytes(CFG.fc1_fmt, 2 * CFG.I, CFG.H, CFG.block)
FC2_BYTES = expert_bytes(CFG.fc2_fmt, CFG.H, CFG.I, CFG.block)


def active_experts(logits_row: np.ndarray) -> list[int]:
    order = np.argsort(-logits_row.astype(np.float64), kind="stable")
    return sorted(int(e) for e in order[: CFG.k]) + [CFG.E + j for j in range(CFG.n_shared)]


def layer_bytes(logits: np.ndarray) -> dict:
    """Algorithmic bytes of one layer forward: weights of the active experts,
    x, y and logits (each read or written once)."""
    T = logits.shape[0]
    act = set()
    for t in range(T):
        act.update(active_experts(logits[t]))
    n = len(act)
    io = T * CFG.H * 2 * 2 + T * CFG.E * 4
    return {"total": n * (FC1_BYTES + FC2_BYTES) + io, "fc1": n * FC1_BYTES + T * CFG.H * 2, "experts": n}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ GPU arm

def _to_dev(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def pack_moe(qmoe, torch, rotate: int):
    """Pack the layer once on the host, then replicate it `rotate` times on the device."""
    n = CFG.E + CFG.n_shared
    f1, f2 = qmoe.FMT[CFG.fc1_fmt], qmoe.FMT[CFG.fc2_fmt]
    c1, s1 = qmoe.pack_stack(f1, qmoe.ROWS_GATE_UP, (synth.expert_fc1(CFG, SEED, e) for e in range(n)), CFG.block)
    c2, s2 = qmoe.pack_stack(f2, qmoe.ROWS_KSPLIT, (synth.expert_fc2(CFG, SEED, e) for e in range(n)), CFG.block)
    dev = [_to_dev(torch, a) for a in (c1, s1, c2, s2)]
    layers, keep = [], []
    for r in range(rotate):
        copies = dev if r == 0 else [t.clone() for t in dev]
        keep.append(copies)
        w1 = qmoe.make_weights(f1, CFG.block, copies[0], copies[1], None, qmoe.ROWS_GATE_UP)
        w2 = qmoe.make_weights(f2, CFG.block, copies[2], copies[3], None, qmoe.ROWS_KSPLIT)
        layers.append(qmoe.make_layer(CFG.H, CFG.I, CFG.E, CFG.k, CFG.n_shared, w1, w2))
    return layers, keep


def graph_of(torch, fn, count: int):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0, 1)  # one eager call on the capture stream (allocations, attributes)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        for i in range(count):
            fn(i, count)
    return g


class Steps:
    """K forward calls as graph replays: full graphs of `rotate` calls plus a tail graph."""

    def __init__(self, torch, fn, rotate: int):
        self.torch, self.fn, self.rotate = torch, fn, rotate
        self.full = graph_of(torch, fn, rotate)
        self.tails = {}

    def prepare(self, *ks: int):
        for k in ks:
            rem = k % self.rotate
            if rem and rem not in self.tails:
                self.tails[rem] = graph_of(self.torch, self.fn, rem)

    def run(self, k: int):
        for _ in range(k // self.rotate):
            self.full.replay()
        rem = k % self.rotate
        if rem:
            if rem not in self.tails:
                self.tails[rem] = graph_of(self.torch, self.fn, rem)
            self.tails[rem].replay()


def reduce_ranks(torch, dist, ms: float, nbytes: float, device: str = "cuda"):
    """Whole-job aggregation: the slowest rank's time and the bytes all ranks moved."""
    if dist is None:
        return ms, nbytes
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    b = torch.tensor([nbytes], dtype=torch.float64, device=device)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


def time_steps(torch, dist, steps: Steps, k: int) -> float:
    """ms for k steps, device-timed with events, max over ranks."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    steps.run(k)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def moe_inputs(torch, M: int, rotate: int):
    xs = [_to_dev(torch, synth.tokens(CFG.H, SEED, M, index=r)) for r in range(rotate)]
    rows = synth.router_logits(CFG, SEED, rotate, index=7)
    lgs_np = [np.repeat(rows[r:r + 1], M, axis=0) for r in range(rotate)]
    lgs = [torch.from_numpy(l).cuda() for l in lgs_np]
    return xs, lgs, lgs_np


def run_profile(args):
    """A handful of eager forwards and linears on one GPU: small enough for ncu."""
    import torch
    from skinny_gemm_top_b200 import qmoe
    layers, keep = pack_moe(qmoe, torch, 1)
    for M in (1, 8):
        xs, lgs, _ = moe_inputs(torch, M, 1)
        ws = torch.empty(qmoe.workspace_size(layers[0], M), dtype=torch.uint8, device="cuda")
        y = torch.empty((M, CFG.H), dtype=torch.int16, device="cuda")
        for _ in range(args.steps):
            qmoe.forward(layers[0], xs[0], lgs[0], y, ws)
            torch.cuda.synchronize()
    N, K = 17408, 5120
    c, s = qmoe.pack(qmoe.INT2, qmoe.ROWS_PLAIN, synth.linear_weight(SEED, N, K), 128)
    dc, ds = _to_dev(torch, c), _to_dev(torch, s)
    w = qmoe.make_weights(qmoe.INT2, 128, dc, ds)
    x = _to_dev(torch, synth.tokens(K, SEED, 1))
    y = torch.empty((1, N), dtype=torch.int16, device="cuda")
    ws = torch.empty(qmoe.linear_workspace_size(N, K, 1), dtype=torch.uint8, device="cuda")
    for _ in range(args.steps):
        qmoe.linear(w, N, K, x, y, ws)
        torch.cuda.synchronize()
    print("profile run done", flush=True)


def run_profile_prefill(args):
    """Two eager forwards of the prefill layer (T = 4096, 128 experts top-8) with a full workspace (one row tile)."""
    import torch
    from skinny_gemm_top_b200 import qmoe
    cfg = synth.PREFILL
    layer, keep = pack_cfg(qmoe, torch, cfg)
    T = 4096
    x = _to_dev(torch, synth.tokens(cfg.H, SEED, T))
    lg = torch.from_numpy(np.ascontiguousarray(synth.router_logits(cfg, SEED, T, index=100))).cuda()
    ws = torch.empty(qmoe.workspace_size(layer, T), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    for _ in range(2):
        qmoe.forward(layer, x, lg, y, ws)
        torch.cuda.synchronize()
    assert qmoe.get_stats().device_status == 0
    del keep
    print("prefill profile run done", flush=True)


def run_profile_ternary(args):
    """A few eager forwards of the ternary layer (H=2048, I=6144, 128 experts top-1) at T = 1."""
    import torch
    from skinny_gemm_top_b200 import qmoe
    cfg = synth.TERNARY
    layer, keep = pack_cfg(qmoe, torch, cfg, distinct=8)
    x = _to_dev(torch, synth.tokens(cfg.H, SEED, 1))
    ws = torch.empty(qmoe.workspace_size(layer, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty((1, cfg.H), dtype=torch.int16, device="cuda")
    for r in range(max(args.steps, 1)):
        lg = torch.from_numpy(np.ascontiguousarray(synth.router_logits(cfg, SEED, 1, index=100 + r))).cuda()
        qmoe.forward(layer, x, lg, y, ws)
        torch.cuda.synchronize()
    assert qmoe.get_stats().device_status == 0
    del keep
    print("ternary profile run done", flush=True)


# ------------------------------------------------------------------ channel-selective layer

CHAN_BUDGETS = (0.13, 0.18, 1.0)  # the explainer's 13% and 18% read budgets, and every channel


def pack_chan(qmoe, torch, cfg, copies: int = 1):
    """Channel layer of `cfg` (records, sketches, norms, signs) packed once on the
    host, `copies` device copies (so that consecutive steps do not reuse L2)."""
    f1, f2 = qmoe.FMT[cfg.fc1_fmt], qmoe.FMT[cfg.fc2_fmt]
    signs = synth.rht_signs(SEED, cfg.H)
    recs, sks, dns = [], [], []
    for e in range(cfg.E + cfg.n_shared):
        routed = e < cfg.E
        r, s, d = qmoe.chan_pack(f1, f2, synth.expert_fc1(cfg, SEED, e), synth.expert_fc2(cfg, SEED, e), cfg.block,
                                 signs if routed else None, sketch=routed)
        recs.append(r)
        if routed:
            sks.append(s)
            dns.append(d)
    host = [np.concatenate(recs), np.concatenate(sks), np.concatenate(dns), signs]
    layers, keep = [], []
    for _ in range(copies):
        dev = [_to_dev(torch, a) for a in host]
        keep.append(dev)
        layers.append(qmoe.make_chan_layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.n_shared, f1, f2, cfg.block, *dev))
    R, SK = qmoe.chan_sizes(f1, f2, cfg.H, cfg.block)
    return layers, keep, R, SK


def chan_step_bytes(cfg, logits: np.ndarray, n_keep: int, R: int, SK: int) -> int:
    """Algorithmic bytes of one channel-layer forward: the sketch records and
    norms of the active routed experts, the selected and shared channel
    records, x, y and the logits."""
    T = logits.shape[0]
    act = set()
    for t in range(T):
        act.update(int(e) for e in np.argsort(-logits[t].astype(np.float64), kind="stable")[:cfg.k])
    return (len(act) * cfg.I * (SK + 4) + T * n_keep * R + cfg.n_shared * cfg.I * R
            + 2 * T * cfg.H * 2 + T * cfg.E * 4)


def chan_sweep(qmoe, torch, dist, args, cfg, Ts, rotate: int = 16, copies: int = 3) -> dict:
    """The channel-selective layer on `cfg` for each T and read budget."""
    layers, keep, R, SK = pack_chan(qmoe, torch, cfg, copies)
    out = {"config": f"{cfg.name}: H={cfg.H} I={cfg.I} E={cfg.E} top-{cfg.k} + {cfg.n_shared} shared, "
                     f"FC1 {cfg.fc1_fmt} / FC2 {cfg.fc2_fmt} (columns), block {cfg.block}; sketch 2-bit trits, "
                     f"block 128; {copies} device copies rotated", "record_bytes": R, "sketch_bytes": SK, "runs": []}
    for T in Ts:
        xs = [_to_dev(torch, synth.tokens(cfg.H, SEED, T, index=r)) for r in range(rotate)]
        lgs_np = [synth.router_logits(cfg, SEED, T, index=100 + r) for r in range(rotate)]
        lgs = [torch.from_numpy(np.ascontiguousarray(l)).cuda() for l in lgs_np]
        ys = [torch.empty((T, cfg.H), dtype=torch.int16, device="cuda") for _ in range(rotate)]
        for b in CHAN_BUDGETS:
            n_keep = int(round(b * cfg.k * cfg.I))
            ws = torch.empty(qmoe.chan_workspace_size(layers[0], T, n_keep), dtype=torch.uint8, device="cuda")
            nrot = max(rotate, copies)

            def fn(i, n, xs=xs, lgs=lgs, ys=ys, ws=ws, n_keep=n_keep):
                r = i % rotate
                qmoe.chan_forward(layers[i % copies], xs[r], lgs[r], n_keep, ys[r], ws)

            steps = Steps(torch, fn, nrot)
            k = max(nrot, (args.steps // nrot) * nrot)
            steps.prepare(k, args.warmup)
            steps.run(max(args.warmup, 3))
            ms = reduce_ranks(torch, dist, time_steps(torch, dist, steps, k), 0.0)[0] / k
            nbytes = statistics.mean(chan_step_bytes(cfg, l, n_keep, R, SK) for l in lgs_np)
            out["runs"].append({"T": T, "budget": b, "n_keep": n_keep, "us": round(ms * 1e3, 3),
                                "GBps": round(nbytes / (ms * 1e6), 1), "bytes": int(nbytes)})
    assert qmoe.get_stats().device_status == 0
    del keep, layers
    return out


def run_profile_chan(args):
    """A few eager forwards of the channel-selective layer (V2-Lite shapes, T = 1, 18% of the routed channels)."""
    import torch
    from skinny_gemm_top_b200 import qmoe
    cfg = synth.V2LITE
    layers, keep, _, _ = pack_chan(qmoe, torch, cfg, 1)
    n_keep = int(round(0.18 * cfg.k * cfg.I))
    x = _to_dev(torch, synth.tokens(cfg.H, SEED, 1))
    ws = torch.empty(qmoe.chan_workspace_size(layers[0], 1, n_keep), dtype=torch.uint8, device="cuda")
    y = torch.empty((1, cfg.H), dtype=torch.int16, device="cuda")
    for r in range(max(args.steps, 1)):
        lg = torch.from_numpy(np.ascontiguousarray(synth.router_logits(cfg, SEED, 1, index=100 + r))).cuda()
        qmoe.chan_forward(layers[0], x, lg, n_keep, y, ws)
        torch.cuda.synchronize()
    assert qmoe.get_stats().device_status == 0
    del keep
    print("channel profile run done", flush=True)


def run_ours(args):
    import torch
    from skinny_gemm_top_b200 import qmoe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev_index = torch.cuda.current_device()
    layers, keep = pack_moe(qmoe, torch, ROTATE)

    def measure_moe(M: int, k: int, w: int, trace: bool = False, clocks: ClockSampler | None = None):
        xs, lgs, lgs_np = moe_inputs(torch, M, ROTATE)
        ws = torch.empty(qmoe.workspace_size(layers[0], M), dtype=torch.uint8, device="cuda")
        ys = [torch.empty((M, CFG.H), dtype=torch.int16, device="cuda") for _ in range(ROTATE)]

        def fn(i, n):
            r = i % ROTATE
            qmoe.forward(layers[r], xs[r], lgs[r], ys[r], ws)

        # launches of one forward call (traced eager call)
        qmoe.trace_start(64)
        fn(0, 1)
        qmoe.trace_stop()
        per_call = len(qmoe.trace_read(64))
        steps = Steps(torch, fn, ROTATE)
        steps.prepare(k, w)
        if clocks is not None:  # settle clocks under this load before the timed region
            t_end = time.time() + 1.5
            while time.time() < t_end:
                steps.run(ROTATE * 64)
                torch.cuda.synchronize()
        steps.run(w)
        ms = time_steps(torch, dist, steps, k)
        per = [layer_bytes(l) for l in lgs_np]
        local_bytes = statistics.mean(p["total"] for p in per)
        ms, job_bytes = reduce_ranks(torch, dist, ms, local_bytes)
        out = {"ms_per_step": ms / k, "bytes": local_bytes, "job_bytes": job_bytes,
               "fc1_bytes": statistics.mean(p["fc1"] for p in per), "launches_per_step": per_call}
        if trace:
            # Per-kernel device time: a second graph of the same ROTATE calls with CUDA
            # events around every launch (the eager call of graph_of takes per_call records).
            qmoe.trace_start(per_call * (ROTATE + 1))
            traced = Steps(torch, fn, ROTATE)
            qmoe.trace_stop()
            traced.run(w)
            t0 = time.time()
            while time.time() - t0 < 0.2:  # the timed region of the trace: replays of the traced graph
                traced.run(k)
            torch.cuda.synchronize()
            rec = qmoe.trace_read(per_call * (ROTATE + 1))[per_call:]
            out["kernels"] = {n: statistics.mean(t for m, t in rec if m == n) for n in sorted({n for n, _ in rec})}
            del traced
        return out

    sampler = ClockSampler(dev_index)
    sampler.start()
    head = measure_moe(1, args.steps, args.warmup, trace=True, clocks=sampler)
    clocks = sampler.stop()

    result_sweep = []
    if not args.quick:
        for M in [int(m) for m in args.sweep.split(",")]:
            r = measure_moe(M, max(args.steps, 64), args.warmup)
            result_sweep.append({"M": M, "us": round(r["ms_per_step"] * 1e3, 3),
                                 "GBps": round(r["bytes"] / (r["ms_per_step"] * 1e6), 1),
                                 "tokens_per_s": round(M / (r["ms_per_step"] * 1e-3), 1)})
    linear = [] if args.quick else linear_sweep(qmoe, torch, dist, args)
    lmhead = [] if args.quick else lmhead_sweep(qmoe, torch, dist, args)
    decoder_layer = [] if args.quick else model_layer_sweep(qmoe, torch, dist, args)
    # tiny layer (T = 1; 64 weight copies, 4 MB each, rotated past L2); the V2-Lite layer at
    # its own batches T = 1, 2, 4, 8 with hot-expert routing; the ternary layer (H=2048,
    # I=6144, 128 experts top-1; 8 distinct experts' bytes tiled over the 128) at
    # T = 1, 8, 32, 128; the prefill layer (T = 4096, 128 experts top-8, tcgen05 grouped
    # path, 256 MiB workspace with row tiling)
    tiny = [] if args.quick else cfg_sweep(qmoe, torch, dist, args, synth.TINY, (1,), rotate=8, copies=64)
    v2lite_batches = [] if args.quick else cfg_sweep(qmoe, torch, dist, args, synth.V2LITE, (1, 2, 4, 8), rotate=8)
    ternary = [] if args.quick else cfg_sweep(qmoe, torch, dist, args, synth.TERNARY, (1, 8, 32, 128), rotate=32,
                                              distinct=8)
    prefill = [] if args.quick else cfg_sweep(qmoe, torch, dist, args, synth.PREFILL, (4096,), rotate=1,
                                              ws_cap=256 << 20)
    # the channel-selective layer on the V2-Lite shapes (13% / 18% / all routed channels)
    chan = [] if args.quick else chan_sweep(qmoe, torch, dist, args, synth.V2LITE, (1, 2, 4, 8))
    e2e = measure_e2e(qmoe, torch, dist, layers[0], args.steps, args.warmup)

    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    # Dominant kernel: the fused decode launch (routing, FC1, FC2 and the combine of
    # the whole layer), or FC1 when the layer runs as two expert launches.
    if "decode_layer" in head["kernels"]:
        dom, dom_bytes = "decode_layer", head["bytes"]
        dom_desc = "decode_layer (routing + FC1 dequant/gate-up MMA/SwiGLU + FC2 MMA + combine, one launch)"
    else:
        dom, dom_bytes = "fc1_small", head["fc1_bytes"]
        dom_desc = "fc1_small (dequant + gate/up MMA + SwiGLU)"
    # Kernel time for the roofline: in the clean graph the layer is the decode
    # kernel plus an 8-CTA reset launch that runs under the previous layer's
    # tail (programmatic dependent launch), so the step time bounds the decode
    # kernel's time from above; events around each launch (a traced graph)
    # break that overlap and are kept only as a breakdown.
    dom_ms = min(head["kernels"][dom], head["ms_per_step"]) if dom != "decode_layer" else head["ms_per_step"]
    dom_gbps = dom_bytes / (dom_ms * 1e6)
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        traffic = json.load(open(tpath)).get(f"{dom}_v2lite_M1_bytes_per_launch")

    value = head["job_bytes"] / (head["ms_per_step"] * 1e6)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(head["ms_per_step"], 6),
        "us_per_layer": round(head["ms_per_step"] * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4-weights/bf16-act/fp32-acc",
        "data": "synthetic",
        "config": headline_config(world),
        "bytes_per_step": int(head["bytes"]),
        "pct_of_hbm_peak": round(100 * value / world / hbm_peak, 1),
        "pct_of_nominal_8TBps": round(100 * value / world / 8000, 1),
        "roofline": {"bound": "hbm", "kernel": dom_desc,
                     "achieved": round(dom_gbps, 1), "peak": hbm_peak, "peak_source": peak_src,
                     "unit": "GB/s", "frac": round(dom_gbps / hbm_peak, 3), "traffic": traffic,
                     "bytes_per_launch": int(dom_bytes), "launch_us": round(dom_ms * 1e3, 3),
                     "launch_us_source": "ms_per_step (bounds the kernel; the reset launch overlaps the previous "
                                         "layer)" if dom == "decode_layer" else "traced launch, capped at ms_per_step",
                     "kernels_us_traced": {k: round(v * 1e3, 3) for k, v in head["kernels"].items()}},
        "sweep_tokens_per_expert": result_sweep,
        "linear_5120x17408_g128": linear,
        "linear_5120x248320_g128": lmhead,
        "decoder_layer_linears_g128": {"shapes": [{"name": n, "N": N, "K": K, "count": c}
                                                  for n, N, K, c in DECODER_LINEARS],
                                       "note": "q, k, v, o taken as 5120x5120 (the pages give no attention shapes); "
                                               "per-forward bill = layers x layer_us + lm_head",
                                       "rows": decoder_layer},
        "tiny_layer": tiny,
        "v2lite_decode_batches": v2lite_batches,
        "ternary_layer": ternary,
        "prefill_layer": prefill,
        "channel_select_layer": chan,
        "e2e": e2e,
        "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(head["bytes"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    del keep
    if dist is not None:
        dist.destroy_process_group()


def measure_e2e(qmoe, torch, dist, layer, k: int, w: int) -> dict:
    """Through the public API with pinned host buffers: each step copies x and
    logits host->device, runs the layer and reads y back."""
    M = 1
    x_h = torch.from_numpy(synth.tokens(CFG.H, SEED, M, index=99).view(np.int16)).pin_memory()
    rows = synth.router_logits(CFG, SEED, 16, index=9)
    lg_h = [torch.from_numpy(np.ascontiguousarray(rows[i:i + 1])).pin_memory() for i in range(16)]
    y_h = torch.empty((M, CFG.H), dtype=torch.int16).pin_memory()
    x_d = torch.empty((M, CFG.H), dtype=torch.int16, device="cuda")
    lg_d = torch.empty((M, CFG.E), dtype=torch.float32, device="cuda")
    y_d = torch.empty_like(x_d)
    ws = torch.empty(qmoe.workspace_size(layer, M), dtype=torch.uint8, device="cuda")

    def step(i):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h[i % 16], non_blocking=True)
        qmoe.forward(layer, x_d, lg_d, y_d, ws)
        y_h.copy_(y_d, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    for i in range(w):
        step(i)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(k):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / k
    nbytes = statistics.mean(layer_bytes(rows[i:i + 1])["total"] for i in range(16))
    return {"value": round(nbytes / (ms * 1e6), 1), "unit": "GB/s", "us_per_layer": round(ms * 1e3, 2),
            "h2d_bytes_per_step": M * CFG.H * 2 + M * CFG.E * 4, "d2h_bytes_per_step": M * CFG.H * 2,
            "note": "unfused single layer incl. launch latency (no graph) and a host sync per step"}


def linear_sweep(qmoe, torch, dist, args) -> list:
    N, K, block = 17408, 5120, 128
    wb = synth.linear_weight(SEED, N, K)
    out = []
    for fmt in ("int2", "int4"):
        c, s = qmoe.pack(qmoe.FMT[fmt], qmoe.ROWS_PLAIN, wb, block)
        nbytes = c.nbytes + s.nbytes
        rot = max(2, int(np.ceil(2 * 126e6 / nbytes)) + 1)
        dc, ds = _to_dev(torch, c), _to_dev(torch, s)
        copies = [(dc, ds)] + [(dc.clone(), ds.clone()) for _ in range(rot - 1)]
        ws_list = [qmoe.make_weights(qmoe.FMT[fmt], block, a, b) for a, b in copies]
        row = {"fmt": fmt, "bytes_M1": nbytes + K * 2 + N * 2, "copies_rotated": rot, "M": []}
        for M in [int(m) for m in args.linear_sweep.split(",")]:
            x = _to_dev(torch, synth.tokens(K, SEED, M))
            y = torch.empty((M, N), dtype=torch.int16, device="cuda")
            ws = torch.empty(qmoe.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")

            def fn(i, n, M=M, x=x, y=y, ws=ws):
                qmoe.linear(ws_list[i % rot], N, K, x, y, ws)

            steps = Steps(torch, fn, rot)
            k = max(args.steps, 64)
            steps.prepare(k, args.warmup)
            steps.run(args.warmup)
            ms = reduce_ranks(torch, dist, time_steps(torch, dist, steps, k), 0.0)[0] / k
            b = nbytes + M * K * 2 + M * N * 2
            row["M"].append({"M": M, "us": round(ms * 1e3, 3), "GBps": round(b / (ms * 1e6), 1)})
        out.append(row)
    return out


def cfg_layer_bytes(cfg, logits: np.ndarray) -> tuple[int, int]:
    """(algorithmic bytes, active experts) of one forward of `cfg` on these logits."""
    f1 = expert_bytes(cfg.fc1_fmt, 2 * cfg.I, cfg.H, cfg.block) + (2 * cfg.I * 2 if cfg.bias else 0)
    f2 = expert_bytes(cfg.fc2_fmt, cfg.H, cfg.I, cfg.block) + (cfg.H * 2 if cfg.bias else 0)
    T = logits.shape[0]
    top = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, : cfg.k]
    n = len(set(top.ravel().tolist())) + cfg.n_shared
    return n * (f1 + f2) + T * cfg.H * 2 * 2 + T * cfg.E * 4, n


def pack_cfg(qmoe, torch, cfg, distinct: int | None = None):
    """Device layer for `cfg`.  With `distinct`, only that many experts are
    drawn and quantized; expert e holds the packed bytes of expert e % distinct
    (same sizes and layout, for timing a layer whose weights take minutes to draw)."""
    n = cfg.E + cfg.n_shared
    d = n if distinct is None else min(n, distinct)
    f1, f2 = qmoe.FMT[cfg.fc1_fmt], qmoe.FMT[cfg.fc2_fmt]
    c1, s1 = qmoe.pack_stack(f1, qmoe.ROWS_GATE_UP, (synth.expert_fc1(cfg, SEED, e) for e in range(d)), cfg.block)
    c2, s2 = qmoe.pack_stack(f2, qmoe.ROWS_KSPLIT, (synth.expert_fc2(cfg, SEED, e) for e in range(d)), cfg.block)
    if d < n:
        reps = -(-n // d)
        c1, s1, c2, s2 = (np.tile(a.reshape(d, -1), (reps, 1))[:n].reshape(-1) for a in (c1, s1, c2, s2))
    keep = [_to_dev(torch, a) for a in (c1, s1, c2, s2)]
    b1 = b2 = None
    if cfg.bias:
        b1 = _to_dev(torch, np.stack([synth.expert_b1(cfg, SEED, e) for e in range(n)]))
        b2 = _to_dev(torch, np.stack([synth.expert_b2(cfg, SEED, e) for e in range(n)]))
        keep += [b1, b2]
    w1 = qmoe.make_weights(f1, cfg.block, keep[0], keep[1], b1, qmoe.ROWS_GATE_UP)
    w2 = qmoe.make_weights(f2, cfg.block, keep[2], keep[3], b2, qmoe.ROWS_KSPLIT)
    return qmoe.make_layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.n_shared, w1, w2), keep


def cfg_sweep(qmoe, torch, dist, args, cfg, Ts, rotate: int, ws_cap: int | None = None, copies: int = 1,
              distinct: int | None = None) -> dict:
    """One layer forward per step on `cfg` for each T; router rows rotate over
    `rotate` seeded draws so that consecutive steps touch different experts,
    and over `copies` device copies of the weights (a layer smaller than L2)."""
    layer0, keep = pack_cfg(qmoe, torch, cfg, distinct)
    layers = [layer0]
    base = list(keep)  # codes, scales of FC1 and FC2 (and the biases)
    for _ in range(copies - 1):
        cp = [a.clone() for a in base]
        keep += cp
        b1, b2 = (cp[4], cp[5]) if cfg.bias else (None, None)
        w1 = qmoe.make_weights(qmoe.FMT[cfg.fc1_fmt], cfg.block, cp[0], cp[1], b1, qmoe.ROWS_GATE_UP)
        w2 = qmoe.make_weights(qmoe.FMT[cfg.fc2_fmt], cfg.block, cp[2], cp[3], b2, qmoe.ROWS_KSPLIT)
        layers.append(qmoe.make_layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.n_shared, w1, w2))
    layer = layer0
    out = {"config": f"{cfg.name}: H={cfg.H} I={cfg.I} E={cfg.E} top-{cfg.k}"
                     f"{' + %d shared' % cfg.n_shared if cfg.n_shared else ''}, "
                     f"FC1 {cfg.fc1_fmt} / FC2 {cfg.fc2_fmt}, block {cfg.block}", "T": []}
    for T in Ts:
        xs = [_to_dev(torch, synth.tokens(cfg.H, SEED, T, index=r)) for r in range(rotate)]
        lgs_np = [synth.router_logits(cfg, SEED, T, index=100 + r) for r in range(rotate)]
        lgs = [torch.from_numpy(np.ascontiguousarray(l)).cuda() for l in lgs_np]
        need = qmoe.workspace_size(layer, T)
        ws = torch.empty(min(need, ws_cap) if ws_cap else need, dtype=torch.uint8, device="cuda")
        ys = [torch.empty((T, cfg.H), dtype=torch.int16, device="cuda") for _ in range(rotate)]

        nrot = max(rotate, copies)

        def fn(i, n, xs=xs, lgs=lgs, ys=ys, ws=ws):
            r = i % rotate
            qmoe.forward(layers[i % copies], xs[r], lgs[r], ys[r], ws)

        steps = Steps(torch, fn, nrot)
        k = max(nrot, (args.steps // nrot) * nrot) if T <= 64 else nrot * 2
        steps.prepare(k, args.warmup)
        steps.run(max(args.warmup, 3))
        ms = reduce_ranks(torch, dist, time_steps(torch, dist, steps, k), 0.0)[0] / k
        per = [cfg_layer_bytes(cfg, l) for l in lgs_np]
        nbytes = statistics.mean(b for b, _ in per)
        flops = 2.0 * T * cfg.k * (2 * cfg.I * cfg.H + cfg.H * cfg.I) + 2.0 * T * cfg.n_shared * 3 * cfg.I * cfg.H
        out["T"].append({"T": T, "us": round(ms * 1e3, 3), "tokens_per_s": round(T / (ms * 1e-3), 1),
                         "active_experts": round(statistics.mean(a for _, a in per), 1),
                         "GBps": round(nbytes / (ms * 1e6), 1), "TFLOPs": round(flops / (ms * 1e9), 2),
                         "workspace_bytes": ws.numel(), "row_tiles": qmoe.get_stats().row_tiles})
    if copies > 1:
        out["weight_copies_rotated"] = copies
    if distinct is not None:
        out["distinct_experts"] = f"{distinct} drawn and quantized; expert e holds the bytes of expert e % {distinct}"
    del keep, layers
    return out


# One decoder layer of the model the MLX issue bills per forward (hidden 5120, MLP
# intermediate 17408, vocabulary 248320).  The pages give no attention shapes; the
# plainest reading, full multi-head attention with q, k, v and o all 5120 x 5120, is
# taken here.  (N, K, count) per layer.
DECODER_LINEARS = (("q_k_v_o", 5120, 5120, 4), ("gate_up", 17408, 5120, 2), ("down", 5120, 17408, 1))


def model_layer_sweep(qmoe, torch, dist, args) -> list:
    """Every linear of one decoder layer at widths M = 1..6 (the speculative-verify
    window), group 128, INT2 and INT4: the per-layer bill of the MLX issue's per-forward
    sum.  Each shape's weights rotate over copies past L2."""
    out = []
    for fmt in ("int2", "int4"):
        per_shape = {}
        for name, N, K, count in DECODER_LINEARS:
            wb = synth.linear_weight(SEED, N, K)
            c, s = qmoe.pack(qmoe.FMT[fmt], qmoe.ROWS_PLAIN, wb, 128)
            nbytes = c.nbytes + s.nbytes
            rot = max(2, int(np.ceil(2 * 126e6 / nbytes)) + 1)
            dc, ds = _to_dev(torch, c), _to_dev(torch, s)
            copies = [(dc, ds)] + [(dc.clone(), ds.clone()) for _ in range(rot - 1)]
            wl = [qmoe.make_weights(qmoe.FMT[fmt], 128, a, b) for a, b in copies]
            per_shape[name] = []
            for M in range(1, 7):
                x = _to_dev(torch, synth.tokens(K, SEED, M))
                y = torch.empty((M, N), dtype=torch.int16, device="cuda")
                ws = torch.empty(qmoe.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")

                def fn(i, n, x=x, y=y, ws=ws, N=N, K=K):
                    qmoe.linear(wl[i % rot], N, K, x, y, ws)

                steps = Steps(torch, fn, rot)
                k = max(args.steps, 64)
                steps.prepare(k, args.warmup)
                steps.run(args.warmup)
                per_shape[name].append(reduce_ranks(torch, dist, time_steps(torch, dist, steps, k), 0.0)[0] / k)
            del copies, wl, dc, ds
        layer_us = [sum(per_shape[n][m] * cnt for n, _, _, cnt in DECODER_LINEARS) * 1e3 for m in range(6)]
        out.append({"fmt": fmt, "M": list(range(1, 7)),
                    "per_linear_us": {n: [round(v * 1e3, 3) for v in per_shape[n]] for n, _, _, _ in DECODER_LINEARS},
                    "layer_us": [round(v, 2) for v in layer_us],
                    "layer_slope_vs_M1": [round(v / layer_us[0], 3) for v in layer_us]})
    return out


def lmhead_sweep(qmoe, torch, dist, args) -> list:
    """Single quantized linear 5120 -> 248320, g128: one copy is > 2x L2."""
    N, K, block = 248320, 5120, 128
    wb = synth.linear_weight(SEED, N, K)
    out = []
    for fmt in ("int2", "int4"):
        c, s = qmoe.pack(qmoe.FMT[fmt], qmoe.ROWS_PLAIN, wb, block)
        nbytes = c.nbytes + s.nbytes
        dc, ds = _to_dev(torch, c), _to_dev(torch, s)
        del c, s
        w = qmoe.make_weights(qmoe.FMT[fmt], block, dc, ds)
        row = {"fmt": fmt, "bytes_M1": nbytes + K * 2 + N * 2, "M": []}
        for M in range(1, 9):
            x = _to_dev(torch, synth.tokens(K, SEED, M))
            y = torch.empty((M, N), dtype=torch.int16, device="cuda")
            ws = torch.empty(qmoe.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")

            def fn(i, n, x=x, y=y, ws=ws):
                qmoe.linear(w, N, K, x, y, ws)

            steps = Steps(torch, fn, 4)
            k = 40
            steps.prepare(k, args.warmup)
            steps.run(args.warmup)
            ms = reduce_ranks(torch, dist, time_steps(torch, dist, steps, k), 0.0)[0] / k
            b = nbytes + M * K * 2 + M * N * 2
            row["M"].append({"M": M, "us": round(ms * 1e3, 3), "GBps": round(b / (ms * 1e6), 1)})
        out.append(row)
        del dc, ds, w
    del wb
    return out


# ------------------------------------------------------------------ CPU oracle

def _oracle_bank():
    from oracle import qmoe_oracle as Q

    def q(fmt, wbits):
        w = Q.bf16_bits_to_f64(wbits)
        return Q.quantize_ternary(w, CFG.block) if fmt == "ternary" else Q.quantize_sym(
            w, 2 if fmt == "int2" else 4, CFG.block)

    return Q, Q.QuantExpertBank(CFG.H, CFG.I, CFG.E, CFG.n_shared, CFG.block,
                                lambda e: q(CFG.fc1_fmt, synth.expert_fc1(CFG, SEED, e)),
                                lambda e: q(CFG.fc2_fmt, synth.expert_fc2(CFG, SEED, e)), cache=16)


def _cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(gpu_bytes_per_step: float, budget_s: float = 12.0, single_s: float = 8.0) -> dict:
    """The oracle as it stands, one M=1 layer step at a time, for about budget_s
    seconds on all host threads, then for about single_s seconds on one thread."""
    out = _cpu_baseline_run(budget_s)
    out["cores"] = _cores()
    if single_s > 0:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            one = _cpu_baseline_run(single_s)
        out["single_thread"] = {"value": one["value"], "unit": "GB/s", "cores": 1, "sample": one["sample"],
                                "us_per_layer": one["us_per_layer"]}
    return out


def _cpu_baseline_run(budget_s: float) -> dict:
    Q, bank = _oracle_bank()
    rows = synth.router_logits(CFG, SEED, 64, index=7)
    x = Q.bf16_bits_to_f64(synth.tokens(CFG.H, SEED, 1))
    t0 = time.perf_counter()
    n = 0
    nbytes = 0.0
    while time.perf_counter() - t0 < budget_s or n == 0:
        Q.moe_token(x[0], rows[n % 64], CFG.k, bank)
        nbytes += layer_bytes(rows[n % 64:n % 64 + 1])["total"]
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / (dt * 1e9), 4), "unit": "GB/s", "kind": "oracle",
            "sample": f"{n} single-token layer steps (M=1, rotating router rows), {dt:.1f} s",
            "us_per_layer": round(dt / n * 1e6, 1)}


def headline_config(world: int) -> dict:
    """The workload the headline line (and the reference arm's line) is quoted on."""
    return {
        "workload": "v2lite-decode-moe-layer: H=2048 I=1408 E=64 top-6 + 2 shared, INT4 FC1/FC2 block 64, "
                    "M=1 token per expert",
        "tokens_per_expert": 1,
        "global_batch": world,
        "parallelism": f"replicas x{world} (independent decode batches, no data-path collective)",
        "l2": "8 weight copies (2.4 GB) rotated step by step: inputs larger than L2",
        "graph": "CUDA graphs of forward calls",
    }


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    Q, bank = _oracle_bank()
    rows = synth.router_logits(CFG, SEED, 64, index=7)
    x = Q.bf16_bits_to_f64(synth.tokens(CFG.H, SEED, 1))
    for i in range(args.warmup):
        Q.moe_token(x[0], rows[i % 64], CFG.k, bank)
    t0 = time.perf_counter()
    nbytes = 0.0
    for i in range(args.steps):
        r = (args.warmup + i) % 64
        Q.moe_token(x[0], rows[r], CFG.k, bank)
        nbytes += layer_bytes(rows[r:r + 1])["total"]
    dt = time.perf_counter() - t0
    value = nbytes / (dt * 1e9)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(world),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"{args.steps} single-token layer steps after {args.warmup} warm-up steps"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.profile:
        run_profile(args)
    elif args.profile_prefill:
        run_profile_prefill(args)
    elif args.profile_ternary:
        run_profile_ternary(args)
    elif args.profile_chan:
        run_profile_chan(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
