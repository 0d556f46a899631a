#!/usr/bin/env python
"""Benchmark of the packed ternary-weight decode GEMV on B200.

Default workload: the BitNet b1.58-2B decode layer set -- 30 layers x 7
projections (q/o 2560x2560, k/v 640x2560, gate/up 6912x2560, down
2560x6912), batch 1, single ternary plane with a per-tensor scale, int8
per-token absmax activations, fp32 output, each GEMV with its own seeded
weights and activations. One step = the layer set's 210 GEMVs, which have no
data dependencies on one another: one grouped launch per input width (the
180 GEMVs with K = 2560, then the 30 down projections), every GEMV quantising
its bf16 activation per token inside the kernel (521 MB of packed weights, so every step streams from HBM: inputs
larger than L2). The same GEMVs run in decode order -- per layer [q,k,v] ->
o -> [gate,up] -> down, each launch waiting for the previous one -- are
reported alongside as "decode_chain".

Metric: achieved HBM GB/s over the step (algorithmic bytes: packed weights,
activations read and written, outputs) and its fraction of the measured copy
bandwidth; per-shape figures are reported alongside.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  torchrun --nproc-per-node N bench.py --gpus N ...   (independent replicas)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from packed_ternary_weight_b200 import synth  # noqa: E402

METRIC = "decode GEMV achieved HBM GB/s and % of B200 roofline per layer shape, 1 GPU"
WORKLOAD = ("BitNet b1.58-2B decode layer set: 30 layers x 7 projections (q,o 2560x2560; k,v 640x2560; "
            "gate,up 6912x2560; down 2560x6912), batch 1, single ternary plane, per-tensor scale 0.02, "
            "int8 per-token absmax activations, fp32 out, distinct seeds")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=synth.BITNET_2B_LAYERS)
    ap.add_argument("--config", default="bitnet2b", choices=("bitnet2b", "single", "tq3p", "bt3", "tq2p"),
                    help="bitnet2b: the headline layer set; single: one 512x1024 GEMV; tq3p / bt3: "
                         "Llama-3.1-8B shapes; tq2p: the batched sweep (per-shape tables only)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' per-shape rows in the default line")
    ap.add_argument("--profile", default=None,
                    help="run only one case eagerly for a profiler: step | decode | <shape>_indep | <shape>_chain "
                         "(headline workload); with --config tq3p|bt3|tq2p|single: <shape>:<m> (the copies "
                         "launched one after another) or <shape>:1:indep (one grouped launch)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--ceiling", action="store_true",
                    help="measure the read ceiling (tern_stream_read) for a few access shapes and exit")
    return ap.parse_args()


def measured_bf16_tflops():
    """Dense bf16 tensor throughput (burst) measured on this machine, else the fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def header_scale_digits(buf) -> int:
    """Digit count the packer stored in the header (u32 at byte 72)."""
    return int(np.asarray(buf[72:76]).view("<u4")[0])


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        self.gpu = gpu_index
        if not enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def clock_verdict(clk):
    """Why a timed region's clock record rejects its number, or None: hardware or thermal slowdown
    active, or the SM clock held well below its maximum with no reason given (a leftover clock lock).
    sw_power_cap alone is the normal state of a 1 kW part under load and is kept."""
    if not clk or not clk.get("samples"):
        return None
    bad = [r for r in clk.get("reasons", []) if r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")]
    if bad:
        return "throttled: " + ", ".join(bad)
    sm, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if sm and mx and sm < 0.75 * mx and not clk.get("reasons"):
        return "SM clock %.0f of %.0f MHz with no reason" % (sm, mx)
    return None


# ------------------------------------------------------------ rank plumbing
def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank calls this, in the same order."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_gbs(step_bytes: float, ms_step: float, world: int) -> float:
    """Whole-job throughput of N replicas: every rank's bytes over the slowest rank's time."""
    return world * step_bytes / (ms_step * 1e-3) / 1e9


def parity_checks(n_layers: int):
    """(layer, projection) of the GEMVs the bench's spot check samples: start, middle and end."""
    return [(0, "q_proj"), (n_layers // 2, "k_proj"), (n_layers - 1, "down_proj")]


def parity_samples(y_host, by, n_layers: int, rows_per_gemv: int = 256) -> bool:
    """Bit-exact comparison of sampled output rows of the layer set's step (y_host: every GEMV's fp32
    outputs, GEMV L at offset L["yoff"]) with the oracle on the same seeded weights and activations."""
    import oracle
    names = [nm for nm, _, _ in synth.BITNET_2B_SHAPES]
    ok = True
    for li, nm in parity_checks(n_layers):
        L = by[(li, nm)]
        lay = synth.bitnet_layer(L["n"], L["k"], synth.bitnet_layer_set_seed(li, names.index(nm)), 0.02)
        rows = np.sort(np.random.default_rng(li).choice(L["n"], min(L["n"], rows_per_gemv), replace=False))
        q, s = oracle.quantize_act(synth.draw_x_bf16(lay.seed, 1, lay.k))
        yref = oracle.gemv_bitnet_int8(lay.trits[:, rows], q, s, lay.tensor_scale)[0]
        got = np.ascontiguousarray(y_host[L["yoff"] + rows], dtype=np.float32)
        ok = ok and bool(np.array_equal(got.view(np.uint32), yref.view(np.uint32)))
    return ok


# --------------------------------------------------------------- our impl
STAGES = (("q_proj", "k_proj", "v_proj"), ("o_proj",), ("gate_proj", "up_proj"), ("down_proj",))


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    from packed_ternary_weight_b200 import tern

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream()
    layers = []           # per GEMV: name, shape, desc, packed weights, offsets into x/y
    x_host = []
    k_tot = n_tot = 0
    for lay in synth.bitnet_layer_set(args.layers):
        d, buf = tern.pack_layer(lay, flags=tern.F_PDL)
        x_host.append(synth.draw_x_bf16(lay.seed, 1, lay.k)[0])
        layers.append(dict(name=lay.name.split(".", 1)[1], layer=int(lay.name[1:].split(".")[0]), n=lay.n, k=lay.k,
                           desc=d, packed=torch.from_numpy(buf).to(dev), wbytes=len(buf) - 256, xoff=k_tot,
                           yoff=n_tot))
        k_tot += lay.k
        n_tot += lay.n
        del lay
    x_all_host = torch.from_numpy(np.concatenate(x_host).view(np.int16)).pin_memory()
    y_all_host = torch.empty(n_tot, dtype=torch.float32).pin_memory()
    x_all = x_all_host.to(dev)
    y_all = torch.empty(n_tot, dtype=torch.float32, device=dev)
    xv = lambda L: x_all[L["xoff"]:L["xoff"] + L["k"]]          # noqa: E731
    yv = lambda L: y_all[L["yoff"]:L["yoff"] + L["n"]]          # noqa: E731
    by = {(L["layer"], L["name"]): L for L in layers}

    def grouped(Ls):
        return tern.Grouped([L["desc"] for L in Ls], [L["packed"] for L in Ls], tern.ACT_BF16_Q8,
                            [xv(L) for L in Ls], None, tern.OUT_F32, [yv(L) for L in Ls])

    # per shape: the 30 copies as one dependent chain of single launches, and
    # as one launch of 30 independent GEMVs
    chain = {nm: [grouped([L]) for L in layers if L["name"] == nm] for nm, _, _ in synth.BITNET_2B_SHAPES}
    indep = {nm: grouped([L for L in layers if L["name"] == nm]) for nm, _, _ in synth.BITNET_2B_SHAPES}

    # per shape, the timing protocol for independent GEMVs: a pool of distinct
    # weight copies of at least 512 MB (four times L2: the layer set's 30 copies,
    # cloned further), grouped launches of up to 256, four back-to-back rounds
    # per captured graph
    pools = {}
    for nm, _, _ in ([] if args.profile else synth.BITNET_2B_SHAPES):
        Ls = [L for L in layers if L["name"] == nm]
        copies = max(len(Ls), -(-512_000_000 // Ls[0]["wbytes"]))
        pk = [Ls[i]["packed"] if i < len(Ls) else Ls[i % len(Ls)]["packed"].clone() for i in range(copies)]
        ys_p = [torch.empty(Ls[0]["n"], dtype=torch.float32, device=dev) for _ in range(copies)]
        launches = [tern.Grouped([Ls[0]["desc"]] * len(pk[i:i + 256]), pk[i:i + 256], tern.ACT_BF16_Q8,
                                 [xv(Ls[j % len(Ls)]) for j in range(i, min(i + 256, copies))], None, tern.OUT_F32,
                                 ys_p[i:i + 256]) for i in range(0, copies, 256)]
        pools[nm] = (launches, copies, pk, ys_p)

    # the step: the layer set's 210 independent GEMVs in one grouped launch
    # (ordered by input width K: the 180 with K = 2560, then the 30 down
    # projections with K = 6912; the kernel balances CTAs by columns),
    # activations quantised per token inside each GEMV
    step_launches = [grouped(sorted(layers, key=lambda L: L["k"]))]

    def step():
        for g in step_launches:
            g.launch(stream)

    # the same GEMVs in decode order, each launch waiting for the previous one:
    # per layer [q,k,v] -> o -> [gate,up] -> down
    chain_launches = [grouped([by[(li, nm)] for nm in st]) for li in range(args.layers) for st in STAGES]

    def chain_step():
        for g in chain_launches:
            g.launch(stream)

    # bytes that must move per step (algorithmic): packed weights, the bf16
    # activations read, the fp32 outputs written
    gbytes = lambda L: L["wbytes"] + 2 * L["k"] + 4 * L["n"]    # noqa: E731
    step_bytes = sum(gbytes(L) for L in layers)

    if args.profile == "decode":
        run_decode(tern, torch, stream, {(L["layer"], L["name"]): L["packed"] for L in layers}, args.layers,
                   reps=args.reps, clocks=False)
        return None
    if args.profile:
        cases = {"step": step, "chain_step": chain_step}
        for nm, _, _ in synth.BITNET_2B_SHAPES:
            short = nm.split("_")[0]
            cases[f"{short}_indep"] = indep[nm].launch
            cases[f"{short}_chain"] = (lambda gs=chain[nm]: [g.launch(stream) for g in gs])
        fn = cases[args.profile]
        with torch.cuda.stream(stream):
            for _ in range(args.reps):
                fn(stream) if args.profile.endswith("_indep") else fn()
            torch.cuda.synchronize()
        assert tern.device_error(stream) == tern.OK
        return None

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    with torch.cuda.stream(stream):
        step()                      # eager warm-up, sets kernel attributes
        torch.cuda.synchronize()
        assert tern.device_error(stream) == tern.OK
        g_step = capture(step)
        # the timed steps: back-to-back launches captured in one graph (the
        # launches carry programmatic dependent launch, so each one's start
        # overlaps the previous one's tail); spb steps per graph, spb | steps
        spb = max(d for d in range(1, min(args.steps, 25) + 1) if args.steps % d == 0)
        g_steps = capture(lambda: [step() for _ in range(spb)])
        g_chain_step = capture(chain_step)
        g_chain = {nm: capture(lambda gs=gs: [g.launch(stream) for g in gs]) for nm, gs in chain.items()}
        g_pool = {nm: capture(lambda ls=pl[0]: [g.launch(stream) for _ in range(4) for g in ls])
                  for nm, pl in pools.items()}
    torch.cuda.synchronize()

    # parity spot check of the captured step against the oracle: sampled rows of
    # GEMVs at the start, middle and end of the launch
    parity = None
    if rank == 0:
        y_all.fill_(float("nan"))
        g_step.replay()
        torch.cuda.synchronize()
        parity = parity_samples(y_all.cpu().numpy(), by, args.layers)

    def timed(graph, reps):
        with torch.cuda.stream(stream):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                graph.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
            if world > 1:
                dist.barrier()
        return ms

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
        torch.cuda.synchronize()

    def measure():
        clocks = ClockSampler(dev.index, not args.no_clocks and rank == 0)
        t_end = time.time() + (1.0 if not args.no_clocks else 0.0)   # soak so the clock samples see this load
        with torch.cuda.stream(stream):
            while time.time() < t_end:
                for _ in range(20):
                    g_step.replay()
                torch.cuda.synchronize()
        ms = timed(g_steps, args.steps // spb)
        return ms, clocks.stop()

    ms_total, clk = measure()
    # a record that rejects the number: measure once more (every rank takes the same decision)
    why = clock_verdict(clk)
    if max_over_ranks(1.0 if why else 0.0, world, dev) > 0:
        ms_total, clk = measure()
        if clk is not None:
            clk["remeasured_after"] = why
    ms_step = ms_total / args.steps

    peak, peak_kind = measured_peaks()
    reps = max(3, min(args.steps, 100))
    ms_chain_step = timed(g_chain_step, reps) / reps
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)       # twice the L2

    def single_launch_us(g):
        """One launch timed alone with events after the L2 was flushed: the median of five."""
        out = []
        with torch.cuda.stream(stream):
            for _ in range(5):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.launch(stream)
                e1.record(stream)
                torch.cuda.synchronize()
                out.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(out)

    per_shape = []
    for nm, n, k in synth.BITNET_2B_SHAPES:
        Ls = [L for L in layers if L["name"] == nm]
        b = sum(gbytes(L) for L in Ls)
        ms_c = timed(g_chain[nm], reps) / reps
        t1 = single_launch_us(chain[nm][0])
        launches, copies = pools[nm][0], pools[nm][1]
        ms_i = timed(g_pool[nm], 3) / (3 * 4)
        bp = (b // len(Ls)) * copies
        per_shape.append(dict(shape=f"{nm} {n}x{k}", bytes_per_gemv=b // len(Ls),
                              chain_us_per_gemv=round(ms_c * 1e3 / len(Ls), 3),
                              chain_gbs=round(b / (ms_c * 1e-3) / 1e9, 1),
                              single_launch_us=round(t1, 2),
                              single_launch_gbs=round(b / len(Ls) / (t1 * 1e-6) / 1e9, 1),
                              independent_gbs=round(bp / (ms_i * 1e-3) / 1e9, 1),
                              independent_frac=round(bp / (ms_i * 1e-3) / 1e9 / peak, 4),
                              independent_pool="%d copies (%.0f MB) in %d launch(es), 4 rounds per graph" % (
                                  copies, bp / 1e6, len(launches))))

    # the whole decode step of a token (every layer, attention included), one launch per token
    decode = run_decode(tern, torch, stream, {(L["layer"], L["name"]): L["packed"] for L in layers}, args.layers,
                        reps=max(3, min(args.steps, 100)), clocks=not args.no_clocks and rank == 0)

    # end to end through the public API, pipelined as a server runs it: every
    # step copies its bf16 activations in from pinned host memory and its fp32
    # outputs back out; step i's input copy (copy stream) overlaps step i-1's
    # compute, and step i-1's output copy (another copy stream) overlaps step
    # i's; two device buffer sets alternate, each reused only after the copies
    # that read or fill it have finished
    h2d = x_all_host.numel() * 2
    d2h = y_all_host.numel() * 4
    x_b = [x_all, torch.empty_like(x_all)]
    y_b = [y_all, torch.empty_like(y_all)]
    x_h = [x_all_host, x_all_host.clone().pin_memory()]
    y_h = [y_all_host, torch.empty_like(y_all_host).pin_memory()]

    def step_on(xbuf, ybuf):
        Ls = sorted(layers, key=lambda L: L["k"])
        return tern.Grouped([L["desc"] for L in Ls], [L["packed"] for L in Ls], tern.ACT_BF16_Q8,
                            [xbuf[L["xoff"]:L["xoff"] + L["k"]] for L in Ls], None, tern.OUT_F32,
                            [ybuf[L["yoff"]:L["yoff"] + L["n"]] for L in Ls])

    with torch.cuda.stream(stream):
        g_b = [g_step, capture(lambda g=step_on(x_b[1], y_b[1]): g.launch(stream))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "done", "out")}

    def e2e_pipeline(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev["done"][b])          # step i-2 has read x_b[b]
            with torch.cuda.stream(s_in):
                x_b[b].copy_(x_h[b], non_blocking=True)
                ev["in"][b].record(s_in)
            stream.wait_event(ev["in"][b])
            if i >= 2:
                stream.wait_event(ev["out"][b])         # step i-2's outputs have left y_b[b]
            with torch.cuda.stream(stream):
                g_b[b].replay()
                ev["done"][b].record(stream)
            s_out.wait_event(ev["done"][b])
            with torch.cuda.stream(s_out):
                y_h[b].copy_(y_b[b], non_blocking=True)
                ev["out"][b].record(s_out)

    e2e_pipeline(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_pipeline(reps)
    s_out.wait_event(ev["out"][(reps - 1) & 1])
    e1.record(s_out)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / reps, world, dev)
    assert tern.device_error(stream) == tern.OK
    # the last step's outputs reached the host intact
    e2e_ok = bool(torch.equal(y_h[(reps - 1) & 1], y_all.cpu())) if rank == 0 else None

    value = replica_gbs(step_bytes, ms_step, world)
    achieved = step_bytes / (ms_step * 1e-3) / 1e9     # every launch of the step is the GEMV kernel
    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded ternary weights P(-1)=P(+1)=0.3, bf16 N(0,1) activations)",
        "config": {"workload": WORKLOAD, "layers": args.layers, "gemvs_per_step": len(layers),
                   "launches_per_step": len(step_launches),
                   "order": "one grouped launch of the 210 independent GEMVs (the 180 with K = 2560, then the "
                            "30 down projections with K = 6912; the layer set's GEMVs have no data "
                            "dependencies); decode-order figures in decode_chain, per-shape launches in per_shape",
                   "l2": "inputs larger than L2 (packed weights per step %.1f MB vs 126 MB L2)" % (
                       sum(L["wbytes"] for L in layers) / 1e6),
                   "graph": "%d steps per captured graph, programmatic dependent launch between launches" % spb,
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": committed_traffic(),
                     "kernel": "gemv2w_kernel<bf16->int8 in-kernel, 1 plane, per-tensor scale> (one CTA per SM)",
                     "peak_kind": peak_kind,
                     "achieved_basis": "algorithmic bytes of the step's GEMV launches (weights, bf16 activations, "
                                       "fp32 outputs) / their duration; every launch of the step is this kernel"},
        "per_shape": per_shape,
        "decode_chain": {"launches_per_step": len(chain_launches),
                         "order": "per layer [q,k,v] -> o -> [gate,up] -> down, each launch waiting for the previous "
                                  "one (programmatic dependent launch: weights prefetched before the wait)",
                         "ms_per_step": round(ms_chain_step, 4),
                         "gbs": round(step_bytes / (ms_chain_step * 1e-3) / 1e9, 1)},
        "tokens_per_s_equiv": {"independent": round(world * 1e3 / ms_step, 1),
                               "decode_step": decode["tokens_per_s"],
                               "decode_chain": round(world * 1e3 / ms_chain_step, 1),
                               "basis": "a step's GEMVs are the projection layers one decoded token at batch 1 "
                                        "streams (attention, norms and the output head are not on this path); "
                                        "tokens per second = steps per second, summed over replicas"},
        "decode_step": decode,
        "e2e": {"value": round(replica_gbs(step_bytes, ms_e2e, world), 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4),
                "pipeline": "per step: pinned H2D of the bf16 activations (copy stream), the captured step, D2H "
                            "of the fp32 outputs (second copy stream); two buffer sets, copies of step i "
                            "overlapping the compute of steps i-1 and i+1",
                "outputs_match": e2e_ok},
        "gpu_launches": args.steps * len(step_launches),
        "parity_bit_exact": parity,
        "parity_sample": "%d rows of each of %s in the timed launch, against the oracle" % (
            256, ", ".join("layer %d %s" % c for c in parity_checks(args.layers))),
    }
    if clk is not None:
        out["clocks"] = clk
        if clk.get("sm_mhz"):
            # clock-normalised step: thousands of SM cycles per step at the median sampled clock
            out["sm_kcycles_per_step"] = round(ms_step * clk["sm_mhz"], 1)
    if rank == 0 and world == 1 and not args.no_configs:
        out["configs"] = run_all_configs(args)
    if rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline(args.layers)
    return out


def model_token_rate(rows, layers: int):
    """Tokens/s-equivalent of a decode step that runs every shape of `rows` once per layer at batch 1
    (projections only): from the per-shape chain times (each GEMV waiting for the previous one) and
    from the per-shape independent throughputs (all bytes streamed at each shape's rate). None where a
    row lacks the figure."""
    one = [r for r in rows if r.get("m", 1) == 1]
    if not one:
        return None
    out = {"layers": layers, "shapes_per_layer": len(one)}
    if all("chain_us_per_gemv" in r for r in one):
        out["decode_chain"] = round(1e6 / (layers * sum(r["chain_us_per_gemv"] for r in one)), 1)
    if all("independent_gbs" in r for r in one):
        s_per_layer = sum(r["bytes_per_gemv"] / (r["independent_gbs"] * 1e9) for r in one)
        out["independent"] = round(1.0 / (layers * s_per_layer), 1)
    return out


DECODE_POS = 1023
DECODE_WORKLOAD = ("BitNet b1.58-2B decode step at batch 1: 30 layers (RMSNorm, q/k/v, RoPE theta 500000, GQA 20/5 x "
                   "128 over a bf16 KV cache, attn_sub_norm, o_proj, residual, RMSNorm, gate/up, relu^2 * up, "
                   "ffn_sub_norm, down_proj, residual), token at position %d (%d cached positions), the layer set's "
                   "packed weights, synthetic gains, cache and residual stream" % (DECODE_POS, DECODE_POS))


def run_decode(tern, torch, stream, packed_by, n_layers: int, reps: int, pos: int = DECODE_POS, clocks=True):
    """The whole decode step of one token (one cooperative launch per token), timed with events over
    back-to-back launches. packed_by: (layer, projection name) -> packed device buffer."""
    m = synth.decode_model(n_layers=n_layers, pos=pos, max_pos=pos + 1)
    names = [nm for nm, _, _ in synth.BITNET_2B_SHAPES]
    packed = [packed_by[(li, nm)] for li in range(n_layers) for nm in names]
    dev = torch.device("cuda", torch.cuda.current_device())
    gains = torch.from_numpy(np.concatenate([np.concatenate(g) for g in m.gains]).astype(np.float32)).to(dev)
    kc = torch.from_numpy(m.kcache.view(np.int16)).to(dev)
    vc = torch.from_numpy(m.vcache.view(np.int16)).to(dev)
    rope = torch.from_numpy(tern.decode_rope_table(m.max_pos)).to(dev)
    model = tern.DecodeModel(packed, gains, kc, vc, rope, m.D, m.F, m.H, m.KVH, m.max_pos)
    ws = torch.zeros(model.workspace_size(), dtype=torch.uint8, device=dev)
    h_in = torch.from_numpy(m.h0).to(dev)
    h_out = torch.empty_like(h_in)
    with torch.cuda.stream(stream):
        for _ in range(3):
            model.step(pos, h_in, h_out, ws, stream=stream)
        torch.cuda.synchronize()
        assert tern.device_error(stream) == tern.OK
        clk = ClockSampler(dev.index, clocks)
        t_end = time.time() + (0.5 if clocks else 0.0)
        while time.time() < t_end:
            for _ in range(20):
                model.step(pos, h_in, h_out, ws, stream=stream)
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            model.step(pos, h_in, h_out, ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ck = clk.stop()
    assert tern.device_error(stream) == tern.OK
    ms = e0.elapsed_time(e1) / reps
    wbytes = sum(int(p.numel()) - 256 for p in packed)
    kv_read = 2 * n_layers * m.KVH * pos * 128 * 2
    other = gains.numel() * 4 + 2 * n_layers * m.KVH * 128 * 2 + rope.shape[1] * 8
    total = wbytes + kv_read + other
    peak, _ = measured_peaks()
    out = {"workload": DECODE_WORKLOAD, "launches_per_token": 1, "ms_per_token": round(ms, 4),
           "tokens_per_s": round(1e3 / ms, 1), "bytes_per_token": total,
           "bytes_basis": "packed ternary weights %.1f MB + cached keys and values read %.1f MB + gains, RoPE row "
                          "and the new cache entries %.2f MB" % (wbytes / 1e6, kv_read / 1e6, other / 1e6),
           "gbs": round(total / (ms * 1e-3) / 1e9, 1), "frac": round(total / (ms * 1e-3) / 1e9 / peak, 4),
           "timing": "%d back-to-back launches (one per token), CUDA events" % reps}
    if ck is not None:
        out["clocks"] = ck
    return out


CONFIG_WORKLOADS = {
    "single": "single ternary GEMV 512x1024, BitNet layout, tensor scale 0.02, int8 per-token absmax "
              "activations (quantised in the kernel), fp32 out, seed 0",
    "tq3p": "TQ3P (3 planes, g = 256, fp16 scales |N(0,1)|*0.02*3^-p) at Llama-3.1-8B shapes, batch 1, bf16 "
            "activations, fp32 out",
    "bt3": "balanced ternary d = 3 (27 levels, group 16, 27-entry log codebook 1e-4..1e-1) at Llama-3.1-8B "
           "shapes, batch 1, bf16 activations, fp32 out",
    "tq2p": "TQ2P (2 planes, g = 32) 14336x4096 and 4096x14336, M = 1, 2, 4, 8 (CUDA cores) and 16, 64, 256 "
            "(tcgen05 int8 tensor cores), int8 activations, fp32 out",
}


def run_config(args, name=None):
    """Per-shape rows of one of the other workloads (rank 0, one GPU).

    Each shape's packed layer is replicated on the device until the pool holds
    at least 512 MB (4x L2), so every launch streams from HBM. Per row:
    "chain" launches the copies one after another (each waiting for the
    previous one, programmatic dependent launch); "independent" (one token)
    puts all copies in grouped launches of up to 256, four rounds per captured
    graph; "single_launch_us" is one launch timed alone with events after the
    L2 was flushed (the median of five).
    """
    import torch

    from packed_ternary_weight_b200 import tern

    name = name or args.config
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")       # twice the L2
    if name == "single":
        layers = [synth.single_gemv_layer()]
        act = tern.ACT_BF16_Q8
    elif name == "tq3p":
        layers = synth.tq3p_llama_layers()
        act = tern.ACT_BF16
    elif name == "bt3":
        layers = synth.bt3_llama_layers()
        act = tern.ACT_BF16
    else:
        layers = synth.tq2p_prefill_layers()
        act = tern.ACT_INT8
    peak, _ = measured_peaks()
    bf16_peak = measured_bf16_tflops()
    rows = []
    reps = max(3, min(args.steps, 50))
    for lay in layers:
        d, buf = tern.pack_layer(lay, flags=tern.F_PDL)
        wbytes = len(buf) - 256
        copies = max(2, min(256, -(-512_000_000 // wbytes)))
        pk = torch.from_numpy(buf).cuda()
        packs = [pk] + [pk.clone() for _ in range(copies - 1)]
        del lay.trits
        if name == "tq2p":
            tokens = synth.PREFILL_TOKENS
        elif name == "bt3" and lay.name in ("q_proj", "gate_proj"):
            tokens = (1, 2, 4, 8)        # weights read once for the tokens of a pass
        elif name == "tq3p" and lay.name == "gate_proj":
            tokens = (1, 2)              # bf16 over 2-bit planes: one pass per token
        else:
            tokens = (1,)
        for m in tokens:
            x = synth.draw_x_bf16(lay.seed, m, lay.k)
            xd = torch.from_numpy(x.view(np.int16)).cuda()
            ys = [torch.empty((m, lay.n), dtype=torch.float32, device="cuda") for _ in range(copies)]
            xq = torch.empty((m, lay.k), dtype=torch.int8, device="cuda")
            sx = torch.empty((m,), dtype=torch.float32, device="cuda")
            tern.quantize_act(xd, xq, sx, stream)
            ws = torch.zeros(max(16, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda")
            xin = xq if act == tern.ACT_INT8 else xd
            sin = sx if act == tern.ACT_INT8 else None
            x_bytes = m * lay.k * 2 if act != tern.ACT_INT8 else m * (lay.k + 4)
            algo = wbytes + x_bytes + 4 * m * lay.n

            def chain():
                for pkc, y in zip(packs, ys):
                    tern.gemm_batched(d, pkc, m, act, xin, sin, tern.OUT_F32, y, ws, stream)

            indep = None
            if m == 1:   # grouped launches of up to 256 independent GEMVs
                G = 256
                indep = [tern.Grouped([d] * len(packs[i:i + G]), packs[i:i + G], act,
                                      [xin.view(-1)] * len(packs[i:i + G]),
                                      None if sin is None else [sin] * len(packs[i:i + G]), tern.OUT_F32,
                                      [y.view(-1) for y in ys[i:i + G]]) for i in range(0, copies, G)]

            def timed(fn):
                with torch.cuda.stream(stream):
                    fn()
                    torch.cuda.synchronize()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        fn()
                    for _ in range(2):
                        g.replay()
                    torch.cuda.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    for _ in range(reps):
                        g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize()
                return e0.elapsed_time(e1) / reps

            def single_launch_us():
                out = []
                with torch.cuda.stream(stream):
                    for _ in range(5):
                        flush.zero_()
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record(stream)
                        tern.gemm_batched(d, packs[0], m, act, xin, sin, tern.OUT_F32, ys[0], ws, stream)
                        e1.record(stream)
                        torch.cuda.synchronize()
                        out.append(e0.elapsed_time(e1) * 1e3)
                return statistics.median(out)

            if args.profile:
                case = f"{lay.name}:{m}"
                if args.profile in (case, case + ":indep"):
                    fn = (lambda: [g.launch(stream) for g in indep]) if args.profile.endswith(":indep") else chain
                    with torch.cuda.stream(stream):
                        for _ in range(args.reps):
                            fn()
                    torch.cuda.synchronize()
                    assert tern.device_error(stream) == tern.OK
                    return None
                continue
            ms_c = timed(chain)
            row = dict(shape=f"{lay.name} {lay.n}x{lay.k}", m=m, bytes_per_gemv=algo, copies=copies,
                       chain_us_per_gemv=round(ms_c * 1e3 / copies, 3),
                       chain_gbs=round(algo * copies / (ms_c * 1e-3) / 1e9, 1),
                       chain_frac=round(algo * copies / (ms_c * 1e-3) / 1e9 / peak, 4))
            t1 = single_launch_us()
            row.update(single_launch_us=round(t1, 2), single_launch_gbs=round(algo / (t1 * 1e-6) / 1e9, 1))
            if m >= 16:
                # tensor-core path: algorithmic int8 ops 2 m N K P (both planes' MACs)
                ops = 2.0 * m * lay.n * lay.k * lay.planes
                tops = ops * copies / (ms_c * 1e-3) / 1e12
                row.update(path="tcgen05 kind::i8 (activation staging + GEMM per call)",
                           tops=round(tops, 1), int8_peak_tops=round(2 * bf16_peak, 1),
                           tensor_frac=round(tops / (2 * bf16_peak), 4),
                           scale_digits=int(header_scale_digits(buf)))
            if indep is not None:
                # four back-to-back rounds per captured graph (each round streams >= 512 MB of
                # distinct weights, four times L2; PDL between launches)
                ms_i = timed(lambda: [g.launch(stream) for _ in range(4) for g in indep]) / 4
                row["independent_gbs"] = round(algo * copies / (ms_i * 1e-3) / 1e9, 1)
                row["independent_frac"] = round(row["independent_gbs"] / peak, 4)
                row["independent_graph"] = "4 rounds of %d launch(es) per graph" % len(indep)
            rows.append(row)
        del packs
        torch.cuda.empty_cache()
    assert tern.device_error(stream) == tern.OK
    out = {"metric": METRIC, "config": {"workload": CONFIG_WORKLOADS[name]}, "unit": "GB/s", "peak": peak,
           "per_shape": rows}
    if name in ("tq3p", "bt3"):   # the seven projections of one Llama-3.1-8B layer
        out["tokens_per_s_equiv"] = model_token_rate(rows, synth.LLAMA_8B_LAYERS)
    return out


def run_fit(args):
    """Dense -> ternary fits on the GPU of a Llama-3.1-8B gate_proj-shaped fp32 matrix (14336 x 4096,
    N(0, 0.02^2)): TQ3P at g = 256 and balanced ternary d = 3, time per matrix (CUDA events)."""
    import torch

    from packed_ternary_weight_b200 import tern
    n, k = 14336, 4096
    g = torch.Generator(device="cuda").manual_seed(5)
    w = torch.randn((n, k), device="cuda", generator=g) * 0.02
    out = {"shape": "%dx%d fp32" % (n, k)}
    t3 = torch.empty((3, n, k), dtype=torch.int8, device="cuda")
    s3 = torch.empty((3, n, k // 256), dtype=torch.int16, device="cuda")
    ix = torch.empty((n, k // 16), dtype=torch.uint8, device="cuda")
    cb = torch.from_numpy(synth.codebook27()).cuda()
    for nm, fn in (("tq3p_g256", lambda: tern.fit_tq(w, 3, 256, t3, s3)),
                   ("bt_d3", lambda: tern.fit_bt(w, 3, cb, t3, ix))):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 3
        out[nm] = {"ms_per_matrix": round(ms, 3), "gweights_per_s": round(n * k / (ms * 1e-3) / 1e9, 2)}
    assert tern.device_error() == tern.OK
    return out


def run_all_configs(args):
    """The other workloads' per-shape rows, for the default bench line, with the SM clock sampled
    while they run."""
    clocks = ClockSampler(0, not args.no_clocks)
    t0 = time.time()
    out = {nm: run_config(args, nm) for nm in ("single", "tq3p", "bt3", "tq2p")}
    for v in out.values():
        v.pop("metric", None)
        v.pop("peak", None)
    out["fit"] = run_fit(args)
    out["seconds"] = round(time.time() - t0, 1)
    clk = clocks.stop()
    if clk is not None:
        out["clocks"] = clk
    return out


def run_ceiling(args):
    """Read-ceiling sweep: stream a 2 GiB buffer once per launch with several access shapes."""
    import torch

    from packed_ternary_weight_b200 import tern

    torch.cuda.set_device(0)
    buf = torch.empty(2 << 30, dtype=torch.uint8, device="cuda")
    buf.random_(0, 255)
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    shapes = [(0, 16, d, cps, w) for w, cps in ((8, 4), (16, 4)) for d in (1, 4, 8)]
    shapes += [(1, c, d, cps, w) for c in (2048, 4096, 8192) for d in (2, 3, 4) for w, cps in ((4, 2), (4, 1), (8, 1))
               if w * d * c * cps <= 220 * 1024]
    shapes += [(2, c, d, cps, w) for c in (8192, 16384, 32768) for d in (2, 4) for w, cps in ((4, 1), (4, 2), (8, 2))
               if d * c * cps <= 220 * 1024]
    rows = []
    for mode, chunk, depth, cps, warps in shapes:
        tern.stream_read(buf, mode, chunk, depth, cps, warps, sink)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            tern.stream_read(buf, mode, chunk, depth, cps, warps, sink)
        e1.record()
        torch.cuda.synchronize()
        gbs = buf.numel() / (e0.elapsed_time(e1) / 5 * 1e-3) / 1e9
        rows.append(dict(mode=mode, chunk=chunk, depth=depth, ctas_per_sm=cps, warps=warps, gbs=round(gbs, 1)))
    assert tern.device_error() == tern.OK
    return {"metric": "read ceiling", "unit": "GB/s", "bytes": buf.numel(), "rows": rows,
            "best": max(r["gbs"] for r in rows)}


def code_hash(path: str) -> str:
    """First 16 hex digits of the SHA-256 of a C++/CUDA source with its comments removed and its
    whitespace collapsed: edits to comments alone keep the hash, any change to the code changes it."""
    src = open(path, encoding="utf-8").read()
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":                                    # string or character literal, kept whole
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    code = " ".join("".join(out).split())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def committed_traffic():
    """DRAM bytes (read + written) per launch of the step from a committed ncu summary, if the summary
    was taken on the current kernel code (else None)."""
    p = os.path.join(ROOT, "profiles", "gemv2w_bitnet2b_step_traffic.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                vals[key.strip()] = val.strip()
    src = os.path.join(ROOT, "packed_ternary_weight_b200", "csrc", "tern_gemv2w_kernel.cuh")
    if vals.get("kernel_code_sha256_16") != code_hash(src):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------- CPU baseline
# The oracle timed on the host cores. Its inputs are the layer set's logical
# weights and activations drawn by the seeded generators (nothing of the CUDA
# library is loaded on this leg); the timed work per GEMV is the oracle's
# per-token quantisation and exact integer GEMV with the scale at the end.
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def layer_set_items(n_layers: int):
    """(layer, projection index, N, K) of every GEMV of the layer set, in layer order."""
    return [(li, pi, n, k) for li in range(n_layers) for pi, (_, n, k) in enumerate(synth.BITNET_2B_SHAPES)]


def gemv_algo_bytes(n: int, k: int) -> int:
    """Algorithmic bytes of one layer-set GEMV: packed 2-bit weights, bf16 activations, fp32 outputs."""
    return n * k // 4 + 2 * k + 4 * n


def _oracle_inputs(items):
    out = []
    for li, pi, n, k in items:
        lay = synth.bitnet_layer(n, k, synth.bitnet_layer_set_seed(li, pi), 0.02)
        out.append((lay.trits, synth.draw_x_bf16(lay.seed, 1, k), lay.tensor_scale, gemv_algo_bytes(n, k)))
    return out


def _oracle_gemv(inp):
    import oracle
    trits, x, scale, _ = inp
    q, s = oracle.quantize_act(x)
    oracle.gemv_bitnet_int8(trits, q, s, scale)


def _oracle_worker(items, cmd_q, res_q):
    """One process of the all-core oracle: draws its share of the layer set once, then runs the
    GEMVs it is told to on one thread and reports its bytes."""
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)
    data = _oracle_inputs(items)
    res_q.put(("ready", 0))
    while True:
        cmd = cmd_q.get()
        if cmd is None:
            return
        done = 0
        for j in cmd:
            _oracle_gemv(data[j])
            done += data[j][3]
        res_q.put(("done", done))


class OraclePool:
    """The oracle on all host cores: one spawned process per core (never forked after CUDA use),
    each owning a round-robin share of the layer set's GEMVs."""

    def __init__(self, n_layers: int, workers: int):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        items = layer_set_items(n_layers)
        self.workers = max(1, min(workers, len(items)))
        self.shares = [items[w::self.workers] for w in range(self.workers)]
        self.res_q = ctx.Queue()
        self.cmd_qs = [ctx.Queue() for _ in range(self.workers)]
        self.procs = [ctx.Process(target=_oracle_worker, args=(self.shares[w], self.cmd_qs[w], self.res_q),
                                  daemon=True) for w in range(self.workers)]
        for pr in self.procs:
            pr.start()
        for _ in range(self.workers):
            self.res_q.get()

    def run(self, frac: float = 1.0):
        """Every worker runs the first `frac` of its share; returns (bytes, wall seconds)."""
        t0 = time.perf_counter()
        for w, q in enumerate(self.cmd_qs):
            q.put(list(range(max(1, int(round(len(self.shares[w]) * frac))))))
        done = sum(self.res_q.get()[1] for _ in range(self.workers))
        return done, time.perf_counter() - t0

    def close(self):
        for q in self.cmd_qs:
            q.put(None)
        for pr in self.procs:
            pr.join(timeout=10)


def cpu_baseline(n_layers: int, budget_s: float = 8.0, max_workers: int = 64):
    """The oracle as it stands, on bounded samples of the layer set: one thread on the first GEMVs
    in layer order (about budget_s of work), then every host core (up to max_workers processes) on
    whole passes over the layer set."""
    from threadpoolctl import threadpool_limits
    done, t_used, gemvs = 0, 0.0, 0
    with threadpool_limits(limits=1):
        for it in layer_set_items(n_layers):
            inp = _oracle_inputs([it])[0]
            t0 = time.perf_counter()
            _oracle_gemv(inp)
            t_used += time.perf_counter() - t0
            done += inp[3]
            gemvs += 1
            if t_used > budget_s:
                break
    one = done / t_used / 1e9
    cores = host_cores()
    pool = OraclePool(n_layers, min(cores, max_workers))
    try:
        pool.run(0.0)                                   # warm-up: one GEMV per worker
        b, dt = pool.run(1.0)
    finally:
        pool.close()
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
            "host_cores": cores, "cpu_model": cpu_model(),
            "sample": "all %d GEMVs of the layer set, one pass, split over %d single-threaded processes (%.1f s "
                      "wall); inputs drawn by the seeded generators, timed work = per-token quantisation + exact "
                      "integer GEMV + scales (numpy)" % (len(layer_set_items(n_layers)), pool.workers, dt),
            "single_thread": {"value": round(one, 4), "unit": "GB/s", "cores": 1,
                              "sample": "first %d GEMVs of the layer set in layer order, %.1f s" % (gemvs, t_used)}}


# ------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    """The oracle as the reference arm, on the host cores, on the headline workload: each step is
    one pass over the layer set (or, where the host's cores cannot finish the run within a few
    minutes, the same fraction of every process's share, stated in the sample)."""
    if rank != 0:
        return None
    cores = host_cores()
    pool = OraclePool(args.layers, min(cores, 64))
    try:
        b1, t1 = pool.run(1.0)                          # one full pass, untimed: sizes the sample
        budget = 150.0
        frac = min(1.0, budget / (args.steps + args.warmup) / t1)
        for _ in range(args.warmup):
            pool.run(frac)
        done, t_tot = 0, 0.0
        for _ in range(args.steps):
            b, dt = pool.run(frac)
            done += b
            t_tot += dt
    finally:
        pool.close()
    v = done / t_tot / 1e9
    full_bytes = sum(gemv_algo_bytes(n, k) for _, _, n, k in layer_set_items(args.layers))
    sample = ("%s of the layer set per step (%.0f of %.0f MB algorithmic bytes), split over %d single-threaded "
              "processes; inputs drawn by the seeded generators; timed work = per-token quantisation + exact "
              "integer GEMV + scales (numpy); host: %s" % (
                  "all" if frac >= 1.0 else "%.1f%%" % (100 * frac), done / args.steps / 1e6, full_bytes / 1e6,
                  pool.workers, cpu_model()))
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_tot * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": {"workload": WORKLOAD, "reference": "CPU oracle",
                                            "same_config": frac >= 1.0},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.impl == "ours" and args.ceiling:
        out = run_ceiling(args) if rank == 0 else None
    elif args.impl == "ours" and args.config != "bitnet2b":
        out = run_config(args) if rank == 0 else None
    else:
        out = run_reference(args, rank, world) if args.impl == "reference" else run_ours(args, rank, world)
    if rank == 0 and out is not None:
        print(json.dumps(out))
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
