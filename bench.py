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
    ap.add_argument("--profile", default=None,
                    help="run only one case eagerly for a profiler: step | <shape>_indep | <shape>_chain "
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
    per_shape = []
    for nm, n, k in synth.BITNET_2B_SHAPES:
        Ls = [L for L in layers if L["name"] == nm]
        b = sum(gbytes(L) for L in Ls)
        ms_c = timed(g_chain[nm], reps) / reps
        launches, copies = pools[nm][0], pools[nm][1]
        ms_i = timed(g_pool[nm], 3) / (3 * 4)
        bp = (b // len(Ls)) * copies
        per_shape.append(dict(shape=f"{nm} {n}x{k}", bytes_per_gemv=b // len(Ls),
                              chain_us_per_gemv=round(ms_c * 1e3 / len(Ls), 3),
                              chain_gbs=round(b / (ms_c * 1e-3) / 1e9, 1),
                              independent_gbs=round(bp / (ms_i * 1e-3) / 1e9, 1),
                              independent_frac=round(bp / (ms_i * 1e-3) / 1e9 / peak, 4),
                              independent_pool="%d copies (%.0f MB) in %d launch(es), 4 rounds per graph" % (
                                  copies, bp / 1e6, len(launches))))

    # end to end through the public API: pinned H2D of the step's activations,
    # the captured step, D2H of the step's outputs
    h2d = x_all_host.numel() * 2
    d2h = y_all_host.numel() * 4
    with torch.cuda.stream(stream):
        def e2e_step():
            x_all.copy_(x_all_host, non_blocking=True)
            g_step.replay()
            y_all_host.copy_(y_all, non_blocking=True)
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = e0.elapsed_time(e1) / reps
    ms_e2e = max_over_ranks(ms_e2e, world, dev)
    assert tern.device_error(stream) == tern.OK

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
                               "decode_chain": round(world * 1e3 / ms_chain_step, 1),
                               "basis": "a step's GEMVs are the projection layers one decoded token at batch 1 "
                                        "streams (attention, norms and the output head are not on this path); "
                                        "tokens per second = steps per second, summed over replicas"},
        "e2e": {"value": round(replica_gbs(step_bytes, ms_e2e, world), 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * len(step_launches),
        "parity_bit_exact": parity,
        "parity_sample": "%d rows of each of %s in the timed launch, against the oracle" % (
            256, ", ".join("layer %d %s" % c for c in parity_checks(args.layers))),
    }
    if clk is not None:
        out["clocks"] = clk
    if rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline(budget_s=12.0)
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


def run_config(args):
    """Per-shape tables for the other workloads (one JSON line, rank 0, one GPU).

    Each shape's packed layer is replicated on the device until the pool holds
    at least 512 MB (4x L2), so every launch streams from HBM; "independent" is
    one grouped launch over all copies, "chain" launches the copies one after
    another with programmatic dependent launch.
    """
    import torch

    from packed_ternary_weight_b200 import tern

    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    if args.config == "single":
        layers = [synth.single_gemv_layer()]
        act = tern.ACT_BF16_Q8
    elif args.config == "tq3p":
        layers = list(synth.tq3p_llama_layers())
        act = tern.ACT_BF16
    elif args.config == "bt3":
        layers = list(synth.bt3_llama_layers())
        act = tern.ACT_BF16
    else:
        layers = list(synth.tq2p_prefill_layers())
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
        tokens = synth.PREFILL_TOKENS if args.config == "tq2p" else (1,)
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
            algo = wbytes + m * lay.k * (1 if act == tern.ACT_INT8 else 2) + 4 * m * lay.n

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
                       chain_gbs=round(algo * copies / (ms_c * 1e-3) / 1e9, 1))
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
    out = {"metric": METRIC, "config": {"workload": args.config}, "unit": "GB/s", "peak": peak, "per_shape": rows}
    if args.config in ("tq3p", "bt3"):   # the seven projections of one Llama-3.1-8B layer
        out["tokens_per_s_equiv"] = model_token_rate(rows, synth.LLAMA_8B_LAYERS)
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
def cpu_baseline(budget_s: float):
    """The oracle as it stands on a bounded sample of the same workload."""
    import oracle
    from packed_ternary_weight_b200 import tern
    from threadpoolctl import threadpool_limits
    done_bytes, t_used, gemvs = 0, 0.0, 0
    with threadpool_limits(limits=1):
        for lay in synth.bitnet_layer_set():
            _, buf = tern.pack_layer(lay)
            x = synth.draw_x_bf16(lay.seed, 1, lay.k)
            t0 = time.perf_counter()
            u = oracle.unpack(buf)
            q, s = oracle.quantize_act(x)
            oracle.gemv_bitnet_int8(u["trits"], q, s, u["tensor_scale"])
            t_used += time.perf_counter() - t0
            done_bytes += (len(buf) - 256) + 2 * lay.k + 4 * lay.n
            gemvs += 1
            if t_used > budget_s:
                break
    return {"value": round(done_bytes / t_used / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {gemvs} GEMVs of the layer set in layer order (unpack + quantise + exact "
                      f"integer GEMV, numpy, one thread), {t_used:.1f} s"}


# ------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    """The oracle as the reference arm: bounded samples of the workload on host cores."""
    if rank != 0:
        return None
    import oracle
    from packed_ternary_weight_b200 import tern
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)
    total_steps = args.steps + args.warmup
    budget = 90.0
    lay = synth.bitnet_layer(2560, 6912, synth.bitnet_layer_set_seed(0, 6))   # down_proj of layer 0
    _, buf = tern.pack_layer(lay)
    x = synth.draw_x_bf16(lay.seed, 1, lay.k)
    # rows per step so that all steps fit the budget (one 32-row tile minimum)
    t0 = time.perf_counter()
    u = oracle.unpack(buf)
    q, s = oracle.quantize_act(x)
    oracle.gemv_bitnet_int8(u["trits"], q, s, u["tensor_scale"])
    full = time.perf_counter() - t0
    frac = min(1.0, budget / total_steps / full)
    rows = max(32, int(lay.n * frac) // 32 * 32)
    tiles = rows // 32
    hdr = oracle.parse_header(buf)
    cols = hdr["cols"]
    tile_bytes = cols * 512
    sub = np.concatenate([buf[:256], buf[256:256 + tiles * tile_bytes]])
    hd = sub[:256].copy().view("<u4")
    hd[3] = rows                     # N of the sub-buffer (whole row tiles)
    hd[8] = tiles
    sub[:256] = hd.view(np.uint8)
    sub[48:56] = np.frombuffer(np.uint64(tiles * tile_bytes).tobytes(), np.uint8)
    sub[56:64] = np.frombuffer(np.uint64(256 + tiles * tile_bytes).tobytes(), np.uint8)
    step_bytes = tiles * tile_bytes + 2 * lay.k + 4 * rows

    def one():
        uu = oracle.unpack(sub)
        qq, ss = oracle.quantize_act(x)
        oracle.gemv_bitnet_int8(uu["trits"], qq, ss, uu["tensor_scale"])

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    v = step_bytes * args.steps / dt / 1e9
    sample = f"{rows} of 2560 rows of down_proj 2560x6912 per step (unpack + quantise + exact integer GEMV, numpy, 1 thread)"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": {"workload": WORKLOAD, "reference": "CPU oracle"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
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
