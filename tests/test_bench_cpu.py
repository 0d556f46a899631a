"""bench.py's host logic on CPU: the key that ties the committed DRAM-traffic
summary to the kernel it was captured on (comment edits keep it, code edits
change it), the token-rate arithmetic, the clock verdict, and the reference
arm's JSON line."""
import bench


def _hash(tmp_path, text):
    p = tmp_path / "k.cuh"
    p.write_text(text)
    return bench.code_hash(str(p))


BASE = '''// a kernel
__device__ int f(int x) {  /* body */
  asm volatile("mov.u32 %0, %1; // not a comment" : "=r"(x) : "r"(x));
  return x + 1;   // increment
}
'''


def test_comment_edits_keep_the_key(tmp_path):
    a = _hash(tmp_path, BASE)
    b = _hash(tmp_path, BASE.replace("// a kernel", "// the kernel, reworded\n// over two lines")
              .replace("/* body */", "/* a\n   longer body comment */").replace("// increment", ""))
    assert a == b


def test_code_edits_change_the_key(tmp_path):
    a = _hash(tmp_path, BASE)
    assert _hash(tmp_path, BASE.replace("x + 1", "x + 2")) != a
    # text inside a string literal is code, even when it looks like a comment
    assert _hash(tmp_path, BASE.replace("// not a comment", "// changed")) != a
    assert _hash(tmp_path, BASE.replace("return x", "return  x")) == a       # whitespace only


def test_committed_summary_parses():
    v = bench.committed_traffic()
    assert v is None or v > 0


def test_model_token_rate():
    # two shapes per layer, 2 layers: chain 10 + 30 us per layer -> 80 us per token
    rows = [dict(m=1, bytes_per_gemv=1e6, chain_us_per_gemv=10.0, independent_gbs=1000.0),
            dict(m=1, bytes_per_gemv=3e6, chain_us_per_gemv=30.0, independent_gbs=3000.0),
            dict(m=4, bytes_per_gemv=9e9, chain_us_per_gemv=1.0)]          # batched rows are not part of it
    r = bench.model_token_rate(rows, 2)
    assert r["decode_chain"] == 12500.0                # 1e6 / 80
    assert r["independent"] == 250000.0                # 2 layers x (1 us + 1 us) per token
    assert r["shapes_per_layer"] == 2
    assert "independent" not in bench.model_token_rate([dict(m=1, bytes_per_gemv=1, chain_us_per_gemv=1.0)], 1)


def test_clock_verdict():
    ok = dict(sm_mhz=1800.0, sm_max_mhz=1965.0, reasons=["sw_power_cap"], samples=10)
    assert bench.clock_verdict(ok) is None                                  # the power cap is kept
    assert bench.clock_verdict(None) is None and bench.clock_verdict(dict(samples=0)) is None
    hot = dict(ok, reasons=["hw_thermal_slowdown", "sw_power_cap"])
    assert bench.clock_verdict(hot) == "throttled: hw_thermal_slowdown"
    locked = dict(sm_mhz=1200.0, sm_max_mhz=1965.0, reasons=[], samples=10)
    assert "no reason" in bench.clock_verdict(locked)
    capped_low = dict(locked, reasons=["sw_power_cap"])                   # low, but with a reason
    assert bench.clock_verdict(capped_low) is None


def test_reference_arm_line():
    # the reference arm is the oracle on host cores (spawned processes, oracle code only): its JSON
    # line carries the contract's keys; two layers keep the test short
    import argparse
    import sys
    args = argparse.Namespace(steps=1, warmup=0, layers=2)
    out = bench.run_reference(args, 0, 1)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["value"] > 0 and out["unit"] == "GB/s"
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["config"]["same_config"] is True               # a whole pass of the (two-layer) set
    assert out["e2e"]["value"] == out["value"] and out["e2e"]["h2d_bytes_per_step"] == 0
    assert bench.run_reference(args, 1, 2) is None            # other ranks do no work
    # the product library is not loaded on this leg (checked in a fresh interpreter)
    code = ("import argparse, sys, bench; bench.run_reference(argparse.Namespace(steps=1, warmup=0, layers=1), 0, 1); "
            "assert 'packed_ternary_weight_b200.tern' not in sys.modules")
    import subprocess
    r = subprocess.run([sys.executable, "-c", code], cwd=bench.ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr


def test_oracle_pool_covers_the_layer_set():
    # every GEMV of the layer set is in exactly one worker's share, and a full pass counts all bytes
    items = bench.layer_set_items(2)
    assert len(items) == 14
    pool = bench.OraclePool(2, 3)
    try:
        shares = [it for sh in pool.shares for it in sh]
        assert sorted(shares) == sorted(items)
        b, dt = pool.run(1.0)
        assert b == sum(bench.gemv_algo_bytes(n, k) for _, _, n, k in items) and dt > 0
    finally:
        pool.close()


def test_parity_samples_plumbing():
    # the bench's spot check finds each sampled GEMV's rows at its own offset of the step's outputs
    import numpy as np

    import oracle
    from packed_ternary_weight_b200 import synth
    n_layers = 30
    by, off = {}, 0
    for li in range(n_layers):
        for nm, n, k in synth.BITNET_2B_SHAPES:
            by[(li, nm)] = dict(n=n, k=k, yoff=off)
            off += n
    y = np.full(off, np.nan, np.float32)
    names = [nm for nm, _, _ in synth.BITNET_2B_SHAPES]
    for li, nm in bench.parity_checks(n_layers):
        L = by[(li, nm)]
        lay = synth.bitnet_layer(L["n"], L["k"], synth.bitnet_layer_set_seed(li, names.index(nm)), 0.02)
        q, s = oracle.quantize_act(synth.draw_x_bf16(lay.seed, 1, lay.k))
        y[L["yoff"]:L["yoff"] + L["n"]] = oracle.gemv_bitnet_int8(lay.trits, q, s, 0.02)[0]
    assert bench.parity_samples(y, by, n_layers)
    li, nm = bench.parity_checks(n_layers)[-1]
    rows = np.sort(np.random.default_rng(li).choice(by[(li, nm)]["n"], 256, replace=False))
    y[by[(li, nm)]["yoff"] + rows[7]] += 1.0                     # one wrong output in the last sample
    assert not bench.parity_samples(y, by, n_layers)
