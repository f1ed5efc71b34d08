"""The benchmark's CPU legs (the oracle's baseline and the reference arm)
run without a GPU: they must handle every workload shape, shared experts
included, and print the documented JSON line."""
import json
import os
import subprocess
import sys

import bench
from expert_dispatch_gemm_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_cpu_baseline_covers_shared_experts():
    w = wl.SMALL[4]  # grouped sigmoid routing with a shared expert
    assert w.n_shared == 1
    inp = wl.make_inputs(w, "cpu")
    res = bench.cpu_baseline(w, inp, steps=1)
    assert res["kind"] == "oracle" and res["cores"] == 1 and res["value"] > 0
    assert res["tokens_per_step"] == bench.oracle_sample_tokens(w)


def test_oracle_sample_rule():
    """One rule sizes both CPU legs: about 8 GFLOP of expert FFN per step,
    the whole batch when that is less; token choice without a capacity
    routes each token alone, so its steps need no extrapolation."""
    assert bench.oracle_sample_tokens(wl.EC_FP32) == wl.EC_FP32.n
    for w in wl.FULL[1:]:
        m = bench.oracle_sample_tokens(w)
        assert 4 <= m < w.n
    assert bench.routes_per_token(wl.TC_SIGMOID_GROUPED)
    assert bench.routes_per_token(wl.TC_DROPLESS)
    assert not bench.routes_per_token(wl.TC_TOP2_CAP)  # capacity: needs the whole batch
    assert not bench.routes_per_token(wl.EC_BF16)


def test_sampled_oracle_step_equals_full_batch_rows():
    """Routing a sample of tokens alone gives those tokens the same layer
    output as routing the whole batch (token choice without a capacity), so
    the reference arm's sampled step is the layer on those tokens."""
    import numpy as np
    import oracle
    w = wl.SMALL[4]
    X, Wg, lb, sb, weights, shared = bench._host_inputs(w, wl.make_inputs(w, "cpu"))
    spec = oracle.spec_of(w)
    toks = [3, 17, 150, 299]
    _, S, lse = oracle.router(X, Wg, lb, spec["score"])
    full = oracle.layer_forward(spec, X, oracle.route(spec, S, lse, sb), weights, shared,
                                tokens=toks)
    _, S2, lse2 = oracle.router(X[toks], Wg, lb, spec["score"])
    part = oracle.layer_forward(spec, X[toks], oracle.route(spec, S2, lse2, sb), weights, shared)
    np.testing.assert_array_equal(full, part)


def test_reference_arm_prints_one_json_line():
    w = wl.SMALL[4]
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", w.name, "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["config"] == bench.config_dict(w, 1)
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0
    # ms_per_step is time that elapsed: the timed steps fit in the run
    assert j["ms_per_step"] * j["steps"] / 1e3 <= j["wall_s"]
    assert j["tokens_per_step"] == bench.oracle_sample_tokens(w)


def test_training_cpu_baseline_and_flop_count():
    """The training line's CPU baseline (the oracle's backward on sampled
    tokens) runs for a layer with a shared expert, and the backward's GEMM
    FLOPs count the recompute only for fp32 layers (bf16 layers keep U, V, H
    from the training forward)."""
    import torch
    w = wl.SMALL[4]
    inp = wl.make_inputs(w, "cpu")
    dout = torch.randn((w.n, w.d)).to(w.torch_dtype)
    res = bench.cpu_baseline_train(w, inp, dout, budget_s=2.0)
    assert res["kind"] == "oracle" and res["value"] > 0
    bf = bench.backward_flops(w, 2400)
    assert "recompute" not in bf
    rows = 2400 + w.n
    assert bf["dw13"] == 2 * (2.0 * rows * w.d * w.h)  # SwiGLU: W1 and W3
    assert "recompute" in bench.backward_flops(wl.EC_FP32, 1024)


def test_reference_arm_other_ranks_exit_without_output():
    """Under torchrun the reference arm runs on rank 0 alone; the other ranks
    exit 0 without work or output."""
    w = wl.SMALL[4]
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", w.name, "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


def test_clock_summary_reads_nvml_masks_and_smi_lines():
    """The clock record: median SM clock under load, the maximum, and every
    clock-event reason seen in any sample, from NVML bitmasks (hw slowdown
    0x8, sw power cap 0x4, ...) or from nvidia-smi's csv fields."""
    c = bench.ClockSampler(0)
    c.samples = [(1700, 1965, 0x4), (1650, 1965, 0x4 | 0x8), (1750, 1965, 0x0)]
    c.lines = []
    s = c.summary()
    assert s["sm_mhz"] == 1700.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    c = bench.ClockSampler(0)
    c.lines = ["0, 1800, 1965, 950.1, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1900, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    s = c.summary()
    assert s["sm_mhz"] == 1850.0 and s["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler(0).summary()["reasons"] == ["unsampled"]
