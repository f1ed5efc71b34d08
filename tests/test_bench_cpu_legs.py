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
    res = bench.cpu_baseline(w, inp, budget_s=2.0)
    assert res["kind"] == "oracle" and res["cores"] == 1 and res["value"] > 0


def test_reference_arm_prints_one_json_line():
    w = wl.SMALL[4]
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", w.name, "--steps", "1", "--warmup", "3",
                          "--ref-sample", "4"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["config"]["workload"] == w.name
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0


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
