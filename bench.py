"""Benchmark of the MoE routing-and-dispatch layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--pass forward|train]

One step = one moe_layer_forward call over one batch: moe_route (router GEMM
+ scores + top-k + capacity scan) -> moe_dispatch (gather) -> moe_expert_ffn
(tcgen05 grouped GEMM, up + down) -> moe_combine. Inputs and weights are
resident in HBM before timing; L2 (126 MB) is flushed by writing a 256 MB
buffer between timed steps, outside the timed events. Steps are timed with
CUDA events on the launching stream; a second pass calls the four stages one
by one with an event between them for the per-stage figures.

Default workload: the largest configuration, the DeepSeek-V3-shaped layer
("MoE routing strategies explained", sections 3-5: 256 routed experts plus
one shared, sigmoid scores with a selection-only bias, 8 groups keep 4,
top-8, normalised weights; 8,192 tokens, d 7168, SwiGLU h 2048, bf16).

e2e: the same layer through moe_layer_forward_host, the C call that takes
host X and host out (page-locked) and copies them itself on the caller's
stream; two such calls alternate on two streams so that one call's copies
overlap the other's kernels.

Multi-GPU: the layer does not shard ("replicas only"): each rank runs an
independent replica, no collective touches the data path, and the timed
region is the max over ranks.

--impl reference times the CPU oracle as it stands (single thread) on the
same workload, a bounded sample of tokens per step (the rule of
oracle_sample_tokens, shared with the cpu_baseline leg).

--pass train times forward + backward (moe_layer_forward_train then
moe_layer_backward_train: gradients of X, W_g and every expert weight) per
step, with the backward's grouped-GEMM FLOPs against the tensor-core peak.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from expert_dispatch_gemm_b200 import workloads as wl  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200; route/dispatch HBM GB/s; expert-GEMM TC util %"
DEFAULT = wl.TC_SIGMOID_GROUPED
L2_FLUSH_BYTES = 256 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# multi-rank plumbing (replicas only: no collective touches the data path)
# ---------------------------------------------------------------------------

def max_over_ranks(value_ms: float, device=None) -> float:
    """The slowest rank's time: every rank calls this in the same order."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value_ms)
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Units all ranks processed per second over the max-over-ranks time."""
    return units_per_rank * world * steps / (total_ms * 1e-3)


# ---------------------------------------------------------------------------
# algorithmic work per stage (each input read once, each output written once)
# ---------------------------------------------------------------------------

def algorithmic(w: wl.Workload, k_eff: int, rows_gathered: int, expert_rows):
    """bytes per stage and FLOPs of the grouped GEMM."""
    xb = 4 if w.dtype == "f32" else 2
    n, d, E, h = w.n, w.d, w.E, w.h
    slots = E * k_eff if w.mode == "ec" else n * k_eff
    route = n * d * xb + d * E * 4 + slots * 8
    if w.mode == "ec":
        route += 2 * n * E * 4  # the score matrix is written and read back (one global pass)
    A = rows_gathered
    dispatch = n * d * xb + A * d * xb
    nproj = 3 if w.act == "swiglu" else 2
    active = int(sum(1 for m in expert_rows if m > 0))
    weights = (active + w.n_shared) * nproj * h * d * xb
    rows_all = A + w.n_shared * n
    ffn_bytes = weights + rows_all * d * xb + 2 * rows_all * h * xb + rows_all * d * xb
    flops = 2.0 * rows_all * d * h * nproj
    combine = A * d * xb + w.n_shared * n * d * xb + n * d * xb
    return dict(route=route, dispatch=dispatch, ffn=ffn_bytes, combine=combine), flops


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock, its maximum and the active clock-event reasons during the
    timed region: NVML polled every 10 ms from a thread (the GPU matched by
    its PCI bus id), else `nvidia-smi -lms 100` as a subprocess."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.thread = None
        self.samples = []
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self._stop = threading.Event()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

            def poll():
                while not self._stop.is_set():
                    try:
                        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx,
                                             nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except Exception:
                        pass
                    self._stop.wait(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 100 ms"
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        for clk, m, mask in self.samples:
            sm.append(float(clk))
            mx = float(m)
            for nm, bit in self.REASONS:
                if mask & bit:
                    reasons.add(nm)
        names = [nm for nm, _ in self.REASONS]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def ffma_peak_tflops(dev, detail: dict = None) -> float:
    """FP32 FMA throughput of this device, measured with the probe kernels in
    libmoe_probe.so (the router's roof; not among the measured HBM / tensor
    peaks): single FFMAs and packed fp32x2 FMAs, the faster of the two. Median
    of 5 timed launches after 2 warm-ups each."""
    import ctypes
    lib = ctypes.CDLL(os.path.join(ROOT, "expert_dispatch_gemm_b200", "libmoe_probe.so"))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks, iters = sms * 8, 2048
    out = torch.empty(blocks, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = 2.0 * blocks * 256 * iters * 16
    rates = {}
    for name in ("moe_probe_ffma", "moe_probe_ffma2"):
        fn = getattr(lib, name)
        fn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        times = []
        for i in range(7):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rc = fn(blocks, iters, out.data_ptr(), ctypes.c_void_p(stream.cuda_stream))
            e1.record(stream)
            if rc != 0:
                raise RuntimeError(f"{name} launch failed: {rc}")
            torch.cuda.synchronize(dev)
            if i >= 2:
                times.append(e0.elapsed_time(e1))
        rates[name] = flops / (float(np.median(times)) * 1e-3) / 1e12
    if detail is not None:
        detail.update({"ffma_TFLOP/s": round(rates["moe_probe_ffma"], 1),
                       "ffma2_TFLOP/s": round(rates["moe_probe_ffma2"], 1)})
    return max(rates.values())


def source_sha(name: str) -> str:
    """Hash of a CUDA source's device code (the file up to its '// host side'
    marker, or all of it), to tell whether a committed capture still holds."""
    code = open(os.path.join(ROOT, "expert_dispatch_gemm_b200", "csrc", name), "rb").read()
    return hashlib.sha256(code.split(b"// host side")[0]).hexdigest()[:16]


def traffic_for(workload: str):
    """DRAM bytes per launch of the grouped GEMM from the committed ncu summary
    (profiles/gemm_traffic.json), or None when the device code of a source it
    was captured from changed since, or the workload was not captured."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec["bytes_per_launch"][workload]
        for src, sha in entry["sources"].items():
            if source_sha(src) != sha:
                return None
        return entry["bytes"]
    except Exception:
        return None


def routing_stats(w, cfg, inp, rb, ws, moe, stream) -> dict:
    """The per-workload routing figures: expert choice, the experts-per-token
    histogram (the pages: most tokens on 1-2 experts, about 23% on 3-4, 3% on
    more); a capacity, the dropped fractions; the balance and z losses; with a
    selection bias, MaxVio over the simulated bias-update steps (moe_route
    then moe_bias_update, the same X and W_g each step)."""
    aux = rb.aux_dict()
    out = {}
    n, K = w.n, w.K
    if w.mode == "ec":
        h = rb.ec_hist.cpu().numpy().astype(np.int64)
        out["experts_per_token"] = {"0": int(h[0]), "1-2": int(h[1:3].sum()),
                                    "3-4": int(h[3:5].sum()), ">4": int(h[5:].sum())}
        out["experts_per_token_frac"] = {k: round(v / n, 4)
                                         for k, v in out["experts_per_token"].items()}
        return out
    if w.capacity_factor > 0:
        out["dropped_assignment_frac"] = round(aux["dropped_assignments"] / (n * K), 4)
        out["tokens_some_dropped_frac"] = round(aux["tokens_some_dropped"] / n, 4)
        out["tokens_all_dropped_frac"] = round(aux["tokens_all_dropped"] / n, 4)
    out["lb_loss"] = round(aux["lb_loss"], 6)
    out["z_loss"] = round(aux["z_loss"], 6)
    out["maxvio"] = round(aux["maxvio"], 4)
    if inp.get("sel_bias") is not None and w.bias_steps > 0:
        bias = torch.zeros_like(inp["sel_bias"])
        rb2 = moe.RouteBuffers(cfg, inp["X"].device, logits=False)
        per_step = []
        for _ in range(w.bias_steps):
            moe.moe_route(cfg, inp["X"], inp["Wg"], inp["logit_bias"], bias, rb2, ws, stream)
            moe.moe_bias_update(cfg, rb2.load, w.bias_rate, bias, stream)
            per_step.append(round(float(rb2.aux[moe.AUX_NAMES.index("maxvio")].item()), 4))
        out["maxvio_per_bias_step"] = per_step
    return out


def config_dict(w: wl.Workload, world: int, **extra) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": w.name, "tokens": w.n, "d_model": w.d, "experts": w.E, "hidden": w.h,
            "shared_experts": w.n_shared,
            "routing": ("expert-choice c=%g" % w.c if w.mode == "ec"
                        else "token-choice top-%d" % w.K),
            "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
            "l2": "flushed between timed steps (256 MB write, outside the events)", **extra}


def run_gpu(args, w: wl.Workload):
    import torch.distributed as dist

    from expert_dispatch_gemm_b200 import moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    inp = wl.make_inputs(w, dev)
    cfg = moe.config(w)
    sz = moe.sizes(cfg)
    layer = moe.Layer(w, inp, dev)           # the timed calls: moe_layer_forward
    rb = moe.RouteBuffers(cfg, dev)          # the stage pass: the four calls one by one
    ws = moe.workspace(cfg, dev, layer=False)
    dt = w.torch_dtype
    X_perm = torch.empty((sz.rows, w.d), dtype=dt, device=dev)
    H = torch.empty((sz.rows, w.h), dtype=dt, device=dev)
    Y = torch.empty((sz.rows, w.d), dtype=dt, device=dev)
    out = torch.empty((w.n, w.d), dtype=dt, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sb = inp["sel_bias"]
    fused = args.fused_combine
    if fused:
        acc = torch.empty((w.n, w.d), dtype=torch.float32, device=dev)
        row_gate = torch.empty(max(sz.rows, 1), dtype=torch.float32, device=dev)

    def step():
        """One pass of the layer: one moe_layer_forward call (with
        --fused-combine: the four calls, the combine inside the down
        projection's epilogue by moe_expert_ffn_combined)."""
        if fused:
            staged()
        else:
            layer.forward(stream=stream)

    def staged(ev=None):
        """The calls moe_layer_forward makes, one by one: route -> dispatch
        gather -> grouped expert FFN -> combine, with an event between them."""
        X = inp["X"]
        if ev: ev[0].record(stream)
        moe.moe_route(cfg, X, inp["Wg"], inp["logit_bias"], sb, rb, ws, stream)
        if ev: ev[1].record(stream)
        moe.moe_dispatch(cfg, X, rb, X_perm, stream)
        if ev: ev[2].record(stream)
        if fused:
            moe.moe_expert_ffn_combined(cfg, X, X_perm, rb, inp["W1"], inp["W3"], inp["W2"],
                                        inp.get("sW1"), inp.get("sW3"), inp.get("sW2"), H, acc,
                                        row_gate, out, ws, stream)
            if ev: ev[3].record(stream)
        else:
            moe.moe_expert_ffn(cfg, X, X_perm, rb.offsets, inp["W1"], inp["W3"], inp["W2"],
                               inp.get("sW1"), inp.get("sW3"), inp.get("sW2"), H, Y, ws, stream,
                               counts=rb.counts)
            if ev: ev[3].record(stream)
            moe.moe_combine(cfg, Y, rb, out, stream)
        if ev: ev[4].record(stream)

    def check_errors(when):
        for wsp in (layer.ws, ws):
            st, detail = moe.moe_read_error(wsp)
            if st != moe.MOE_OK:
                raise RuntimeError(f"device error {when}: {detail:#x}")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    check_errors("after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()  # outside the timed events: L2 starts cold every step
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall0
    if world > 1:
        dist.barrier()
    step_ms = np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps)])
    total_ms = float(step_ms.sum())
    total_ms = max_over_ranks(total_ms, dev)
    # per-stage breakdown: a second pass with an event between the stages
    # (those events keep a stage's kernels from overlapping the previous
    # stage's tail, so the stages add up to a little more than a step)
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        staged(sevs[i])
    torch.cuda.synchronize(dev)
    stage_ms = np.array([[sevs[i][j].elapsed_time(sevs[i][j + 1]) for j in range(4)]
                         for i in range(args.steps)])
    check_errors("in the timed region")

    # ---- a floor for the two copy-like stages: a plain device-to-device copy
    # (torch, the copy engine's kernel) moving the same bytes as the stage
    # (half read, half written), timed the same way (L2 flushed before each,
    # events around it); a stage at the copy's time is at what this size allows
    def copy_floor_ms(nbytes):
        half = max(16, int(nbytes // 2) // 16 * 16)
        src = torch.empty(half, dtype=torch.uint8, device=dev)
        dst = torch.empty_like(src)
        ts = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dst.copy_(src)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                ts.append(e0.elapsed_time(e1))
        del src, dst
        return float(np.median(ts))

    # ---- end to end through the C call that takes host buffers
    # (moe_layer_forward_host): every step uploads X from page-locked host
    # memory and downloads out into page-locked host memory, the library
    # issuing both copies on the call's stream. Two lanes (stream, device
    # buffers, routing, workspace, host output) alternate, so one call's
    # copies overlap the other lane's kernels.
    Xh = inp["X"].cpu().pin_memory()
    lanes = []
    for _ in range(2):
        lanes.append(dict(s=torch.cuda.Stream(dev), Xd=torch.empty_like(inp["X"]),
                          od=torch.empty_like(out), rb=moe.RouteBuffers(cfg, dev, logits=False),
                          ws=moe.workspace(cfg, dev, layer=True),
                          oh=torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                          done=torch.cuda.Event()))

    def e2e_run(nsteps):
        for i in range(nsteps):
            ln = lanes[i & 1]
            moe.moe_layer_forward_host(cfg, Xh, inp["Wg"], inp["logit_bias"], sb, inp["W1"],
                                       inp.get("W3"), inp["W2"], inp.get("sW1"), inp.get("sW3"),
                                       inp.get("sW2"), ln["oh"], ln["Xd"], ln["od"], ln["rb"],
                                       ln["ws"], ln["s"])
            ln["done"].record(ln["s"])

    torch.cuda.synchronize(dev)
    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for ln in lanes:
        ln["s"].wait_event(e0)
    e2e_run(args.steps)
    for ln in lanes:
        stream.wait_event(ln["done"])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    for ln in lanes:
        st, detail = moe.moe_read_error(ln["ws"], ln["s"])
        if st != moe.MOE_OK:
            raise RuntimeError(f"device error in the end-to-end run: {detail:#x}")
    # the host copy of the last step's output is the layer's output
    if not torch.equal(lanes[(args.steps - 1) & 1]["oh"], layer.out.cpu()):
        raise RuntimeError("moe_layer_forward_host returned a different output")

    # ---- routing statistics the workload statements ask for (from the last
    # step's routing outputs; untimed)
    routing = routing_stats(w, cfg, inp, rb, ws, moe, stream)

    # ---- algorithmic work and rooflines
    counts = rb.counts.cpu().numpy()
    rows_gathered = int(counts.sum())
    k_eff = sz.k
    bytes_, flops = algorithmic(w, k_eff, rows_gathered, counts)
    hbm, tc_burst, tc_sust, src = peaks()
    med = np.median(stage_ms, 0)
    names = ["route", "dispatch", "ffn", "combine"]
    stages = {}
    for j, nm in enumerate(names):
        gbs = bytes_[nm] / (med[j] * 1e-3) / 1e9
        stages[nm] = {"ms": round(float(med[j]), 4), "GB/s": round(gbs, 1),
                      "hbm_frac": round(gbs / hbm, 3)}
    # The burst tensor peak fits a GEMM that runs alone at full clock; when the
    # power cap held the clocks down during the timed steps, the GEMM ran as
    # part of a long power-capped loop and the sustained peak is the fair one.
    clocks = clk.summary()
    capped = "sw_power_cap" in clocks.get("reasons", [])
    use_sust = bool(capped and tc_sust)
    tc_peak = tc_sust if use_sust else tc_burst
    tc_peak_kind = "sustained (sw_power_cap active)" if use_sust else "burst"
    # the router contraction runs on FP32 FFMA: its roof is that pipe, taken
    # here over the whole route stage (router + selection kernels)
    probes = {}
    ffma_peak = ffma_peak_tflops(dev, probes)
    router_flops = 2.0 * w.n * w.d * w.E
    route_tflops = router_flops / (med[0] * 1e-3) / 1e12
    stages["route"].update({"router_FLOP": router_flops, "FFMA_TFLOP/s": round(route_tflops, 2),
                            "ffma_peak_TFLOP/s": round(ffma_peak, 1),
                            "ffma_probes": probes,
                            "ffma_frac": round(route_tflops / ffma_peak, 3)})
    for nm in ("dispatch", "combine"):
        fl = copy_floor_ms(bytes_[nm])
        stages[nm].update({"copy_floor_ms": round(fl, 4),
                           "frac_of_copy": round(fl / stages[nm]["ms"], 3)})
    ffn_tflops = flops / (med[2] * 1e-3) / 1e12
    stages["ffn"]["TFLOP/s"] = round(ffn_tflops, 1)
    stages["ffn"]["tc_frac"] = round(ffn_tflops / tc_peak, 3)
    # dominant kernel: the grouped GEMM (2 launches per step: up and down)
    t_hbm = bytes_["ffn"] / (hbm * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    per_launch_ms = float(med[2]) / 2.0
    traffic = traffic_for(w.name) if w.dtype == "bf16" else None
    if t_hbm >= t_tc:
        ach = bytes_["ffn"] / 2 / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 3)}
    else:
        ach = flops / 2 / (per_launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(ach / tc_peak, 3),
                "peak_kind": tc_peak_kind}
    roof.update({"traffic": traffic, "kernel": "grouped expert GEMM (up + down launches, avg)",
                 "peak_source": src,
                 "algorithmic_per_launch": bytes_["ffn"] / 2 if roof["bound"] == "hbm"
                 else flops / 2})

    value = whole_job_rate(w.n, world, args.steps, total_ms)
    e2e_value = whole_job_rate(w.n, world, args.steps, e2e_ms)
    # route: router (+ split-k reduce) + select_ec + ec_finish (EC) or + hist +
    # scan + scatter (TC); dispatch: gather; expert FFN: up + down; combine
    launches_per_step = sum(moe.launch_counts(cfg).values())
    if fused:
        launches_per_step += 1  # prep + up + down + finish replace up + down + combine
    xbytes = int(Xh.numel() * Xh.element_size())
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) activations, random-init weights)",
        "config": config_dict(w, world, **(
            {"combine": "fused into the down projection (moe_expert_ffn_combined); "
                        "the ffn stage includes it"} if fused else {})),
        "roofline": roof,
        "stages": stages,
        "routing": routing,
        "stages_note": "medians of a second pass with an event between stages; value and "
                       "ms_per_step come from whole-step events around moe_layer_forward; "
                       "copy_floor_ms: a plain device-to-device copy moving the stage's bytes "
                       "(half read, half written) from a cold L2, frac_of_copy = its time / "
                       "the stage's",
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": xbytes, "d2h_bytes_per_step": xbytes,
                "note": "moe_layer_forward_host (C ABI): page-locked host X -> device -> "
                        "layer -> page-locked host out every step, the copies issued by the "
                        "library on the call's stream; two calls alternate on two streams; "
                        "no L2 flush"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 4),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, inp)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# ---------------------------------------------------------------------------
# training step: forward + backward (--pass train)
# ---------------------------------------------------------------------------

METRIC_TRAIN = ("MoE-layer fwd+bwd tokens/s on 1 B200 (gradients of X, W_g and every expert "
                "weight); backward grouped-GEMM TC util %")


def backward_flops(w: wl.Workload, rows_gathered: int) -> dict:
    """FLOPs of the backward's grouped GEMMs and of the router's two FFMA
    contractions, over the kept rows (and the shared experts' n rows). bf16
    layers keep U, V and H from the training forward, so their backward runs
    four GEMMs; fp32 layers recompute the up projection."""
    g = 2 if w.act == "swiglu" else 1  # up projections per expert
    rows = rows_gathered + w.n_shared * w.n
    unit = 2.0 * rows * w.d * w.h
    out = {"dact": unit, "dx": unit * g, "dw2": unit, "dw13": unit * g,
           "router": 4.0 * w.n * w.d * w.E}
    if w.dtype == "f32":
        out["recompute"] = unit * g
    return out


def run_gpu_train(args, w: wl.Workload):
    import torch.distributed as dist

    from expert_dispatch_gemm_b200 import moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = wl.make_inputs(w, dev)
    layer = moe.Layer(w, inp, dev)
    gen = torch.Generator(device=dev).manual_seed(w.seed + 99)
    dout = torch.randn((w.n, w.d), generator=gen, device=dev).to(w.torch_dtype)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    layer.grads()

    def step(X=None, d=None, ev=None):
        """The training pair: the forward keeps U, V and H for the backward
        (bf16 layers; fp32 layers recompute them)."""
        layer.forward_train(X=X, stream=stream)
        if ev is not None:
            ev.record(stream)
        layer.backward_train(dout if d is None else d, X=X, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    for ws in (layer.ws, layer._bws):
        st, detail = moe.moe_read_error(ws)
        if st != moe.MOE_OK:
            raise RuntimeError(f"device error after warm-up: {detail:#x}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step(ev=evs[i][1])
            evs[i][2].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = np.array([evs[i][0].elapsed_time(evs[i][2]) for i in range(args.steps)])
    fwd_ms = np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps)])
    bwd_ms = np.array([evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps)])
    total_ms = max_over_ranks(float(step_ms.sum()), dev)
    for ws in (layer.ws, layer._bws):
        st, detail = moe.moe_read_error(ws)
        if st != moe.MOE_OK:
            raise RuntimeError(f"device error in the timed region: {detail:#x}")

    # end to end: X and dout up from pinned host memory, dX back, every step
    Xh = inp["X"].cpu().pin_memory()
    dh = dout.cpu().pin_memory()
    dXh = torch.empty(inp["X"].shape, dtype=inp["X"].dtype).pin_memory()
    Xd, dd = torch.empty_like(inp["X"]), torch.empty_like(dout)

    def e2e_step():
        Xd.copy_(Xh, non_blocking=True)
        dd.copy_(dh, non_blocking=True)
        step(X=Xd, d=dd)
        dXh.copy_(layer.grads()["dX"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)

    rows_gathered = int(layer.route.counts.sum().item())
    bf = backward_flops(w, rows_gathered)
    gemm_flops = sum(v for k, v in bf.items() if k != "router")
    hbm, tc_burst, tc_sust, src = peaks()
    clocks = clk.summary()
    capped = "sw_power_cap" in clocks.get("reasons", [])
    tc_peak = tc_sust if (capped and tc_sust) else tc_burst
    bwd_med = float(np.median(bwd_ms))
    ach = gemm_flops / (bwd_med * 1e-3) / 1e12
    if w.dtype == "f32":
        # the fp32 layer's GEMMs run on FFMA: their roof is that pipe
        fpk = ffma_peak_tflops(dev)
        roof = {"bound": "alu", "achieved": round(ach, 2), "peak": round(fpk, 1),
                "unit": "TFLOP/s", "frac": round(ach / fpk, 3),
                "peak_kind": "FP32 FFMA, measured by the probe kernel"}
    else:
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(ach / tc_peak, 3),
                "peak_kind": "sustained (sw_power_cap active)" if (capped and tc_sust)
                else "burst"}
    roof.update({"traffic": None, "peak_source": src,
                 "kernel": "moe_layer_backward_train as a whole: its grouped GEMMs' FLOPs over "
                           "the whole call (its non-GEMM kernels included in the time)",
                 "algorithmic_per_launch": gemm_flops})
    fwd_launches, bwd_launches = moe.train_launch_counts(layer.cfg)
    res = {
        "metric": METRIC_TRAIN,
        "value": round(whole_job_rate(w.n, world, args.steps, total_ms), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) activations and output gradient, random-init weights)",
        "config": config_dict(w, world, **{"pass": "forward + backward"}),
        "roofline": roof,
        "stages": {"forward": {"ms": round(float(np.median(fwd_ms)), 4)},
                   "backward": {"ms": round(bwd_med, 4),
                                "gemm_TFLOP": round(gemm_flops / 1e12, 3),
                                "router_FFMA_GFLOP": round(bf["router"] / 1e9, 2)}},
        "e2e": {"value": round(whole_job_rate(w.n, world, args.steps, e2e_ms), 1),
                "unit": "tokens/s",
                "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size() +
                                          dh.numel() * dh.element_size()),
                "d2h_bytes_per_step": int(dXh.numel() * dXh.element_size()),
                "note": "pinned host X and dout -> device -> forward + backward -> host dX "
                        "every step, on the compute stream; no L2 flush"},
        "gpu_launches": (fwd_launches + bwd_launches) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_train(w, inp, dout, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def cpu_baseline_train(w, inp, dout, budget_s=20.0):
    """The oracle's forward routing plus its backward on sampled tokens (each
    token's dX needs only its own pairs; their expert rows also carry the
    weight-gradient work), extrapolated to the batch."""
    import oracle
    X, Wg, lb, sb, weights, sw = _host_inputs(w, inp)
    spec = oracle.spec_of(w)
    dh = dout.float().cpu().numpy()
    rng = np.random.default_rng(0)
    t0 = time.perf_counter()
    logits, S, lse = oracle.router(X, Wg, lb, spec["score"])
    r = oracle.route(spec, S, lse, sb)
    t_route = time.perf_counter() - t0

    def run(toks):
        t1 = time.perf_counter()
        oracle.layer_backward(spec, X, Wg, dh, weights, sw, lb, sb, tokens=toks,
                              pre=(logits, S, lse, r))
        return time.perf_counter() - t1

    probe = sorted(rng.choice(w.n, size=min(2, w.n), replace=False).tolist())
    t_probe = run(probe)
    sample = int(max(2, min(w.n, (budget_s - t_route) / max(t_probe / len(probe), 1e-6) * 0.5)))
    toks = sorted(rng.choice(w.n, size=min(sample, w.n), replace=False).tolist())
    t = run(toks)
    est = t_route + t / len(toks) * w.n
    return {"value": round(w.n / est, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": (f"oracle routing of all {w.n} tokens ({t_route:.2f} s) plus the "
                       f"chain-rule backward of {len(toks)} seeded tokens (their expert rows, "
                       f"weight-gradient work included; {t:.2f} s), extrapolated to {w.n} "
                       "tokens; single-threaded C oracle, fp64")}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

ORACLE_STEP_FLOP = 8e9  # expert-FFN FLOPs of one oracle step (seconds of one core)


def oracle_sample_tokens(w: wl.Workload) -> int:
    """Tokens whose expert FFN and combine one oracle step computes: about
    ORACLE_STEP_FLOP of expert FFN, the whole batch when that is smaller.
    A fixed rule, shared by the reference arm and the cpu_baseline leg, so
    that both time the same work."""
    nproj = 3 if w.act == "swiglu" else 2
    per_token = w.c if w.mode == "ec" else w.K
    flop = 2.0 * nproj * w.d * w.h * (per_token + w.n_shared)
    return int(max(4, min(w.n, ORACLE_STEP_FLOP // flop)))


def routes_per_token(w: wl.Workload) -> bool:
    """Token choice without a capacity routes each token from its own row
    alone ("MoE token-choice routing": no batch coordination), so a sample
    of tokens is a complete layer call on those tokens. Expert choice and a
    capacity buffer need the whole batch's scores."""
    return w.mode == "tc" and w.capacity_factor <= 0


def _oracle_step(w, X, Wg, lb, sb, weights, shared, toks):
    """One oracle step over the tokens `toks`: (seconds routing, seconds of
    expert FFN + combine). Token choice without a capacity routes only the
    sampled tokens; otherwise the whole batch is routed and the FFN and
    combine run for the sample. The expert weights the sample needs are
    converted to the oracle's fp32 arrays before the clock starts (input
    marshalling, not the oracle's work)."""
    import oracle
    spec = oracle.spec_of(w)
    Xs = X[toks] if routes_per_token(w) else X
    t0 = time.perf_counter()
    _, S, lse = oracle.router(Xs, Wg, lb, spec["score"])
    r = oracle.route(spec, S, lse, sb)
    t_route = time.perf_counter() - t0
    local = list(range(len(toks))) if routes_per_token(w) else toks
    need = sorted({e for _, e, _ in oracle.token_pairs(spec, r, Xs.shape[0], local)})
    cache = {e: weights(e) for e in need}
    t0 = time.perf_counter()
    oracle.layer_forward(spec, Xs, r, cache.__getitem__, shared, tokens=local)
    t_ffn = time.perf_counter() - t0
    return t_route, t_ffn


def oracle_steps(w, host, steps: int, warmup: int = 0, seed: int = 0):
    """`warmup` untimed then `steps` timed oracle steps on the sample rule's
    token count, a fresh seeded sample each step. Returns (value tokens/s,
    measured seconds per step, tokens per step, extrapolated, description)."""
    X, Wg, lb, sb, weights, shared = host
    rng = np.random.default_rng(seed)
    m = oracle_sample_tokens(w)
    per_tok = routes_per_token(w)
    times, full = [], []
    for i in range(warmup + steps):
        toks = sorted(rng.choice(w.n, size=m, replace=False).tolist())
        t_route, t_ffn = _oracle_step(w, X, Wg, lb, sb, weights, shared, toks)
        if i >= warmup:
            times.append(t_route + t_ffn)
            full.append(t_route + t_ffn / m * w.n)
    sec = float(np.mean(times))
    if per_tok or m == w.n:
        value, extrap = m / sec, False
        what = (f"per step: the whole layer (router, grouped top-k, expert FFN incl. shared, "
                f"combine) for {m} seeded tokens of the {w.n}-token batch (each token routes "
                "from its own row alone), timed as it runs")
        if m == w.n:
            what = f"per step: the whole {w.n}-token batch, timed as it runs"
    else:
        value, extrap = w.n / float(np.mean(full)), True
        what = (f"per step: routing of all {w.n} tokens (it needs the whole batch) plus the "
                f"expert FFN and combine of {m} seeded tokens; value extrapolates the FFN and "
                f"combine to {w.n} tokens")
    return value, sec, m, extrap, what + "; single-threaded C oracle, fp64 accumulation"


def _host_inputs(w, inp=None):
    if inp is None:
        inp = wl.make_inputs(w, "cuda" if torch.cuda.is_available() else "cpu")

    def h(t):
        return None if t is None else t.detach().float().cpu().numpy()
    X, Wg, lb, sb = h(inp["X"]), h(inp["Wg"]), h(inp.get("logit_bias")), h(inp.get("sel_bias"))
    W1, W3, W2 = inp["W1"], inp.get("W3"), inp["W2"]

    def weights(e):
        return h(W1[e]), None if W3 is None else h(W3[e]), h(W2[e])

    shared = None
    if w.n_shared:
        def shared(s):
            return (h(inp["sW1"][s]), None if inp.get("sW3") is None else h(inp["sW3"][s]),
                    h(inp["sW2"][s]))
    return X, Wg, lb, sb, weights, shared


def cpu_baseline(w, inp=None, steps: int = 2):
    """The GPU arm's cpu_baseline leg: the reference arm's oracle step (same
    sample rule), `steps` times."""
    value, sec, m, extrap, what = oracle_steps(w, _host_inputs(w, inp), steps)
    return {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{what}; mean of {steps} steps of {sec:.2f} s",
            "tokens_per_step": m, "extrapolated": extrap}


def run_reference(args, w):
    """The reference arm: the oracle as it stands, on the host's cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = _host_inputs(w)
    t0 = time.perf_counter()
    value, sec, m, extrap, what = oracle_steps(w, host, args.steps, args.warmup, seed=1)
    wall = time.perf_counter() - t0
    cb = {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
          "sample": what, "tokens_per_step": m, "extrapolated": extrap}
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
           "config": config_dict(w, world),
           "tokens_per_step": m,
           "ms_per_step_note": ("measured oracle time per step (its routing, FFN and combine; "
                                "the conversion of the weights it reads is excluded)"),
           "wall_s": round(wall, 2),
           "cpu_baseline": cb,
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT.name, choices=sorted(wl.BY_NAME))
    ap.add_argument("--impl", default="libmoe", choices=["libmoe", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="--pass train: seconds of the oracle's backward baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fused-combine", action="store_true",
                    help="forward: the combine inside the down projection's epilogue")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "train"],
                    help="forward: the layer's forward (default); train: forward + backward")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = wl.BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    elif args.pass_ == "train":
        run_gpu_train(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
