#!/usr/bin/env python
"""Benchmark of the stacked MoE FFN forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = one moe_forward over the whole synthetic batch of the workload
(router -> CSR build -> gather -> gate_up GEMM + activation -> down GEMM +
weight -> combine), inputs resident in HBM.  Prints ONE JSON line on rank 0.

Multi-GPU: the layer is independent per token batch, so N ranks run N
independent replicas of the workload (weak scaling, no data-path
collective); the only collectives are the barrier and the max over ranks of
the device-timed region.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on the host cores, on a bounded sample of the same workload per step.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_ffn_token_b200 import abi  # noqa: E402
from mixture_experts_ffn_token_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE FFN tokens/s and achieved TFLOP/s (or HBM GB/s) vs B200 roofline"
UNIT = "tokens/s"
DEFAULT_CONFIG = "mixtral"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "gemm_gate_up": "mixture_experts_ffn_token_b200/csrc/grouped_gemm.cu",
    "gemm_down": "mixture_experts_ffn_token_b200/csrc/grouped_gemm.cu",
    "router": "mixture_experts_ffn_token_b200/csrc/router.cu",
    "gather": "mixture_experts_ffn_token_b200/csrc/csr.cu",
    "combine": "mixture_experts_ffn_token_b200/csrc/csr.cu",
}


# ------------------------------------------------------------------ helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_bytes(wl):
    """Algorithmic HBM bytes of one step: touched expert weights are counted
    by the caller; this is x + logits + out (+ biases)."""
    T, H = wl.num_tokens, wl.hidden_dim
    b = T * H * 2 * 2 + T * (wl.num_experts + wl.num_sink) * 4
    if wl.has_bias:
        b += wl.num_experts * (2 * wl.moe_dim + H) * 2
    return b


def touched_expert_bytes(wl, idx):
    used = torch.unique(idx.reshape(-1)).numel()
    return used * 3 * wl.hidden_dim * wl.moe_dim * 2, used


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            target = []
        self.cmd = ["nvidia-smi", *target, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(self.cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.25)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        mx = [num(r[1]) for r in rows if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[2]) or 0.0) for r in rows)}


def kernel_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken from the current source of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    ent = data.get(kernel)
    if not ent:
        return None
    src = os.path.join(ROOT, KERNEL_SOURCES.get(kernel, ""))
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    if ent.get("source_sha256_16") != digest:
        return None
    return ent.get("bytes_per_launch_full_size")


# ---------------------------------------------------------------- oracle arm
def oracle_sample_rate(wl, inp_host, n_tokens, seed=0):
    """Time the oracle (router over the sampled tokens, FFN for them) -> (tokens/s, threads)."""
    import numpy as np

    import oracle
    from mixture_experts_ffn_token_b200.workloads import bf16_bits
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(wl.num_tokens, size=n_tokens, replace=False)).astype(np.int64)
    logits = inp_host["logits"][torch.from_numpy(toks)].numpy()
    t0 = time.perf_counter()
    if wl.router == "softmax_topk":
        idx, w = oracle.route_softmax_topk(logits, wl.num_experts, wl.top_k)
    else:
        bias = None if inp_host["expert_bias"] is None else inp_host["expert_bias"].numpy()
        idx, w, _ = oracle.route_sigmoid_sink(logits, wl.num_experts, wl.num_sink, wl.top_k, bias,
                                              wl.route_scale, float(inp_host["global_scale"][0]))
    full_idx = np.zeros((wl.num_tokens, wl.top_k), np.int32)
    full_w = np.zeros((wl.num_tokens, wl.top_k))
    full_idx[toks] = idx
    full_w[toks] = w
    oracle.expert_ffn(inp_host["x_bits"], full_idx, full_w, inp_host["W_gu_bits"], inp_host["W_d_bits"],
                      inp_host["b_gu_bits"], inp_host["b_d_bits"], wl.gate_up_format, wl.activation, wl.alpha,
                      wl.limit, tokens=toks)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, oracle.num_threads()


def host_inputs_for_oracle(wl, seed, device):
    from mixture_experts_ffn_token_b200.workloads import bf16_bits
    inp = make_inputs(wl, seed, device=device)
    host = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    host["x_bits"] = bf16_bits(host["x"])
    host["W_gu_bits"] = bf16_bits(host["W_gu"])
    host["W_d_bits"] = bf16_bits(host["W_d"])
    host["b_gu_bits"] = bf16_bits(host["b_gu"])
    host["b_d_bits"] = bf16_bits(host["b_d"])
    return inp, host


def calibrated_sample(wl, host, seconds):
    """Smallest sample that takes about `seconds` of oracle time (>= 1 token)."""
    rate, dt, thr = oracle_sample_rate(wl, host, 1, seed=99)
    n = max(1, min(wl.num_tokens, int(rate * seconds)))
    return n, rate, thr


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    device = "cuda" if torch.cuda.is_available() else "cpu"
    _, host = host_inputs_for_oracle(wl, 0, device)
    budget = 150.0  # seconds of oracle time for the whole run
    per_step = budget / max(1, args.steps + args.warmup)
    n, _, threads = calibrated_sample(wl, host, per_step)
    for i in range(args.warmup):
        oracle_sample_rate(wl, host, n, seed=i)
    times = []
    for i in range(args.steps):
        r, dt, threads = oracle_sample_rate(wl, host, n, seed=1000 + i)
        times.append(dt)
    total = sum(times)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n} of {wl.num_tokens} tokens per step (router + expert FFN, fp64)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(wl, world):
    big = 3 * wl.num_experts * wl.hidden_dim * wl.moe_dim * 2
    return {"workload": wl.name, "num_tokens": wl.num_tokens, "hidden_dim": wl.hidden_dim,
            "num_experts": wl.num_experts, "top_k": wl.top_k, "moe_dim": wl.moe_dim, "num_sink": wl.num_sink,
            "router": wl.router, "gate_up_format": wl.gate_up_format, "activation": wl.activation,
            "has_bias": wl.has_bias, "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2 (expert weights {big / 1e9:.2f} GB)" if big > 2 * L2_BYTES
                   else "L2 flushed between timed steps (256 MiB write)")}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, wl):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    abi.load_library()
    peaks, peak_kind = load_peaks()
    cfg = abi.make_config(wl)
    inp = make_inputs(wl, seed=rank, device="cuda")
    T, H, k, S, E = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink, wl.num_experts
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    sink = torch.empty((T, S), dtype=torch.float32, device="cuda") if S > 0 else None
    stream = torch.cuda.current_stream()
    big_inputs = 3 * E * H * wl.moe_dim * 2 > 2 * L2_BYTES
    flush = None if big_inputs else torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    kw = dict(gate_up_b=inp["b_gu"], down_b=inp["b_d"], expert_bias=inp["expert_bias"],
              global_scale=inp["global_scale"], expert_indices_out=idx, expert_weights_out=w, sink_weights_out=sink)

    def step(evs=None):
        if evs is None:
            abi.moe_forward(cfg, inp["x"], inp["logits"], inp["W_gu"], inp["W_d"], out, ws, **kw)
        else:
            abi.moe_forward_timed(cfg, evs, inp["x"], inp["logits"], inp["W_gu"], inp["W_d"], out, ws, **kw)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.fill_(1)
    torch.cuda.synchronize()
    if abi.moe_device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")

    # ---------------- timed region: K steps; every step records its own stage
    # events on the launching stream, read after the region
    n_ev = abi.NUM_STAGE_EVENTS
    ev_sets = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if flush is None:
            start.record(stream)
            for i in range(args.steps):
                step(ev_sets[i])
            stop.record(stream)
            torch.cuda.synchronize()
            elapsed_ms = start.elapsed_time(stop)
        else:
            elapsed_ms = 0.0
            for i in range(args.steps):
                flush.fill_(1)
                start.record(stream)
                step(ev_sets[i])
                stop.record(stream)
                torch.cuda.synchronize()
                elapsed_ms += start.elapsed_time(stop)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    stage_ms = [sum(evs[i].elapsed_time(evs[i + 1]) for evs in ev_sets) / args.steps for i in range(n_ev - 1)]
    status = abi.moe_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the timed region")
    if dist is not None:
        t = torch.tensor([elapsed_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())
    ms_per_step = elapsed_ms / args.steps
    value = world * T / (ms_per_step / 1000.0)

    # ---------------- e2e: host buffers, H2D inputs + D2H output inside the region
    x_h = inp["x"].cpu().pin_memory()
    lg_h = inp["logits"].cpu().pin_memory()
    out_h = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(inp["x"])
    lg_d = torch.empty_like(inp["logits"])
    for _ in range(max(1, args.warmup // 2)):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        abi.moe_forward(cfg, x_d, lg_d, inp["W_gu"], inp["W_d"], out, ws, **kw)
        out_h.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        abi.moe_forward(cfg, x_d, lg_d, inp["W_gu"], inp["W_d"], out, ws, **kw)
        out_h.copy_(out, non_blocking=True)
    e_stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_stop)
    if dist is not None:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * T / (e2e_ms / args.steps / 1000.0)

    # ---------------- roofline of the dominant kernel
    names = abi.STAGE_NAMES
    flops = wl.flops()
    wbytes, used = touched_expert_bytes(wl, idx)
    gate_up_flops = 4 * T * k * H * wl.moe_dim
    down_flops = 2 * T * k * H * wl.moe_dim
    dom = max(range(len(names)), key=lambda i: stage_ms[i])
    dom_name = names[dom]
    sustained = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    if dom_name in ("gemm_gate_up", "gemm_down"):
        kflops = gate_up_flops if dom_name == "gemm_gate_up" else down_flops
        kbytes = (2 if dom_name == "gemm_gate_up" else 1) * used * H * wl.moe_dim * 2
        t_flop = kflops / (sustained * 1e12)
        t_byte = kbytes / (peaks["hbm_gbs"] * 1e9)
        if t_flop >= t_byte:
            achieved = kflops / (stage_ms[dom] / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                    "peak_kind": f"{peak_kind} bf16 sustained"}
        else:
            achieved = kbytes / (stage_ms[dom] / 1e3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "peak_kind": f"{peak_kind} hbm copy"}
    else:
        kb = workload_bytes(wl)
        achieved = kb / (stage_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_kind": f"{peak_kind} hbm copy"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom_name
    roof["traffic"] = kernel_traffic(dom_name)
    roof["kernel_ms"] = stage_ms[dom]

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; random-init expert weights N(0,0.02))",
        "config": config_block(wl, world),
        "tflops": flops / (ms_per_step / 1e3) / 1e12,
        "weight_gbs": (wbytes + workload_bytes(wl)) / (ms_per_step / 1e3) / 1e9,
        "experts_touched": used,
        "stages_ms": {n: round(v, 5) for n, v in zip(names, stage_ms)},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": x_h.numel() * 2 + lg_h.numel() * 4,
                "d2h_bytes_per_step": out_h.numel() * 2},
        "gpu_launches": 8 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def cpu_baseline(wl):
    _, host = host_inputs_for_oracle(wl, 0, "cuda")
    n, _, _ = calibrated_sample(wl, host, 15.0)
    rate, dt, threads = oracle_sample_rate(wl, host, n, seed=7)
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} of {wl.num_tokens} tokens (router + expert FFN, fp64), {dt:.1f} s"}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.config]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
