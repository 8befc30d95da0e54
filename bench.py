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
import re
import statistics
import sys
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
# e2e: a step shorter than this on the device runs its copies on the launching
# stream (host-bound), a longer one on double-buffered copy streams
SHORT_STEP_MS = 0.1
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the B200 data-sheet figures, for context beside the measured fractions:
# dense bf16 tensor throughput and HGX HBM3e bandwidth
NOMINAL_PEAKS = {"TFLOP/s": 2250.0, "GB/s": 7700.0}


# ------------------------------------------------------------------ helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def roofline(wl, stage, kernel_ms, peaks, peak_kind, clock_summary, used_experts, region_s=0.0):
    """The dominant stage's roofline entry: its algorithmic FLOPs (GEMM
    stages) or bytes over its live time `kernel_ms`, against the peak that
    bounds it. A GEMM stage is tensor-bound when its FLOPs at the bf16 peak
    take longer than its touched experts' weight bytes at the HBM copy
    bandwidth, else HBM-bound. `frac` is taken against the burst bf16 figure
    (a timed region shorter than a second never settles at the power-capped
    clock); only a region of a second or more that NVML saw under
    `sw_power_cap` is compared with the sustained figure. `frac_sustained`
    (the achieved rate over the sustained figure) is given beside it for
    tensor-bound kernels."""
    capped = "sw_power_cap" in clock_summary.get("reasons", [])
    use_sustained = capped and region_s >= 1.0 and "bf16_tflops_sustained" in peaks
    bf16_peak = peaks["bf16_tflops_sustained"] if use_sustained else peaks["bf16_tflops"]
    bf16_kind = "sustained" if use_sustained else "burst"
    T, k, H = wl.num_tokens, wl.top_k, wl.hidden_dim
    gemm_stages = ("gemm_gate_up", "gemm_down", "shared_gemm_gate_up", "shared_gemm_down", "mega_ffn",
                   "shared_mega_ffn")
    if stage in gemm_stages:
        # FLOP / weight-byte multipliers: gate_up 4 / 2, down 2 / 1, both 6 / 3
        fm, bm = (6, 3) if stage.endswith("mega_ffn") else (4, 2) if stage.endswith("gate_up") else (2, 1)
        if stage.startswith("shared"):
            kflops = fm * T * wl.num_shared * H * wl.shared_dim
            kbytes = bm * wl.num_shared * H * wl.shared_dim * 2
        else:
            kflops = fm * T * k * H * wl.moe_dim
            kbytes = bm * used_experts * H * wl.moe_dim * 2
        t_flop = kflops / (bf16_peak * 1e12)
        t_byte = kbytes / (peaks["hbm_gbs"] * 1e9)
        if t_flop >= t_byte:
            achieved = kflops / (kernel_ms / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                    "peak_kind": f"{peak_kind} bf16 {bf16_kind}"}
            if "bf16_tflops_sustained" in peaks:
                roof["frac_sustained"] = achieved / peaks["bf16_tflops_sustained"]
        else:
            achieved = kbytes / (kernel_ms / 1e3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "peak_kind": f"{peak_kind} hbm copy"}
    else:
        achieved = workload_bytes(wl) / (kernel_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_kind": f"{peak_kind} hbm copy"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_of_nominal"] = roof["achieved"] / NOMINAL_PEAKS[roof["unit"]]
    return roof


def check_world(gpus, world):
    """--gpus N must match the number of ranks the launcher started."""
    if gpus != world:
        raise SystemExit(f"--gpus {gpus} but {world} rank(s) were started: run N > 1 GPUs as "
                         f"python -m torch.distributed.run --nproc-per-node {gpus} bench.py --gpus {gpus}")


def max_over_ranks(x, dist_mod, device):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist_mod is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def launches_per_step(wl, single_launch, csr_fused=False, fused_gather=False):
    """Kernels one call launches: the router and the CSR build (one kernel
    together when T*k <= 2048 and E <= 512; else the router plus one
    cooperative CSR kernel when `csr_fused`, or plus count, scan and
    scatter), the gather (none when the gate_up GEMM gathers its rows itself
    and the router weight does not scale them), the two grouped GEMMs (one
    launch when fused), the combine, and with shared experts their index
    kernel and GEMMs (plus their gather only when the router weight scales
    the input: otherwise their gate_up GEMM reads x directly)."""
    small = wl.num_tokens * wl.top_k <= 2048 and wl.num_experts <= 512
    gemms = 1 if single_launch else 2
    shared = (1 + (1 if wl.weight_first else 0) + gemms) if wl.num_shared > 0 else 0
    route_csr = 1 if small else (2 if csr_fused else 4)
    gather = 0 if (fused_gather and not wl.weight_first) else 1
    return route_csr + gather + gemms + shared + 1


def csr_fused_active(wl, num_sms):
    """Whether the library builds the CSR in one launch for this workload:
    its chunks of 2048 slots fit on the GPU at once (MOE_B200_CSR_FUSED=0
    turns it off)."""
    if os.environ.get("MOE_B200_CSR_FUSED", "1").startswith("0"):
        return False
    return 0 < -(-wl.num_tokens * wl.top_k // 2048) <= num_sms


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens/s: every rank runs its own batch of tokens_per_rank."""
    return world * tokens_per_rank / (ms_per_step / 1000.0)


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
    shared = wl.num_shared * 3 * wl.hidden_dim * wl.shared_dim * 2
    return used * 3 * wl.hidden_dim * wl.moe_dim * 2 + shared, used


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled every few
    milliseconds by a host thread through NVML (the counters nvidia-smi
    reads) while the timed region runs."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index, period_s=0.005):
        import threading
        self.period = period_s
        self.samples = []
        self.error = None
        self.stop_evt = threading.Event()
        self.thread = None
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            try:  # read only, to tell a lowered power limit from the usual one
                self.limit_w = pynvml.nvmlDeviceGetEnforcedPowerLimit(self.handle) / 1000.0
            except Exception:
                self.limit_w = None
            self.nvml = pynvml
        except Exception as exc:  # no NVML: report it instead of guessing
            self.error = f"nvml unavailable: {exc}"

    def _run(self):
        p = self.nvml
        while not self.stop_evt.is_set():
            try:
                mhz = p.nvmlDeviceGetClockInfo(self.handle, p.NVML_CLOCK_SM)
                mask = p.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                watts = p.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.samples.append((mhz, mask, watts))
            except Exception as exc:
                self.error = str(exc)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            import threading
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"]}
        p = self.nvml
        reasons = sorted({name for name, attr in self.REASONS for (_, mask, _) in self.samples
                          if mask & getattr(p, attr)})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml",
                # NVML's power reading is averaged over about a second, so
                # over a short timed region it stays below the limit even
                # while sw_power_cap is active
                "power_w_max": max(s[2] for s in self.samples), "power_limit_w": self.limit_w}


def kernel_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary (profiles/traffic.json), if it was captured from the kernel's
    current source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        ent = json.load(f).get(workload, {}).get(kernel)
    if not ent:
        return None
    src = os.path.join(ROOT, ent.get("source", ""))
    if not os.path.isfile(src):
        return None
    if ent.get("code_sha256_16") != code_digest(src):
        return None
    return ent.get("bytes_per_launch")


def dram_frac(traffic, kernel_ms, peaks):
    """The dominant kernel's measured DRAM traffic per launch over its live
    time, as a fraction of the measured HBM copy bandwidth. Beside a
    tensor-bound `frac` it shows how close the kernel also runs to the
    memory roof (a kernel near the ridge point needs both at once)."""
    return traffic / (kernel_ms / 1e3) / (peaks["hbm_gbs"] * 1e9)


_C_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/|\s+', re.S)


def code_digest(path):
    """sha256[:16] of a C/C++/CUDA source with its comments and whitespace
    removed (string and character literals kept): it changes when the code
    changes, not when a comment does."""
    with open(path, encoding="utf-8") as f:
        text = f.read()

    def keep(m):
        tok = m.group(0)
        if tok.startswith(("//", "/*")) or tok.isspace():
            return " "
        return tok

    code = " ".join(_C_TOKENS.sub(keep, text).split())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


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
        idx, w, sw = oracle.route_sigmoid_sink(logits, wl.num_experts, wl.num_sink, wl.top_k, bias,
                                               wl.route_scale, float(inp_host["global_scale"][0]))
    full_idx = np.zeros((wl.num_tokens, wl.top_k), np.int32)
    full_w = np.zeros((wl.num_tokens, wl.top_k))
    full_idx[toks] = idx
    full_w[toks] = w
    mask = None if inp_host.get("token_mask") is None else inp_host["token_mask"].numpy()
    oracle.expert_ffn(inp_host["x_bits"], full_idx, full_w, inp_host["W_gu_bits"], inp_host["W_d_bits"],
                      inp_host["b_gu_bits"], inp_host["b_d_bits"], wl.gate_up_format, wl.activation, wl.alpha,
                      wl.limit, tokens=toks, weight_first=wl.weight_first, token_mask=mask)
    if wl.num_shared > 0:
        gates = np.ones((wl.num_tokens, wl.num_shared))
        if wl.router == "sigmoid_sink":
            gates[toks] = sw
        oracle.shared_expert_ffn(inp_host["x_bits"], gates, bf16_bits(inp_host["Ws_gu"]), bf16_bits(inp_host["Ws_d"]),
                                 bf16_bits(inp_host.get("bs_gu")), bf16_bits(inp_host.get("bs_d")),
                                 wl.gate_up_format, wl.activation, wl.alpha, wl.limit, tokens=toks,
                                 weight_first=wl.weight_first, token_mask=mask)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, oracle.num_threads()


def host_inputs_for_oracle(wl, seed, device):
    inp = make_inputs(wl, seed, device=device)
    return inp, host_copy_for_oracle(inp)


def host_copy_for_oracle(inp):
    from mixture_experts_ffn_token_b200.workloads import bf16_bits
    host = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    host["x_bits"] = bf16_bits(host["x"])
    host["W_gu_bits"] = bf16_bits(host["W_gu"])
    host["W_d_bits"] = bf16_bits(host["W_d"])
    host["b_gu_bits"] = bf16_bits(host["b_gu"])
    host["b_d_bits"] = bf16_bits(host["b_d"])
    return host


def calibrated_sample(wl, host, seconds):
    """Grow a token sample until the oracle spends about `seconds` on it
    (the oracle parallelises over the slots of one expert, so its rate grows
    with the sample until the host cores are busy).  Returns (tokens, rate,
    elapsed, threads) of the last, largest measurement."""
    n = 1
    while True:
        rate, dt, thr = oracle_sample_rate(wl, host, n, seed=99)
        if dt >= 0.5 * seconds or n >= wl.num_tokens:
            return n, rate, dt, thr
        grow = min(8.0, max(2.0, 0.8 * seconds / max(dt, 1e-6)))
        n = min(wl.num_tokens, max(n + 1, int(n * grow)))


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    device = "cuda" if torch.cuda.is_available() else "cpu"
    _, host = host_inputs_for_oracle(wl, 0, device)
    budget = 150.0  # seconds of oracle time for the whole run
    per_step = budget / max(1, args.steps + args.warmup)
    n, _, _, threads = calibrated_sample(wl, host, per_step)
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
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"{n} of {wl.num_tokens} tokens per step (router + expert FFN, fp64)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(wl, world, graph=False):
    big = 3 * wl.num_experts * wl.hidden_dim * wl.moe_dim * 2
    return {"workload": wl.name, "launch": "cuda_graph" if graph else "eager", "num_tokens": wl.num_tokens,
            "hidden_dim": wl.hidden_dim,
            "num_experts": wl.num_experts, "top_k": wl.top_k, "moe_dim": wl.moe_dim, "num_sink": wl.num_sink,
            "router": wl.router, "gate_up_format": wl.gate_up_format, "activation": wl.activation,
            "has_bias": wl.has_bias, "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2 (expert weights {big / 1e9:.2f} GB)" if big > 2 * L2_BYTES
                   else "L2 flushed between timed steps (256 MiB write)")}


# ------------------------------------------------------------------ GPU arm
def timed_steps(step, steps, stream, flush):
    """Device time in ms of `steps` calls of step() on `stream`; with `flush`,
    the L2 is overwritten before every step, outside the timed intervals."""
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if flush is None:
        start.record(stream)
        for _ in range(steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(stop)
    total = 0.0
    for _ in range(steps):
        flush.fill_(1)
        start.record(stream)
        step()
        stop.record(stream)
        torch.cuda.synchronize()
        total += start.elapsed_time(stop)
    return total


def run_e2e(args, cfg, inp, kw, ws, stream, dist, make_ex=None, copy_streams=1, steps=None,
            device_ms_per_step=None):
    """K steps of moe_forward (moe_forward_ex when `make_ex` builds its extras
    from a device token mask) fed from, and returning to, pinned host memory.
    Each step's inputs -- x, the logits and, when there is one, the token
    mask -- sit back to back in one pinned staging buffer and cross to the
    device in one copy; its output comes back in one copy.  For a step
    shorter than SHORT_STEP_MS on the device (`device_ms_per_step`, from the
    timed region) the copies run on the launching stream around the call;
    otherwise they run on their own streams (split by bytes or rows
    over `copy_streams` streams, so that several copy engines can share
    them), double-buffered, so that step i's copies overlap the compute of
    its neighbours.  Returns (device time of the whole region in
    ms, max over ranks; host->device bytes per step)."""
    T, H = inp["x"].shape
    has_mask = inp["token_mask"] is not None
    parts = [inp["x"], inp["logits"]] + ([inp["token_mask"]] if has_mask else [])
    offs, size = [], 0
    for t in parts:
        offs.append(size)
        size += (t.numel() * t.element_size() + 255) // 256 * 256
    stage_h = torch.zeros(size, dtype=torch.uint8).pin_memory()
    for t, o in zip(parts, offs):
        nb = t.numel() * t.element_size()
        stage_h[o:o + nb].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
    stage_d = [torch.empty(size, dtype=torch.uint8, device="cuda") for _ in range(2)]

    def view(buf, i):
        t, o = parts[i], offs[i]
        return buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)

    x_d = [view(stage_d[b], 0) for b in range(2)]
    lg_d = [view(stage_d[b], 1) for b in range(2)]
    mask_d = [view(stage_d[b], 2) if has_mask else None for b in range(2)]
    ex_b = [make_ex(mask_d[b]) if make_ex is not None else None for b in range(2)]
    out_h = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    out_d = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    # the layer call for each buffer set, marshalled once (abi.BoundForward
    # still runs the whole C entry point every call)
    calls = [abi.BoundForward(cfg, x_d[b], lg_d[b], inp["W_gu"], inp["W_d"], out_d[b], ws, extras=ex_b[b],
                              stream=stream, **kw) for b in range(2)]
    n = max(1, min(copy_streams, T))
    h2d = [torch.cuda.Stream() for _ in range(n)]
    d2h = [torch.cuda.Stream() for _ in range(n)]
    bcut = [size * q // n // 256 * 256 for q in range(n)] + [size]  # byte ranges of the split input copy
    cut = [T * q // n for q in range(n + 1)]                         # row ranges of the split output copy

    def region_in_stream(steps):
        # small transfers: copy in, compute and copy out on the launching
        # stream, one step after another (no cross-stream events to wait on)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(steps):
            b = i % 2
            stage_d[b].copy_(stage_h, non_blocking=True)
            calls[b]()
            out_h[b].copy_(out_d[b], non_blocking=True)
        stop.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(stop)

    def region(steps):
        in_ready = [[torch.cuda.Event() for _ in range(n)] for _ in range(steps)]
        fwd_done = [torch.cuda.Event() for _ in range(steps)]
        out_done = [[torch.cuda.Event() for _ in range(n)] for _ in range(steps)]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for st in h2d + d2h:
            st.wait_event(start)
        for i in range(steps):
            b = i % 2
            for q, st in enumerate(h2d):
                lo, hi = bcut[q], bcut[q + 1]
                with torch.cuda.stream(st):
                    if i >= 2:
                        st.wait_event(fwd_done[i - 2])      # buffer b no longer read by step i-2
                    stage_d[b][lo:hi].copy_(stage_h[lo:hi], non_blocking=True)
                    in_ready[i][q].record(st)
            for ev in in_ready[i]:
                stream.wait_event(ev)
            if i >= 2:
                for ev in out_done[i - 2]:
                    stream.wait_event(ev)                   # out_d[b] copied out by step i-2
            calls[b]()
            fwd_done[i].record(stream)
            for q, st in enumerate(d2h):
                lo, hi = cut[q], cut[q + 1]
                with torch.cuda.stream(st):
                    st.wait_event(fwd_done[i])
                    out_h[b][lo:hi].copy_(out_d[b][lo:hi], non_blocking=True)
                    out_done[i][q].record(st)
        for i in range(max(0, steps - 2), steps):
            for ev in out_done[i]:
                stream.wait_event(ev)
        stop.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(stop)

    steps = args.steps if steps is None else steps
    # a step shorter on the device than SHORT_STEP_MS (tiny) is bound by the
    # host's work per step, which the cross-stream events of the overlapped
    # form add to: its copies run on the launching stream; longer steps
    # overlap their copies with the neighbouring steps' compute
    in_stream = (device_ms_per_step is not None and device_ms_per_step < SHORT_STEP_MS and copy_streams == 1)
    run = region_in_stream if in_stream else region
    with torch.cuda.stream(stream):
        run(max(2, args.warmup))
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        ms = run(steps)
    if not torch.equal(out_h[(steps - 1) % 2], out_d[(steps - 1) % 2].cpu()):
        raise RuntimeError("e2e: host copy of the output differs from the device result")
    return max_over_ranks(ms, dist, "cuda"), size


def host_enqueue_us(step, calls, stream):
    """Host microseconds per eager call of step(): the time the calling
    thread spends in `calls` back-to-back calls (the Python binding, the
    library's argument checks, tensor-map encoding and kernel launches).
    Nothing in a call waits for the GPU; the device work is synchronized
    afterwards, outside the timed interval."""
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(calls):
        step()
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    return (t1 - t0) * 1e6 / calls


def measure(args, wl, ctx, steps):
    """Every figure of one workload's bench line (without cpu_baseline):
    warm-up, the stage region, the graph-timed region with the dominant
    kernel's live events, the e2e region and the host enqueue cost.
    Returns (line, inputs)."""
    world, rank, local, dist = ctx["world"], ctx["rank"], ctx["local"], ctx["dist"]
    peaks, peak_kind = ctx["peaks"], ctx["peak_kind"]
    cfg = abi.make_config(wl)
    inp = make_inputs(wl, seed=rank, device="cuda")
    T, H, k, S, E = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink, wl.num_experts
    extras = make_ex = None
    if wl.extended:
        def make_ex(mask):
            return abi.make_extras(token_mask=mask, apply_router_weight_first=wl.weight_first,
                                   shared_gate_up_w=inp.get("Ws_gu"), shared_down_w=inp.get("Ws_d"),
                                   shared_gate_up_b=inp.get("bs_gu"), shared_down_b=inp.get("bs_d"))
        extras = make_ex(inp["token_mask"])
        ws_bytes = abi.moe_workspace_size_ex(cfg, extras)
    else:
        ws_bytes = abi.moe_workspace_size(cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
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
        if extras is not None:
            abi.moe_forward_ex(cfg, extras, inp["x"], inp["logits"], inp["W_gu"], inp["W_d"], out, ws, events=evs,
                               **kw)
        elif evs is None:
            abi.moe_forward(cfg, inp["x"], inp["logits"], inp["W_gu"], inp["W_d"], out, ws, **kw)
        else:
            abi.moe_forward_timed(cfg, evs, inp["x"], inp["logits"], inp["W_gu"], inp["W_d"], out, ws, **kw)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.fill_(1)
    torch.cuda.synchronize()
    if abi.moe_device_status(ws) != 0:
        raise RuntimeError(f"{wl.name}: device status set during warm-up")

    # ---------------- stage region: K eager steps through moe_forward_timed,
    # each recording its own events between all stages (a timing event
    # between two kernels stops them overlapping, so these per-stage times are
    # a breakdown, not the step time); it picks the dominant stage
    names = list(abi.STAGE_NAMES_EX if extras is not None else abi.STAGE_NAMES)
    n_ev = len(names) + 1
    ev_sets = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    for evs in ev_sets:          # create the CUDA events outside the region
        for ev in evs:
            ev.record(stream)
    torch.cuda.synchronize()
    it = iter(ev_sets)
    timed_steps(lambda: step(next(it)), steps, stream, flush)
    stage_ms = [sum(evs[i].elapsed_time(evs[i + 1]) for evs in ev_sets) / steps for i in range(n_ev - 1)]
    dom = max(range(len(names)), key=lambda i: stage_ms[i])
    if abi.moe_device_status(ws) != 0:
        raise RuntimeError(f"{wl.name}: device status set during the stage region")

    # ---------------- timed region: K steps between two CUDA events on the
    # launching stream (max over ranks); L2 flushed between steps when the
    # inputs would fit in it.  With --graph (default) the K steps are captured
    # in one CUDA graph and replayed, which takes the host's launch work off
    # the timeline; the kernels are the same.  Every 10th step (the last one
    # if K < 10) also records a pair of events around the dominant stage:
    # that kernel's live duration for roofline.achieved, taken in the same
    # region (and thermal state) as the step time, from few enough steps that
    # the events barely touch it.
    def ext_event():  # recorded as an event node when captured in a graph
        return torch.cuda.Event(enable_timing=True, external=True)

    pair_steps = [i for i in range(steps) if i % 10 == 9] or [steps - 1]
    pairs = {i: (ext_event(), ext_event()) for i in pair_steps}
    marks = [(ext_event(), ext_event()) for _ in range(steps)]
    for a, b in list(pairs.values()) + marks:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()

    def step_events(i):
        if i not in pairs:
            return None
        evs = [None] * n_ev
        evs[dom], evs[dom + 1] = pairs[i]
        return evs

    def body():
        for i in range(steps):
            if flush is not None:
                flush.fill_(1)
                marks[i][0].record()
            step(step_events(i))
            if flush is not None:
                marks[i][1].record()

    run = body
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            body()
        graph.replay()           # untimed warm replay
        torch.cuda.synchronize()
        if abi.moe_device_status(ws) != 0:
            raise RuntimeError(f"{wl.name}: device status set by the captured steps")
        run = graph.replay
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record(stream)
        run()
        stop.record(stream)
        torch.cuda.synchronize()
    region_ms = start.elapsed_time(stop)
    if flush is None:
        elapsed_ms = region_ms
    else:
        elapsed_ms = sum(a.elapsed_time(b) for a, b in marks)
    kernel_ms = sum(a.elapsed_time(b) for a, b in pairs.values()) / len(pairs)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    status = abi.moe_device_status(ws)
    if status != 0:
        raise RuntimeError(f"{wl.name}: device status {status:#x} after the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dist, "cuda")
    ms_per_step = elapsed_ms / steps
    value = job_throughput(world, T, ms_per_step)
    del graph

    # ---------------- e2e: host buffers; every step copies its inputs host->device
    # from pinned memory and its output device->host inside the timed region.
    # Copies run on their own streams, double-buffered, so step i's copies
    # overlap the compute of its neighbours.
    e2e_ms, x_h_bytes = run_e2e(args, cfg, inp, kw, ws, stream, dist, make_ex, copy_streams=args.copy_streams,
                                steps=steps, device_ms_per_step=ms_per_step)
    e2e_value = job_throughput(world, T, e2e_ms / steps)
    out_bytes = T * H * 2

    # ---------------- host cost of one eager call (the public Python entry
    # point and the library's enqueue work, no GPU wait), and of the
    # library's C entry point alone (arguments marshalled once beforehand)
    host_us = host_enqueue_us(step, min(steps, 20), stream)
    host_lib_us = None
    if extras is None:
        import ctypes
        lib = abi.load_library()
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        c_args = (ctypes.byref(cfg), p(inp["x"]), p(inp["logits"]), p(inp["expert_bias"]), p(inp["global_scale"]),
                p(inp["W_gu"]), p(inp["b_gu"]), p(inp["W_d"]), p(inp["b_d"]), p(out), p(idx), p(w), p(sink),
                p(ws), ws.numel(), stream.cuda_stream)
        fwd = lib.moe_forward

        def c_step():
            if fwd(*c_args) != 0:
                raise RuntimeError("moe_forward failed")
        host_lib_us = host_enqueue_us(c_step, min(steps, 20), stream)

    # ---------------- roofline of the dominant kernel, timed live by its event
    # pair in the timed region
    fused = abi.moe_single_launch_ffn()
    if fused:
        # the "gate_up" stage is the single launch of both GEMMs; "down" is empty
        names = [{"gemm_gate_up": "mega_ffn", "gemm_down": "(fused)", "shared_gemm_gate_up": "shared_mega_ffn",
                  "shared_gemm_down": "(shared fused)"}.get(n, n) for n in names]
    csr_fused = csr_fused_active(wl, torch.cuda.get_device_properties(local).multi_processor_count)
    small = wl.num_tokens * wl.top_k <= 2048 and wl.num_experts <= 512
    if small:
        # routing and the CSR build are one kernel, timed as the router stage
        names = [{"router": "route_csr_small", "csr_count": "(csr in route)", "csr_scan": "(csr scan in route)",
                  "csr_scatter": "(csr scatter in route)"}.get(n, n) for n in names]
    elif csr_fused:
        # the one-launch CSR build is timed as the first CSR stage
        names = [{"csr_count": "csr_build", "csr_scan": "(csr scan in build)",
                  "csr_scatter": "(csr scatter in build)"}.get(n, n) for n in names]
    flops = wl.flops()
    wbytes, used = touched_expert_bytes(wl, idx)
    fused_gather = os.environ.get("MOE_B200_FUSED_GATHER", "0").startswith("1")
    dom_name = names[dom]
    clock_summary = clocks.summary()
    roof = roofline(wl, dom_name, kernel_ms, peaks, peak_kind, clock_summary, used, region_s=region_ms / 1e3)
    roof["kernel"] = dom_name
    roof["traffic"] = kernel_traffic(wl.name, dom_name)
    if roof["traffic"] is not None:
        roof["dram_frac"] = dram_frac(roof["traffic"], kernel_ms, peaks)
    roof["kernel_ms"] = kernel_ms                # live, in the timed region
    roof["kernel_ms_stage_region"] = stage_ms[dom]

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; random-init expert weights N(0,0.02))",
        "config": config_block(wl, world, graph=args.graph),
        "tflops": flops / (ms_per_step / 1e3) / 1e12,
        "weight_gbs": (wbytes + workload_bytes(wl)) / (ms_per_step / 1e3) / 1e9,
        "experts_touched": used,
        "stages_ms": {n: round(v, 5) for n, v in zip(names, stage_ms)},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": x_h_bytes,
                "d2h_bytes_per_step": out_bytes},
        "host_us_per_call": host_us,
        "host_us_per_call_c_abi": host_lib_us,
        "gpu_launches": launches_per_step(wl, fused, csr_fused, fused_gather) * steps,
        "single_launch_ffn": fused,
        "clocks": clock_summary,
    }
    return line, inp


# the other workloads of the per-config object, measured after the headline one
PER_CONFIG = ("tiny", "gptoss", "sink", "decode")


def per_config_enabled(flag, world):
    """--per-config / --no-per-config, else on with one GPU only (with
    several GPUs every rank would hold its GPU through four more workloads)."""
    return flag if flag is not None else world == 1


def compact(line):
    """The per-config entry: the figures of a full line that describe one workload."""
    keep = ("value", "unit", "ms_per_step", "steps", "tflops", "weight_gbs", "experts_touched", "roofline", "e2e",
            "host_us_per_call", "host_us_per_call_c_abi", "gpu_launches", "clocks", "stages_ms")
    ent = {k: line[k] for k in keep}
    ent["workload"] = line["config"]["workload"]
    ent["l2"] = line["config"]["l2"]
    return ent


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
    ctx = {"world": world, "rank": rank, "local": local, "dist": dist, "peaks": peaks, "peak_kind": peak_kind}
    line, inp = measure(args, wl, ctx, args.steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, inp)
    del inp
    if per_config_enabled(args.per_config, world):
        line["per_config"] = {}
        for name in PER_CONFIG:
            if name == wl.name:
                continue
            torch.cuda.empty_cache()
            sub, sub_inp = measure(args, WORKLOADS[name], ctx, args.steps)
            del sub_inp
            line["per_config"][name] = compact(sub)
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def apply_overrides(wl, items):
    """The workload with each FIELD=VALUE of `items` applied (converted to the
    field's type) and its name extended by them, so that a changed workload
    never picks up figures recorded for the named one."""
    if not items:
        return wl
    kw = {}
    for item in items:
        field, sep, value = item.partition("=")
        if not sep or field == "name" or not hasattr(wl, field):
            raise SystemExit(f"--override: not a workload field assignment: {item!r}")
        cur = getattr(wl, field)
        if isinstance(cur, bool):
            kw[field] = value.lower() in ("1", "true", "yes")
        else:
            kw[field] = type(cur)(value)
    return wl.replace(name=wl.name + "+" + ",".join(items), **kw)


def cpu_model():
    """The host CPU's model name (Linux), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(wl, inp):
    host = host_copy_for_oracle(inp)
    n, rate, dt, threads = calibrated_sample(wl, host, 15.0)
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{n} of {wl.num_tokens} tokens (router + expert FFN, fp64), {dt:.1f} s"}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copy-streams", type=int, default=1,
                    help="streams per direction that share each e2e step's host<->device copies")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="time replays of a CUDA graph of one step (default) or eager calls")
    ap.add_argument("--per-config", action=argparse.BooleanOptionalAction, default=None,
                    help="also measure tiny, gptoss, sink and decode into the line's per_config object "
                         "(default: on with one GPU, off with several)")
    ap.add_argument("--override", action="append", default=[], metavar="FIELD=VALUE",
                    help="change one field of the named workload (repeatable), e.g. moe_dim=7168; "
                         "the line's workload name records every override")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = apply_overrides(WORKLOADS[args.config], args.override)
    check_world(args.gpus, dist_env()[0])
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
