"""Named workloads and the seeded synthetic input generator.

This module holds no arithmetic of the MoE method: it only draws inputs of
the shapes and value distributions the layer is exercised on.  It is the one
module shared by the CUDA-path tests, the oracle tests and the benchmark.

Distributions (stated once here, used everywhere):
  * x ~ N(0, 1) in bf16 (round to nearest even from fp32).
  * expert weights ~ N(0, 0.02) in bf16 (the NeMo experts page's init_std).
  * projection biases ~ N(0, 0.01) in bf16 (GptOss-shaped workload).
  * router logits in fp32: N(0, sigma^2) with sigma = 0.02*sqrt(hidden) for
    the softmax workloads whose gate is a projection of x by N(0, 0.02)
    weights, sigma = 2 for the GptOss-shaped workload, N(0, 1) for the sink
    router; the decode workload draws z[t, e] = ln p_e + Gumbel(0, 1) with
    Zipf popularity p_e ~ rank^-1.2 over a seeded expert permutation, so a
    softmax top-k is sampling without replacement by popularity.
  * sink-router selection bias ~ U(-0.1, 0.1) in fp32.
Large tensors are drawn on the requested device with torch's seeded
generator for that device, in per-expert chunks.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_tokens: int          # T
    hidden_dim: int          # H
    num_experts: int         # E (routed)
    top_k: int               # k
    moe_dim: int             # D
    router: str = "softmax_topk"      # or "sigmoid_sink"
    num_sink: int = 0                 # S
    gate_up_format: str = "concatenated"   # or "interleaved"
    activation: str = "silu"          # "silu" | "swigluoai" | "gelu_tanh"
    alpha: float = 0.0
    limit: float = 0.0
    has_bias: bool = False
    logits_kind: str = "normal"       # or "zipf_gumbel"
    logits_std: float = 1.0
    zipf_s: float = 1.2
    expert_bias_range: float = 0.0    # U(-r, r) selection bias (sink router)
    route_scale: float = 1.0
    global_scale: float = 1.0
    weight_std: float = 0.02
    bias_std: float = 0.01
    # extensions (moe_forward_ex)
    num_shared: int = 0               # shared experts (gated by the sink lanes under the sink router)
    shared_dim: int = 0
    weight_first: bool = False        # apply_router_weight_first
    mask_frac: float = 0.0            # fraction of tokens masked out (token_mask)

    @property
    def extended(self) -> bool:
        return self.num_shared > 0 or self.weight_first or self.mask_frac > 0

    @property
    def rows(self) -> int:
        return self.num_tokens * self.top_k

    @property
    def logits_cols(self) -> int:
        return self.num_experts + self.num_sink

    def flops(self) -> int:
        """Algorithmic FLOPs of the grouped contractions: 2*R*H*2D + 2*R*D*H,
        plus the same for the T*Ns rows of the shared experts."""
        return 6 * self.hidden_dim * (self.rows * self.moe_dim + self.num_tokens * self.num_shared * self.shared_dim)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 8, 2, 512, logits_std=0.02 * math.sqrt(256)),
    "mixtral": Workload("mixtral", 4096, 4096, 8, 2, 14336, logits_std=0.02 * math.sqrt(4096)),
    "gptoss": Workload("gptoss", 2048, 2880, 128, 4, 2880, gate_up_format="interleaved",
                       activation="swigluoai", alpha=1.702, limit=7.0, has_bias=True, logits_std=2.0),
    "sink": Workload("sink", 8192, 2048, 128, 6, 768, router="sigmoid_sink", num_sink=2,
                     logits_std=1.0, expert_bias_range=0.1, route_scale=2.5, global_scale=1.0),
    "decode": Workload("decode", 32, 4096, 64, 8, 1536, activation="gelu_tanh",
                       logits_kind="zipf_gumbel"),
}
# The sink-router workload with its two sink lanes as gated shared experts
# (moe_dim-sized), and the Mixtral-shaped one with the router weight applied
# before the experts: the two extension rows, measured by bench.py.
WORKLOADS["sink_shared"] = WORKLOADS["sink"].replace(name="sink_shared", num_shared=2, shared_dim=768)
WORKLOADS["mixtral_wfirst"] = WORKLOADS["mixtral"].replace(name="mixtral_wfirst", weight_first=True)


def _normal(shape, std, gen, device, out_dtype=torch.bfloat16):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(out_dtype)


def make_inputs(wl: Workload, seed: int = 0, device: str | torch.device = "cpu",
                with_weights: bool = True) -> dict:
    """Draw every input of one layer call.

    Returns a dict of tensors on `device`: x [T,H] bf16, logits [T,E+S] fp32,
    W_gu [E,H,2D] bf16, W_d [E,D,H] bf16, b_gu [E,2D] / b_d [E,H] bf16 or None,
    expert_bias [E] fp32 or None, global_scale [1] fp32, token_mask [T] uint8
    or None, and with shared experts Ws_gu [Ns,H,2Ds], Ws_d [Ns,Ds,H] (and
    bs_gu / bs_d with biases).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, H, E, k, D, S = wl.num_tokens, wl.hidden_dim, wl.num_experts, wl.top_k, wl.moe_dim, wl.num_sink
    out = {}
    out["x"] = _normal((T, H), 1.0, gen, device)
    if wl.logits_kind == "normal":
        out["logits"] = _normal((T, E + S), wl.logits_std, gen, device, torch.float32)
    elif wl.logits_kind == "zipf_gumbel":
        ranks = torch.randperm(E, generator=gen, device=device).to(torch.float64) + 1.0
        p = ranks.pow(-wl.zipf_s)
        p = p / p.sum()
        u = torch.rand((T, E + S), generator=gen, device=device, dtype=torch.float64)
        u = u.clamp_(min=1e-300)
        gumbel = -torch.log(-torch.log(u))
        base = torch.zeros(E + S, dtype=torch.float64, device=device)
        base[:E] = torch.log(p)
        out["logits"] = (base + gumbel).to(torch.float32)
    else:
        raise ValueError(wl.logits_kind)
    if wl.expert_bias_range > 0:
        r = wl.expert_bias_range
        out["expert_bias"] = (torch.rand(E, generator=gen, device=device) * (2 * r) - r).to(torch.float32)
    else:
        out["expert_bias"] = None
    out["global_scale"] = torch.full((1,), wl.global_scale, dtype=torch.float32, device=device)
    if with_weights:
        W_gu = torch.empty((E, H, 2 * D), dtype=torch.bfloat16, device=device)
        W_d = torch.empty((E, D, H), dtype=torch.bfloat16, device=device)
        for e in range(E):
            W_gu[e] = _normal((H, 2 * D), wl.weight_std, gen, device)
            W_d[e] = _normal((D, H), wl.weight_std, gen, device)
        out["W_gu"], out["W_d"] = W_gu, W_d
        if wl.has_bias:
            out["b_gu"] = _normal((E, 2 * D), wl.bias_std, gen, device)
            out["b_d"] = _normal((E, H), wl.bias_std, gen, device)
        else:
            out["b_gu"] = out["b_d"] = None
        if wl.num_shared > 0:
            Ns, Ds = wl.num_shared, wl.shared_dim
            out["Ws_gu"] = _normal((Ns, H, 2 * Ds), wl.weight_std, gen, device)
            out["Ws_d"] = _normal((Ns, Ds, H), wl.weight_std, gen, device)
            if wl.has_bias:
                out["bs_gu"] = _normal((Ns, 2 * Ds), wl.bias_std, gen, device)
                out["bs_d"] = _normal((Ns, H), wl.bias_std, gen, device)
            else:
                out["bs_gu"] = out["bs_d"] = None
    if wl.mask_frac > 0:
        out["token_mask"] = (torch.rand(T, generator=gen, device=device) >= wl.mask_frac).to(torch.uint8)
    else:
        out["token_mask"] = None
    return out


def bf16_bits(t: Optional[torch.Tensor]):
    """A bf16 tensor's bit patterns as a numpy uint16 array (host copy)."""
    if t is None:
        return None
    import numpy as np
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
