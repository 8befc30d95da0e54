"""Shared pieces of the GPU parity tests: run the CUDA path through the C ABI
and compute the matching fp64 oracle result on the same seeded inputs."""
import numpy as np
import torch

import oracle
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import bf16_bits, make_inputs

# Tolerances, stated once.  Routing and indexing are compared bit-exactly.
FFN_TOL = 2e-2      # max |gpu - ref| <= FFN_TOL * max |ref|  (bf16 output, fp32 accumulation)
WEIGHT_RTOL = 1e-5  # router weights (fp32) relative to the fp64 oracle
WEIGHT_ATOL = 1e-30


def every_tile_tokens(idx, num_experts, piece=128, token_mask=None):
    """Token ids whose routed rows reach every tile of the grouped GEMMs.

    A tile is (expert, row piece of `piece` permuted rows, output column
    block), and a token's output row reads every column block of the pieces
    its slots sit in, so one compared row per piece compares every tile of
    both contractions.  Taken per expert segment of the CSR (slots sorted by
    expert, stable; masked tokens' slots take no place): the first and last
    row of every piece, and every row of the segment's last, ragged piece.
    Pieces of 128 rows also cover the 256-row pieces of the CTA-pair
    variant (each holds two of them)."""
    idx = np.asarray(idx)
    k = idx.shape[1]
    flat = idx.reshape(-1)
    slots = np.arange(flat.size)
    if token_mask is not None:
        slots = slots[np.asarray(token_mask)[slots // k] != 0]
    order = slots[np.argsort(flat[slots], kind="stable")]
    off = np.concatenate([[0], np.cumsum(np.bincount(flat[slots], minlength=num_experts))])
    rows = []
    for e in range(num_experts):
        lo, hi = int(off[e]), int(off[e + 1])
        for p0 in range(lo, hi, piece):
            p1 = min(p0 + piece, hi)
            rows += [p0, p1 - 1]
            if p1 == hi:
                rows += list(range(p0, p1))
    return np.unique(order[np.asarray(rows, dtype=np.int64)] // k)


def to_dev(inp, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def oracle_route(wl, inp):
    logits = inp["logits"].cpu().numpy()
    if wl.router == "softmax_topk":
        idx, w = oracle.route_softmax_topk(logits, wl.num_experts, wl.top_k)
        return idx, w, np.zeros((idx.shape[0], 0))
    bias = None if inp["expert_bias"] is None else inp["expert_bias"].cpu().numpy()
    return oracle.route_sigmoid_sink(logits, wl.num_experts, wl.num_sink, wl.top_k, bias, wl.route_scale,
                                     float(inp["global_scale"][0]))


def oracle_ffn(wl, inp, idx, w, tokens=None):
    return oracle.expert_ffn(bf16_bits(inp["x"]), idx, w, bf16_bits(inp["W_gu"]), bf16_bits(inp["W_d"]),
                             bf16_bits(inp["b_gu"]), bf16_bits(inp["b_d"]), wl.gate_up_format, wl.activation,
                             wl.alpha, wl.limit, tokens=tokens)


class LayerRun:
    """One moe_forward call with every output kept for comparison."""

    def __init__(self, wl, d, out_guard=0):
        T, H, k, S = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink
        self.cfg = abi.make_config(wl)
        self.ws = torch.empty(abi.moe_workspace_size(self.cfg), dtype=torch.uint8, device="cuda")
        self.out_full = torch.full((T * H + out_guard,), -7.0, dtype=torch.bfloat16, device="cuda")
        self.out = self.out_full[:T * H].view(T, H)
        self.idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        self.w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
        self.sink = torch.full((T, S), -1.0, dtype=torch.float32, device="cuda") if S > 0 else None
        abi.moe_forward(self.cfg, d["x"], d["logits"], d["W_gu"], d["W_d"], self.out, self.ws, gate_up_b=d["b_gu"],
                        down_b=d["b_d"], expert_bias=d["expert_bias"], global_scale=d["global_scale"],
                        expert_indices_out=self.idx, expert_weights_out=self.w, sink_weights_out=self.sink)
        torch.cuda.synchronize()
        self.status = abi.moe_device_status(self.ws)


def ffn_error(got, ref):
    """max |got - ref| / max |ref|."""
    got = np.asarray(got, dtype=np.float64)
    scale = np.abs(ref).max()
    return float(np.abs(got - ref).max() / max(scale, 1e-30))


def check_weights(got, ref):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    assert (err <= WEIGHT_RTOL * np.abs(ref) + WEIGHT_ATOL).all(), float((err / np.maximum(np.abs(ref), 1e-30)).max())


def run_and_check(wl, seed=0, device_inputs=False, sample_tokens=None, out_guard=64):
    """moe_forward against the oracle: routing bit-exact, weights 1e-5, output FFN_TOL."""
    inp = make_inputs(wl, seed, device="cuda" if device_inputs else "cpu")
    d = to_dev(inp)
    run = LayerRun(wl, d, out_guard=out_guard)
    assert run.status == 0, f"device status {run.status:#x}"
    idx_ref, w_ref, s_ref = oracle_route(wl, inp)
    idx = run.idx.cpu().numpy()
    assert np.array_equal(idx, idx_ref), f"{int((idx != idx_ref).sum())} routing mismatches"
    check_weights(run.w.cpu().numpy(), w_ref)
    if wl.num_sink > 0:
        check_weights(run.sink.cpu().numpy(), s_ref)
    tokens = None if sample_tokens is None else np.asarray(sample_tokens, dtype=np.int64)
    ref = oracle_ffn(wl, inp, idx_ref, w_ref, tokens)
    got = run.out.float().cpu().numpy()
    if tokens is not None:
        got = got[tokens]
    err = ffn_error(got, ref)
    assert err <= FFN_TOL, f"ffn error {err:.3e} > {FFN_TOL}"
    if out_guard:
        guard = run.out_full[wl.num_tokens * wl.hidden_dim:].float()
        assert (guard == -7.0).all(), "output guard overwritten"
    return run, err


def run_and_check_ex(wl, seed=0, device_inputs=False, sample_tokens=None):
    """moe_forward_ex (mask / weight first / shared experts) against the oracle."""
    inp = make_inputs(wl, seed, device="cuda" if device_inputs else "cpu")
    d = to_dev(inp)
    T, H, k, S = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink
    ex = abi.make_extras(token_mask=d["token_mask"], apply_router_weight_first=wl.weight_first,
                         shared_gate_up_w=d.get("Ws_gu"), shared_down_w=d.get("Ws_d"),
                         shared_gate_up_b=d.get("bs_gu"), shared_down_b=d.get("bs_d"))
    cfg = abi.make_config(wl)
    ws = torch.empty(abi.moe_workspace_size_ex(cfg, ex), dtype=torch.uint8, device="cuda")
    out = torch.full((T, H), -7.0, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    sink = torch.empty((T, S), dtype=torch.float32, device="cuda") if S > 0 else None
    abi.moe_forward_ex(cfg, ex, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, gate_up_b=d["b_gu"],
                       down_b=d["b_d"], expert_bias=d["expert_bias"], global_scale=d["global_scale"],
                       expert_indices_out=idx, expert_weights_out=w, sink_weights_out=sink)
    torch.cuda.synchronize()
    assert abi.moe_device_status(ws) == 0
    idx_ref, w_ref, s_ref = oracle_route(wl, inp)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_weights(w.cpu().numpy(), w_ref)
    tokens = None if sample_tokens is None else np.asarray(sample_tokens, dtype=np.int64)
    mask = None if inp["token_mask"] is None else inp["token_mask"].cpu().numpy()
    ref = oracle.expert_ffn(bf16_bits(inp["x"]), idx_ref, w_ref, bf16_bits(inp["W_gu"]), bf16_bits(inp["W_d"]),
                            bf16_bits(inp["b_gu"]), bf16_bits(inp["b_d"]), wl.gate_up_format, wl.activation,
                            wl.alpha, wl.limit, tokens=tokens, weight_first=wl.weight_first, token_mask=mask)
    if wl.num_shared > 0:
        gates = s_ref if wl.router == "sigmoid_sink" else np.ones((T, wl.num_shared))
        ref = ref + oracle.shared_expert_ffn(bf16_bits(inp["x"]), gates, bf16_bits(inp["Ws_gu"]),
                                             bf16_bits(inp["Ws_d"]), bf16_bits(inp.get("bs_gu")),
                                             bf16_bits(inp.get("bs_d")), wl.gate_up_format, wl.activation,
                                             wl.alpha, wl.limit, tokens=tokens, weight_first=wl.weight_first,
                                             token_mask=mask)
    got = out.float().cpu().numpy()
    if tokens is not None:
        got = got[tokens]
    err = ffn_error(got, ref)
    assert err <= FFN_TOL, f"ffn error {err:.3e} > {FFN_TOL}"
    if mask is not None:
        masked = (mask == 0) if tokens is None else (mask[tokens] == 0)
        assert (got[masked] == 0).all(), "masked tokens must give zero rows"
    return err
