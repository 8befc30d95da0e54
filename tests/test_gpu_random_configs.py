"""A seeded sweep of random small layer configurations (tests/random_configs.py)
through moe_forward / moe_forward_ex against the fp64 oracle, cycling the
launch forms: single launch in static and dynamic tile order, two launches,
CTA pairs in both, four-box B copies, and the gate_up GEMM gathering its
own rows (row f1) in one and in two launches. Same bars as every parity test:
routing bit-exact, router weights 1e-5 relative, output 2e-2 * max|ref|."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (FFN_TOL, LayerRun, check_weights, every_tile_tokens, ffn_error, oracle_ffn, oracle_route,
                         run_and_check, run_and_check_ex, to_dev)
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import make_inputs
from random_configs import NUM_CASES, NUM_MIDSIZE, random_midsize_workload, random_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("i", range(NUM_CASES))
def test_random_config(i, monkeypatch):
    wl, form = random_workload(i)
    for key, value in form.items():
        monkeypatch.setenv(key, value)
    if wl.extended:
        run_and_check_ex(wl, seed=i)
    else:
        run_and_check(wl, seed=i)


@pytest.mark.parametrize("i", range(0, NUM_CASES, 4))
def test_random_config_stages(i, monkeypatch):
    """The staged entry points on every fourth draw (without the extensions,
    which only moe_forward_ex takes): moe_route -> moe_create_indices (with
    the inverse) -> moe_grouped_ffn give moe_forward's routing and output bit
    for bit, and the CSR is the oracle's counting sort."""
    wl, form = random_workload(i)
    wl = wl.replace(mask_frac=0.0, weight_first=False, num_shared=0, shared_dim=0)
    for key, value in form.items():
        monkeypatch.setenv(key, value)
    inp = make_inputs(wl, seed=i)
    d = to_dev(inp)
    run = LayerRun(wl, d)
    assert run.status == 0
    T, k, E, S = wl.num_tokens, wl.top_k, wl.num_experts, wl.num_sink
    cfg = run.cfg
    ws = torch.empty_like(run.ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    sink = torch.empty((T, S), dtype=torch.float32, device="cuda") if S > 0 else None
    abi.moe_route(cfg, d["logits"], idx, w, sink_weights=sink, expert_bias=d["expert_bias"],
                  global_scale=d["global_scale"])
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    abi.moe_create_indices(cfg, idx, off, perm, inv, ws)
    out = torch.empty((T, wl.hidden_dim), dtype=torch.bfloat16, device="cuda")
    abi.moe_grouped_ffn(cfg, d["x"], d["W_gu"], d["b_gu"], d["W_d"], d["b_d"], off, perm, w, out, ws)
    torch.cuda.synchronize()
    assert abi.moe_device_status(ws) == 0
    assert torch.equal(idx, run.idx) and torch.equal(w, run.w)
    if S > 0:
        assert torch.equal(sink, run.sink)
    _, o_ref, p_ref, i_ref = oracle.create_indices(idx.cpu().numpy(), E)
    assert np.array_equal(off.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)
    assert np.array_equal(inv.cpu().numpy(), i_ref)
    assert torch.equal(out, run.out)


@pytest.mark.parametrize("i", range(NUM_MIDSIZE))
def test_random_midsize_every_tile(i, monkeypatch):
    """Mid-size random draws, the layer output compared on the tokens whose
    rows reach every 128-row piece of every expert (so every tile of both
    contractions has rows compared), routing on every token."""
    wl, form = random_midsize_workload(i)
    for key, value in form.items():
        monkeypatch.setenv(key, value)
    inp = make_inputs(wl, seed=i)
    idx_ref, _, _ = oracle_route(wl, inp)
    tokens = every_tile_tokens(idx_ref, wl.num_experts)
    run_and_check(wl, seed=i, sample_tokens=tokens)


@pytest.mark.parametrize("i", range(2, NUM_CASES, 4))
def test_random_config_bf16_wide_logits(i, monkeypatch):
    """moe_forward on every fourth draw (offset 2, no extensions) with bf16
    logits in rows wider than E + S, the extra columns NaN: routing bit-exact
    against the oracle reading the same bf16 bits, the output at the usual
    bar."""
    wl, form = random_workload(i)
    wl = wl.replace(mask_frac=0.0, weight_first=False, num_shared=0, shared_dim=0)
    for key, value in form.items():
        monkeypatch.setenv(key, value)
    inp = make_inputs(wl, seed=i)
    T, C = inp["logits"].shape
    pad = 1 + i % 9
    wide = torch.full((T, C + pad), float("nan")).to(torch.bfloat16)
    wide[:, :C] = inp["logits"].to(torch.bfloat16)
    cfg = abi.make_config(wl, logits_dtype=torch.bfloat16, logits_row_stride=C + pad)
    d = to_dev(inp)
    k, S = wl.top_k, wl.num_sink
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, wl.hidden_dim), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    sink = torch.empty((T, S), dtype=torch.float32, device="cuda") if S > 0 else None
    abi.moe_forward(cfg, d["x"], wide.cuda(), d["W_gu"], d["W_d"], out, ws, gate_up_b=d["b_gu"], down_b=d["b_d"],
                    expert_bias=d["expert_bias"], global_scale=d["global_scale"], expert_indices_out=idx,
                    expert_weights_out=w, sink_weights_out=sink)
    torch.cuda.synchronize()
    assert abi.moe_device_status(ws) == 0
    bits = wide.view(torch.int16).numpy().view(np.uint16)
    if wl.router == "softmax_topk":
        i_ref, w_ref = oracle.route_softmax_topk(bits, wl.num_experts, k)
        s_ref = None
    else:
        bias = None if inp["expert_bias"] is None else inp["expert_bias"].numpy()
        i_ref, w_ref, s_ref = oracle.route_sigmoid_sink(bits, wl.num_experts, S, k, bias, wl.route_scale,
                                                        float(inp["global_scale"][0]))
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    check_weights(w.cpu().numpy(), w_ref)
    if S > 0:
        check_weights(sink.cpu().numpy(), s_ref)
    ref = oracle_ffn(wl, inp, i_ref, w_ref)
    err = ffn_error(out.float().cpu().numpy(), ref)
    assert err <= FFN_TOL, f"ffn error {err:.3e} > {FFN_TOL}"
