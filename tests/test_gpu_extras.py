"""moe_forward_ex -- token mask, router weight before the experts, shared
experts gated by the sink lanes (or ungated) -- against the fp64 oracle on
seeded inputs; same bars as the core path."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import LayerRun, every_tile_tokens, oracle_route, run_and_check_ex, to_dev
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

MIX = WORKLOADS["mixtral"].replace(num_tokens=256, hidden_dim=512, moe_dim=384, logits_std=0.02 * math.sqrt(512))
GPT = WORKLOADS["gptoss"].replace(num_tokens=96, hidden_dim=328, num_experts=16, moe_dim=200)
SNK = WORKLOADS["sink"].replace(num_tokens=300, hidden_dim=256, num_experts=32, moe_dim=136)
DEC = WORKLOADS["decode"].replace(num_tokens=8, hidden_dim=512, num_experts=16, moe_dim=192)


@pytest.mark.parametrize("wl", [MIX, GPT, DEC, SNK.replace(num_tokens=1200)], ids=["mix", "gpt", "dec", "snk_big"])
def test_weight_first(wl):
    run_and_check_ex(wl.replace(weight_first=True), seed=1)


@pytest.mark.parametrize("wl", [MIX, SNK, SNK.replace(num_tokens=1200), WORKLOADS["tiny"]],
                         ids=["mix", "snk", "snk_big", "tiny"])
def test_token_mask(wl):
    run_and_check_ex(wl.replace(mask_frac=0.3), seed=2)


# GEMM variants (the default single launch, two launches, CTA pairs): the
# shared experts' gate_up GEMM reads x directly in each of them.
GEMM_VARIANTS = {"single_launch": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1"},
                 "two_launches": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "1"},
                 "cta_pair": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "2"},
                 "single_launch_cta_pair": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "2"},
                 # row f1 in the routed pass (the shared pass reads x directly,
                 # and a router weight applied first keeps the gather kernel)
                 "fused_gather": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1",
                                  "MOE_B200_FUSED_GATHER": "1"},
                 "fused_gather_two_launches": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "1",
                                               "MOE_B200_FUSED_GATHER": "1"}}


@pytest.mark.parametrize("variant", sorted(GEMM_VARIANTS))
@pytest.mark.parametrize("wl", [SNK.replace(num_shared=2, shared_dim=136),
                                MIX.replace(num_shared=1, shared_dim=256),
                                GPT.replace(num_shared=1, shared_dim=96),
                                SNK.replace(num_tokens=1200, num_shared=2, shared_dim=72)],
                         ids=["sink_gated", "softmax_ungated", "gpt_bias", "sink_big"])
def test_shared_experts(wl, variant, monkeypatch):
    for k, v in GEMM_VARIANTS[variant].items():
        monkeypatch.setenv(k, v)
    run_and_check_ex(wl, seed=3)


@pytest.mark.parametrize("variant", sorted(GEMM_VARIANTS))
def test_everything_together(variant, monkeypatch):
    for k, v in GEMM_VARIANTS[variant].items():
        monkeypatch.setenv(k, v)
    run_and_check_ex(SNK.replace(num_shared=2, shared_dim=136, weight_first=True, mask_frac=0.25), seed=4)
    run_and_check_ex(GPT.replace(num_shared=1, shared_dim=200, weight_first=True, mask_frac=0.5), seed=5)
    # shared experts reading x directly (no router weight first), with a mask
    run_and_check_ex(SNK.replace(num_shared=2, shared_dim=136, mask_frac=0.25), seed=6)


def test_no_extras_equals_forward():
    """moe_forward_ex with no extensions gives moe_forward's output bit for bit."""
    wl = SNK.replace(num_tokens=1200)
    d = to_dev(make_inputs(wl, 6))
    run = LayerRun(wl, d)
    out = torch.empty_like(run.out)
    sink = torch.empty_like(run.sink)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(abi.NUM_STAGE_EVENTS_EX)]
    abi.moe_forward_ex(run.cfg, None, d["x"], d["logits"], d["W_gu"], d["W_d"], out, run.ws,
                       expert_bias=d["expert_bias"], global_scale=d["global_scale"], sink_weights_out=sink,
                       events=events)
    torch.cuda.synchronize()
    assert torch.equal(out, run.out) and torch.equal(sink, run.sink)
    assert sum(events[i].elapsed_time(events[i + 1]) for i in range(abi.NUM_STAGE_EVENTS_EX - 1)) > 0


@pytest.mark.parametrize("name", ["sink_shared", "mixtral_wfirst", "sink_masked", "mixtral_masked"])
def test_extension_workloads_full_size_every_tile(name):
    """The extension workloads at full size: every token of the sink-shaped
    ones; on the Mixtral-shaped ones the tokens whose rows reach every
    128-row piece of every expert (masked tokens take no row, and the
    masked rows must be exactly zero)."""
    wl = WORKLOADS[name] if name in WORKLOADS else WORKLOADS[name.split("_")[0]].replace(mask_frac=0.3)
    sample = None
    if wl.name.startswith("mixtral"):
        inp = make_inputs(wl, 0, device="cuda")
        idx_ref, _, _ = oracle_route(wl, inp)
        mask = None if inp["token_mask"] is None else inp["token_mask"].cpu().numpy()
        sample = every_tile_tokens(idx_ref, wl.num_experts, token_mask=mask)
        if mask is not None:  # some masked tokens too
            sample = np.union1d(sample, np.flatnonzero(mask == 0)[:16])
    run_and_check_ex(wl, seed=0, device_inputs=True, sample_tokens=sample)


def test_bound_forward_equals_forward():
    """abi.BoundForward (arguments marshalled once, the C entry point run on
    every call) gives moe_forward's and moe_forward_ex's bits, call after call."""
    wl = SNK.replace(num_tokens=1200)
    d = to_dev(make_inputs(wl, 9))
    run = LayerRun(wl, d)
    out = torch.zeros_like(run.out)
    ws = torch.empty_like(run.ws)
    kw = dict(expert_bias=d["expert_bias"], global_scale=d["global_scale"])
    call = abi.BoundForward(run.cfg, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, **kw)
    for _ in range(2):
        out.zero_()
        call()
        torch.cuda.synchronize()
        assert torch.equal(out, run.out)
    wl2 = SNK.replace(num_tokens=1200, num_shared=2, shared_dim=136, mask_frac=0.25)
    d2 = to_dev(make_inputs(wl2, 10))
    ex = abi.make_extras(token_mask=d2["token_mask"], shared_gate_up_w=d2["Ws_gu"], shared_down_w=d2["Ws_d"])
    cfg2 = abi.make_config(wl2)
    ws2 = torch.empty(abi.moe_workspace_size_ex(cfg2, ex), dtype=torch.uint8, device="cuda")
    ref = torch.empty((wl2.num_tokens, wl2.hidden_dim), dtype=torch.bfloat16, device="cuda")
    abi.moe_forward_ex(cfg2, ex, d2["x"], d2["logits"], d2["W_gu"], d2["W_d"], ref, ws2,
                       expert_bias=d2["expert_bias"], global_scale=d2["global_scale"])
    got = torch.zeros_like(ref)
    abi.BoundForward(cfg2, d2["x"], d2["logits"], d2["W_gu"], d2["W_d"], got, ws2, extras=ex,
                     expert_bias=d2["expert_bias"], global_scale=d2["global_scale"])()
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
