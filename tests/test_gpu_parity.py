"""CUDA path against the fp64 oracle, element by element, on seeded inputs.

Bars (stated in gpu_helpers): expert indices, CSR offsets and permutation
bit-exact; router weights within 1e-5 relative; layer output within
2e-2 * max|ref| (bf16 output, fp32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (FFN_TOL, LayerRun, check_weights, every_tile_tokens, ffn_error, oracle_ffn, oracle_route,
                         run_and_check, to_dev)
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# Scaled-down versions of every named workload: several tiles in M and N,
# ragged row pieces, K and N tails (hidden 328 and moe_dim 200/136 are not
# multiples of the 64/128/256 tile edges).
SMALL = {
    "tiny": WORKLOADS["tiny"],
    "mixtral_small": WORKLOADS["mixtral"].replace(num_tokens=256, hidden_dim=512, moe_dim=384,
                                                   logits_std=0.02 * math.sqrt(512)),
    "gptoss_small": WORKLOADS["gptoss"].replace(num_tokens=96, hidden_dim=328, num_experts=16, moe_dim=200),
    "sink_small": WORKLOADS["sink"].replace(num_tokens=300, hidden_dim=256, num_experts=32, moe_dim=136),
    "decode_small": WORKLOADS["decode"].replace(num_tokens=8, hidden_dim=512, num_experts=16, moe_dim=192),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_small(name):
    run_and_check(SMALL[name], seed=0)


# GEMM variants: both contractions in one cooperative launch (default), two
# launches of one CTA per 128x256 tile, or two launches of a CTA pair per
# 256x256 tile (tcgen05 cta_group::2); B stage tiles in one copy (default
# where the column count allows) or in four 64-column copies; the single
# launch's tiles in static or dynamic (atomic counter) order.
VARIANTS = {"single_launch": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1", "MOE_B200_B_ONE_BOX": "1",
                              "MOE_B200_TILE_SCHEDULE": "static"},
            "single_launch_dynamic": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1",
                                      "MOE_B200_B_ONE_BOX": "1", "MOE_B200_TILE_SCHEDULE": "dynamic"},
            "single_launch_four_box": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1",
                                       "MOE_B200_B_ONE_BOX": "0"},
            "two_launches": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "1", "MOE_B200_B_ONE_BOX": "1"},
            "two_launches_cta_pair": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "2"},
            "single_launch_cta_pair": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "2",
                                       "MOE_B200_B_ONE_BOX": "1"},
            "single_launch_cta_pair_four_box": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "2",
                                                "MOE_B200_B_ONE_BOX": "0"},
            # row f1: the gate_up GEMM gathers its rows of x itself (tile::gather4)
            "single_launch_fused_gather": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1",
                                           "MOE_B200_B_ONE_BOX": "1", "MOE_B200_FUSED_GATHER": "1"},
            "single_launch_fused_gather_dynamic": {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "1",
                                                   "MOE_B200_FUSED_GATHER": "1", "MOE_B200_TILE_SCHEDULE": "dynamic"},
            "two_launches_fused_gather_four_box": {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "1",
                                                   "MOE_B200_B_ONE_BOX": "0", "MOE_B200_FUSED_GATHER": "1"}}


def set_variant(monkeypatch, variant):
    for k, v in VARIANTS[variant].items():
        monkeypatch.setenv(k, v)


@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_small_each_gemm_variant(name, variant, monkeypatch):
    set_variant(monkeypatch, variant)
    assert abi.moe_single_launch_ffn() == variant.startswith("single_launch")
    run_and_check(SMALL[name], seed=1)


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_forward_mixtral_shape_each_gemm_variant(variant, monkeypatch):
    set_variant(monkeypatch, variant)
    wl = WORKLOADS["mixtral"].replace(num_tokens=1024, hidden_dim=1024, moe_dim=1536,
                                      logits_std=0.02 * math.sqrt(1024))
    run_and_check(wl, seed=2)


# column counts that are multiples of 64 (one-copy B tiles) in every layout
ALIGNED = {
    "concat_silu": WORKLOADS["sink"].replace(num_tokens=2000, hidden_dim=512, moe_dim=256),
    "interleaved_bias": WORKLOADS["gptoss"].replace(num_tokens=160, hidden_dim=384, num_experts=16, moe_dim=160),
    "concat_gelu_ragged_k": WORKLOADS["decode"].replace(num_tokens=24, hidden_dim=328, num_experts=16, moe_dim=192),
}


@pytest.mark.parametrize("name", sorted(SMALL) + sorted(ALIGNED))
def test_single_launch_equals_two_launches(name, monkeypatch):
    """The single launch does the same tiles, MMAs and epilogues as the two
    launches, only scheduled differently (statically or from a tile counter);
    a one-copy B stage tile has the same
    shared-memory image as four 64-column copies: every variant's output is
    identical bit for bit."""
    wl = SMALL.get(name) or ALIGNED[name]
    d = to_dev(make_inputs(wl, 11))
    outs = []
    for single, one_box, order in (("1", "1", "static"), ("1", "1", "dynamic"), ("0", "1", "static"),
                                   ("1", "0", "dynamic"), ("0", "0", "static")):
        monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", single)
        monkeypatch.setenv("MOE_B200_B_ONE_BOX", one_box)
        monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order)
        run = LayerRun(wl, d)
        assert run.status == 0
        outs.append(run.out.clone())
    for o in outs[1:]:
        assert torch.equal(outs[0], o)


@pytest.mark.parametrize("name", sorted(ALIGNED))
def test_cta_pair_one_copy_equals_two_copies(name, monkeypatch):
    """In the CTA-pair variant each CTA's 128-column half of B arrives in one
    copy or in two 64-column copies: the same shared-memory image, the same bits."""
    wl = ALIGNED[name]
    d = to_dev(make_inputs(wl, 14))
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "0")
    monkeypatch.setenv("MOE_B200_CTA_PAIR", "2")
    outs = []
    for one_box in ("1", "0"):
        monkeypatch.setenv("MOE_B200_B_ONE_BOX", one_box)
        run = LayerRun(wl, d)
        assert run.status == 0
        outs.append(run.out.clone())
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("name", ["tiny", "sink_small", "gptoss_small"])
def test_programmatic_launch_changes_nothing(name, monkeypatch):
    """Kernels launched to overlap their predecessor's tail (programmatic
    dependent launch) wait for its results first: the same bits either way."""
    wl = SMALL[name]
    d = to_dev(make_inputs(wl, 13))
    outs = []
    # every launch programmatic; none; every launch but the two cooperative
    # ones (CSR build, FFN)
    for pdl, coop in (("1", "1"), ("0", "1"), ("1", "0")):
        monkeypatch.setenv("MOE_B200_PDL", pdl)
        monkeypatch.setenv("MOE_B200_PDL_COOP", coop)
        run = LayerRun(wl, d)
        assert run.status == 0
        outs.append((run.out.clone(), run.idx.clone(), run.w.clone()))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["sink_small", "mixtral_small"])
def test_single_launch_pair_without_cooperative_attribute(name, monkeypatch):
    """MOE_B200_PAIR_COOP=0: the single-launch CTA-pair FFN as a plain
    clustered launch, its grid sized by the cluster occupancy query, gives
    the cooperative launch's bits (on an idle GPU every cluster is resident)."""
    wl = SMALL[name]
    d = to_dev(make_inputs(wl, 14))
    set_variant(monkeypatch, "single_launch_cta_pair")
    outs = []
    for coop in ("1", "0"):
        monkeypatch.setenv("MOE_B200_PAIR_COOP", coop)
        run = LayerRun(wl, d)
        assert run.status == 0, f"device status {run.status:#x}"
        outs.append(run.out.clone())
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("name", sorted(ALIGNED))
def test_one_box_layouts_against_oracle(name, monkeypatch):
    monkeypatch.setenv("MOE_B200_B_ONE_BOX", "1")
    run_and_check(ALIGNED[name], seed=12)


@pytest.mark.parametrize("seed", [1, 2])
def test_forward_tiny_seeds(seed):
    run_and_check(WORKLOADS["tiny"], seed=seed)


EDGE_CASES = [
    dict(num_tokens=1), dict(top_k=1), dict(num_tokens=3, top_k=8), dict(num_experts=37, logits_std=1.0),
    dict(num_experts=64, num_tokens=4),                         # most experts empty
    dict(gate_up_format="interleaved"), dict(activation="gelu_tanh"),
    dict(activation="silu", limit=0.05),                        # clamps active on N(0,.) projections
    dict(activation="swigluoai", alpha=1.702, limit=0.05, has_bias=True),
    dict(num_tokens=200, hidden_dim=8, moe_dim=8),              # single partial K block, tiny N
    dict(num_tokens=1100),                                      # R > 2048: separate router and CSR kernels
    dict(num_experts=600, num_tokens=40, logits_std=1.0),       # E > 512: separate router and CSR kernels
    dict(num_experts=1024, top_k=32, num_tokens=40, logits_std=1.0),  # the library's largest E and k
    dict(num_tokens=64, hidden_dim=8192, moe_dim=64),           # long gate_up K (128 K blocks), tiny down K
    dict(num_tokens=48, hidden_dim=64, moe_dim=8192),           # long down K, 64 gate_up column blocks
]


@pytest.mark.parametrize("variant", EDGE_CASES)
def test_forward_edge_cases(variant):
    run_and_check(WORKLOADS["tiny"].replace(**variant), seed=3)


@pytest.mark.parametrize("variant", EDGE_CASES)
def test_forward_edge_cases_cta_pair(variant, monkeypatch):
    """The same shapes on CTA pairs: 256-row pieces, tails of at most 128
    rows as M = 128 pair MMAs, gate/up-paired B halves."""
    set_variant(monkeypatch, "two_launches_cta_pair")
    run_and_check(WORKLOADS["tiny"].replace(**variant), seed=3)


def test_sink_router_largest_shape():
    """Sink router at its limits: 1024 routed experts, k + S = 32 lanes."""
    wl = WORKLOADS["sink"].replace(num_tokens=50, hidden_dim=128, num_experts=1024, top_k=30, num_sink=2,
                                   moe_dim=64)
    run_and_check(wl, seed=9)


def test_all_tokens_on_one_expert():
    wl = WORKLOADS["tiny"].replace(num_tokens=150, top_k=2)
    inp = make_inputs(wl, 4)
    inp["logits"][:, 5] += 100.0        # expert 5 first for every token; every other segment is short or empty
    d = to_dev(inp)
    run = LayerRun(wl, d)
    idx_ref, w_ref, _ = oracle_route(wl, inp)
    assert (idx_ref[:, 0] == 5).all()
    assert np.array_equal(run.idx.cpu().numpy(), idx_ref)
    ref = oracle_ffn(wl, inp, idx_ref, w_ref)
    assert ffn_error(run.out.float().cpu().numpy(), ref) <= FFN_TOL


def test_bf16_logits_and_wide_rows():
    wl = WORKLOADS["sink"].replace(num_tokens=77, hidden_dim=64, num_experts=20, moe_dim=64)
    inp = make_inputs(wl, 5)
    T, C = inp["logits"].shape
    wide = torch.full((T, C + 9), float("nan"))
    wide[:, :C] = inp["logits"].to(torch.bfloat16).float()
    cfg = abi.make_config(wl, logits_dtype=torch.bfloat16, logits_row_stride=C + 9)
    lg = wide.to(torch.bfloat16).cuda()
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    sw = torch.empty((T, wl.num_sink), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, lg, idx, w, sw, inp["expert_bias"].cuda(), inp["global_scale"].cuda())
    bits = wide.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    i_ref, w_ref, s_ref = oracle.route_sigmoid_sink(bits, wl.num_experts, wl.num_sink, wl.top_k,
                                                    inp["expert_bias"].numpy(), wl.route_scale, 1.0)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    check_weights(w.cpu().numpy(), w_ref)
    check_weights(sw.cpu().numpy(), s_ref)


@pytest.mark.parametrize("E,k,logits_dtype", [(8, 2, torch.float32), (37, 5, torch.bfloat16), (128, 4, torch.float32),
                                             (1024, 32, torch.float32), (1, 1, torch.float32)])
def test_softmax_router(E, k, logits_dtype):
    T = 513
    g = torch.Generator().manual_seed(E * 7 + k)
    logits = (torch.randn(T, E, generator=g) * 2).to(logits_dtype)
    logits[7, :] = 0.5                    # all ties: lowest indices, in order
    logits[9, :] = float("-inf")          # one finite logit, then -inf ties by lowest index
    logits[9, E // 2] = 1.0
    logits[10, :] = 0.0                   # +0 and -0 compare equal: lowest indices
    logits[10, 1::2] = -0.0
    wl = WORKLOADS["tiny"].replace(num_experts=E, top_k=k, num_tokens=T)
    cfg = abi.make_config(wl, logits_dtype=logits_dtype)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, logits.cuda(), idx, w)
    host = logits.float().numpy() if logits_dtype == torch.float32 else \
        logits.view(torch.int16).numpy().view(np.uint16)
    i_ref, w_ref = oracle.route_softmax_topk(host, E, k)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert idx[7].tolist() == list(range(k))
    assert idx[10].tolist() == list(range(k))
    assert idx[9, 0].item() == E // 2
    check_weights(w.cpu().numpy(), w_ref)


def test_sink_router_extremes():
    wl = WORKLOADS["sink"].replace(num_tokens=64, num_experts=40, top_k=6, num_sink=2)
    g = torch.Generator().manual_seed(9)
    logits = torch.randn(64, 42, generator=g) * 30          # sigmoids saturate and underflow
    logits[3] = -850.0                                     # every sigmoid underflows: log-space weights
    bias = (torch.rand(40, generator=g) * 0.2 - 0.1)
    cfg = abi.make_config(wl)
    idx = torch.empty((64, 6), dtype=torch.int32, device="cuda")
    w = torch.empty((64, 6), dtype=torch.float32, device="cuda")
    sw = torch.empty((64, 2), dtype=torch.float32, device="cuda")
    gs = torch.tensor([0.75], device="cuda")
    abi.moe_route(cfg, logits.cuda(), idx, w, sw, bias.cuda(), gs)
    i_ref, w_ref, s_ref = oracle.route_sigmoid_sink(logits.numpy(), 40, 2, 6, bias.numpy(), wl.route_scale, 0.75)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    check_weights(w.cpu().numpy(), w_ref)
    check_weights(sw.cpu().numpy(), s_ref)
    tot = w.double().sum(1) + sw.double().sum(1)
    assert torch.allclose(tot.cpu(), torch.full((64,), 2.5 * 0.75, dtype=torch.float64), rtol=1e-6)


@pytest.mark.parametrize("fused", ["1", "0"])
@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (1000, 16, 4), (4096, 128, 6), (7, 1024, 3), (50000, 8, 2),
                                   (8192, 1024, 6), (160000, 64, 2),
                                   # 148 and 149 chunks of 2048 slots: the most the
                                   # one-launch form takes on a 148-SM B200, and one more
                                   (151552, 16, 2), (151553, 16, 2)])
def test_create_indices(T, E, k, fused, monkeypatch):
    """Both forms of the CSR build (one cooperative launch, or count -> scan
    -> scatter) against the oracle's counting sort, bit for bit.  Problems of
    more chunks than SMs always take three launches."""
    monkeypatch.setenv("MOE_B200_CSR_FUSED", fused)
    g = torch.Generator().manual_seed(T + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32) if T < 5000 else \
        torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :k].to(torch.int32)
    wl = WORKLOADS["tiny"].replace(num_tokens=T, num_experts=E, top_k=k)
    cfg = abi.make_config(wl)
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    abi.moe_create_indices(cfg, idx.cuda(), off, perm, inv, ws)
    counts, o_ref, p_ref, i_ref = oracle.create_indices(idx.numpy(), E)
    assert np.array_equal(off.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)
    assert np.array_equal(inv.cpu().numpy(), i_ref)
    assert abi.moe_device_status(ws) == 0


@pytest.mark.parametrize("fused", ["1", "0"])
def test_create_indices_flags_bad_expert(fused, monkeypatch):
    monkeypatch.setenv("MOE_B200_CSR_FUSED", fused)
    wl = WORKLOADS["tiny"].replace(num_tokens=10, num_experts=8, top_k=2)
    cfg = abi.make_config(wl)
    idx = torch.randint(0, 8, (10, 2), dtype=torch.int32)
    idx[4, 1] = 8
    idx[6, 0] = -3
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    off = torch.empty(9, dtype=torch.int32, device="cuda")
    perm = torch.full((20,), -1, dtype=torch.int32, device="cuda")
    abi.moe_create_indices(cfg, idx.cuda(), off, perm, None, ws)
    assert abi.moe_device_status(ws) & abi.DEVICE_ERR_EXPERT_INDEX
    assert int(off[-1]) == 18                      # the two bad slots are left out


def test_stages_compose_to_forward():
    """moe_route -> moe_create_indices -> moe_grouped_ffn equals moe_forward bit for bit."""
    wl = SMALL["gptoss_small"]
    inp = make_inputs(wl, 6)
    d = to_dev(inp)
    run = LayerRun(wl, d)
    T, k, E = wl.num_tokens, wl.top_k, wl.num_experts
    cfg = run.cfg
    ws = torch.empty_like(run.ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, d["logits"], idx, w)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    abi.moe_create_indices(cfg, idx, off, perm, None, ws)
    out = torch.empty((T, wl.hidden_dim), dtype=torch.bfloat16, device="cuda")
    abi.moe_grouped_ffn(cfg, d["x"], d["W_gu"], d["b_gu"], d["W_d"], d["b_d"], off, perm, w, out, ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, run.idx) and torch.equal(w, run.w)
    assert torch.equal(out, run.out)
    again = LayerRun(wl, d)
    assert torch.equal(again.out, run.out)         # deterministic


def test_forward_timed_matches_forward():
    wl = SMALL["sink_small"]
    d = to_dev(make_inputs(wl, 8))
    run = LayerRun(wl, d)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(abi.NUM_STAGE_EVENTS)]
    out = torch.empty_like(run.out)
    sink = torch.empty_like(run.sink)
    abi.moe_forward_timed(run.cfg, events, d["x"], d["logits"], d["W_gu"], d["W_d"], out, run.ws,
                          expert_bias=d["expert_bias"], global_scale=d["global_scale"], sink_weights_out=sink)
    torch.cuda.synchronize()
    assert torch.equal(out, run.out) and torch.equal(sink, run.sink)
    times = [events[i].elapsed_time(events[i + 1]) for i in range(abi.NUM_STAGE_EVENTS - 1)]
    assert all(t >= 0 for t in times) and sum(times) > 0


def test_grouped_ffn_rejects_inconsistent_csr():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, 7)
    d = to_dev(inp)
    cfg = abi.make_config(wl)
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    off = torch.tensor([0, 10, 5, 40, 60, 80, 100, 120, 128], dtype=torch.int32, device="cuda")  # not monotone
    perm = torch.arange(128, dtype=torch.int32, device="cuda")
    w = torch.ones((64, 2), dtype=torch.float32, device="cuda")
    out = torch.empty((64, 256), dtype=torch.bfloat16, device="cuda")
    abi.moe_grouped_ffn(cfg, d["x"], d["W_gu"], None, d["W_d"], None, off, perm, w, out, ws)
    assert abi.moe_device_status(ws) & abi.DEVICE_ERR_CSR


def test_zero_tokens():
    wl = WORKLOADS["tiny"].replace(num_tokens=0)
    cfg = abi.make_config(wl)
    ws = torch.zeros(abi.moe_workspace_size(cfg) + 256, dtype=torch.uint8, device="cuda")
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    W = make_inputs(WORKLOADS["tiny"], 0, device="cuda")
    out = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    abi.moe_forward(cfg, x, lg, W["W_gu"], W["W_d"], out, ws)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- full size
# Every workload at full size in the benchmark's launch configuration (the
# default single launch), in both tile orders: routing and weights for every
# token; the layer output for every token where the oracle finishes in
# seconds (tiny, gptoss, sink, decode: up to 464 GFLOP in fp64) and for
# tokens whose rows reach every tile where it would take minutes (mixtral:
# about 600 of 4096 tokens).
FULL_EVERY_TOKEN = ("tiny", "gptoss", "sink", "decode")


def full_size_reference(wl):
    inp = make_inputs(wl, seed=0, device="cuda")
    idx_ref, w_ref, s_ref = oracle_route(wl, inp)
    tokens = None if wl.name in FULL_EVERY_TOKEN else every_tile_tokens(idx_ref, wl.num_experts)
    ref = oracle_ffn(wl, inp, idx_ref, w_ref, tokens)
    return inp, (idx_ref, w_ref, s_ref), tokens, ref


def check_full_size_run(wl, inp, route_ref, tokens, ref):
    idx_ref, w_ref, s_ref = route_ref
    run = LayerRun(wl, inp, out_guard=64)
    assert run.status == 0, f"device status {run.status:#x}"
    assert np.array_equal(run.idx.cpu().numpy(), idx_ref)
    check_weights(run.w.cpu().numpy(), w_ref)
    if wl.num_sink > 0:
        check_weights(run.sink.cpu().numpy(), s_ref)
    got = run.out.float().cpu().numpy()
    if tokens is not None:
        got = got[tokens]
    err = ffn_error(got, ref)
    assert err <= FFN_TOL, f"ffn error {err:.3e} > {FFN_TOL}"
    assert (run.out_full[wl.num_tokens * wl.hidden_dim:].float() == -7.0).all(), "output guard overwritten"
    return err


@pytest.mark.parametrize("name", ["tiny", "mixtral", "gptoss", "sink", "decode"])
def test_forward_full_size_every_tile(name, monkeypatch):
    """Both tile orders of the default single launch against one oracle
    result: every 128-row piece of every expert has rows compared."""
    wl = WORKLOADS[name]
    inp, route_ref, tokens, ref = full_size_reference(wl)
    if tokens is not None:
        assert len(tokens) >= wl.num_experts and len(tokens) < wl.num_tokens
    for order in ("static", "dynamic"):
        monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order)
        check_full_size_run(wl, inp, route_ref, tokens, ref)


@pytest.mark.parametrize("variant", ["two_launches_cta_pair", "single_launch_cta_pair"])
@pytest.mark.parametrize("name", ["mixtral", "sink"])
def test_forward_full_size_every_tile_cta_pair(name, variant, monkeypatch):
    """The selectable CTA-pair variants at full size, as two launches and as
    one: 256-row pieces and M = 128 pair tails over every expert of the
    workload."""
    set_variant(monkeypatch, variant)
    wl = WORKLOADS[name]
    inp, route_ref, tokens, ref = full_size_reference(wl)
    check_full_size_run(wl, inp, route_ref, tokens, ref)


@pytest.mark.parametrize("name,order", [("gptoss", "dynamic"), ("sink", "static"), ("sink", "dynamic")])
def test_full_size_runs_are_bit_identical(name, order, monkeypatch):
    """Which CTA computes which tile changes from run to run (the dynamic
    order draws tiles from an atomic counter); what each tile computes, and
    the combine's summation order, do not: repeated full-size calls give the
    same bits, in the workload's default tile order and in the other."""
    monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order)
    wl = WORKLOADS[name]
    d = to_dev(make_inputs(wl, 21, device="cuda"))
    first = LayerRun(wl, d)
    assert first.status == 0
    for _ in range(2):
        again = LayerRun(wl, d)
        assert again.status == 0
        assert torch.equal(first.out, again.out) and torch.equal(first.idx, again.idx)
        assert torch.equal(first.w, again.w)


def test_nvtx_ranges_change_nothing():
    """With MOE_B200_NVTX=1 (read once per process) every API call and kernel
    enqueue is wrapped in an NVTX range; the layer still matches the oracle."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    script = ("import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
              "from gpu_helpers import run_and_check\n"
              "from test_gpu_parity import SMALL\n"
              "run_and_check(SMALL['sink_small'], seed=15)\n"
              "run_and_check(SMALL['decode_small'], seed=15)\n"
              "print('ok')\n") % (here, os.path.dirname(here))
    env = dict(os.environ, MOE_B200_NVTX="1")
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stderr[-2000:]


@pytest.mark.parametrize("name", ["sink_small", "gptoss_small", "decode_small"])
def test_cuda_graph_capture(name):
    """moe_forward allocates nothing and never synchronizes, so it can be
    captured in a CUDA graph (cooperative single launch and programmatic
    dependent launches included); every replay gives the eager result."""
    wl = SMALL[name]
    d = to_dev(make_inputs(wl, 16))
    eager = LayerRun(wl, d)
    assert eager.status == 0
    T, H, k, S = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink
    ws = torch.empty_like(eager.ws)
    out = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    kw = dict(gate_up_b=d["b_gu"], down_b=d["b_d"], expert_bias=d["expert_bias"], global_scale=d["global_scale"],
              expert_indices_out=idx)
    abi.moe_forward(eager.cfg, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, **kw)  # warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        abi.moe_forward(eager.cfg, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, **kw)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert abi.moe_device_status(ws) == 0
        assert torch.equal(out, eager.out) and torch.equal(idx, eager.idx)
    del g


def test_stage_events_inside_a_cuda_graph():
    """moe_forward_timed with only the GEMM stage's pair of events set (the
    other slots NULL), captured in a CUDA graph: every replay records that
    pair, and the stage time is positive and shorter than the whole step."""
    wl = SMALL["sink_small"]
    d = to_dev(make_inputs(wl, 17))
    eager = LayerRun(wl, d)
    ws = torch.empty_like(eager.ws)
    out = torch.empty_like(eager.out)
    kw = dict(expert_bias=d["expert_bias"], global_scale=d["global_scale"])
    a, b = torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)
    s0, s1 = torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)
    evs = [None] * abi.NUM_STAGE_EVENTS
    evs[5], evs[6] = a, b                       # around the gate_up stage (the single launch by default)
    for ev in (a, b, s0, s1):
        ev.record()
    abi.moe_forward_timed(eager.cfg, evs, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, **kw)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        s0.record()
        abi.moe_forward_timed(eager.cfg, evs, d["x"], d["logits"], d["W_gu"], d["W_d"], out, ws, **kw)
        s1.record()
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        stage, whole = a.elapsed_time(b), s0.elapsed_time(s1)
        assert 0.0 < stage < whole, (stage, whole)
        assert torch.equal(out, eager.out)
    del g


@pytest.mark.parametrize("name", ["sink_small", "gptoss_small", "decode_small", "mixtral_small"])
@pytest.mark.parametrize("single_launch", ["1", "0"])
def test_no_writes_past_any_buffer(name, single_launch, monkeypatch):
    """Canaries after the workspace and after every routing output: the
    kernels write only inside the sizes the API states."""
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", single_launch)
    wl = SMALL[name]
    d = to_dev(make_inputs(wl, 18))
    cfg = abi.make_config(wl)
    T, H, k, S = wl.num_tokens, wl.hidden_dim, wl.top_k, wl.num_sink
    guard = 4096
    need = abi.moe_workspace_size(cfg)
    ws_full = torch.full((need + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = ws_full[:need]
    idx_full = torch.full((T * k + guard,), -12345, dtype=torch.int32, device="cuda")
    w_full = torch.full((T * k + guard,), -3.0, dtype=torch.float32, device="cuda")
    sink_full = torch.full((T * S + guard,), -5.0, dtype=torch.float32, device="cuda")
    out_full = torch.full((T * H + guard,), -7.0, dtype=torch.bfloat16, device="cuda")
    abi.moe_forward(cfg, d["x"], d["logits"], d["W_gu"], d["W_d"], out_full[:T * H].view(T, H), ws,
                    gate_up_b=d["b_gu"], down_b=d["b_d"], expert_bias=d["expert_bias"],
                    global_scale=d["global_scale"], expert_indices_out=idx_full[:T * k].view(T, k),
                    expert_weights_out=w_full[:T * k].view(T, k),
                    sink_weights_out=sink_full[:T * S].view(T, S) if S > 0 else None)
    torch.cuda.synchronize()
    assert abi.moe_device_status(ws) == 0
    assert (ws_full[need:] == 0xA5).all(), "workspace guard overwritten"
    assert (idx_full[T * k:] == -12345).all() and (w_full[T * k:] == -3.0).all()
    assert (sink_full[T * S:] == -5.0).all()
    assert (out_full[T * H:] == -7.0).all()


@pytest.mark.parametrize("order", ["static", "dynamic"])
@pytest.mark.parametrize("name", sorted(SMALL) + sorted(ALIGNED))
def test_fused_gather_equals_gather_kernel(name, order, monkeypatch):
    """Row f1: the gate_up GEMM reading its rows of x by tile::gather4 gives
    the same bits as the separate gather kernel followed by the GEMM (both
    multiply the same bf16 rows), in one launch and in two."""
    wl = {**SMALL, **ALIGNED}[name]
    d = to_dev(make_inputs(wl, 31))
    monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order)
    for single in ("1", "0"):
        monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", single)
        monkeypatch.setenv("MOE_B200_FUSED_GATHER", "0")
        ref = LayerRun(wl, d)
        monkeypatch.setenv("MOE_B200_FUSED_GATHER", "1")
        got = LayerRun(wl, d)
        assert ref.status == 0 and got.status == 0
        assert torch.equal(got.out, ref.out), (name, single)


@pytest.mark.parametrize("name", ["mixtral", "sink", "gptoss"])
def test_fused_gather_full_size_equals_gather_kernel(name, monkeypatch):
    """Row f1 at full size in the single launch: bit-identical to the default
    path, whose every tile is compared with the oracle above."""
    wl = WORKLOADS[name]
    d = to_dev(make_inputs(wl, 0, device="cuda"))
    monkeypatch.setenv("MOE_B200_FUSED_GATHER", "0")
    ref = LayerRun(wl, d)
    monkeypatch.setenv("MOE_B200_FUSED_GATHER", "1")
    got = LayerRun(wl, d)
    assert ref.status == 0 and got.status == 0
    assert torch.equal(got.out, ref.out)


@pytest.mark.parametrize("name", ["sink", "mixtral", "gptoss"])
def test_csr_forms_give_the_same_forward(name, monkeypatch):
    """The full-size forward with the one-launch CSR build (default) and with
    three launches: identical routing, permutation and output bits."""
    wl = WORKLOADS[name]
    d = to_dev(make_inputs(wl, 3, device="cuda"))
    monkeypatch.setenv("MOE_B200_CSR_FUSED", "1")
    a = LayerRun(wl, d)
    monkeypatch.setenv("MOE_B200_CSR_FUSED", "0")
    b = LayerRun(wl, d)
    assert a.status == 0 and b.status == 0
    assert torch.equal(a.out, b.out) and torch.equal(a.idx, b.idx)
