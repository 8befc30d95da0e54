"""Seeded random layer configurations for the randomized parity sweep.

Each draw is a small Workload that the library accepts: any hidden and
moe_dim that are multiples of 8 (so K and N tails of every size), 1 to 130
experts, both routers (k + S a power of two for the sink router), both
gate/up layouts, the three activations with and without clamps and bias,
and, for some draws, the moe_forward_ex extensions (token mask, router
weight first, shared experts). Sizes stay small enough for the fp64 oracle
to finish each case in about a second.
"""
import random

from mixture_experts_ffn_token_b200.workloads import WORKLOADS

# launch forms the sweep cycles through (MOE_B200_* switches)
LAUNCH_FORMS = [
    {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_TILE_SCHEDULE": "static"},
    {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_TILE_SCHEDULE": "dynamic"},
    {"MOE_B200_SINGLE_LAUNCH": "0"},
    {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_CTA_PAIR": "2"},
    {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_CTA_PAIR": "2"},
    {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_B_ONE_BOX": "0"},
    # row f1: the gate_up GEMM gathers its rows of x itself (the gather
    # kernel still runs where the router weight scales the rows)
    {"MOE_B200_SINGLE_LAUNCH": "1", "MOE_B200_FUSED_GATHER": "1", "MOE_B200_TILE_SCHEDULE": "static"},
    {"MOE_B200_SINGLE_LAUNCH": "0", "MOE_B200_FUSED_GATHER": "1"},
]

NUM_CASES = 256


def random_workload(i):
    """The i-th configuration of the sweep (deterministic in i)."""
    r = random.Random(7919 * (i + 1))
    router = r.choice(["softmax_topk", "sigmoid_sink"])
    E = r.choice([1, 2, 3, 5, 8, 13, 32, 64, 130])
    if router == "sigmoid_sink":
        lanes = r.choice([1, 2, 4, 8, 16, 32])
        k = r.randint(1, min(E, lanes))
        S = lanes - k
    else:
        k = r.randint(1, min(E, 8))
        S = 0
    T = r.choice([1, 2, 7, 33, 100, 257])
    H = 8 * r.randint(1, 64)
    D = 8 * r.randint(1, 64)
    activation = r.choice(["silu", "swigluoai", "gelu_tanh"])
    alpha = 1.702 if activation == "swigluoai" else 0.0
    limit = 0.0 if activation == "gelu_tanh" else r.choice([0.0, 0.05, 7.0])
    kw = dict(name=f"random{i}", num_tokens=T, hidden_dim=H, num_experts=E, top_k=k, moe_dim=D, router=router,
              num_sink=S, gate_up_format=r.choice(["concatenated", "interleaved"]), activation=activation,
              alpha=alpha, limit=limit, has_bias=r.random() < 0.5, logits_kind="normal",
              logits_std=r.choice([0.5, 1.0, 2.0]))
    if router == "sigmoid_sink":
        kw.update(expert_bias_range=0.1, route_scale=r.choice([0.5, 1.0, 2.5]), global_scale=r.choice([1.0, 0.7]))
    else:
        kw.update(expert_bias_range=0.0, route_scale=1.0, global_scale=1.0)
    # extensions on about a third of the draws
    if r.random() < 0.35:
        kw["mask_frac"] = r.choice([0.0, 0.3])
        kw["weight_first"] = r.random() < 0.5
        if router == "softmax_topk":
            kw["num_shared"] = r.choice([0, 1, 2])
        else:
            kw["num_shared"] = r.choice([0, S])  # shared expert i is gated by sink lane i
        kw["shared_dim"] = 8 * r.randint(1, 48) if kw["num_shared"] > 0 else 0
    return WORKLOADS["tiny"].replace(**kw), LAUNCH_FORMS[i % len(LAUNCH_FORMS)]


NUM_MIDSIZE = 48


def random_midsize_workload(i):
    """The i-th mid-size draw: a few thousand routed rows, so each launch has
    hundreds to thousands of tiles over ragged expert segments (several tiles
    per CTA, every wrap of the tile-number ring, the dynamic counter under
    contention), at sizes whose oracle over the every-tile token sample
    still takes seconds. No extensions."""
    r = random.Random(104729 * (i + 1))
    router = r.choice(["softmax_topk", "sigmoid_sink"])
    E = r.choice([4, 8, 16, 40, 64, 128, 160])
    if router == "sigmoid_sink":
        lanes = r.choice([4, 8, 16])
        k = r.randint(1, min(E, lanes, 8))
        S = lanes - k
    else:
        k = r.randint(1, min(E, 8))
        S = 0
    T = r.randint(400, max(400, 6000 // k))
    H = 8 * r.randint(32, 128)
    D = 8 * r.randint(32, 128)
    activation = r.choice(["silu", "swigluoai", "gelu_tanh"])
    kw = dict(name=f"midsize{i}", num_tokens=T, hidden_dim=H, num_experts=E, top_k=k, moe_dim=D, router=router,
              num_sink=S, gate_up_format=r.choice(["concatenated", "interleaved"]), activation=activation,
              alpha=1.702 if activation == "swigluoai" else 0.0,
              limit=0.0 if activation == "gelu_tanh" else r.choice([0.0, 7.0]), has_bias=r.random() < 0.5,
              logits_kind="normal", logits_std=r.choice([0.5, 1.0, 2.0]),
              expert_bias_range=0.1 if router == "sigmoid_sink" else 0.0,
              route_scale=2.5 if router == "sigmoid_sink" else 1.0)
    return WORKLOADS["tiny"].replace(**kw), LAUNCH_FORMS[i % len(LAUNCH_FORMS)]
