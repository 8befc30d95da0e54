"""The randomized sweep's generator (tests/random_configs.py), on the CPU:
deterministic, inside the library's accepted configurations, and spread
over the cases it is there to reach."""
from mixture_experts_ffn_token_b200 import abi
from random_configs import LAUNCH_FORMS, NUM_CASES, NUM_MIDSIZE, random_midsize_workload, random_workload


def test_draws_are_deterministic():
    assert [random_workload(i) for i in range(NUM_CASES)] == [random_workload(i) for i in range(NUM_CASES)]


def test_every_draw_is_accepted_by_the_library():
    for i in range(NUM_CASES):
        wl, form = random_workload(i)
        assert abi.moe_workspace_size(abi.make_config(wl)) > 0
        assert form in LAUNCH_FORMS
        assert wl.hidden_dim % 8 == 0 and wl.moe_dim % 8 == 0 and 1 <= wl.top_k <= wl.num_experts
        if wl.router == "sigmoid_sink":
            lanes = wl.top_k + wl.num_sink
            assert lanes & (lanes - 1) == 0 and lanes <= 32
            assert wl.num_shared in (0, wl.num_sink)
        else:
            assert wl.num_sink == 0


def test_sweep_reaches_its_cases():
    draws = [random_workload(i)[0] for i in range(NUM_CASES)]
    assert {w.router for w in draws} == {"softmax_topk", "sigmoid_sink"}
    assert {w.gate_up_format for w in draws} == {"concatenated", "interleaved"}
    assert {w.activation for w in draws} == {"silu", "swigluoai", "gelu_tanh"}
    assert any(w.has_bias for w in draws) and not all(w.has_bias for w in draws)
    assert any(w.hidden_dim % 64 for w in draws) and any(w.moe_dim % 128 for w in draws)  # K and N tails
    assert any(w.extended for w in draws) and not all(w.extended for w in draws)
    assert any(w.limit > 0 for w in draws)


def test_midsize_draws_are_accepted_and_large_enough():
    for i in range(NUM_MIDSIZE):
        wl, form = random_midsize_workload(i)
        assert random_midsize_workload(i) == (wl, form)
        assert abi.moe_workspace_size(abi.make_config(wl)) > 0
        assert form in LAUNCH_FORMS and not wl.extended
        assert wl.num_tokens >= 400 and wl.num_tokens * wl.top_k <= 6000 and wl.hidden_dim % 8 == 0
        if wl.router == "sigmoid_sink":
            lanes = wl.top_k + wl.num_sink
            assert lanes & (lanes - 1) == 0
