"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/moe.h declares, sizes its workspace, and rejects bad
arguments before it touches the device."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.build import build
from mixture_experts_ffn_token_b200.workloads import WORKLOADS

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")

INVALID, UNSUPPORTED, SMALL = 1, 2, 3
FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced by these calls


@pytest.fixture(scope="module")
def lib():
    build()
    return abi.load_library()


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|moe_status_t)\s+(moe_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_entry_points()
    assert set(names) == set(abi.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in abi.STATUS_NAMES.items():
        assert abi.moe_status_string(code) == name


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workspace_size_covers_intermediates(lib, name):
    wl = WORKLOADS[name]
    n = abi.moe_workspace_size(abi.make_config(wl))
    R = wl.num_tokens * wl.top_k
    assert n >= R * wl.hidden_dim * 2 + R * wl.moe_dim * 2 + R * 12
    assert n % 256 == 0


def status_of(lib, cfg):
    n = ctypes.c_size_t(0)
    return lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n))


def cfg_for(name="tiny", **kw):
    c = abi.make_config(WORKLOADS[name])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,expected", [
    ("num_tokens", -1, INVALID), ("hidden_dim", 0, INVALID), ("num_experts", 0, INVALID),
    ("top_k", 0, INVALID), ("top_k", 9, INVALID), ("moe_dim", -8, INVALID),
    ("num_sink", 1, INVALID),                      # sinks need the sigmoid router
    ("logits_row_stride", 7, INVALID), ("router", 5, INVALID), ("logits_dtype", 3, INVALID),
    ("gate_up_format", 2, INVALID), ("activation", 7, INVALID), ("has_bias", 2, INVALID),
    ("alpha", 1.702, INVALID),                     # alpha only for swigluoai
    ("limit", -1.0, INVALID),
    ("hidden_dim", 260, UNSUPPORTED), ("moe_dim", 500, UNSUPPORTED),
])
def test_config_validation(lib, field, value, expected):
    assert status_of(lib, cfg_for(**{field: value})) == expected


def test_expert_count_limit(lib):
    assert status_of(lib, cfg_for(num_experts=1024, logits_row_stride=1024)) == 0
    assert status_of(lib, cfg_for(num_experts=2048, logits_row_stride=2048)) == UNSUPPORTED


def test_activation_parameter_rules(lib):
    assert status_of(lib, cfg_for(activation=2, limit=7.0)) == INVALID       # limit must be 0 for gelu_tanh
    assert status_of(lib, cfg_for(activation=1, alpha=1.702, limit=7.0)) == 0
    assert status_of(lib, cfg_for(activation=0, limit=7.0)) == 0             # clamped silu
    assert status_of(lib, cfg_for(activation=0, alpha=float("nan"))) == INVALID


def test_sink_router_rules(lib):
    base = cfg_for("sink")
    assert status_of(lib, base) == 0
    assert status_of(lib, cfg_for("sink", num_sink=3, logits_row_stride=131)) == UNSUPPORTED        # 6 + 3 is not a power of two
    assert status_of(lib, cfg_for("sink", top_k=32, num_sink=2)) == UNSUPPORTED
    assert status_of(lib, cfg_for("sink", logits_row_stride=129)) == INVALID
    assert status_of(lib, cfg_for("sink", logits_row_stride=200)) == 0       # a wider row is fine
    assert status_of(lib, cfg_for("sink", route_scale=float("inf"))) == INVALID


def test_entry_points_reject_before_device(lib):
    cfg = cfg_for("tiny")
    need = abi.moe_workspace_size(cfg)
    by = ctypes.byref
    # moe_forward: null x, misaligned weights, small workspace, stray bias
    assert lib.moe_forward(by(cfg), None, FAKE, None, None, FAKE, None, FAKE, None, FAKE, None, None, None,
                           FAKE, need, None) == INVALID
    assert lib.moe_forward(by(cfg), FAKE, FAKE, None, None, FAKE + 2, None, FAKE, None, FAKE, None, None, None,
                           FAKE, need, None) == INVALID
    assert lib.moe_forward(by(cfg), FAKE, FAKE, None, None, FAKE, None, FAKE, None, FAKE, None, None, None,
                           FAKE, need - 1, None) == SMALL
    assert lib.moe_forward(by(cfg), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                           FAKE, need, None) == INVALID
    # moe_grouped_ffn without routing arrays
    assert lib.moe_grouped_ffn(by(cfg), FAKE, FAKE, None, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, need,
                               None) == INVALID
    # moe_create_indices with a small workspace
    assert lib.moe_create_indices(by(cfg), FAKE, FAKE, FAKE, None, FAKE, 16, None) == SMALL
    # moe_route: the sink router needs sink_weights when S > 0
    scfg = cfg_for("sink")
    assert lib.moe_route(by(scfg), FAKE, None, None, FAKE, FAKE, None, None) == INVALID
    # moe_forward_timed needs its events
    assert lib.moe_forward_timed(by(cfg), FAKE, FAKE, None, None, FAKE, None, FAKE, None, FAKE, None, None, None,
                                 FAKE, need, None, None) == INVALID
    assert lib.moe_device_status(None, None, None) == INVALID


def test_zero_tokens_is_a_no_op(lib):
    cfg = cfg_for("tiny", num_tokens=0)
    need = abi.moe_workspace_size(cfg)
    # returns before any device call: nothing to do
    assert lib.moe_forward(ctypes.byref(cfg), FAKE, FAKE, None, None, FAKE, None, FAKE, None, FAKE, None, None,
                           None, FAKE, need, None) == 0


def test_extras_validation(lib):
    by = ctypes.byref
    n = ctypes.c_size_t(0)
    cfg = cfg_for("tiny")
    base = abi.moe_workspace_size(cfg)
    assert lib.moe_workspace_size_ex(by(cfg), None, by(n)) == 0 and n.value == base
    ex = abi.MoEExtras()
    ex.num_shared, ex.shared_dim = 2, 64
    ex.shared_gate_up_w = ex.shared_down_w = FAKE
    assert lib.moe_workspace_size_ex(by(cfg), by(ex), by(n)) == 0 and n.value > base
    ex.shared_dim = 12
    assert lib.moe_workspace_size_ex(by(cfg), by(ex), by(n)) == UNSUPPORTED
    ex.shared_dim = 0
    assert lib.moe_workspace_size_ex(by(cfg), by(ex), by(n)) == INVALID
    ex = abi.MoEExtras()
    ex.apply_router_weight_first = 2
    assert lib.moe_workspace_size_ex(by(cfg), by(ex), by(n)) == INVALID
    # the sink router gates its shared experts with the sink lanes: counts must agree
    scfg = cfg_for("sink")
    ex = abi.MoEExtras()
    ex.num_shared, ex.shared_dim = 1, 64
    ex.shared_gate_up_w = ex.shared_down_w = FAKE
    assert lib.moe_workspace_size_ex(by(scfg), by(ex), by(n)) == INVALID
    ex.num_shared = 2
    assert lib.moe_workspace_size_ex(by(scfg), by(ex), by(n)) == 0
    # shared experts need their weights
    ex.shared_down_w = None
    need = abi.moe_workspace_size(scfg)
    assert lib.moe_forward_ex(by(scfg), by(ex), FAKE, FAKE, None, None, FAKE, None, FAKE, None, FAKE, None, None,
                              None, FAKE, need * 4, None, None) == INVALID


def test_switches_are_read_on_every_call(lib, monkeypatch):
    """Each entry point takes its own snapshot of the MOE_B200_* switches (one
    pass over the environment), so a change between two calls takes effect
    at the next call; unrelated and malformed entries are ignored."""
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "0")
    assert abi.moe_single_launch_ffn() is False
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "1")
    assert abi.moe_single_launch_ffn() is True
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH_X", "0")      # a longer name is another variable
    monkeypatch.setenv("MOE_B200_", "0")
    assert abi.moe_single_launch_ffn() is True
    monkeypatch.delenv("MOE_B200_SINGLE_LAUNCH")
    assert abi.moe_single_launch_ffn() is True
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "")        # empty: the default
    assert abi.moe_single_launch_ffn() is True
