"""The single launch's cross-CTA waits are bounded: when a down tile's
dependency never completes, the launch gives up, records its timeout bits in
the workspace status word, and ends normally; the next call runs as usual.

The wait is made to run out with a test hook that asks for one arrival more
than any gate_up tile will deliver (nothing faults, traps or hangs)."""
import pytest
import torch

from gpu_helpers import GpuRun, run_and_check, to_dev
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

SINK = WORKLOADS["sink"].replace(num_tokens=300, hidden_dim=256, num_experts=32, moe_dim=136)
GPT = WORKLOADS["gptoss"].replace(num_tokens=96, hidden_dim=328, num_experts=16, moe_dim=200)
TIMEOUT_BITS = abi.DEVICE_ERR_TIMEOUT_GEMM1 | abi.DEVICE_ERR_TIMEOUT_GEMM2


@pytest.mark.parametrize("order", ["static", "dynamic"])
@pytest.mark.parametrize("wl", [SINK, GPT], ids=["sink", "gptoss"])
def test_down_tile_wait_gives_up_and_recovers(wl, order, monkeypatch):
    d = to_dev(make_inputs(wl, 21))
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "1")
    monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order)
    monkeypatch.setenv("MOE_B200_TEST_STALL_DOWN_TILES_MS", "20")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    run = GpuRun(wl, d)
    stop.record()
    torch.cuda.synchronize()
    assert run.status & TIMEOUT_BITS == TIMEOUT_BITS, f"status {run.status:#x}"
    # every CTA stopped within a few of its 20 ms limits, not the 2 s default
    assert start.elapsed_time(stop) < 1000.0
    # the C entry point reports the timeout as a status code
    import ctypes
    v = ctypes.c_int32(0)
    st = abi.load_library().moe_device_status(run.ws.data_ptr(), ctypes.byref(v), None)
    assert st == abi.MOE_ERR_DEVICE_TIMEOUT and v.value & TIMEOUT_BITS == TIMEOUT_BITS
    # the context is intact: the same call without the hook is correct again
    monkeypatch.delenv("MOE_B200_TEST_STALL_DOWN_TILES_MS")
    run_and_check(wl, seed=21)
