"""The single launch's cross-CTA waits are bounded: when a down tile's
dependency never completes, the launch gives up, records its timeout bits in
the workspace status word, and ends normally; the next call runs as usual.

The wait is made to run out with a test hook that asks for one arrival more
than any gate_up tile will deliver (nothing faults, traps or hangs)."""
import pytest
import torch

from gpu_helpers import LayerRun, run_and_check, to_dev
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

SINK = WORKLOADS["sink"].replace(num_tokens=300, hidden_dim=256, num_experts=32, moe_dim=136)
GPT = WORKLOADS["gptoss"].replace(num_tokens=96, hidden_dim=328, num_experts=16, moe_dim=200)
TIMEOUT_BITS = abi.DEVICE_ERR_TIMEOUT_GEMM1 | abi.DEVICE_ERR_TIMEOUT_GEMM2


@pytest.mark.parametrize("order", ["static", "dynamic", "static_cta_pair"])
@pytest.mark.parametrize("wl", [SINK, GPT], ids=["sink", "gptoss"])
def test_down_tile_wait_gives_up_and_recovers(wl, order, monkeypatch):
    d = to_dev(make_inputs(wl, 21))
    monkeypatch.setenv("MOE_B200_SINGLE_LAUNCH", "1")
    monkeypatch.setenv("MOE_B200_TILE_SCHEDULE", order.split("_")[0])
    monkeypatch.setenv("MOE_B200_CTA_PAIR", "2" if order.endswith("cta_pair") else "1")
    monkeypatch.setenv("MOE_B200_TEST_STALL_DOWN_TILES_MS", "20")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    run = LayerRun(wl, d)
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


def test_csr_grid_barrier_gives_up_and_recovers(monkeypatch):
    """The one-launch CSR build waits at a grid barrier for every chunk's
    counts; with one arrival more requested than any launch delivers, every
    CTA gives up after the hook's limit, records MOE_DEVICE_ERR_TIMEOUT_CSR
    and returns; the next call, without the hook, matches the oracle."""
    import numpy as np

    import oracle
    T, E, k = 8192, 128, 6
    wl = WORKLOADS["tiny"].replace(num_tokens=T, num_experts=E, top_k=k)
    cfg = abi.make_config(wl)
    g = torch.Generator().manual_seed(5)
    idx = torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :k].to(torch.int32).cuda()
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("MOE_B200_CSR_FUSED", "1")
    monkeypatch.setenv("MOE_B200_TEST_STALL_CSR_MS", "20")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    abi.moe_create_indices(cfg, idx, off, perm, None, ws)
    stop.record()
    torch.cuda.synchronize()
    assert abi.moe_device_status(ws) & abi.DEVICE_ERR_TIMEOUT_CSR
    assert start.elapsed_time(stop) < 1000.0
    monkeypatch.delenv("MOE_B200_TEST_STALL_CSR_MS")
    abi.moe_create_indices(cfg, idx, off, perm, None, ws)
    assert abi.moe_device_status(ws) == 0
    _, o_ref, p_ref, _ = oracle.create_indices(idx.cpu().numpy(), E)
    assert np.array_equal(off.cpu().numpy(), o_ref) and np.array_equal(perm.cpu().numpy(), p_ref)
