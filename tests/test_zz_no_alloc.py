"""moe_create_indices_noalloc: the CSR build for callers that cannot allocate
device memory (a host runtime that owns all device memory and gives plugins
no allocator, or a latency-critical path that cannot afford cudaMalloc's
implicit synchronisation).  Its scratch is one fixed array in device memory
that every call shares, so the test makes several calls in a row and checks
each against moe_create_indices (which takes a caller workspace) and against
the oracle's counting sort: offsets, permutation and inverse must be
identical, as for any index output.  It also checks the property the entry
point exists for: once the first call has set it up, further calls change
neither the free device memory nor torch's allocations.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_token_b200 import abi
from mixture_experts_ffn_token_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :k].to(torch.int32).cuda()


def _with_workspace(cfg, idx, E, R):
    ws = torch.empty(abi.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    abi.moe_create_indices(cfg, idx, off, perm, inv, ws)
    return off, perm, inv


def _without_workspace(cfg, idx, E, R):
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    perm = torch.full((R,), -1, dtype=torch.int32, device="cuda")
    inv = torch.full((R,), -1, dtype=torch.int32, device="cuda")
    abi.moe_create_indices_noalloc(cfg, idx, off, perm, inv)
    return off, perm, inv


def _check_against_oracle(got, idx, E):
    _, off_ref, perm_ref, inv_ref = oracle.create_indices(idx.cpu().numpy(), E)
    off, perm, inv = (t.cpu().numpy() for t in got)
    assert np.array_equal(off, off_ref)
    assert np.array_equal(perm, perm_ref)
    assert np.array_equal(inv, inv_ref)


def test_noalloc_matches_workspace_version_and_oracle_on_consecutive_calls():
    # large, small, then large again: each call must not see the previous
    # call's leftovers in the shared scratch
    cases = [(8192, 128, 6, 11), (300, 16, 4, 12), (8192, 128, 6, 13), (1, 1, 1, 14)]
    for T, E, k, seed in cases:
        wl = WORKLOADS["tiny"].replace(num_tokens=T, num_experts=E, top_k=k)
        cfg = abi.make_config(wl)
        idx = _routing(T, E, k, seed)
        ref = _with_workspace(cfg, idx, E, T * k)
        got = _without_workspace(cfg, idx, E, T * k)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b), (T, E, k)
        _check_against_oracle(got, idx, E)


def test_noalloc_calls_allocate_nothing():
    T, E, k = 8192, 128, 6
    wl = WORKLOADS["tiny"].replace(num_tokens=T, num_experts=E, top_k=k)
    cfg = abi.make_config(wl)
    idx = _routing(T, E, k, 16)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    abi.moe_create_indices_noalloc(cfg, idx, off, perm, inv)  # set-up call
    torch.cuda.synchronize()
    free0, allocated0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(5):
        abi.moe_create_indices_noalloc(cfg, idx, off, perm, inv)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == allocated0
    _check_against_oracle((off, perm, inv), idx, E)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = abi.load_library()
    # ceil(R / 2048) * E = 513 * 128 > 65536 cells
    wl = WORKLOADS["tiny"].replace(num_tokens=175104, num_experts=128, top_k=6)
    cfg = abi.make_config(wl)
    fake = ctypes.c_void_p(0x10000)
    st = lib.moe_create_indices_noalloc(ctypes.byref(cfg), fake, fake, fake, None, None)
    assert st == 3  # MOE_ERR_WORKSPACE_TOO_SMALL, before anything is enqueued
    # exactly at the limit is accepted (512 chunks x 128 experts)
    wl = WORKLOADS["tiny"].replace(num_tokens=174762, num_experts=128, top_k=6)
    cfg = abi.make_config(wl)
    idx = _routing(174762, 128, 6, 15)
    got = _without_workspace(cfg, idx, 128, 174762 * 6)
    ref = _with_workspace(cfg, idx, 128, 174762 * 6)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    _check_against_oracle(got, idx, 128)
