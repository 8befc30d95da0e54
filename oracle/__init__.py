"""fp64 CPU oracle for the stacked MoE FFN forward pass.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py may import this package.  The product library
(mixture_experts_ffn_token_b200) never imports it and shares no code with it.

Thin numpy wrappers around moe_oracle.cpp (argument marshalling only; all
arithmetic is in the C++ file, which cites the documentation pages it
follows).
"""
import ctypes
import os

import numpy as np

from .build import build_oracle

_lib = None

ACT_CODES = {"silu": 0, "swigluoai": 1, "gelu_tanh": 2}
FORMAT_CODES = {"concatenated": 0, "interleaved": 1}


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_oracle())
        c_i64, c_int, c_dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        _lib.oracle_activation.restype = c_dbl
        _lib.oracle_activation.argtypes = [c_int, c_dbl, c_dbl, c_dbl, c_dbl]
        _lib.oracle_route_softmax_topk.restype = c_int
        _lib.oracle_route_softmax_topk.argtypes = [c_i64, c_int, c_int, vp, c_int, c_i64, vp, vp]
        _lib.oracle_route_sigmoid_sink.restype = c_int
        _lib.oracle_route_sigmoid_sink.argtypes = [c_i64, c_int, c_int, c_int, vp, c_int, c_i64, vp,
                                                   c_dbl, c_dbl, vp, vp, vp]
        _lib.oracle_create_indices.restype = c_int
        _lib.oracle_create_indices.argtypes = [c_i64, c_int, vp, vp, vp, vp, vp]
        _lib.oracle_expert_ffn.restype = c_int
        _lib.oracle_expert_ffn.argtypes = [c_i64, c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp,
                                           c_int, c_int, c_dbl, c_dbl, c_i64, vp, c_int, vp]
        _lib.oracle_expert_ffn_ex.restype = c_int
        _lib.oracle_expert_ffn_ex.argtypes = [c_i64, c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp,
                                              c_int, c_int, c_dbl, c_dbl, c_i64, vp, c_int, c_int, vp, vp]
        _lib.oracle_num_threads.restype = c_int
        _lib.oracle_num_threads.argtypes = []
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a):
    """bf16 data as a contiguous uint16 array of its bit patterns."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return a


def _logits(logits):
    a = np.ascontiguousarray(logits)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.uint16:
        return a, 1
    raise TypeError("logits must be float32 or bf16 bit patterns (uint16)")


def num_threads() -> int:
    return _load().oracle_num_threads()


def activation(kind: str, g: float, u: float, alpha: float = 0.0, limit: float = 0.0) -> float:
    return _load().oracle_activation(ACT_CODES[kind], g, u, alpha, limit)


def route_softmax_topk(logits, num_experts: int, top_k: int):
    """logits [T, stride] (float32, or uint16 bf16 bits) -> (idx [T,k] int32, w [T,k] fp64)."""
    a, is_bf16 = _logits(logits)
    T, stride = a.shape
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    rc = _load().oracle_route_softmax_topk(T, num_experts, top_k, _ptr(a), is_bf16, stride, _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("oracle_route_softmax_topk: bad arguments")
    return idx, w


def route_sigmoid_sink(logits, num_experts: int, num_sink: int, top_k: int, bias=None,
                       route_scale: float = 1.0, global_scale: float = 1.0):
    """-> (idx [T,k] int32, w [T,k] fp64, sink_w [T,S] fp64)."""
    a, is_bf16 = _logits(logits)
    T, stride = a.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    sw = np.empty((T, max(num_sink, 0)), np.float64)
    rc = _load().oracle_route_sigmoid_sink(T, num_experts, num_sink, top_k, _ptr(a), is_bf16, stride, _ptr(b),
                                           route_scale, global_scale, _ptr(idx), _ptr(w), _ptr(sw))
    if rc != 0:
        raise ValueError("oracle_route_sigmoid_sink: bad arguments")
    return idx, w, sw


def create_indices(idx, num_experts: int):
    """idx [T,k] or [R] int32 -> (counts [E], offsets [E+1], perm [R], inv [R])."""
    flat = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1)
    R = flat.size
    counts = np.empty(num_experts, np.int32)
    offsets = np.empty(num_experts + 1, np.int32)
    perm = np.empty(R, np.int32)
    inv = np.empty(R, np.int32)
    rc = _load().oracle_create_indices(R, num_experts, _ptr(flat), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("oracle_create_indices: index out of range")
    return counts, offsets, perm, inv


def expert_ffn(x, idx, w, W_gu, W_d, b_gu=None, b_d=None, gate_up_format="concatenated",
               activation="silu", alpha=0.0, limit=0.0, tokens=None, round_h_bf16=False,
               weight_first=False, token_mask=None):
    """Grouped expert FFN in fp64.

    x [T,H], W_gu [E,H,2D], W_d [E,D,H], b_gu [E,2D], b_d [E,H]: bf16 bit
    patterns (uint16).  idx [T,k] int32, w [T,k] (any float dtype, used as
    fp64).  tokens: optional token ids; the result then has one row per id.
    Returns fp64 [T or len(tokens), H].
    """
    x = _bits16(x)
    T, H = x.shape
    E, H2, N1 = W_gu.shape
    D = N1 // 2
    k = idx.shape[1]
    assert H2 == H and W_d.shape == (E, D, H)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    sel = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n_out = T if sel is None else sel.size
    out = np.empty((n_out, H), np.float64)
    mask = None if token_mask is None else np.ascontiguousarray(token_mask, dtype=np.uint8)
    if mask is not None and mask.size != T:
        raise ValueError("token_mask must have one byte per token")
    rc = _load().oracle_expert_ffn_ex(T, H, E, k, D, _ptr(x), _ptr(idx), _ptr(w), _ptr(_bits16(W_gu)),
                                      _ptr(_bits16(b_gu)), _ptr(_bits16(W_d)), _ptr(_bits16(b_d)),
                                      FORMAT_CODES[gate_up_format], ACT_CODES[activation], alpha, limit,
                                      0 if sel is None else sel.size, _ptr(sel), int(bool(round_h_bf16)),
                                      int(bool(weight_first)), _ptr(mask), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_expert_ffn: bad arguments")
    return out


def shared_expert_ffn(x, gates, Ws_gu, Ws_d, bs_gu=None, bs_d=None, gate_up_format="concatenated",
                      activation="silu", alpha=0.0, limit=0.0, tokens=None, weight_first=False, token_mask=None):
    """Shared experts (StackedMoE has_shared_experts): every token goes through
    all Ns of them; gates [T, Ns] weight them like routing weights (the sink
    router's sink weights, or ones).  Evaluated as the routed FFN with every
    token routed to experts 0..Ns-1."""
    T = x.shape[0]
    Ns = Ws_gu.shape[0]
    idx = np.tile(np.arange(Ns, dtype=np.int32), (T, 1))
    return expert_ffn(x, idx, gates, Ws_gu, Ws_d, bs_gu, bs_d, gate_up_format, activation, alpha, limit,
                      tokens, weight_first=weight_first, token_mask=token_mask)


def forward(x, logits, W_gu, W_d, b_gu=None, b_d=None, *, num_experts, top_k, router="softmax_topk",
            num_sink=0, expert_bias=None, route_scale=1.0, global_scale=1.0, gate_up_format="concatenated",
            activation="silu", alpha=0.0, limit=0.0, tokens=None, weight_first=False, token_mask=None,
            shared=None):
    """Whole layer: router -> expert FFN (+ shared experts).  `shared` is None
    or a dict with Ws_gu, Ws_d (and optional bs_gu, bs_d) of the shared
    experts; their gates are the sink weights (sink router) or ones.
    Returns (out, idx, w, sink_w)."""
    if router == "softmax_topk":
        idx, w = route_softmax_topk(logits, num_experts, top_k)
        sw = np.zeros((idx.shape[0], 0))
    else:
        idx, w, sw = route_sigmoid_sink(logits, num_experts, num_sink, top_k, expert_bias, route_scale, global_scale)
    out = expert_ffn(x, idx, w, W_gu, W_d, b_gu, b_d, gate_up_format, activation, alpha, limit, tokens,
                     weight_first=weight_first, token_mask=token_mask)
    if shared is not None:
        Ns = shared["Ws_gu"].shape[0]
        gates = sw if router == "sigmoid_sink" else np.ones((idx.shape[0], Ns))
        out = out + shared_expert_ffn(x, gates, shared["Ws_gu"], shared["Ws_d"], shared.get("bs_gu"),
                                      shared.get("bs_d"), gate_up_format, activation, alpha, limit, tokens,
                                      weight_first, token_mask)
    return out, idx, w, sw
