"""ctypes binding of the C ABI in include/moe.h.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of libmoe_b200.so.  Tensors are torch tensors already on the device; their
data pointers and the current CUDA stream are passed through unchanged.
There is no fallback: if the library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_DEVICE_TIMEOUT = 5
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT"}
ROUTERS = {"softmax_topk": 0, "sigmoid_sink": 1}
FORMATS = {"concatenated": 0, "interleaved": 1}
ACTIVATIONS = {"silu": 0, "swigluoai": 1, "gelu_tanh": 2}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
DEVICE_ERR_EXPERT_INDEX = 0x1
DEVICE_ERR_CSR = 0x2
DEVICE_ERR_TIMEOUT_GEMM1 = 0x4
DEVICE_ERR_TIMEOUT_GEMM2 = 0x8
DEVICE_ERR_TIMEOUT_CSR = 0x10
DEVICE_ERR_LAUNCH = 0x20
NUM_STAGE_EVENTS = 9
STAGE_NAMES = ("router", "csr_count", "csr_scan", "csr_scatter", "gather", "gemm_gate_up", "gemm_down", "combine")

EXPORTED = ("moe_status_string", "moe_workspace_size", "moe_route", "moe_create_indices", "moe_grouped_ffn",
            "moe_forward", "moe_forward_timed", "moe_device_status", "moe_create_indices_noalloc",
            "moe_workspace_size_ex", "moe_forward_ex", "moe_single_launch_ffn")
NUM_STAGE_EVENTS_EX = 13
STAGE_NAMES_EX = ("router", "csr_count", "csr_scan", "csr_scatter", "gather", "gemm_gate_up", "gemm_down",
                  "shared_index", "shared_gather", "shared_gemm_gate_up", "shared_gemm_down", "combine")


class MoEConfig(ctypes.Structure):
    """moe_config_t."""
    _fields_ = [
        ("num_tokens", ctypes.c_int32),
        ("hidden_dim", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("moe_dim", ctypes.c_int32),
        ("num_sink", ctypes.c_int32),
        ("router", ctypes.c_int),
        ("logits_dtype", ctypes.c_int),
        ("logits_row_stride", ctypes.c_int64),
        ("route_scale", ctypes.c_float),
        ("gate_up_format", ctypes.c_int),
        ("activation", ctypes.c_int),
        ("alpha", ctypes.c_float),
        ("limit", ctypes.c_float),
        ("has_bias", ctypes.c_int32),
    ]


class MoEExtras(ctypes.Structure):
    """moe_extras_t."""
    _fields_ = [
        ("token_mask", ctypes.c_void_p),
        ("apply_router_weight_first", ctypes.c_int32),
        ("num_shared", ctypes.c_int32),
        ("shared_dim", ctypes.c_int32),
        ("shared_gate_up_w", ctypes.c_void_p),
        ("shared_gate_up_b", ctypes.c_void_p),
        ("shared_down_w", ctypes.c_void_p),
        ("shared_down_b", ctypes.c_void_p),
    ]


def make_extras(token_mask=None, apply_router_weight_first=False, shared_gate_up_w=None, shared_down_w=None,
                shared_gate_up_b=None, shared_down_b=None) -> MoEExtras:
    """moe_extras_t from torch tensors (shared weights [Ns, H, 2Ds] / [Ns, Ds, H])."""
    ex = MoEExtras()
    ex.token_mask = None if token_mask is None else token_mask.data_ptr()
    ex.apply_router_weight_first = 1 if apply_router_weight_first else 0
    if shared_gate_up_w is not None:
        ex.num_shared = shared_gate_up_w.shape[0]
        ex.shared_dim = shared_gate_up_w.shape[2] // 2
        ex.shared_gate_up_w = shared_gate_up_w.data_ptr()
        ex.shared_down_w = shared_down_w.data_ptr()
        ex.shared_gate_up_b = None if shared_gate_up_b is None else shared_gate_up_b.data_ptr()
        ex.shared_down_b = None if shared_down_b is None else shared_down_b.data_ptr()
    return ex


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load_library():
    """Load libmoe_b200.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError(f"{LIB_PATH} is missing: build it with `python -m mixture_experts_ffn_token_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, cfgp, sz = ctypes.c_void_p, ctypes.POINTER(MoEConfig), ctypes.c_size_t
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_workspace_size.restype = ctypes.c_int
    lib.moe_workspace_size.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_route.restype = ctypes.c_int
    lib.moe_route.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp]
    lib.moe_create_indices.restype = ctypes.c_int
    lib.moe_create_indices.argtypes = [cfgp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_grouped_ffn.restype = ctypes.c_int
    lib.moe_grouped_ffn.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_forward.restype = ctypes.c_int
    lib.moe_forward.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_forward_timed.restype = ctypes.c_int
    lib.moe_forward_timed.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.moe_device_status.restype = ctypes.c_int
    lib.moe_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
    lib.moe_create_indices_noalloc.restype = ctypes.c_int
    lib.moe_create_indices_noalloc.argtypes = [cfgp, vp, vp, vp, vp, vp]
    exp = ctypes.POINTER(MoEExtras)
    lib.moe_workspace_size_ex.restype = ctypes.c_int
    lib.moe_workspace_size_ex.argtypes = [cfgp, exp, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_forward_ex.restype = ctypes.c_int
    lib.moe_forward_ex.argtypes = [cfgp, exp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.moe_single_launch_ffn.restype = ctypes.c_int
    lib.moe_single_launch_ffn.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    _lib = lib
    return lib


def config(num_tokens: int, hidden_dim: int, num_experts: int, top_k: int, moe_dim: int, *,
           router: str = "softmax_topk", num_sink: int = 0, logits_dtype=torch.float32,
           logits_row_stride: Optional[int] = None, route_scale: float = 1.0,
           gate_up_format: str = "concatenated", activation: str = "silu", alpha: float = 0.0,
           limit: float = 0.0, has_bias: bool = False) -> MoEConfig:
    """moe_config_t from keyword arguments (names as in include/moe.h; router
    "softmax_topk" | "sigmoid_sink", gate_up_format "concatenated" |
    "interleaved", activation "silu" | "swigluoai" | "gelu_tanh")."""
    c = MoEConfig()
    c.num_tokens = num_tokens
    c.hidden_dim = hidden_dim
    c.num_experts = num_experts
    c.top_k = top_k
    c.moe_dim = moe_dim
    c.num_sink = num_sink
    c.router = ROUTERS[router]
    c.logits_dtype = DTYPES[logits_dtype]
    c.logits_row_stride = num_experts + num_sink if logits_row_stride is None else logits_row_stride
    c.route_scale = route_scale
    c.gate_up_format = FORMATS[gate_up_format]
    c.activation = ACTIVATIONS[activation]
    c.alpha = alpha
    c.limit = limit
    c.has_bias = 1 if has_bias else 0
    return c


def make_config(wl, num_tokens: Optional[int] = None, logits_dtype=torch.float32,
                logits_row_stride: Optional[int] = None) -> MoEConfig:
    """moe_config_t for a workloads.Workload (num_tokens overrides wl's T)."""
    return config(wl.num_tokens if num_tokens is None else num_tokens, wl.hidden_dim, wl.num_experts, wl.top_k,
                  wl.moe_dim, router=wl.router, num_sink=wl.num_sink, logits_dtype=logits_dtype,
                  logits_row_stride=logits_row_stride, route_scale=wl.route_scale,
                  gate_up_format=wl.gate_up_format, activation=wl.activation, alpha=wl.alpha, limit=wl.limit,
                  has_bias=wl.has_bias)


def _p(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_status_string(status: int) -> str:
    return load_library().moe_status_string(status).decode()


def moe_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_route(cfg, logits, expert_indices, expert_weights, sink_weights=None, expert_bias=None,
              global_scale=None, stream=None):
    _check(load_library().moe_route(ctypes.byref(cfg), _p(logits), _p(expert_bias), _p(global_scale),
                                    _p(expert_indices), _p(expert_weights), _p(sink_weights), _stream(stream)),
           "moe_route")


def moe_create_indices(cfg, expert_indices, expert_offsets, permutation, inverse, workspace, stream=None):
    _check(load_library().moe_create_indices(ctypes.byref(cfg), _p(expert_indices), _p(expert_offsets),
                                             _p(permutation), _p(inverse), _p(workspace), workspace.numel(),
                                             _stream(stream)), "moe_create_indices")


def moe_create_indices_noalloc(cfg, expert_indices, expert_offsets, permutation, inverse=None, stream=None):
    """moe_create_indices with its scratch in the library's fixed device array
    (for callers that cannot allocate a workspace)."""
    _check(load_library().moe_create_indices_noalloc(ctypes.byref(cfg), _p(expert_indices), _p(expert_offsets),
                                                     _p(permutation), _p(inverse), _stream(stream)),
           "moe_create_indices_noalloc")


def moe_grouped_ffn(cfg, x, gate_up_w, gate_up_b, down_w, down_b, expert_offsets, permutation, expert_weights,
                    out, workspace, stream=None):
    _check(load_library().moe_grouped_ffn(ctypes.byref(cfg), _p(x), _p(gate_up_w), _p(gate_up_b), _p(down_w),
                                          _p(down_b), _p(expert_offsets), _p(permutation), _p(expert_weights),
                                          _p(out), _p(workspace), workspace.numel(), _stream(stream)),
           "moe_grouped_ffn")


def moe_forward(cfg, x, logits, gate_up_w, down_w, out, workspace, gate_up_b=None, down_b=None, expert_bias=None,
                global_scale=None, expert_indices_out=None, expert_weights_out=None, sink_weights_out=None,
                stream=None):
    _check(load_library().moe_forward(ctypes.byref(cfg), _p(x), _p(logits), _p(expert_bias), _p(global_scale),
                                      _p(gate_up_w), _p(gate_up_b), _p(down_w), _p(down_b), _p(out),
                                      _p(expert_indices_out), _p(expert_weights_out), _p(sink_weights_out),
                                      _p(workspace), workspace.numel(), _stream(stream)), "moe_forward")


class BoundForward:
    """moe_forward (or, with `extras`, moe_forward_ex) bound to fixed tensors
    and a stream: the argument marshalling happens once, and each call()
    runs the C entry point itself -- validation, workspace checks and every
    kernel launch happen on every call, as with moe_forward.  The object
    keeps its tensors alive; bind again for other buffers or another
    stream."""

    def __init__(self, cfg, x, logits, gate_up_w, down_w, out, workspace, gate_up_b=None, down_b=None,
                 expert_bias=None, global_scale=None, expert_indices_out=None, expert_weights_out=None,
                 sink_weights_out=None, extras=None, stream=None):
        lib = load_library()
        self._keep = (cfg, x, logits, gate_up_w, down_w, out, workspace, gate_up_b, down_b, expert_bias,
                      global_scale, expert_indices_out, expert_weights_out, sink_weights_out, extras)
        common = (_p(x), _p(logits), _p(expert_bias), _p(global_scale), _p(gate_up_w), _p(gate_up_b), _p(down_w),
                  _p(down_b), _p(out), _p(expert_indices_out), _p(expert_weights_out), _p(sink_weights_out),
                  _p(workspace), workspace.numel(), _stream(stream))
        if extras is None:
            self._fn, self._where = lib.moe_forward, "moe_forward"
            self._args = (ctypes.byref(cfg),) + common
        else:
            self._fn, self._where = lib.moe_forward_ex, "moe_forward_ex"
            self._args = (ctypes.byref(cfg), ctypes.byref(extras)) + common + (None,)

    def __call__(self):
        st = self._fn(*self._args)
        if st != MOE_OK:
            raise MoEError(st, self._where)


def _event_handles(events, stream):
    """cudaEvent_t handles of torch.cuda.Event objects (None stays NULL)."""
    handles = []
    for ev in events:
        if ev is None:
            handles.append(None)
            continue
        if ev.cuda_event == 0:      # torch creates the CUDA event on its first record
            ev.record(stream)
        handles.append(ev.cuda_event)
    return handles


def moe_forward_timed(cfg, events, x, logits, gate_up_w, down_w, out, workspace, gate_up_b=None, down_b=None,
                      expert_bias=None, global_scale=None, expert_indices_out=None, expert_weights_out=None,
                      sink_weights_out=None, stream=None):
    """moe_forward recording torch.cuda.Event objects `events` (9, None
    entries skipped) between stages."""
    if len(events) != NUM_STAGE_EVENTS:
        raise ValueError(f"moe_forward_timed needs {NUM_STAGE_EVENTS} events")
    arr = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*_event_handles(events, stream))
    _check(load_library().moe_forward_timed(ctypes.byref(cfg), _p(x), _p(logits), _p(expert_bias),
                                            _p(global_scale), _p(gate_up_w), _p(gate_up_b), _p(down_w), _p(down_b),
                                            _p(out), _p(expert_indices_out), _p(expert_weights_out),
                                            _p(sink_weights_out), _p(workspace), workspace.numel(),
                                            _stream(stream), arr), "moe_forward_timed")


def moe_single_launch_ffn() -> bool:
    """Whether the two grouped GEMMs run as one launch in this process (set
    MOE_B200_SINGLE_LAUNCH=0 in the environment for two launches)."""
    v = ctypes.c_int32(0)
    _check(load_library().moe_single_launch_ffn(ctypes.byref(v)), "moe_single_launch_ffn")
    return bool(v.value)


def moe_workspace_size_ex(cfg: MoEConfig, extras: Optional[MoEExtras]) -> int:
    n = ctypes.c_size_t(0)
    ex = None if extras is None else ctypes.byref(extras)
    _check(load_library().moe_workspace_size_ex(ctypes.byref(cfg), ex, ctypes.byref(n)), "moe_workspace_size_ex")
    return n.value


def moe_forward_ex(cfg, extras, x, logits, gate_up_w, down_w, out, workspace, gate_up_b=None, down_b=None,
                   expert_bias=None, global_scale=None, expert_indices_out=None, expert_weights_out=None,
                   sink_weights_out=None, events=None, stream=None):
    """moe_forward with token mask / router weight first / shared experts
    (`extras`, a MoEExtras or None); `events`: None or 13 torch.cuda.Event."""
    arr = None
    if events is not None:
        if len(events) != NUM_STAGE_EVENTS_EX:
            raise ValueError(f"moe_forward_ex needs {NUM_STAGE_EVENTS_EX} events")
        arr = (ctypes.c_void_p * NUM_STAGE_EVENTS_EX)(*_event_handles(events, stream))
    ex = None if extras is None else ctypes.byref(extras)
    _check(load_library().moe_forward_ex(ctypes.byref(cfg), ex, _p(x), _p(logits), _p(expert_bias),
                                         _p(global_scale), _p(gate_up_w), _p(gate_up_b), _p(down_w), _p(down_b),
                                         _p(out), _p(expert_indices_out), _p(expert_weights_out),
                                         _p(sink_weights_out), _p(workspace), workspace.numel(), _stream(stream),
                                         arr), "moe_forward_ex")


def moe_device_status(workspace, stream=None) -> int:
    """The device fault bits recorded in the workspace (synchronizes the stream)."""
    v = ctypes.c_int32(0)
    st = load_library().moe_device_status(_p(workspace), ctypes.byref(v), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE_TIMEOUT):
        raise MoEError(st, "moe_device_status")
    return v.value
