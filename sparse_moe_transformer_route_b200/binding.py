"""ctypes binding of libmoe_b200.so, with the C ABI's names (include/moe.h).

Argument marshalling only: every function checks that tensors have the dtype,
device and contiguity the C side expects, passes raw pointers and the current
CUDA stream, and turns a non-zero status into MoeError. No step of the layer
runs here. The library must be built (python -m sparse_moe_transformer_route_b200.build);
without it every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

ABI_VERSION = 6  # MOE_ABI_VERSION of include/moe.h this binding marshals for
MOE_BF16 = 0
MOE_FP32 = 1
MOE_ROUTER_SOFTMAX_TOPK = 0
MOE_ROUTER_RENORM = 1
ROW_ALIGN = 128

STATUS_NAMES = {
    0: "MOE_OK",
    1: "MOE_ERR_INVALID_ARG",
    2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL",
    4: "MOE_ERR_CUDA",
    5: "MOE_ERR_DEVICE_CHECK",
    6: "MOE_ERR_NO_DEVICE",
}

# Every symbol the header declares, in declaration order.
EXPORTS = (
    "moe_status_string", "moe_abi_version", "moe_check_config", "moe_padded_rows",
    "moe_workspace_bytes", "moe_workspace_init", "moe_route", "moe_route_static", "moe_dispatch",
    "moe_expert_gate_up", "moe_expert_down", "moe_expert_ffn", "moe_combine", "moe_forward",
    "moe_forward_decode", "moe_forward_host", "moe_forward_host_async", "moe_backward", "moe_rmsnorm", "moe_combine_residual",
    "moe_stack_forward", "moe_stack_forward_trace", "moe_expert_choice_capacity", "moe_route_expert_choice",
    "moe_forward_expert_choice", "moe_set_stage_events", "moe_get_device_status",
)
STAGE_EVENTS = 6
STAGES = ("router", "dispatch", "gate_up", "down", "combine")


class MoeError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class moe_config(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("d_model", ctypes.c_int32),
        ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("d_ff", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("alpha_lb", ctypes.c_float),
        ("beta_z", ctypes.c_float),
        ("grad_dtype", ctypes.c_int32),
        ("router_mode", ctypes.c_int32),
    ]


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(moe_config)
_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "moe_abi_version": (ctypes.c_int32, []),
    "moe_check_config": (ctypes.c_int, [_CFG]),
    "moe_padded_rows": (ctypes.c_int64, [_CFG]),
    "moe_workspace_bytes": (ctypes.c_size_t, [_CFG, ctypes.c_int32]),
    "moe_workspace_init": (ctypes.c_int, [_P, _P]),
    "moe_route": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_route_static": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_gate_up": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_down": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P,
                                   ctypes.c_size_t, _P]),
    "moe_forward_decode": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_forward_host": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_forward_host_async": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_backward": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_rmsnorm": (ctypes.c_int, [_CFG, _P, _P, ctypes.c_float, _P, _P]),
    "moe_combine_residual": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
    "moe_stack_forward": (ctypes.c_int, [_CFG, ctypes.c_int32, _P, _P, _P, _P, _P, _P,
                                         ctypes.c_size_t, _P]),
    "moe_stack_forward_trace": (ctypes.c_int, [_CFG, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               ctypes.c_size_t, _P]),
    "moe_expert_choice_capacity": (ctypes.c_int64, [_CFG]),
    "moe_route_expert_choice": (ctypes.c_int, [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               ctypes.c_size_t, _P]),
    "moe_forward_expert_choice": (ctypes.c_int, [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                 ctypes.c_size_t, _P]),
    "moe_set_stage_events": (ctypes.c_int, [_P]),
    "moe_get_device_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
}


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m sparse_moe_transformer_route_b200.build`"
            )
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.moe_abi_version() != ABI_VERSION:
            raise RuntimeError(f"{LIB_PATH} implements ABI {L.moe_abi_version()}, this binding ABI {ABI_VERSION}: "
                               "rebuild with `python -m sparse_moe_transformer_route_b200.build`")
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(status, where):
    if status != 0:
        raise MoeError(status, where)


def config(T, d_model, n_experts, top_k, d_ff, dtype=torch.bfloat16, alpha_lb=0.01, beta_z=0.001,
           grad_dtype=None, renorm=False):
    """A moe_config. `dtype` is torch.bfloat16 or torch.float32; `grad_dtype`, the
    type of the weight gradients moe_backward writes, defaults to `dtype`;
    `renorm` selects the renormalised top-k weights (MOE_ROUTER_RENORM)."""
    grad_dtype = dtype if grad_dtype is None else grad_dtype
    for t in (dtype, grad_dtype):
        if t not in (torch.bfloat16, torch.float32):
            raise ValueError("dtypes must be torch.bfloat16 or torch.float32")
    code = lambda t: MOE_BF16 if t == torch.bfloat16 else MOE_FP32
    return moe_config(int(T), int(d_model), int(n_experts), int(top_k), int(d_ff), code(dtype), float(alpha_lb),
                      float(beta_z), code(grad_dtype), 1 if renorm else 0)


def torch_dtype(cfg) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == MOE_BF16 else torch.float32


def grad_torch_dtype(cfg) -> torch.dtype:
    """The dtype of the weight gradients moe_backward writes for `cfg`."""
    return torch.float32 if (cfg.dtype == MOE_FP32 or cfg.grad_dtype == MOE_FP32) else torch.bfloat16


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, dtype=None, shape=None, name="tensor", allow_none=False, device=True):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not device and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    return ctypes.c_void_p(t.data_ptr())


def _cfgp(cfg):
    return ctypes.byref(cfg)


# ---------------------------------------------------------------- sizes


def moe_check_config(cfg) -> int:
    return lib().moe_check_config(_cfgp(cfg))


def moe_padded_rows(cfg) -> int:
    return lib().moe_padded_rows(_cfgp(cfg))


def moe_workspace_bytes(cfg, for_backward=False) -> int:
    return lib().moe_workspace_bytes(_cfgp(cfg), 1 if for_backward else 0)


def moe_workspace_init(ws, stream=None):
    _check(lib().moe_workspace_init(_ptr(ws, torch.uint8, name="ws"), _stream(stream)), "moe_workspace_init")


def workspace(cfg, for_backward=False, device="cuda"):
    """Allocate (torch) and initialise a workspace for cfg."""
    n = moe_workspace_bytes(cfg, for_backward)
    if n == 0:
        _check(moe_check_config(cfg) or 2, "moe_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


# ---------------------------------------------------------------- stages


def moe_route(cfg, x, w_router, router_bias, topk_idx, topk_w, counts, losses, ws, stream=None):
    dt = torch_dtype(cfg)
    T, d, E, k = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k
    st = lib().moe_route(
        _cfgp(cfg), _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(topk_idx, torch.int32, (T, k), "topk_idx"), _ptr(topk_w, torch.float32, (T, k), "topk_w"),
        _ptr(counts, torch.int32, (E,), "counts", allow_none=True),
        _ptr(losses, torch.float32, (2,), "losses", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_route")


def moe_route_static(cfg, x, w_router, router_bias, topk_idx, topk_w, counts, losses, stream=None):
    """moe_route on the library's own fixed scratch: no workspace, no allocation.
    For callers that cannot provide device memory; see include/moe.h for the
    size limit and the sharing rules (one array per device, calls must not overlap)."""
    dt = torch_dtype(cfg)
    T, d, E, k = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k
    st = lib().moe_route_static(
        _cfgp(cfg), _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(topk_idx, torch.int32, (T, k), "topk_idx"), _ptr(topk_w, torch.float32, (T, k), "topk_w"),
        _ptr(counts, torch.int32, (E,), "counts", allow_none=True),
        _ptr(losses, torch.float32, (2,), "losses", allow_none=True), _stream(stream))
    _check(st, "moe_route_static")


def moe_dispatch(cfg, topk_idx, x, offsets, perm, inv_perm, group_start, x_perm, ws, stream=None):
    dt = torch_dtype(cfg)
    T, d, E, k = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k
    P = moe_padded_rows(cfg)
    st = lib().moe_dispatch(
        _cfgp(cfg), _ptr(topk_idx, torch.int32, (T, k), "topk_idx"), _ptr(x, dt, (T, d), "x"),
        _ptr(offsets, torch.int32, (E + 1,), "offsets"), _ptr(perm, torch.int32, (T * k,), "perm"),
        _ptr(inv_perm, torch.int32, (T * k,), "inv_perm"),
        _ptr(group_start, torch.int32, (E + 1,), "group_start"), _ptr(x_perm, dt, (P, d), "x_perm"),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_dispatch")


def moe_expert_gate_up(cfg, x_perm, group_start, offsets, w_gate_up, h, preact, ws, stream=None):
    dt = torch_dtype(cfg)
    d, E, f = cfg.d_model, cfg.n_experts, cfg.d_ff
    P = moe_padded_rows(cfg)
    st = lib().moe_expert_gate_up(
        _cfgp(cfg), _ptr(x_perm, dt, (P, d), "x_perm"), _ptr(group_start, torch.int32, (E + 1,), "group_start"),
        _ptr(offsets, torch.int32, (E + 1,), "offsets"), _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"),
        _ptr(h, dt, (P, f), "h"), _ptr(preact, torch.float32, (P, 2 * f), "preact", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_expert_gate_up")


def moe_expert_down(cfg, h, group_start, offsets, w_down, o_perm, ws, stream=None):
    dt = torch_dtype(cfg)
    d, E, f = cfg.d_model, cfg.n_experts, cfg.d_ff
    P = moe_padded_rows(cfg)
    st = lib().moe_expert_down(
        _cfgp(cfg), _ptr(h, dt, (P, f), "h"), _ptr(group_start, torch.int32, (E + 1,), "group_start"),
        _ptr(offsets, torch.int32, (E + 1,), "offsets"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(o_perm, dt, (P, d), "o_perm"), _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_expert_down")


def moe_expert_ffn(cfg, x_perm, group_start, offsets, w_gate_up, w_down, h, o_perm, ws, stream=None):
    dt = torch_dtype(cfg)
    d, E, f = cfg.d_model, cfg.n_experts, cfg.d_ff
    P = moe_padded_rows(cfg)
    st = lib().moe_expert_ffn(
        _cfgp(cfg), _ptr(x_perm, dt, (P, d), "x_perm"), _ptr(group_start, torch.int32, (E + 1,), "group_start"),
        _ptr(offsets, torch.int32, (E + 1,), "offsets"), _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"),
        _ptr(w_down, dt, (E, d, f), "w_down"), _ptr(h, dt, (P, f), "h"), _ptr(o_perm, dt, (P, d), "o_perm"),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_expert_ffn")


def moe_combine(cfg, o_perm, inv_perm, topk_w, y, stream=None):
    dt = torch_dtype(cfg)
    T, d, k = cfg.T, cfg.d_model, cfg.top_k
    P = moe_padded_rows(cfg)
    st = lib().moe_combine(
        _cfgp(cfg), _ptr(o_perm, dt, (P, d), "o_perm"), _ptr(inv_perm, torch.int32, (T * k,), "inv_perm"),
        _ptr(topk_w, torch.float32, (T, k), "topk_w"), _ptr(y, dt, (T, d), "y"), _stream(stream))
    _check(st, "moe_combine")


def moe_combine_residual(cfg, o_perm, inv_perm, topk_w, resid, stream=None):
    dt = torch_dtype(cfg)
    T, d, k = cfg.T, cfg.d_model, cfg.top_k
    P = moe_padded_rows(cfg)
    st = lib().moe_combine_residual(
        _cfgp(cfg), _ptr(o_perm, dt, (P, d), "o_perm"), _ptr(inv_perm, torch.int32, (T * k,), "inv_perm"),
        _ptr(topk_w, torch.float32, (T, k), "topk_w"), _ptr(resid, torch.float32, (T, d), "resid"),
        _stream(stream))
    _check(st, "moe_combine_residual")


def moe_rmsnorm(cfg, resid, weight, eps, out, stream=None):
    dt = torch_dtype(cfg)
    T, d = cfg.T, cfg.d_model
    st = lib().moe_rmsnorm(
        _cfgp(cfg), _ptr(resid, torch.float32, (T, d), "resid"),
        _ptr(weight, torch.float32, (d,), "weight", allow_none=True), float(eps), _ptr(out, dt, (T, d), "out"),
        _stream(stream))
    _check(st, "moe_rmsnorm")


# ---------------------------------------------------------------- whole layer


def moe_forward(cfg, x, w_router, router_bias, w_gate_up, w_down, y, losses, topk_idx, topk_w,
                save_for_backward, ws, stream=None):
    dt = torch_dtype(cfg)
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff
    st = lib().moe_forward(
        _cfgp(cfg), _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(y, dt, (T, d), "y"), _ptr(losses, torch.float32, (2,), "losses", allow_none=True),
        _ptr(topk_idx, torch.int32, (T, k), "topk_idx", allow_none=True),
        _ptr(topk_w, torch.float32, (T, k), "topk_w", allow_none=True),
        1 if save_for_backward else 0, _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_forward")


def moe_forward_decode(cfg, x, w_router, router_bias, w_gate_up, w_down, y, losses, topk_idx, topk_w, ws,
                       stream=None):
    """The one-kernel decode layer (T <= 8); moe_forward picks it by itself when
    nothing is saved for the backward."""
    dt = torch_dtype(cfg)
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff
    st = lib().moe_forward_decode(
        _cfgp(cfg), _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(y, dt, (T, d), "y"), _ptr(losses, torch.float32, (2,), "losses", allow_none=True),
        _ptr(topk_idx, torch.int32, (T, k), "topk_idx", allow_none=True),
        _ptr(topk_w, torch.float32, (T, k), "topk_w", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_forward_decode")


def moe_expert_choice_capacity(cfg) -> int:
    """Default expert-choice capacity ceil(T*k/E), capped at T."""
    c = lib().moe_expert_choice_capacity(_cfgp(cfg))
    if c < 0:
        raise MoeError(2, "moe_expert_choice_capacity")
    return c


def moe_route_expert_choice(cfg, x, w_router, router_bias, sel, gates, probs, counts, losses, ws, capacity=0,
                            stream=None):
    dt = torch_dtype(cfg)
    T, d, E = cfg.T, cfg.d_model, cfg.n_experts
    C = capacity if capacity > 0 else moe_expert_choice_capacity(cfg)
    st = lib().moe_route_expert_choice(
        _cfgp(cfg), capacity, _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(sel, torch.int32, (E, C), "sel"), _ptr(gates, torch.float32, (E, C), "gates"),
        _ptr(probs, torch.float32, (T, E), "probs", allow_none=True),
        _ptr(counts, torch.int32, (E,), "counts", allow_none=True),
        _ptr(losses, torch.float32, (2,), "losses", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_route_expert_choice")


def moe_forward_expert_choice(cfg, x, w_router, router_bias, w_gate_up, w_down, y, losses, sel, gates, ws,
                              capacity=0, stream=None):
    dt = torch_dtype(cfg)
    T, d, E, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff
    C = capacity if capacity > 0 else moe_expert_choice_capacity(cfg)
    st = lib().moe_forward_expert_choice(
        _cfgp(cfg), capacity, _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(y, dt, (T, d), "y"), _ptr(losses, torch.float32, (2,), "losses", allow_none=True),
        _ptr(sel, torch.int32, (E, C), "sel", allow_none=True),
        _ptr(gates, torch.float32, (E, C), "gates", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_forward_expert_choice")


def moe_forward_host(cfg, x_host, w_router, router_bias, w_gate_up, w_down, y_host, losses_host, ws,
                     stream=None):
    dt = torch_dtype(cfg)
    T, d, E, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff
    st = lib().moe_forward_host(
        _cfgp(cfg), _ptr(x_host, dt, (T, d), "x_host", device=False), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(y_host, dt, (T, d), "y_host", device=False),
        _ptr(losses_host, torch.float32, (2,), "losses_host", allow_none=True, device=False),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_forward_host")


def moe_forward_host_async(cfg, x_host, w_router, router_bias, w_gate_up, w_down, y_host, losses_host, ws,
                           stream=None):
    """moe_forward_host without the final synchronisation: the results are in
    y_host / losses_host once `stream`'s queued work has completed."""
    dt = torch_dtype(cfg)
    T, d, E, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff
    st = lib().moe_forward_host_async(
        _cfgp(cfg), _ptr(x_host, dt, (T, d), "x_host", device=False), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(router_bias, torch.float32, (E,), "router_bias", allow_none=True),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(y_host, dt, (T, d), "y_host", device=False),
        _ptr(losses_host, torch.float32, (2,), "losses_host", allow_none=True, device=False),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_forward_host_async")


def moe_backward(cfg, dy, x, w_router, w_gate_up, w_down, dx, dw_router, dw_gate_up, dw_down, ws,
                 stream=None):
    dt = torch_dtype(cfg)
    gt = grad_torch_dtype(cfg)
    T, d, E, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff
    st = lib().moe_backward(
        _cfgp(cfg), _ptr(dy, dt, (T, d), "dy"), _ptr(x, dt, (T, d), "x"), _ptr(w_router, dt, (E, d), "w_router"),
        _ptr(w_gate_up, dt, (E, 2 * f, d), "w_gate_up"), _ptr(w_down, dt, (E, d, f), "w_down"),
        _ptr(dx, dt, (T, d), "dx"), _ptr(dw_router, gt, (E, d), "dw_router"),
        _ptr(dw_gate_up, gt, (E, 2 * f, d), "dw_gate_up"), _ptr(dw_down, gt, (E, d, f), "dw_down"),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_backward")


def moe_stack_forward_trace(cfg, layers, resid, ws, counts=None, losses=None, topk_idx=None, stream=None):
    """moe_stack_forward that also fills, when given, counts [L, E] int32,
    losses [L, 2] fp32 and topk_idx [L, T, k] int32 (device tensors)."""
    dt = torch_dtype(cfg)
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff
    n = len(layers)
    arr = ctypes.c_void_p * n
    wr = arr(*[_ptr(L["w_router"], dt, (E, d), "w_router") for L in layers])
    wgu = arr(*[_ptr(L["w_gate_up"], dt, (E, 2 * f, d), "w_gate_up") for L in layers])
    wd = arr(*[_ptr(L["w_down"], dt, (E, d, f), "w_down") for L in layers])
    bs = arr(*[_ptr(L.get("router_bias"), torch.float32, (E,), "router_bias", allow_none=True)
               for L in layers])
    st = lib().moe_stack_forward_trace(
        _cfgp(cfg), n, wr, bs, wgu, wd, _ptr(resid, torch.float32, (T, d), "resid"),
        _ptr(counts, torch.int32, (n, E), "counts", allow_none=True),
        _ptr(losses, torch.float32, (n, 2), "losses", allow_none=True),
        _ptr(topk_idx, torch.int32, (n, T, k), "topk_idx", allow_none=True),
        _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_stack_forward_trace")


def moe_stack_forward(cfg, layers, resid, ws, stream=None):
    """`layers`: list of dicts with w_router, w_gate_up, w_down and optional router_bias
    (device tensors). `resid` [T, d] fp32 is updated in place."""
    dt = torch_dtype(cfg)
    T, d, E, f = cfg.T, cfg.d_model, cfg.n_experts, cfg.d_ff
    n = len(layers)
    arr = ctypes.c_void_p * n
    wr = arr(*[_ptr(L["w_router"], dt, (E, d), "w_router") for L in layers])
    wgu = arr(*[_ptr(L["w_gate_up"], dt, (E, 2 * f, d), "w_gate_up") for L in layers])
    wd = arr(*[_ptr(L["w_down"], dt, (E, d, f), "w_down") for L in layers])
    bs = arr(*[_ptr(L.get("router_bias"), torch.float32, (E,), "router_bias", allow_none=True)
               for L in layers])
    st = lib().moe_stack_forward(_cfgp(cfg), n, wr, bs, wgu, wd, _ptr(resid, torch.float32, (T, d), "resid"),
                                 _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    _check(st, "moe_stack_forward")


def moe_set_stage_events(events):
    """Arm stage timing for the next moe_forward: `events` is a list of
    STAGE_EVENTS torch.cuda.Event(enable_timing=True) (already created), or None."""
    if events is None:
        _check(lib().moe_set_stage_events(None), "moe_set_stage_events")
        return
    if len(events) != STAGE_EVENTS:
        raise ValueError(f"need {STAGE_EVENTS} events")
    arr = (ctypes.c_void_p * STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_set_stage_events(arr), "moe_set_stage_events")


def moe_get_device_status(ws, stream=None) -> int:
    """The workspace status word (0 when no kernel recorded a failure); clears it."""
    code = ctypes.c_int32(0)
    st = lib().moe_get_device_status(_ptr(ws, torch.uint8, name="ws"), ctypes.byref(code), _stream(stream))
    if st not in (0, 5):
        _check(st, "moe_get_device_status")
    return code.value


# ---------------------------------------------------------------- convenience


class MoELayer:
    """One layer's device-resident weights plus a workspace.

    forward(x) -> (y, losses[2]); backward(dy) -> dict of gradients (needs
    forward(..., train=True) first).
    """

    def __init__(self, w_router, w_gate_up, w_down, router_bias=None, top_k=8, alpha_lb=0.01,
                 beta_z=0.001, grad_dtype=None, renorm=False):
        self.w_router, self.w_gate_up, self.w_down = w_router, w_gate_up, w_down
        self.router_bias = router_bias
        self.top_k = top_k
        self.alpha_lb, self.beta_z = alpha_lb, beta_z
        self.grad_dtype = grad_dtype
        self.renorm = renorm
        self._ws = {}

    def cfg(self, T):
        E, d = self.w_router.shape
        f = self.w_down.shape[2]
        return config(T, d, E, self.top_k, f, self.w_router.dtype, self.alpha_lb, self.beta_z, self.grad_dtype,
                      self.renorm)

    def ws(self, T, train):
        key = (T, bool(train))
        if key not in self._ws:
            self._ws = {key: workspace(self.cfg(T), train, self.w_router.device)}
        return self._ws[key]

    def forward(self, x, train=False, return_routing=False):
        T = x.shape[0]
        cfg = self.cfg(T)
        y = torch.empty_like(x)
        losses = torch.empty(2, dtype=torch.float32, device=x.device)
        idx = torch.empty(T, self.top_k, dtype=torch.int32, device=x.device) if return_routing else None
        w = torch.empty(T, self.top_k, dtype=torch.float32, device=x.device) if return_routing else None
        moe_forward(cfg, x, self.w_router, self.router_bias, self.w_gate_up, self.w_down, y, losses, idx, w,
                    train, self.ws(T, train))
        self._x = x
        return (y, losses, idx, w) if return_routing else (y, losses)

    def backward(self, dy):
        x = self._x
        T = x.shape[0]
        cfg = self.cfg(T)
        gt = grad_torch_dtype(cfg)
        g = {
            "dx": torch.empty_like(x),
            "dw_router": torch.empty_like(self.w_router, dtype=gt),
            "dw_gate_up": torch.empty_like(self.w_gate_up, dtype=gt),
            "dw_down": torch.empty_like(self.w_down, dtype=gt),
        }
        moe_backward(cfg, dy, x, self.w_router, self.w_gate_up, self.w_down, g["dx"], g["dw_router"],
                     g["dw_gate_up"], g["dw_down"], self.ws(T, True))
        return g
