"""Python binding of the B200 top-k MoE FFN layer (C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA library
``libmoe_b200.so``; PyTorch supplies device memory and streams.  The functions
carry the C names and take torch tensors (device memory) in place of pointers.
A missing library raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
MOE_F32, MOE_BF16, MOE_INT8, MOE_INT4, MOE_FP8 = range(5)
MOE_BIAS_NONE, MOE_BIAS_LOGIT, MOE_BIAS_SELECT = range(3)
MOE_ROUTE_TOPK, MOE_ROUTE_EXPERT_CHOICE = range(2)
ROUTING_CODE = {"topk": MOE_ROUTE_TOPK, "expert_choice": MOE_ROUTE_EXPERT_CHOICE}

DTYPE_CODE = {"f32": MOE_F32, "bf16": MOE_BF16, "int8": MOE_INT8, "int4": MOE_INT4,
              "fp8": MOE_FP8}
BIAS_CODE = {"none": MOE_BIAS_NONE, "logit": MOE_BIAS_LOGIT, "select": MOE_BIAS_SELECT}


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("renormalize", ctypes.c_int32),
                ("bias_mode", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("act_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("router_dtype", ctypes.c_int32), ("expert_dtype", ctypes.c_int32),
                ("group_size", ctypes.c_int32), ("wait_kcycles", ctypes.c_int32),
                ("routing", ctypes.c_int32), ("prefill_tiles", ctypes.c_int32)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "rms_gamma", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up",
        "s_down", "sh_gate", "sh_up", "sh_down", "sh_s_gate", "sh_s_up", "sh_s_down")]


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


_lib = None
_VP, _SZ, _I32P, _F32P = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfig)
_WTS = ctypes.POINTER(MoeWeights)
_SIGS = {
    "moe_workspace_size": (ctypes.c_size_t, [_CFG]),
    "moe_clear_device_status": (ctypes.c_int, [_VP, _SZ, _VP]),
    "moe_rmsnorm_router": (ctypes.c_int, [_CFG, _WTS, _VP, _VP, _F32P, _VP, _SZ, _VP]),
    "moe_route": (ctypes.c_int, [_CFG, _F32P, _F32P, _I32P, _F32P, _VP]),
    "moe_permute": (ctypes.c_int, [_CFG, _I32P, _I32P, _I32P, _I32P, _I32P, _I32P, _VP, _SZ, _VP]),
    "moe_route_expert_choice": (ctypes.c_int, [_CFG, _F32P, _F32P, _F32P, _I32P, _F32P, _I32P,
                                               _VP, _SZ, _VP]),
    "moe_expert_choice_capacity": (ctypes.c_int32, [_CFG]),
    "moe_permute_static": (ctypes.c_int, [_CFG, _I32P, _I32P, _I32P, _I32P, _I32P, _I32P, _VP]),
    "moe_grouped_ffn": (ctypes.c_int, [_CFG, _WTS, _VP, _I32P, _I32P, _F32P, _F32P, _F32P, _VP, _SZ, _VP]),
    "moe_combine": (ctypes.c_int, [_CFG, _F32P, _I32P, _F32P, _VP, _VP, _VP]),
    "moe_layer_forward": (ctypes.c_int, [_CFG, _WTS, _VP, _VP, _VP, _SZ, _F32P, _I32P, _I32P, _VP]),
    "moe_layer_forward_profiled": (ctypes.c_int, [_CFG, _WTS, _VP, _VP, _VP, _SZ,
                                                   ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, _VP]),
    "moe_get_device_status": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_int32), _VP]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_layer_launch_count": (ctypes.c_int32, [_CFG]),
    "moe_layer_step_count": (ctypes.c_int32, [_CFG]),
}


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m moe_layer_fp32_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().moe_status_string(s).decode()


def _check(fn: str, s: int):
    if s != MOE_OK:
        raise MoeError(fn, s)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.device.type != "cuda":
        raise ValueError("device tensors are required")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_config(shape, T: int, out_dtype: Optional[str] = None) -> MoeConfig:
    """MoeConfig from a shape description with the fields of moe_synth.LayerShape."""
    out = out_dtype or shape.act
    return MoeConfig(T=T, d=shape.d, E=shape.E, k=shape.k, f=shape.f, n_shared=shape.n_shared,
                     capacity_factor=float(shape.capacity_factor),
                     renormalize=int(bool(shape.renormalize)), bias_mode=BIAS_CODE[shape.bias_mode],
                     rms_eps=float(shape.rms_eps), act_dtype=DTYPE_CODE[shape.act],
                     out_dtype=DTYPE_CODE[out], router_dtype=DTYPE_CODE[shape.router],
                     expert_dtype=DTYPE_CODE[shape.expert], group_size=int(shape.group_size),
                     routing=ROUTING_CODE[getattr(shape, "routing", "topk")])


def make_weights(li) -> MoeWeights:
    """MoeWeights from an object with the fields of moe_synth.LayerInputs (on the device)."""
    alias = {"rms_gamma": "gamma"}

    def v(name):
        t = getattr(li, alias.get(name, name), None)
        return None if t is None else t.data_ptr()
    return MoeWeights(**{n: v(n) for n, _ in MoeWeights._fields_})


def moe_workspace_size(cfg: MoeConfig) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg)))


def alloc_workspace(cfg: MoeConfig, device="cuda") -> torch.Tensor:
    n = moe_workspace_size(cfg)
    if n == 0:
        raise MoeError("moe_workspace_size", MOE_ERR_INVALID)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_clear_device_status(ws)
    return ws


def moe_clear_device_status(ws: torch.Tensor, stream=None):
    _check("moe_clear_device_status",
           lib().moe_clear_device_status(_p(ws), ws.numel(), _stream(stream)))


def moe_rmsnorm_router(cfg, w: MoeWeights, x, xn_out, logits, ws, stream=None):
    _check("moe_rmsnorm_router", lib().moe_rmsnorm_router(
        ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(xn_out), _p(logits), _p(ws), ws.numel(),
        _stream(stream)))


def moe_route(cfg, logits, bias, topk_idx, topk_gate, stream=None):
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _p(logits), _p(bias), _p(topk_idx),
                                        _p(topk_gate), _stream(stream)))


def moe_permute(cfg, topk_idx, counts, offsets, perm_assign, slot_of, n_dropped, ws, stream=None):
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(offsets), _p(perm_assign), _p(slot_of),
        _p(n_dropped), _p(ws), ws.numel(), _stream(stream)))


def moe_permute_static(cfg, topk_idx, counts, offsets, perm_assign, slot_of, n_dropped,
                       stream=None):
    """moe_permute for callers that cannot allocate: no workspace argument."""
    _check("moe_permute_static", lib().moe_permute_static(
        ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(offsets), _p(perm_assign), _p(slot_of),
        _p(n_dropped), _stream(stream)))


def moe_route_expert_choice(cfg, logits, bias, scores_out, tok, gate, slot_te, ws, stream=None):
    _check("moe_route_expert_choice", lib().moe_route_expert_choice(
        ctypes.byref(cfg), _p(logits), _p(bias), _p(scores_out), _p(tok), _p(gate), _p(slot_te),
        _p(ws), ws.numel(), _stream(stream)))


def moe_expert_choice_capacity(cfg) -> int:
    return int(lib().moe_expert_choice_capacity(ctypes.byref(cfg)))


def moe_grouped_ffn(cfg, w: MoeWeights, xn, offsets, perm_assign, topk_gate, y_assign, y_shared,
                    ws, stream=None):
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(
        ctypes.byref(cfg), ctypes.byref(w), _p(xn), _p(offsets), _p(perm_assign), _p(topk_gate),
        _p(y_assign), _p(y_shared), _p(ws), ws.numel(), _stream(stream)))


def moe_combine(cfg, y_assign, slot_of, y_shared, residual, out, stream=None):
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(cfg), _p(y_assign), _p(slot_of), _p(y_shared), _p(residual), _p(out),
        _stream(stream)))


def moe_layer_forward(cfg, w: MoeWeights, x, out, ws, logits_out=None, topk_idx_out=None,
                      counts_out=None, stream=None):
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(out), _p(ws), ws.numel(), _p(logits_out),
        _p(topk_idx_out), _p(counts_out), _stream(stream)))


def moe_layer_forward_profiled(cfg, w: MoeWeights, x, out, ws, events, stream=None):
    """``events``: torch.cuda.Event objects (enable_timing) -- one before the first
    kernel and one after each step of the layer (moe_layer_step_count + 1)."""
    for e in events:                     # torch creates the CUDA event on first use
        if not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check("moe_layer_forward_profiled", lib().moe_layer_forward_profiled(
        ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(out), _p(ws), ws.numel(), arr, len(events),
        _stream(stream)))


def moe_get_device_status(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    s = lib().moe_get_device_status(_p(ws), ctypes.byref(code), _stream(stream))
    if s not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoeError("moe_get_device_status", s)
    return int(code.value)


def moe_layer_launch_count(cfg) -> int:
    return int(lib().moe_layer_launch_count(ctypes.byref(cfg)))


def moe_layer_step_count(cfg) -> int:
    return int(lib().moe_layer_step_count(ctypes.byref(cfg)))


class MoELayer:
    """Convenience wrapper: one layer's weights on the device, its config and a
    workspace sized for ``T`` tokens; ``forward(x)`` calls moe_layer_forward."""

    def __init__(self, inputs, T: int, out_dtype: Optional[str] = None):
        self.inputs = inputs
        self.cfg = make_config(inputs.shape, T, out_dtype)
        self.w = make_weights(inputs)
        self.ws = alloc_workspace(self.cfg, inputs.w_router.device)
        odt = torch.float32 if (out_dtype or inputs.shape.act) == "f32" else torch.bfloat16
        self.out_dtype = odt

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, logits=None,
                topk_idx=None, counts=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(x.shape, dtype=self.out_dtype, device=x.device)
        moe_layer_forward(self.cfg, self.w, x, out, self.ws, logits, topk_idx, counts, stream)
        return out
