"""Python binding of libmoe.so, the routed quantized-expert MoE FFN layer for B200.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch supplies device memory and
streams); their data pointers and the current CUDA stream are passed through
the C ABI declared in include/moe_capi.h.  The names mirror that header.

If libmoe.so has not been built this module raises on first use; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence

__all__ = [
    "MoeConfig", "LayerWeights", "MoeError", "load_library", "EXPORTS", "LIB_PATH",
    "moe_workspace_bytes", "moe_route", "moe_layer_forward", "moe_stack_forward",
    "moe_device_status", "moe_dequant_rows", "moe_dequant_rows_scaled", "moe_status_str", "config_of",
    "moe_profile_begin",
    "moe_profile_end", "moe_layer_forward_noalloc", "moe_noalloc_device_status", "NOALLOC_SCRATCH_BYTES",
    "moe_layer_forward_ep", "ep_all_reduce",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

EXPORTS = ("moe_workspace_bytes", "moe_route", "moe_layer_forward", "moe_stack_forward",
           "moe_device_status", "moe_dequant_rows", "moe_status_str", "moe_profile_begin", "moe_profile_end",
           "moe_layer_forward_noalloc", "moe_last_cuda_error", "moe_debug_fused_timing",
           "moe_debug_prefill_timing", "moe_layer_forward_ep", "moe_debug_decode_path", "moe_debug_wait_probe",
           "moe_noalloc_device_status", "moe_dequant_rows_scaled")

MOE_OK = 0


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = f", cudaError {load_library().moe_last_cuda_error()}" if status == -4 else ""
        super().__init__(f"{what}: status {status} ({moe_status_str(status)}{detail})")
        self.status = status


class MoeConfig(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("shared_inter", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("block", ctypes.c_int32), ("half_levels", ctypes.c_int32), ("scale_fmt", ctypes.c_int32)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_up_codes", "gate_up_scales", "down_codes", "down_scales", "shared_gate_up_codes",
        "shared_gate_up_scales", "shared_down_codes", "shared_down_scales", "router_w", "router_bias",
        "shared_gate_w", "gate_up_row_scales", "down_row_scales", "shared_gate_up_row_scales",
        "shared_down_row_scales")]


@dataclasses.dataclass
class LayerWeights:
    """Device tensors of one layer (layouts in include/moe_capi.h).  Scales and
    bf16 tensors may be any dtype of the right element size (fp16 scales 16-bit,
    E4M3 scales 8-bit); only the bytes matter."""
    gate_up_codes: object
    gate_up_scales: object
    down_codes: object
    down_scales: object
    router_w: object
    router_bias: Optional[object] = None
    shared_gate_up_codes: Optional[object] = None
    shared_gate_up_scales: Optional[object] = None
    shared_down_codes: Optional[object] = None
    shared_down_scales: Optional[object] = None
    shared_gate_w: Optional[object] = None      # [H] bf16: shared expert weighted by sigmoid(x . w)
    gate_up_row_scales: Optional[object] = None          # fp8 block scales: fp32 [E][2I]
    down_row_scales: Optional[object] = None             # fp32 [E][H]
    shared_gate_up_row_scales: Optional[object] = None   # fp32 [2I]
    shared_down_row_scales: Optional[object] = None      # fp32 [H]

    def to_c(self) -> _Weights:
        w = _Weights()
        for f in _Weights._fields_:
            t = getattr(self, f[0])
            setattr(w, f[0], _ptr(t))
        return w


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libmoe.so (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m quantized_expert_ffn_moe_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp = ctypes.POINTER(MoeConfig)
    lib.moe_workspace_bytes.argtypes = [cfgp, I32]
    lib.moe_workspace_bytes.restype = SZ
    lib.moe_route.argtypes = [cfgp, P, P, P, I32, P, P, P, P, P, P, SZ, P]
    lib.moe_route.restype = ctypes.c_int
    lib.moe_layer_forward.argtypes = [cfgp, ctypes.POINTER(_Weights), P, I32, P, P, SZ, P]
    lib.moe_layer_forward.restype = ctypes.c_int
    lib.moe_layer_forward_ep.argtypes = [cfgp, ctypes.POINTER(_Weights), P, I32, I32, I32, P, P, SZ, P]
    lib.moe_layer_forward_ep.restype = ctypes.c_int
    lib.moe_stack_forward.argtypes = [cfgp, ctypes.POINTER(_Weights), I32, P, I32, P, P, SZ, P]
    lib.moe_stack_forward.restype = ctypes.c_int
    lib.moe_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
    lib.moe_device_status.restype = ctypes.c_int
    lib.moe_dequant_rows.argtypes = [cfgp, P, P, I32, I32, I32, P, P]
    lib.moe_dequant_rows.restype = ctypes.c_int
    lib.moe_dequant_rows_scaled.argtypes = [cfgp, P, P, P, I32, I32, I32, P, P]
    lib.moe_dequant_rows_scaled.restype = ctypes.c_int
    lib.moe_layer_forward_noalloc.argtypes = [cfgp, ctypes.POINTER(_Weights), P, I32, P, P]
    lib.moe_layer_forward_noalloc.restype = ctypes.c_int
    lib.moe_noalloc_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    lib.moe_noalloc_device_status.restype = ctypes.c_int
    lib.moe_profile_begin.argtypes = [I32]
    lib.moe_profile_begin.restype = ctypes.c_int
    lib.moe_profile_end.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32)]
    lib.moe_profile_end.restype = ctypes.c_int
    lib.moe_debug_fused_timing.argtypes = [P]
    lib.moe_debug_fused_timing.restype = None
    lib.moe_debug_prefill_timing.argtypes = [P]
    lib.moe_debug_decode_path.argtypes = [I32]
    lib.moe_debug_decode_path.restype = None
    lib.moe_debug_wait_probe.argtypes = [P, P]
    lib.moe_debug_wait_probe.restype = ctypes.c_int
    lib.moe_debug_prefill_timing.restype = None
    lib.moe_last_cuda_error.argtypes = []
    lib.moe_last_cuda_error.restype = ctypes.c_int
    lib.moe_status_str.argtypes = [ctypes.c_int]
    lib.moe_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, what: str):
    if st != MOE_OK:
        raise MoeError(st, what)


def config_of(experts, hidden, inter, top_k, shared, bits, block, half_levels=False, fp8_scales=False) -> MoeConfig:
    return MoeConfig(experts, hidden, inter, top_k, inter if shared else 0, bits, block, 1 if half_levels else 0,
                     1 if fp8_scales else 0)


def moe_status_str(status: int) -> str:
    return load_library().moe_status_str(status).decode()


def moe_workspace_bytes(cfg: MoeConfig, max_tokens: int) -> int:
    return int(load_library().moe_workspace_bytes(ctypes.byref(cfg), max_tokens))


def moe_route(cfg: MoeConfig, router_w, router_bias, x, topk_idx, topk_w, workspace, *, counts=None,
              offsets=None, pairs=None, stream=None, check=True) -> int:
    T = int(x.shape[0])
    st = load_library().moe_route(ctypes.byref(cfg), _ptr(router_w), _ptr(router_bias), _ptr(x), T,
                                  _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets), _ptr(pairs),
                                  _ptr(workspace), _nbytes(workspace), _stream(stream))
    if check:
        _check(st, "moe_route")
    return st


def moe_layer_forward(cfg: MoeConfig, w: LayerWeights, x, y, workspace, *, stream=None, check=True,
                      tokens: Optional[int] = None) -> int:
    T = int(x.shape[0]) if tokens is None else tokens
    cw = w.to_c()
    st = load_library().moe_layer_forward(ctypes.byref(cfg), ctypes.byref(cw), _ptr(x), T, _ptr(y),
                                          _ptr(workspace), _nbytes(workspace), _stream(stream))
    if check:
        _check(st, "moe_layer_forward")
    return st


def moe_layer_forward_ep(cfg: MoeConfig, w: LayerWeights, x, y_partial, workspace, ep_rank: int, ep_size: int,
                         *, stream=None, check=True, tokens: Optional[int] = None) -> int:
    """This rank's fp32 partial [T, H] of the layer output: the routed experts
    e with e % ep_size == ep_rank, plus the shared expert on rank 0."""
    T = int(x.shape[0]) if tokens is None else tokens
    cw = w.to_c()
    st = load_library().moe_layer_forward_ep(ctypes.byref(cfg), ctypes.byref(cw), _ptr(x), T, ep_rank, ep_size,
                                             _ptr(y_partial), _ptr(workspace), _nbytes(workspace), _stream(stream))
    if check:
        _check(st, "moe_layer_forward_ep")
    return st


def ep_all_reduce(y_partial, group=None):
    """The exchange step of the expert-parallel layer: sums the ranks' fp32
    partials in place over the torch.distributed process group (NCCL over
    NVLink on GPUs).  Afterwards every rank holds the layer output before its
    bf16 rounding."""
    import torch.distributed as dist
    dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial


def moe_layer_forward_noalloc(cfg: MoeConfig, w: LayerWeights, x, y, *, stream=None, check=True,
                              tokens: Optional[int] = None) -> int:
    """moe_layer_forward without a workspace argument: the library's fixed
    scratch array is used (see include/moe_capi.h for the size limit)."""
    T = int(x.shape[0]) if tokens is None else tokens
    cw = w.to_c()
    st = load_library().moe_layer_forward_noalloc(ctypes.byref(cfg), ctypes.byref(cw), _ptr(x), T, _ptr(y),
                                                  _stream(stream))
    if check:
        _check(st, "moe_layer_forward_noalloc")
    return st


NOALLOC_SCRATCH_BYTES = 4 << 20


def moe_noalloc_device_status() -> int:
    """The device check word of the allocation-free entry point's scratch on
    the current device (synchronises the device); 0 when no kernel reported a
    failed check."""
    code = ctypes.c_int32(0)
    st = load_library().moe_noalloc_device_status(ctypes.byref(code))
    if st not in (MOE_OK, -5):
        _check(st, "moe_noalloc_device_status")
    return int(code.value)


def moe_stack_forward(cfg: MoeConfig, layers: Sequence[LayerWeights], x_inout, workspace, *, topk_trace=None,
                      stream=None, check=True) -> int:
    arr = (_Weights * len(layers))(*[l.to_c() for l in layers])
    T = int(x_inout.shape[0])
    st = load_library().moe_stack_forward(ctypes.byref(cfg), arr, len(layers), _ptr(x_inout), T,
                                          _ptr(topk_trace), _ptr(workspace), _nbytes(workspace),
                                          _stream(stream))
    if check:
        _check(st, "moe_stack_forward")
    return st


def moe_device_status(workspace) -> int:
    code = ctypes.c_int32(0)
    load_library().moe_device_status(_ptr(workspace), ctypes.byref(code))
    return int(code.value)


def moe_dequant_rows(cfg: MoeConfig, codes, scales, row0: int, rows: int, cols: int, out, *, stream=None,
                     check=True) -> int:
    st = load_library().moe_dequant_rows(ctypes.byref(cfg), _ptr(codes), _ptr(scales), row0, rows, cols,
                                         _ptr(out), _stream(stream))
    if check:
        _check(st, "moe_dequant_rows")
    return st


def moe_dequant_rows_scaled(cfg: MoeConfig, codes, scales, row_scales, row0: int, rows: int, cols: int, out, *,
                            stream=None, check=True) -> int:
    st = load_library().moe_dequant_rows_scaled(ctypes.byref(cfg), _ptr(codes), _ptr(scales), _ptr(row_scales),
                                                row0, rows, cols, _ptr(out), _stream(stream))
    if check:
        _check(st, "moe_dequant_rows_scaled")
    return st


def moe_profile_begin(max_calls: int):
    _check(load_library().moe_profile_begin(max_calls), "moe_profile_begin")


def moe_profile_end():
    """Returns ([route, gate_up, down, combine, fused] summed ms, number of calls)."""
    ms = (ctypes.c_float * 5)()
    n = ctypes.c_int32(0)
    _check(load_library().moe_profile_end(ms, ctypes.byref(n)), "moe_profile_end")
    return [float(v) for v in ms], int(n.value)


def _nbytes(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return 0
    return int(t.numel() * t.element_size())
