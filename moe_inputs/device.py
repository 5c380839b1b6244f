"""Device side of the input generator: fills torch CUDA tensors with the same
bytes moe_inputs.gen produces on the host (libmoe_inputs.so)."""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import gen

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_inputs.so")
_lib = None


def load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m moe_inputs.build`")
        lib = ctypes.CDLL(LIB_PATH)
        u64, i32, f32, P = ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        lib.moe_gen_pool.argtypes = [u64, i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, f32, P, P, P, P, P]
        lib.moe_gen_pool.restype = ctypes.c_int
        lib.moe_gen_pool_f8.argtypes = [u64, i32, i32, i32, i32, i32, i32, i32, i32, i32, f32, P, P, P, P, P, P, P]
        lib.moe_gen_pool_f8.restype = ctypes.c_int
        lib.moe_gen_normal_bf16.argtypes = [u64, u64, u64, f32, P, P]
        lib.moe_gen_normal_bf16.restype = ctypes.c_int
        lib.moe_gen_stream_key.argtypes = [u64, i32, i32, i32]
        lib.moe_gen_stream_key.restype = u64
        _lib = lib
    return _lib


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def stream_key(seed: int, layer: int, role: int, expert: int) -> int:
    return int(load().moe_gen_stream_key(seed, layer, role, expert))


def fill_pool(shape: gen.MoeShape, seed: int, layer: int, gu_codes, gu_scales, d_codes, d_scales,
              e0: int = 0, ne: int | None = None, shared: bool = False, gu_rs=None, d_rs=None):
    """Writes experts [e0, e0+ne) (or the shared expert) into the given device
    tensors, which start at the first generated expert (fp8 scales: also the
    fp32 row scales gu_rs, d_rs)."""
    ne = (1 if shared else shape.experts - e0) if ne is None else ne
    if shape.fp8_scales:
        st = load().moe_gen_pool_f8(seed, layer, shape.experts, shape.hidden, shape.inter, shape.bits, shape.block,
                                    e0, ne, 1 if shared else 0, float(gen.C_SIGMA002), gu_codes.data_ptr(),
                                    gu_scales.data_ptr(), d_codes.data_ptr(), d_scales.data_ptr(), gu_rs.data_ptr(),
                                    d_rs.data_ptr(), _stream())
        if st != 0:
            raise RuntimeError(f"moe_gen_pool_f8 failed: {st}")
        return
    st = load().moe_gen_pool(seed, layer, shape.experts, shape.hidden, shape.inter, shape.bits, shape.block,
                             1 if shape.half else 0, e0, ne, 1 if shared else 0, float(gen.C_SIGMA002), gu_codes.data_ptr(),
                             gu_scales.data_ptr(), d_codes.data_ptr(), d_scales.data_ptr(), _stream())
    if st != 0:
        raise RuntimeError(f"moe_gen_pool failed: {st}")


def fill_normal_bf16(key: int, start: int, out, c=gen.C_SIGMA002):
    st = load().moe_gen_normal_bf16(key, start, out.numel(), float(np.float32(c)), out.data_ptr(), _stream())
    if st != 0:
        raise RuntimeError(f"moe_gen_normal_bf16 failed: {st}")


def device_layer_tensors(shape: gen.MoeShape, seed: int, layer: int, zipf: bool = False, device: str = "cuda",
                         shared_gate: bool = False):
    """One layer's inputs generated on the device: a dict of torch tensors named
    like the fields of the C ABI's moe_layer_weights (shared_* absent when the
    shape has no shared expert, router_bias only for the skewed workload,
    shared_gate_w only when asked for)."""
    import torch
    E, H, I, b, bs = shape.experts, shape.hidden, shape.inter, shape.bits, shape.block
    sdt = torch.uint8 if shape.fp8_scales else torch.int16
    t = dict(
        gate_up_codes=torch.empty((E, 2 * I, H * b // 8), dtype=torch.uint8, device=device),
        gate_up_scales=torch.empty((E, 2 * I, H // bs), dtype=sdt, device=device),
        down_codes=torch.empty((E, H, I * b // 8), dtype=torch.uint8, device=device),
        down_scales=torch.empty((E, H, I // bs), dtype=sdt, device=device),
        router_w=torch.empty((E, H), dtype=torch.int16, device=device),
    )
    rs = {}
    if shape.fp8_scales:
        t["gate_up_row_scales"] = torch.empty((E, 2 * I), dtype=torch.float32, device=device)
        t["down_row_scales"] = torch.empty((E, H), dtype=torch.float32, device=device)
        rs = dict(gu_rs=t["gate_up_row_scales"], d_rs=t["down_row_scales"])
    fill_pool(shape, seed, layer, t["gate_up_codes"], t["gate_up_scales"], t["down_codes"], t["down_scales"], **rs)
    fill_normal_bf16(gen.stream_key(seed, layer, gen.ROLE_ROUTER, 0), 0, t["router_w"], gen.C_SIGMA002)
    if shape.shared:
        t.update(
            shared_gate_up_codes=torch.empty((2 * I, H * b // 8), dtype=torch.uint8, device=device),
            shared_gate_up_scales=torch.empty((2 * I, H // bs), dtype=sdt, device=device),
            shared_down_codes=torch.empty((H, I * b // 8), dtype=torch.uint8, device=device),
            shared_down_scales=torch.empty((H, I // bs), dtype=sdt, device=device),
        )
        rs = {}
        if shape.fp8_scales:
            t["shared_gate_up_row_scales"] = torch.empty(2 * I, dtype=torch.float32, device=device)
            t["shared_down_row_scales"] = torch.empty(H, dtype=torch.float32, device=device)
            rs = dict(gu_rs=t["shared_gate_up_row_scales"], d_rs=t["shared_down_row_scales"])
        fill_pool(shape, seed, layer, t["shared_gate_up_codes"], t["shared_gate_up_scales"],
                  t["shared_down_codes"], t["shared_down_scales"], shared=True, **rs)
    if shared_gate and shape.shared:
        t["shared_gate_w"] = torch.empty(H, dtype=torch.int16, device=device)
        fill_normal_bf16(gen.stream_key(seed, layer, gen.ROLE_SH_GATE_W, 0), 0, t["shared_gate_w"], gen.C_SIGMA002)
    if zipf:
        t["router_bias"] = torch.from_numpy(gen.zipf_router_bias(shape, seed, layer)).to(device)
    return t
