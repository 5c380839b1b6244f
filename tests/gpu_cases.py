"""Helpers of the GPU parity tests: put a seeded layer on the device through
the input generator, call the C ABI, and compare with the oracle."""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
import oracle as orc  # noqa: E402
import quantized_expert_ffn_moe_b200 as q  # noqa: E402

GOLDEN = os.path.join(ROOT, "tests", "golden")
TIE_BAND = 1e-5          # oracle k-th vs (k+1)-th logit gap inside which either choice is valid
REL_TOL = 2e-2           # max |err| <= REL_TOL * RMS(oracle output)


def torch():
    import torch as t
    return t


def cfg_of(shape: mi.MoeShape) -> q.MoeConfig:
    return q.config_of(shape.experts, shape.hidden, shape.inter, shape.top_k, shape.shared, shape.bits,
                       shape.block, shape.half, shape.fp8_scales)


def device_layer(shape: mi.MoeShape, seed: int, layer: int, zipf: bool = False,
                 shared_gate: bool = False) -> q.LayerWeights:
    """One layer's packed weights generated on the device (same bytes as the
    host generator), as LayerWeights."""
    import moe_inputs.device as md
    return q.LayerWeights(**md.device_layer_tensors(shape, seed, layer, zipf=zipf, shared_gate=shared_gate))


def to_dev_bits(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).to("cuda")


def bits_to_np(x) -> np.ndarray:
    return x.cpu().numpy().view(np.uint16)


def workspace(cfg, T):
    t = torch()
    n = q.moe_workspace_bytes(cfg, T)
    assert n > 0
    return t.empty(n, dtype=t.uint8, device="cuda")


def run_layer(shape, w, x_bits: np.ndarray):
    t = torch()
    cfg = cfg_of(shape)
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    y = t.empty_like(x)
    ws = workspace(cfg, T)
    q.moe_layer_forward(cfg, w, x, y, ws)
    t.cuda.synchronize()
    assert q.moe_device_status(ws) == 0
    return mi.bf16_bits_to_f32(bits_to_np(y)).astype(np.float64)


def run_route(shape, w, x_bits: np.ndarray):
    t = torch()
    cfg = cfg_of(shape)
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    ws = workspace(cfg, T)
    idx = t.empty((T, shape.top_k), dtype=t.int32, device="cuda")
    wt = t.empty((T, shape.top_k), dtype=t.float32, device="cuda")
    counts = t.empty(shape.experts, dtype=t.int32, device="cuda")
    offsets = t.empty(shape.experts + 1, dtype=t.int32, device="cuda")
    pairs = t.empty(T * shape.top_k, dtype=t.int32, device="cuda")
    q.moe_route(cfg, w.router_w, w.router_bias, x, idx, wt, ws, counts=counts, offsets=offsets, pairs=pairs)
    t.cuda.synchronize()
    return (idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64), counts.cpu().numpy(), offsets.cpu().numpy(),
            pairs.cpu().numpy())


def host_oracle_layer(shape, seed, layer, zipf=False, cache_size=16, shared_gate=False):
    return orc.OracleLayer(
        experts=shape.experts, hidden=shape.hidden, inter=shape.inter, top_k=shape.top_k, bits=shape.bits,
        block=shape.block, router_w_bits=mi.router_weight_bf16(shape, seed, layer),
        router_bias=mi.zipf_router_bias(shape, seed, layer) if zipf else None,
        expert=lambda e: mi.expert_packed(shape, seed, layer, e),
        shared=(lambda: mi.shared_packed(shape, seed, layer)) if shape.shared else (lambda: None),
        cache_size=cache_size,
        shared_gate_w_bits=mi.shared_gate_weight_bf16(shape, seed, layer) if shared_gate else None,
        half_levels=shape.half)


def check_selection(oracle_logits, oracle_idx, gpu_idx, k, band=TIE_BAND):
    """Indices equal the oracle's except inside the tie band; returns the tokens
    whose (valid) selection differs from the oracle's."""
    differ = []
    for t in range(gpu_idx.shape[0]):
        if np.array_equal(gpu_idx[t], oracle_idx[t]):
            continue
        assert orc.tie_band_ok(oracle_logits[t], gpu_idx[t], k, band), (t, gpu_idx[t], oracle_idx[t])
        # the slots still run by descending logit
        sel = oracle_logits[t][gpu_idx[t]]
        assert np.all(np.diff(sel) <= band)
        differ.append(t)
    return differ


def assert_close(got: np.ndarray, ref: np.ndarray, rel=REL_TOL):
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= rel * rms, f"max|err| {err:.3e} > {rel} * rms {rms:.3e} (ratio {err / rms:.3e})"
    return err / rms


# Free-running stack comparisons only (each single layer step is checked at
# REL_TOL): the stack's residual stream is rounded to bf16 after every layer on
# both sides; where the two sums differ in their last bits the rounding flips
# by one bf16 ulp (2^-8 relative).  Over d layers the flips add like a random
# walk, about sqrt(d) * 2^-9 * |x| per element; elements reach ~4 RMS, so d = 48
# gives about 0.05 RMS.  These comparisons use that bound on the largest
# element error and 1e-2 on the root-mean-square error.
STACK_MAX_TOL = 5e-2
STACK_RMS_TOL = 1e-2


def assert_close_stack(got: np.ndarray, ref: np.ndarray):
    rms = float(np.sqrt(np.mean(ref * ref)))
    diff = got - ref
    err = float(np.max(np.abs(diff)))
    rerr = float(np.sqrt(np.mean(diff * diff)))
    assert err <= STACK_MAX_TOL * rms, f"max|err| {err:.3e} > {STACK_MAX_TOL} * rms {rms:.3e}"
    assert rerr <= STACK_RMS_TOL * rms, f"rms err {rerr:.3e} > {STACK_RMS_TOL} * rms {rms:.3e}"
    return err / rms, rerr / rms


def load_case(name):
    path = os.path.join(GOLDEN, f"oracle_{name}.npz")
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} missing: run tests/golden/make_oracle_cases.py {name}")
    return dict(np.load(path))
