"""GPU parity of the layer stack (moe_stack_forward) against the float64 oracle.

Each stack layer is x <- bf16(x + moe(bf16(rmsnorm(x)))); 48 layers of 512
experts ("Strata Open Source Project: Run a 125B Model Locally on a Home PC",
section "How Strata Makes Your Entire PC Work Together": 24,576 experts).

Three kinds of check:

* One layer at a time, at the layer tolerance: for sampled depths l of the
  48-layer stack, layer l runs through moe_stack_forward on its own seeded
  input, and the GPU's selection must equal the oracle's except inside the
  1e-5 tie band, and its new residual stream must be a bf16 rounding of
  x + o for some MoE output o within 2e-2 x RMS of the oracle's (bf16
  rounding is monotone, so the stream must lie between the roundings of
  x + out -/+ that tolerance).  The oracle only ever sees seeded inputs.
* Composition: one launch over L layers equals L one-layer calls, bit for
  bit (decode: the single-launch kernel over up to 64 layers per launch;
  prefill: the per-layer kernels with the next layer's RMSNorm fused into
  the combine).
* Free running over 48 layers (secondary): both sides round the residual
  stream to bf16 every layer, so the two streams drift apart by rounding
  flips; each token is compared up to the first layer where its selection
  differs, and that difference must be explained by the logit shift the
  drifted stream implies.
"""

import numpy as np
import pytest

import gpu_cases as gc
import moe_inputs as mi
import oracle as orc
import quantized_expert_ffn_moe_b200 as q

pytestmark = pytest.mark.gpu

MID4 = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=4, shared=True, bits=4, block=32)
FULL4F8 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=32, fp8_scales=True)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_moe_b200 import build
    from moe_inputs import build as ibuild
    build.build()
    ibuild.build()
    q.load_library()


def _gpu_stack(shape, layers_w, x_bits, trace=True):
    torch = gc.torch()
    cfg = gc.cfg_of(shape)
    T = x_bits.shape[0]
    x = gc.to_dev_bits(x_bits)
    ws = gc.workspace(cfg, T)
    tr = torch.empty((len(layers_w), T, shape.top_k), dtype=torch.int32, device="cuda") if trace else None
    q.moe_stack_forward(cfg, layers_w, x, ws, topk_trace=tr)
    torch.cuda.synchronize()
    assert q.moe_device_status(ws) == 0
    return mi.bf16_bits_to_f32(gc.bits_to_np(x)).astype(np.float64), (tr.cpu().numpy() if trace else None)


def _stack_bits(shape, layers_w, x_bits):
    """The stack's output as raw bf16 bits (for bitwise comparisons)."""
    torch = gc.torch()
    cfg = gc.cfg_of(shape)
    x = gc.to_dev_bits(x_bits)
    ws = gc.workspace(cfg, x_bits.shape[0])
    q.moe_stack_forward(cfg, layers_w, x, ws)
    torch.cuda.synchronize()
    assert q.moe_device_status(ws) == 0
    return gc.bits_to_np(x)


def assert_stack_step(x_in, got, out_ref, rel=gc.REL_TOL):
    """got = bf16(x_in + o) with max |o - out_ref| <= rel * RMS(out_ref)?"""
    eps = rel * float(np.sqrt(np.mean(out_ref * out_ref)))
    lo = orc.round_bf16(x_in + out_ref - eps)
    hi = orc.round_bf16(x_in + out_ref + eps)
    bad = (got < lo) | (got > hi)
    assert not bad.any(), f"{int(bad.sum())} elements outside the rounding of x + out -/+ {rel} RMS; first at " \
                          f"{np.argwhere(bad)[0]}"


# ------------------------------------------------ one layer at a time ---

@pytest.mark.parametrize("name", ["full4_stack_step_t1", "full4_stack_step_t32", "full4_stack_step_t2048"])
def test_stack_layer_steps_stored_oracle(name):
    """Layers 0, 1, ..., 47 of the full-shape 4-bit stack one at a time: the
    single-launch decode kernel (1 token: fewer tokens than warps, so the
    (token, expert) router dots are shared; 32 tokens: every token staged
    once per layer) and the per-layer tensor-core kernels (2048 tokens)."""
    case = gc.load_case(name)
    E, H, I, k, sh, bits, bs = case["shape"].tolist()
    shape = mi.MoeShape(E, H, I, k, bool(sh), bits, bs)
    T, toks = int(case["T"]), case["tokens"]
    for li, l in enumerate(case["steps"].tolist()):
        w = gc.device_layer(shape, 0, l)
        x = mi.hidden_states_bf16(T, H, 0, int(case["batch"]) + l)
        got, trace = _gpu_stack(shape, [w], x)
        ref = case["out_"][li].astype(np.float64)
        differ = gc.check_selection(case["logits"][li], case["idx"][li], trace[0][toks], k)
        if differ:
            lay = gc.host_oracle_layer(shape, 0, l, cache_size=12)
            for i in differ:     # the oracle on the GPU's (valid) selection
                t = int(toks[i])
                ref[i] = orc.layer_forward(lay, x[t:t + 1], rmsnorm=True, topk_override={0: trace[0][t]})["out"][0]
        assert_stack_step(orc.bf16_to_f64(x[toks]), got[toks], ref)


@pytest.mark.parametrize("shape,T", [(mi.TINY, 6), (mi.TINY, 100), (MID4, 129)], ids=["tiny_t6", "tiny_t100", "mid4_t129"])
def test_stack_layer_steps_live_oracle(shape, T):
    """Small shapes (the separate kernels: decode GEMV, and the tensor-core
    path for 129 tokens), two layers, each on its own seeded input."""
    for l in (0, 3):
        w = gc.device_layer(shape, 0, l)
        x = mi.hidden_states_bf16(T, shape.hidden, 0, 60 + l)
        got, trace = _gpu_stack(shape, [w], x)
        lay = gc.host_oracle_layer(shape, 0, l, cache_size=shape.experts + 1)
        r = orc.layer_forward(lay, x, rmsnorm=True)
        differ = gc.check_selection(r["logits"], r["idx"], trace[0], shape.top_k)
        if differ:
            r = orc.layer_forward(lay, x, rmsnorm=True, topk_override={t: trace[0][t] for t in differ})
        assert_stack_step(orc.bf16_to_f64(x), got, r["out"])


@pytest.mark.parametrize("T", [1, 3])
def test_stack_fp8_scales_full_live_oracle(T):
    """fp8 block scales through the stack's single-launch decode kernel
    (RMSNorm in its first phase, the residual in its combine): each of two
    full-shape layers on its own seeded input against the oracle, and the
    two-layer launch equal to two one-layer calls."""
    shape = FULL4F8
    ws = [gc.device_layer(shape, 0, l) for l in range(2)]
    for l in range(2):
        x = mi.hidden_states_bf16(T, shape.hidden, 0, 90 + l)
        got, trace = _gpu_stack(shape, [ws[l]], x)
        lay = gc.host_oracle_layer(shape, 0, l, cache_size=12)
        r = orc.layer_forward(lay, x, rmsnorm=True)
        differ = gc.check_selection(r["logits"], r["idx"], trace[0], shape.top_k)
        if differ:
            r = orc.layer_forward(lay, x, rmsnorm=True, topk_override={t: trace[0][t] for t in differ})
        assert_stack_step(orc.bf16_to_f64(x), got, r["out"])
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 95)
    whole = _stack_bits(shape, ws, x)
    step = x
    for w in ws:
        step = _stack_bits(shape, [w], step)
    np.testing.assert_array_equal(whole, step)


# --------------------------------------------------------- composition ---

@pytest.fixture(scope="module")
def full48():
    return [gc.device_layer(mi.FULL4, 0, l) for l in range(48)]


@pytest.mark.parametrize("T,L", [(1, 48), (32, 48), (1, 70)], ids=["t1_l48", "t32_l48", "t1_l70"])
def test_stack_launch_equals_chained_layers_decode(full48, T, L):
    """One moe_stack_forward over L layers (up to 64 per launch of the decode
    kernel) gives the same bits as L one-layer calls in a row."""
    shape = mi.FULL4
    layers = [full48[l % 48] for l in range(L)]
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 700 + T)
    whole = _stack_bits(shape, layers, x)
    step = x
    for w in layers:
        step = _stack_bits(shape, [w], step)
    np.testing.assert_array_equal(whole, step)


@pytest.mark.parametrize("shape,T,L", [(mi.FULL4, 2048, 4), (mi.TINY, 6, 4), (MID4, 300, 3)],
                         ids=["full4_t2048", "tiny_t6", "mid4_t300"])
def test_stack_launch_equals_chained_layers_separate_kernels(full48, shape, T, L):
    """The per-layer kernels: the next layer's RMSNorm fused into the combine
    gives the same normalised input as the stand-alone RMSNorm kernel."""
    layers = full48[:L] if shape is mi.FULL4 else [gc.device_layer(shape, 0, l) for l in range(L)]
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 800 + T)
    whole = _stack_bits(shape, layers, x)
    step = x
    for w in layers:
        step = _stack_bits(shape, [w], step)
    np.testing.assert_array_equal(whole, step)


# ------------------------------------------------------- free running ---

def _bf16_f64(v):
    return mi.bf16_bits_to_f32(mi.bf16_bits_from_f32(np.asarray(v, dtype=np.float32))).astype(np.float64)


def _implied_logit_shift(x_gpu, x_ref, router_bits):
    """Largest change of any router logit between the normalised inputs of two
    residual streams of one token (RMSNorm with weight 1, eps 1e-6, rounded
    to bf16), plus the 1e-5 tie band."""
    wr = mi.bf16_bits_to_f32(router_bits).astype(np.float64)
    xh = []
    for xs in (x_gpu, x_ref):
        r = 1.0 / np.sqrt(np.mean(xs * xs) + 1e-6)
        xh.append(_bf16_f64(xs * r))
    return float(np.max(np.abs((xh[0] - xh[1]) @ wr.T))) + gc.TIE_BAND


def _free_running(shape, ws, x, oracle_idx, oracle_logits, oracle_x, toks, router_bits, min_depth):
    """oracle_*[l][i]: the oracle's selection, logits and stream after layer l
    for token toks[i].  Returns the depth of the first divergence per token."""
    L = len(ws)
    got, trace = _gpu_stack(shape, ws, x)
    x0 = orc.bf16_to_f64(x)
    streams = {L: got}
    depth = {}
    for i, t in enumerate(toks):
        first = next((l for l in range(L) if not np.array_equal(trace[l, t], oracle_idx[l][i])), None)
        depth[i] = L if first is None else first
    for d in sorted(set(depth.values())):
        if d not in streams:
            streams[d] = x0 if d == 0 else _gpu_stack(shape, ws[:d], x, trace=False)[0]
    for i, t in enumerate(toks):
        d = depth[i]
        ref_in = x0[t] if d == 0 else oracle_x[d - 1][i]
        if d < L:
            band = _implied_logit_shift(streams[d][t], ref_in, router_bits[d])
            assert orc.tie_band_ok(oracle_logits[d][i], trace[d, t], shape.top_k, band), (t, d, band)
        if d > 0:
            gc.assert_close_stack(streams[d][t], np.asarray(oracle_x[d - 1][i], dtype=np.float64))
    assert max(depth.values()) >= min_depth, depth
    return depth


def test_stack_full48_free_running_stored_oracle(full48):
    case = gc.load_case("full4_stack48_decode")
    shape = mi.FULL4
    L = int(case["layers"])
    x = mi.hidden_states_bf16(int(case["T"]), shape.hidden, 0, int(case["batch"]))
    _free_running(shape, full48[:L], x, case["trace_idx"], case["trace_logits"], case["trace_x"],
                  case["tokens"], [mi.router_weight_bf16(shape, 0, l) for l in range(L)], min_depth=4)


def test_stack_tiny_free_running_live_oracle():
    shape = mi.TINY
    L, T = 4, 6
    ws = [gc.device_layer(shape, 0, l) for l in range(L)]
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 2)
    lays = [gc.host_oracle_layer(shape, 0, l, cache_size=shape.experts + 1) for l in range(L)]
    r = orc.stack_forward(lays, x)
    tr = r["trace"]
    _free_running(shape, ws, x, [s["idx"] for s in tr], [s["logits"] for s in tr], [s["x"] for s in tr],
                  np.arange(T), [mi.router_weight_bf16(shape, 0, l) for l in range(L)], min_depth=2)
