"""Pin of the oracle's layer stack (no GPU).

The stack of "Strata Open Source Project: Run a 125B Model Locally on a Home
PC", section "How Strata Makes Your Entire PC Work Together" (24,576 experts
= 48 layers of 512) runs, per layer, x <- bf16(x + moe(bf16(rmsnorm(x))))
with RMSNorm weight 1 and eps 1e-6.  Here that composition is restated
element by element -- plain Python loops, exact rational bf16 rounding, a
decoder written from the format description, top-k by sorting -- and checked
against oracle.stack_forward on a three-layer stack whose middle layer has
every scale zero (its MoE output is exactly zero, so the residual stream
must come out of it unchanged).  A residual added to the normalised input, a
missing per-layer bf16 rounding, the norm skipped before the router, or the
layers applied out of order each break it.
"""
from fractions import Fraction
import math

import numpy as np

import moe_inputs as mi
import oracle as orc

SHAPE = mi.MoeShape(experts=8, hidden=64, inter=32, top_k=2, shared=True, bits=4, block=32)
EPS = 1e-6


def _bf16(v: float) -> float:
    """Nearest bf16 value (8 significant bits, ties to even), by exact
    rational arithmetic."""
    if v == 0.0:
        return 0.0
    f = Fraction(v)
    e = math.floor(math.log2(abs(v)))
    while Fraction(2) ** e > abs(f):
        e -= 1
    while Fraction(2) ** (e + 1) <= abs(f):
        e += 1
    ulp = Fraction(2) ** (e - 7)
    return float(round(f / ulp) * ulp)


def _decode_row(codes_row, scales_row, cols, bits, block):
    """Weights of one packed row: element j sits at bit j*bits of the row,
    lower element in the lower bits, code minus 2^(bits-1), times its
    block's fp16 scale."""
    half = 1 << (bits - 1)
    out = []
    for j in range(cols):
        pos = j * bits
        code = (int(codes_row[pos // 8]) >> (pos % 8)) & ((1 << bits) - 1)
        s = float(np.array([scales_row[j // block]], dtype=np.uint16).view(np.float16)[0])
        out.append((code - half) * s)
    return out


def _expert_ffn(packed, x, H, I):
    gc, gs, dc, ds = packed
    w13 = [_decode_row(gc[r], gs[r], H, SHAPE.bits, SHAPE.block) for r in range(2 * I)]
    wd = [_decode_row(dc[r], ds[r], I, SHAPE.bits, SHAPE.block) for r in range(H)]
    h = []
    for i in range(I):
        g = math.fsum(w13[2 * i][c] * x[c] for c in range(H))
        u = math.fsum(w13[2 * i + 1][c] * x[c] for c in range(H))
        h.append(g / (1.0 + math.exp(-g)) * u)
    return [math.fsum(wd[r][i] * h[i] for i in range(I)) for r in range(H)]


def _layer_step(lay, x):
    """One stack layer for one token, written out: returns the new residual
    stream and the selected experts."""
    H, I, E, k = lay.hidden, lay.inter, lay.experts, lay.top_k
    r = 1.0 / math.sqrt(math.fsum(v * v for v in x) / H + EPS)
    xh = [_bf16(v * r) for v in x]
    wr = mi.bf16_bits_to_f32(lay.router_w_bits).astype(np.float64)
    logits = [math.fsum(float(wr[e, c]) * xh[c] for c in range(H)) for e in range(E)]
    sel = sorted(range(E), key=lambda e: (-logits[e], e))[:k]
    ex = [math.exp(logits[e] - logits[sel[0]]) for e in sel]
    tot = math.fsum(ex)
    out = [0.0] * H
    if lay.shared() is not None:
        out = _expert_ffn(lay.shared(), xh, H, I)
    for j, e in enumerate(sel):
        y = _expert_ffn(lay.expert(e), xh, H, I)
        out = [out[c] + ex[j] / tot * y[c] for c in range(H)]
    return [_bf16(x[c] + out[c]) for c in range(H)], sel, [x[c] + out[c] for c in range(H)]


def _layers():
    lays = []
    for l in range(3):
        pool, sh = mi.layer_packed_pool(SHAPE, 0, l)
        if l == 1:       # every scale zero: this layer's MoE output is exactly 0
            pool = (pool[0], np.zeros_like(pool[1]), pool[2], np.zeros_like(pool[3]))
            sh = (sh[0], np.zeros_like(sh[1]), sh[2], np.zeros_like(sh[3]))
        lays.append(orc.OracleLayer(
            experts=SHAPE.experts, hidden=SHAPE.hidden, inter=SHAPE.inter, top_k=SHAPE.top_k,
            bits=SHAPE.bits, block=SHAPE.block, router_w_bits=mi.router_weight_bf16(SHAPE, 0, l),
            router_bias=None, expert=(lambda e, p=pool: tuple(a[e] for a in p)),
            shared=(lambda s=sh: s), cache_size=SHAPE.experts + 1))
    return lays


def test_bf16_restatement_cases():
    for v, e in [(1.0 + 2 ** -8, 1.0), (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6), (-(1.0 + 2 ** -8), -1.0),
                 (0.7071067811865476, 0.70703125), (3.0, 3.0), (2 ** -20 * 1.00390625, 2 ** -20)]:
        assert _bf16(v) == e


def test_stack_matches_elementwise_restatement():
    lays = _layers()
    xb = mi.hidden_states_bf16(3, SHAPE.hidden, 0, 5)
    r = orc.stack_forward(lays, xb)
    x0 = mi.bf16_bits_to_f32(xb).astype(np.float64)
    for t in range(3):
        x = [float(v) for v in x0[t]]
        for l, lay in enumerate(lays):
            x_new, sel, pre = _layer_step(lay, x)
            assert list(r["trace"][l]["idx"][t]) == sel, (t, l)
            got = r["trace"][l]["x"][t]
            for c in range(SHAPE.hidden):
                if got[c] != x_new[c]:
                    # only a float64 summation-order difference right at a
                    # bf16 rounding boundary may round the other way
                    mid = (got[c] + x_new[c]) / 2
                    assert abs(pre[c] - mid) <= 1e-12 * max(1.0, abs(pre[c])), (t, l, c, got[c], x_new[c])
            if l == 1:
                np.testing.assert_array_equal(got, x)        # zero layer: stream unchanged
            x = list(got)
        np.testing.assert_array_equal(r["x"][t], r["trace"][-1]["x"][t])


def test_zero_layer_leaves_the_stream_exactly():
    lays = _layers()
    xb = mi.hidden_states_bf16(2, SHAPE.hidden, 0, 9)
    only_zero = orc.stack_forward([lays[1]], xb)
    np.testing.assert_array_equal(only_zero["x"], mi.bf16_bits_to_f32(xb).astype(np.float64))


def test_norm_feeds_the_router_and_the_residual_takes_the_raw_stream():
    """Scaling the input stream by a power of two leaves the normalised input,
    hence the routing and the MoE output, unchanged (RMSNorm is scale
    invariant up to eps), while the residual keeps the scaled stream."""
    lays = _layers()[:1]
    xb = mi.hidden_states_bf16(2, SHAPE.hidden, 0, 11)
    x = mi.bf16_bits_to_f32(xb).astype(np.float64)
    a = orc.stack_forward(lays, xb)
    x4 = (x * 4.0).astype(np.float32)
    xb4 = (x4.view(np.uint32) >> 16).astype(np.uint16)
    b = orc.stack_forward(lays, xb4)
    np.testing.assert_array_equal(a["trace"][0]["idx"], b["trace"][0]["idx"])
    out_a = a["x"] - x                       # bf16(x + out) - x
    out_b = b["x"] - 4.0 * x
    # the two increments are the same MoE output, rounded on different grids
    ulp = np.abs(4.0 * x) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(out_a - out_b) <= ulp)
    assert not np.allclose(b["x"], a["x"])
