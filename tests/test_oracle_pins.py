"""Pins of the CPU oracle against facts outside itself (no GPU needed).

Each test fixes one part of the oracle with something that does not reuse
the oracle's own code: hand-decoded bytes, closed forms, brute force over all
candidates, independent element-by-element evaluations, invariants.
"""

import itertools
import math
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([p.split() for p in line.split("|")])
    return rows


# ------------------------------------------------------------ the format ---

def test_format_blocks_hand_decoded():
    rows = _read_golden("format_blocks.txt")
    assert len(rows) == 5
    for (bb, scales, codes, expected) in rows:
        bits, block = int(bb[0]), int(bb[1])
        sc = np.array([int(s, 16) for s in scales], dtype=np.uint16)
        cd = np.array([int(c, 16) for c in codes], dtype=np.uint8)
        exp = np.array([float(v) for v in expected])
        cols = len(sc) * block
        assert exp.size == cols and cd.size == cols * bits // 8
        got = orc.dequantize(cd, sc, 1, cols, bits, block)[0]
        np.testing.assert_array_equal(got, exp)


@pytest.mark.parametrize("bits,block", [(4, 32), (4, 128), (2, 16)])
def test_encoder_roundtrip_bound(bits, block):
    """|w - dequant(encode(w))| <= max(s/2, absmax - qmax*s) per element, where
    the second term covers an fp16 scale rounded below absmax/qmax.  A wrong
    nibble order, offset, scale index or sign in the decoder breaks it."""
    rng_key = mi.stream_key(7, 1, mi.ROLE_GATE, 3)
    rows, cols = 24, 256
    w = mi.normal_f32(rng_key, 0, rows * cols, mi.C_SIGMA002).reshape(rows, cols)
    w[3, :block] = 0.0                      # an all-zero block: scale 0, exact
    w[5, 7] = 0.5                           # an outlier block
    codes, scales = mi.quantize_blocks(w, bits, block)
    qmax = (1 << (bits - 1)) - 1
    c = orc.unpack_codes(codes.reshape(-1), bits, rows * cols)
    assert c.min() >= (1 << (bits - 1)) - qmax and c.max() <= (1 << (bits - 1)) + qmax
    back = orc.dequantize(codes, scales, rows, cols, bits, block)
    s = scales.view(np.float16).astype(np.float64)
    wb = w.astype(np.float64).reshape(rows, cols // block, block)
    amax = np.abs(wb).max(-1)
    bound = np.maximum(s / 2, amax - qmax * s) * (1 + 1e-6) + 1e-12
    err = np.abs(wb - back.reshape(rows, cols // block, block)).max(-1)
    assert np.all(err <= bound)
    np.testing.assert_array_equal(back[3, :block], 0.0)
    # the block holding the outlier reproduces it to within half a step
    assert abs(back[5, 7] - 0.5) <= s[5, 0] / 2 * (1 + 1e-6)


def test_encoder_matches_fp64_definition_away_from_ties():
    """The generator's fp32 encoder agrees with the float64 statement of the
    symmetric quantiser except where w/s sits within fp32 rounding of a
    rounding boundary."""
    w = mi.normal_f32(mi.stream_key(3, 0, mi.ROLE_UP, 9), 0, 64 * 512, mi.C_SIGMA002).reshape(64, 512)
    codes, scales = mi.quantize_blocks(w, 4, 32)
    s = scales.view(np.float16).astype(np.float64).repeat(32, axis=1)
    r = w.astype(np.float64) / s
    q64 = np.clip(np.rint(r), -7, 7)
    q = orc.unpack_codes(codes.reshape(-1), 4, w.size).reshape(w.shape) - 8
    near_tie = np.abs(np.abs(r - np.floor(r)) - 0.5) < 1e-5
    assert np.all((q == q64) | near_tie)
    assert np.mean(q == q64) > 0.9999


# -------------------------------------------------------------- numbers ---

def test_round_bf16_cases():
    cases = {1.0 + 2 ** -8: 1.0, 1.0 + 3 * 2 ** -8: 1.0 + 2 ** -6, -(1.0 + 2 ** -8): -1.0,
             0.0: 0.0, 3.0: 3.0, 1.0 + 2 ** -7: 1.0 + 2 ** -7, 0.7071067811865476: 0.70703125}
    for v, e in cases.items():
        assert orc.round_bf16(np.array([v]))[0] == e


def test_round_bf16_agrees_with_generator_rounding():
    f = mi.normal_f32(mi.stream_key(1, 2, 3, 4), 0, 100000, mi.C_SIGMA1)
    via_gen = mi.bf16_bits_to_f32(mi.bf16_bits_from_f32(f)).astype(np.float64)
    np.testing.assert_array_equal(orc.round_bf16(f.astype(np.float64)), via_gen)


def test_rmsnorm_constant_vectors():
    for c, e in [(3.0, 1.0), (0.0, 0.0), (1e-3, 0.70703125), (-2.0, -1.0)]:
        x = np.full((1, 64), c)
        np.testing.assert_array_equal(orc.rmsnorm_bf16(x), np.full((1, 64), e))


def test_silu_closed_forms():
    assert orc.silu(np.array([0.0]))[0] == 0.0
    assert abs(orc.silu(np.array([50.0]))[0] - 50.0) < 1e-18 * 50 + 1e-12
    assert abs(orc.silu(np.array([-50.0]))[0]) < 1e-19
    assert abs(orc.silu(np.array([1.0]))[0] - 1 / (1 + math.exp(-1))) < 1e-16


def test_swiglu_hand_example():
    wg = np.array([[1.0, 0.0]])
    wu = np.array([[0.0, 2.0]])
    wd = np.array([[1.0], [-1.0]])
    for xs, outs in _read_golden("swiglu_tiny.txt"):
        x = np.array([float(v) for v in xs])
        e = np.array([float(v) for v in outs])
        np.testing.assert_allclose(orc.swiglu_ffn(wg, wu, wd, x), e, rtol=1e-15, atol=0)


# --------------------------------------------------------------- router ---

def _brute_topk(l, k):
    """The ordered k-tuple of distinct experts whose (logit, -index) keys are
    lexicographically largest."""
    best, best_key = None, None
    for tup in itertools.permutations(range(l.size), k):
        key = [(l[a], -a) for a in tup]
        if best_key is None or key > best_key:
            best, best_key = tup, key
    return list(best)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(0)
    cases = [rng.normal(size=6) for _ in range(20)]
    cases += [np.array([1.0, 2.0, 2.0, 0.5, 2.0, -1.0]),       # a three-way tie at the top
              np.array([0.0] * 6),                              # all equal
              np.array([3.0, 1.0, 1.0, 1.0, 0.0, 1.0]),         # tie straddling the cut
              np.array([-1.0, -1.0, 5.0, -1.0, 5.0, -7.0])]
    for l in cases:
        for k in (1, 2, 3):
            got = orc.select_topk(l[None, :], k)[0].tolist()
            assert got == _brute_topk(l, k), (l, k)


def test_gate_weights_closed_form_and_invariants():
    l = np.array([[math.log(3.0), 0.0, -100.0, -100.0]])
    idx = orc.select_topk(l, 2)
    w = orc.gate_weights(l, idx)
    assert idx[0].tolist() == [0, 1]
    np.testing.assert_allclose(w[0], [0.75, 0.25], rtol=1e-14)
    rng = np.random.default_rng(1)
    L = rng.normal(size=(16, 64))
    for k in (1, 4, 10):
        idx = orc.select_topk(L, k)
        w = orc.gate_weights(L, idx)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 1e-15)        # descending with the logits
        if k == 1:
            np.testing.assert_array_equal(w, 1.0)
        # equal to a softmax over the selected logits alone, via log-sum-exp
        for t in range(16):
            sel = L[t, idx[t]]
            lse = max(sel) + math.log(math.fsum(math.exp(v - max(sel)) for v in sel))
            np.testing.assert_allclose(w[t], np.exp(sel - lse), rtol=1e-13)


def test_router_logits_hand_case():
    # 2 tokens x 3 hidden, 4 experts, bf16-exact values, one bias
    x = np.array([[1.0, -2.0, 0.5], [0.25, 0.0, 4.0]])
    wr = np.array([[1.0, 1.0, 1.0], [0.5, -0.5, 2.0], [0.0, 0.0, 0.0], [-1.0, 0.125, 1.0]], dtype=np.float32)
    bits = (wr.view(np.uint32) >> 16).astype(np.uint16)
    bias = np.array([0.0, 1.0, -1.0, 0.5])
    got = orc.router_logits(x, bits, bias)
    exp = np.array([[-0.5, 1.0 + 1.5 + 1.0, -1.0, -1.0 - 0.25 + 0.5 + 0.5],
                    [4.25, 0.125 + 8.0 + 1.0, -1.0, -0.25 + 4.0 + 0.5]])
    np.testing.assert_array_equal(got, exp)


def test_grouping_brute_force():
    rng = np.random.default_rng(2)
    for T, k, E in [(1, 1, 4), (5, 3, 8), (17, 4, 16), (64, 10, 512)]:
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, pairs = orc.group_by_expert(idx, E)
        ref = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
        assert pairs.tolist() == [t * k + j for (_, t, j) in ref]
        for e in range(E):
            assert counts[e] == sum(1 for r in ref if r[0] == e)
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.all(np.diff(offsets) == counts)


def test_tie_band_check():
    l = np.array([5.0, 4.0, 3.0, 3.0 - 5e-6, 1.0])
    assert orc.tie_band_ok(l, [0, 1, 2], 3, 1e-5)
    assert orc.tie_band_ok(l, [0, 1, 3], 3, 1e-5)     # swap inside the band
    assert not orc.tie_band_ok(l, [0, 1, 4], 3, 1e-5)
    assert not orc.tie_band_ok(l, [0, 0, 2], 3, 1e-5)


# ---------------------------------------------------------------- layer ---

def _tiny_layer(shape, seed=0, layer=0, bias=None, shared=True, transform=None):
    pool, sh = mi.layer_packed_pool(shape, seed, layer)
    if transform is not None:
        pool, sh = transform(pool, sh)
    return orc.OracleLayer(
        experts=shape.experts, hidden=shape.hidden, inter=shape.inter, top_k=shape.top_k,
        bits=shape.bits, block=shape.block,
        router_w_bits=mi.router_weight_bf16(shape, seed, layer), router_bias=bias,
        expert=lambda e: tuple(a[e] for a in pool),
        shared=(lambda: sh) if shared else (lambda: None))


def _decode_ref(codes_row, scales_row, cols, bits, block):
    """Element-by-element decoder written separately from the oracle's."""
    out = []
    half = 1 << (bits - 1)
    for j in range(cols):
        bitpos = j * bits
        code = (int(codes_row[bitpos // 8]) >> (bitpos % 8)) & ((1 << bits) - 1)
        s = float(np.array([scales_row[j // block]], dtype=np.uint16).view(np.float16)[0])
        out.append((code - half) * s)
    return out


def test_one_expert_layer_is_dense_swiglu():
    """E = 1, k = 1, no shared expert: the gate weight is exactly 1 and the
    layer is a dense SwiGLU FFN; the reference here is plain Python loops."""
    shape = mi.MoeShape(experts=1, hidden=64, inter=32, top_k=1, shared=False, bits=4, block=32)
    lay = _tiny_layer(shape, seed=5, shared=False)
    x = mi.hidden_states_bf16(3, 64, seed=5)
    r = orc.layer_forward(lay, x)
    gc, gs, dc, ds = lay.expert(0)
    H, I = 64, 32
    w13 = [_decode_ref(gc[i], gs[i], H, 4, 32) for i in range(2 * I)]
    wd = [_decode_ref(dc[i], ds[i], I, 4, 32) for i in range(H)]
    xf = mi.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        hvec = []
        for i in range(I):
            g = math.fsum(w13[2 * i][c] * xf[t, c] for c in range(H))
            u = math.fsum(w13[2 * i + 1][c] * xf[t, c] for c in range(H))
            hvec.append(g / (1 + math.exp(-g)) * u)
        y = [math.fsum(wd[r_][i] * hvec[i] for i in range(I)) for r_ in range(H)]
        np.testing.assert_allclose(r["out"][t], y, rtol=1e-12, atol=1e-15)
    assert np.all(r["w"] == 1.0)


def test_shared_expert_is_added_with_weight_one():
    """Zero every routed expert (all scales 0): the layer equals the shared
    expert's FFN on its own."""
    shape = mi.TINY

    def zero_routed(pool, sh):
        gc, gs, dc, ds = pool
        return (gc, np.zeros_like(gs), dc, np.zeros_like(ds)), sh
    lay = _tiny_layer(shape, transform=zero_routed)
    x = mi.hidden_states_bf16(4, shape.hidden, seed=0)
    r = orc.layer_forward(lay, x)
    gc, gs, dc, ds = lay.shared()
    H, I = shape.hidden, shape.inter
    w13 = np.array([_decode_ref(gc[i], gs[i], H, 4, 32) for i in range(2 * I)])
    wd = np.array([_decode_ref(dc[i], ds[i], I, 4, 32) for i in range(H)])
    xf = mi.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(4):
        g, u = w13[0::2] @ xf[t], w13[1::2] @ xf[t]
        np.testing.assert_allclose(r["out"][t], wd @ (g / (1 + np.exp(-g)) * u), rtol=1e-12, atol=1e-15)


def test_linearity_in_down_weights():
    shape = mi.TINY

    def double_down(pool, sh):
        gc, gs, dc, ds = pool
        d2 = (ds.view(np.float16) * np.float16(2)).view(np.uint16)
        s2 = (sh[3].view(np.float16) * np.float16(2)).view(np.uint16)
        return (gc, gs, dc, d2), (sh[0], sh[1], sh[2], s2)
    x = mi.hidden_states_bf16(8, shape.hidden, seed=0)
    a = orc.layer_forward(_tiny_layer(shape), x)["out"]
    b = orc.layer_forward(_tiny_layer(shape, transform=double_down), x)["out"]
    np.testing.assert_array_equal(b, 2 * a)


def test_permutation_invariance_of_expert_storage():
    shape = mi.TINY
    bias = mi.zipf_router_bias(shape, 0, 0, alpha=0.5)
    base = _tiny_layer(shape, bias=bias)
    perm = np.random.default_rng(3).permutation(shape.experts)     # new slot p holds old expert perm[p]
    pool, sh = mi.layer_packed_pool(shape, 0, 0)
    permuted = orc.OracleLayer(
        experts=shape.experts, hidden=shape.hidden, inter=shape.inter, top_k=shape.top_k,
        bits=shape.bits, block=shape.block,
        router_w_bits=mi.router_weight_bf16(shape, 0, 0)[perm], router_bias=bias[perm],
        expert=lambda e: tuple(a[perm[e]] for a in pool), shared=lambda: sh)
    x = mi.hidden_states_bf16(8, shape.hidden, seed=0)
    a = orc.layer_forward(base, x)
    b = orc.layer_forward(permuted, x)
    np.testing.assert_array_equal(perm[b["idx"]], a["idx"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=1e-12, atol=1e-14)


def test_tiny_layer_runs_fast_and_is_sane():
    import time
    shape = mi.TINY
    lay = _tiny_layer(shape)
    x = mi.hidden_states_bf16(8, shape.hidden, seed=0)
    t0 = time.time()
    r = orc.layer_forward(lay, x)
    assert time.time() - t0 < 1.0
    assert r["out"].shape == (8, shape.hidden) and np.all(np.isfinite(r["out"]))
    np.testing.assert_allclose(r["w"].sum(1), 1.0, atol=1e-12)


def test_zipf_alpha_matches_calibration():
    import json
    with open(os.path.join(GOLDEN, "zipf_alpha.json")) as f:
        cal = json.load(f)
    assert mi.ZIPF_ALPHA == cal["alpha"]
    # a smaller batch lands near the calibrated 95% hot share
    shape = mi.FULL2
    x = mi.hidden_states_bf16(1024, shape.hidden, seed=0, batch=77)
    bias = mi.zipf_router_bias(shape, 0, 0)
    l = orc.router_logits(orc.bf16_to_f64(x), mi.router_weight_bf16(shape, 0, 0), bias)
    idx = orc.select_topk(l, shape.top_k)
    rank = np.rint(np.exp(bias.astype(np.float64) / -mi.ZIPF_ALPHA)).astype(np.int64)
    assert abs(np.mean(rank[idx] <= 102) - 0.95) < 0.02


# ----------------------------------------------- gated shared expert (variant)

def test_shared_gate_weight_closed_form():
    """sigmoid of an exactly representable dot product, evaluated by hand."""
    shape = mi.MoeShape(experts=4, hidden=8, inter=4, top_k=1, shared=True, bits=4, block=4)
    gate = mi.bf16_bits_from_f32(np.array([0.5, -0.25, 1.0, 0, 0, 0, 0, 2.0], dtype=np.float32))
    lay = orc.OracleLayer(experts=4, hidden=8, inter=4, top_k=1, bits=4, block=4,
                          router_w_bits=np.zeros((4, 8), np.uint16), router_bias=None,
                          expert=lambda e: None, shared=lambda: None, shared_gate_w_bits=gate)
    x = np.array([2.0, 4.0, -1.0, 7.0, 7.0, 7.0, 7.0, 0.5])
    z = 0.5 * 2.0 - 0.25 * 4.0 + 1.0 * -1.0 + 2.0 * 0.5          # 1 - 1 - 1 + 1
    assert z == 0.0
    assert lay.shared_weight(x) == 0.5
    x2 = x.copy()
    x2[7] = 3.0                                                     # z = 1 - 1 - 1 + 6 = 5
    assert abs(lay.shared_weight(x2) - 1.0 / (1.0 + math.exp(-5.0))) < 1e-15
    assert _tiny_layer(shape=mi.TINY).shared_weight(x) == 1.0      # no gate: weight 1


def test_zero_gate_halves_the_shared_expert():
    shape = mi.TINY
    x = mi.hidden_states_bf16(6, shape.hidden, seed=9)
    with_sh = orc.layer_forward(_tiny_layer(shape), x)["out"]
    no_sh = orc.layer_forward(_tiny_layer(shape, shared=False), x)["out"]
    zero_gate = _tiny_layer(shape)
    zero_gate.shared_gate_w_bits = np.zeros(shape.hidden, np.uint16)
    half = orc.layer_forward(zero_gate, x)["out"]
    np.testing.assert_allclose(half, no_sh + 0.5 * (with_sh - no_sh), rtol=0, atol=1e-12 * np.abs(with_sh).max())


def test_gated_layer_partials_sum_to_the_layer():
    shape = mi.TINY
    lay = _tiny_layer(shape)
    lay.shared_gate_w_bits = mi.shared_gate_weight_bf16(shape, 0, 0)
    x = mi.hidden_states_bf16(6, shape.hidden, seed=10)
    full = orc.layer_forward(lay, x)["out"]
    parts = [orc.layer_forward_ep(lay, x, r, 3)["partial"] for r in range(3)]
    np.testing.assert_allclose(sum(parts), full, rtol=0, atol=1e-12 * np.abs(full).max())
