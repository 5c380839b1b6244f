"""Pins of the half-integer-level format variant (no GPU).

A 2-bit model keeps each parameter in two bits ("Strata Open Source Project:
Run a 125B Model Locally on a Home PC", section "A Few Things to Keep in
Perspective"); read as four levels, those are the half-integers -3/2, -1/2,
+1/2, +3/2 times the block scale.  The variant generalises to 2**bits levels
q = c - (2**bits - 1)/2 for either bit width.  Pinned here against hand-decoded
bytes, the round-trip bound of the encoder, the float64 statement of the
encoder, and the dense-SwiGLU identity with a decoder written separately from
the oracle's.
"""
import math
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            out.append([p.split() for p in line.split("|")])
    return out


def test_half_level_blocks_hand_decoded():
    rows = _rows("format_blocks_half.txt")
    assert len(rows) == 5
    for bb, scales, codes, expected in rows:
        bits, block = int(bb[0]), int(bb[1])
        sc = np.array([int(s, 16) for s in scales], dtype=np.uint16)
        cd = np.array([int(c, 16) for c in codes], dtype=np.uint8)
        exp = np.array([float(v) for v in expected])
        cols = len(sc) * block
        assert exp.size == cols and cd.size == cols * bits // 8
        np.testing.assert_array_equal(orc.dequantize(cd, sc, 1, cols, bits, block, half=True)[0], exp)


@pytest.mark.parametrize("bits,block", [(2, 16), (4, 32), (4, 128)])
def test_half_level_roundtrip_bound(bits, block):
    """|w - q s| <= max(s/2, absmax - L s) with L = 2**(bits-1) - 1/2 (the
    second term covers an fp16 scale rounded below absmax / L); codes within
    range; an all-zero block decodes to exact zeros; no level is zero."""
    rows, cols = 24, 256
    w = mi.normal_f32(mi.stream_key(11, 2, mi.ROLE_GATE, 1), 0, rows * cols, mi.C_SIGMA002).reshape(rows, cols)
    w[3, :block] = 0.0
    w[5, 7] = 0.5
    codes, scales = mi.quantize_blocks(w, bits, block, half=True)
    L = (1 << (bits - 1)) - 0.5
    c = orc.unpack_codes(codes.reshape(-1), bits, rows * cols)
    assert c.min() >= 0 and c.max() <= (1 << bits) - 1
    back = orc.dequantize(codes, scales, rows, cols, bits, block, half=True)
    s = scales.view(np.float16).astype(np.float64)
    wb = w.astype(np.float64).reshape(rows, cols // block, block)
    amax = np.abs(wb).max(-1)
    bound = np.maximum(s / 2, amax - L * s) * (1 + 1e-6) + 1e-12
    err = np.abs(wb - back.reshape(rows, cols // block, block)).max(-1)
    assert np.all(err <= bound)
    np.testing.assert_array_equal(back[3, :block], 0.0)
    nz = s.repeat(block, axis=1) > 0
    assert np.all(back[nz] != 0.0)                     # half-integer levels: zero is not a level


def test_half_level_encoder_matches_fp64_definition_away_from_boundaries():
    """The generator's fp32 encoder agrees with the float64 statement
    c = clamp(floor(w / s) + 2**(bits-1)) except where w / s sits within fp32
    rounding of an integer (a boundary between two levels)."""
    w = mi.normal_f32(mi.stream_key(5, 0, mi.ROLE_UP, 3), 0, 64 * 512, mi.C_SIGMA002).reshape(64, 512)
    for bits, block in ((2, 16), (4, 32)):
        codes, scales = mi.quantize_blocks(w, bits, block, half=True)
        s = scales.view(np.float16).astype(np.float64).repeat(block, axis=1)
        ratio = w.astype(np.float64) / s
        c64 = np.clip(np.floor(ratio) + (1 << (bits - 1)), 0, (1 << bits) - 1)
        c = orc.unpack_codes(codes.reshape(-1), bits, w.size).reshape(w.shape)
        near = np.abs(ratio - np.rint(ratio)) < 1e-5
        assert np.array_equal(c[~near], c64[~near])
        assert np.mean(near) < 1e-3


def test_two_bit_half_levels_use_all_four_codes():
    w = mi.normal_f32(mi.stream_key(1, 0, mi.ROLE_DOWN, 0), 0, 8 * 2048, mi.C_SIGMA002).reshape(8, 2048)
    codes, _ = mi.quantize_blocks(w, 2, 16, half=True)
    c = orc.unpack_codes(codes.reshape(-1), 2, w.size)
    counts = np.bincount(c, minlength=4)
    # all four levels in use; with s = absmax / (3/2) the outer two hold the
    # elements with |w| >= absmax / (3/2), about a tenth each for these blocks
    assert np.all(counts > 0.05 * w.size)
    assert counts[1] + counts[2] > 0.6 * w.size


def _decode_half(codes_row, scales_row, cols, bits, block):
    """Element-by-element decoder of the half-integer levels, written apart
    from the oracle's."""
    out = []
    for j in range(cols):
        pos = j * bits
        code = (int(codes_row[pos // 8]) >> (pos % 8)) & ((1 << bits) - 1)
        s = float(np.array([scales_row[j // block]], dtype=np.uint16).view(np.float16)[0])
        out.append((2 * code - ((1 << bits) - 1)) / 2.0 * s)
    return out


def test_one_expert_half_level_layer_is_dense_swiglu():
    shape = mi.MoeShape(experts=1, hidden=64, inter=32, top_k=1, shared=False, bits=2, block=16, half=True)
    pool, _ = mi.layer_packed_pool(shape, 7, 0)
    lay = orc.OracleLayer(experts=1, hidden=64, inter=32, top_k=1, bits=2, block=16,
                          router_w_bits=mi.router_weight_bf16(shape, 7, 0), router_bias=None,
                          expert=lambda e: tuple(a[e] for a in pool), shared=lambda: None, half_levels=True)
    x = mi.hidden_states_bf16(3, 64, seed=7)
    r = orc.layer_forward(lay, x)
    gc, gs, dc, ds = lay.expert(0)
    H, I = 64, 32
    w13 = [_decode_half(gc[i], gs[i], H, 2, 16) for i in range(2 * I)]
    wd = [_decode_half(dc[i], ds[i], I, 2, 16) for i in range(H)]
    xf = mi.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        hv = []
        for i in range(I):
            g = math.fsum(w13[2 * i][c] * xf[t, c] for c in range(H))
            u = math.fsum(w13[2 * i + 1][c] * xf[t, c] for c in range(H))
            hv.append(g / (1 + math.exp(-g)) * u)
        y = [math.fsum(wd[rr][i] * hv[i] for i in range(I)) for rr in range(H)]
        np.testing.assert_allclose(r["out"][t], y, rtol=1e-12, atol=1e-15)


def test_integer_and_half_levels_differ():
    """The flag changes the decoded weights (same bytes, different levels)."""
    shape = mi.MoeShape(experts=2, hidden=64, inter=32, top_k=1, shared=False, bits=2, block=16)
    gc, gs, _, _ = mi.expert_packed(shape, 0, 0, 0)
    a = orc.dequantize(gc, gs, 64, 64, 2, 16)
    b = orc.dequantize(gc, gs, 64, 64, 2, 16, half=True)
    s = gs.view(np.float16).astype(np.float64).repeat(16, axis=1)
    np.testing.assert_array_equal(b - a, 0.5 * s)       # q_half = q_int + 1/2 for the same code
