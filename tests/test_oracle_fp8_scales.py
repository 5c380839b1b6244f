"""Pins of the fp8-scale format variant (no GPU).

The pages' grouped symmetric quantiser ("Running Massive Language Models on
Consumer Hardware Without Breaking the Bank", section "Quantization
Techniques That Actually Work") keeps one scale per group; in this variant
that scale is one E4M3 byte (the OCP 8-bit floating-point format: 4 exponent
bits with bias 7, 3 mantissa bits, no infinities, largest finite 448) under
one fp32 scale per weight row, so w = q * e4m3(byte) * row_scale.  Pinned here
against hand-decoded bytes, the values the E4M3 definition prints (largest
finite 448, smallest normal 2^-6, smallest subnormal 2^-9, NaN at 0x7F), the
format's structure (eight evenly spaced values per binade, subnormals
continuing the first binade's spacing), the encoder's round trip and
round-to-nearest-even, the quantiser's error bound, and the dense-SwiGLU
identity with a decoder written separately from the oracle's.
"""
import math
import os
import struct

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


def test_fp8_blocks_hand_decoded():
    rows = _rows("format_blocks_fp8.txt")
    assert len(rows) == 4
    for bb, rs, scales, codes, expected in rows:
        bits, block = int(bb[0]), int(bb[1])
        row_scale = np.array([struct.unpack(">f", bytes.fromhex(rs[0]))[0]], dtype=np.float32)
        sb = np.array([int(s, 16) for s in scales], dtype=np.uint8)
        cd = np.array([int(c, 16) for c in codes], dtype=np.uint8)
        exp = np.array([float(v) for v in expected])
        cols = len(sb) * block
        assert exp.size == cols and cd.size == cols * bits // 8
        got = orc.dequantize(cd, sb, 1, cols, bits, block, row_scale=row_scale)[0]
        np.testing.assert_array_equal(got, exp)


def test_e4m3_printed_values():
    v = orc.e4m3_value
    assert v(0x7E) == 448.0                      # largest finite
    assert v(0x08) == 2.0 ** -6                  # smallest normal
    assert v(0x01) == 2.0 ** -9                  # smallest subnormal
    assert v(0x38) == 1.0 and v(0x40) == 2.0 and v(0x30) == 0.5
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    assert v(0x00) == 0.0 and v(0x80) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    c = np.arange(0x7F)
    np.testing.assert_array_equal(v(c | 0x80), -v(c))


def test_e4m3_structure():
    """Finite non-negative codes are strictly increasing; each binade holds
    eight evenly spaced values with spacing 2^(e-10) and starts at twice the
    previous one; the subnormals continue the first binade's spacing 2^-9."""
    c = np.arange(0x7F)
    val = orc.e4m3_value(c)
    assert np.all(np.diff(val) > 0)
    for e in range(1, 16):
        b = val[e * 8:e * 8 + 8] if e < 15 else val[e * 8:e * 8 + 7]
        np.testing.assert_array_equal(np.diff(b), 2.0 ** (e - 10))
        if e > 1:
            assert val[e * 8] == 2 * val[(e - 1) * 8]
    np.testing.assert_array_equal(np.diff(val[:9]), 2.0 ** -9)


def test_encoder_round_trip_and_nearest_even():
    c = np.arange(0x7F)
    val = orc.e4m3_value(c)
    np.testing.assert_array_equal(mi.gen.e4m3_encode(val.astype(np.float32)), c)
    # midpoints between neighbours go to the even mantissa; other values to the nearest
    mids = ((val[:-1] + val[1:]) / 2).astype(np.float32)
    enc = mi.gen.e4m3_encode(mids)
    want = np.where(c[:-1] % 2 == 0, c[:-1], c[1:])
    np.testing.assert_array_equal(enc, want)
    rng = np.random.default_rng(5)
    t = (rng.random(20000) * 460).astype(np.float32)
    t = np.concatenate([t, (rng.random(2000) * 0.02).astype(np.float32)])
    got = orc.e4m3_value(mi.gen.e4m3_encode(t))
    err = np.abs(got - t.astype(np.float64))
    best = np.min(np.abs(val[None, :] - t.astype(np.float64)[:, None]), axis=1)
    np.testing.assert_array_equal(err, best)     # nearest representable (saturating at 448)


@pytest.mark.parametrize("bits,block", [(4, 32), (2, 16)])
def test_fp8_quantizer_bound(bits, block):
    """|w - q s| <= max(s/2, blockmax - qmax s) with s = e4m3(byte) * S; the
    row scale maps the row's largest block to the largest E4M3 value; codes
    stay in range; an all-zero row decodes to exact zeros."""
    rows, cols = 20, 512
    w = mi.normal_f32(mi.stream_key(4, 1, mi.ROLE_DOWN, 2), 0, rows * cols, mi.C_SIGMA002).reshape(rows, cols)
    w[6] = 0.0
    w[9, 3] = 0.3                                 # one outlier row
    codes, s8, S = mi.gen.quantize_blocks_e4m3(w, bits, block)
    qmax = (1 << (bits - 1)) - 1
    back = orc.dequantize(codes, s8, rows, cols, bits, block, row_scale=S)
    s = orc.e4m3_value(s8) * S.astype(np.float64)[:, None]
    wb = w.astype(np.float64).reshape(rows, cols // block, block)
    amax = np.abs(wb).max(-1)
    bound = np.maximum(s / 2, amax - qmax * s) * (1 + 1e-6) + 1e-12
    err = np.abs(wb - back.reshape(rows, cols // block, block)).max(-1)
    assert np.all(err <= bound)
    np.testing.assert_array_equal(back[6], 0.0)
    assert np.all(s8 <= 0x7E)
    rmax = np.abs(w).max(1).astype(np.float64)
    nz = rmax > 0
    # the block holding the row's maximum gets (about) 448, i.e. byte 0x7E or its neighbour
    top = s8[np.arange(rows), np.argmax(amax, axis=1)]
    assert np.all(top[nz] >= 0x7D)
    np.testing.assert_allclose(S[nz].astype(np.float64) * qmax * 448, rmax[nz], rtol=1e-6)
    c = orc.unpack_codes(codes.reshape(-1), bits, rows * cols)
    assert c.min() >= 1 and c.max() <= (1 << bits) - 1     # q in [-qmax, qmax]


def test_fp8_encoder_matches_fp64_definition_away_from_ties():
    w = mi.normal_f32(mi.stream_key(8, 0, mi.ROLE_UP, 1), 0, 48 * 256, mi.C_SIGMA002).reshape(48, 256)
    for bits, block in ((4, 32), (2, 16)):
        codes, s8, S = mi.gen.quantize_blocks_e4m3(w, bits, block)
        qmax = (1 << (bits - 1)) - 1
        s = (orc.e4m3_value(s8) * S.astype(np.float64)[:, None]).repeat(block, axis=1)
        ratio = w.astype(np.float64) / s
        q64 = np.clip(np.rint(ratio), -qmax, qmax)
        q = orc.unpack_codes(codes.reshape(-1), bits, w.size).reshape(w.shape) - (1 << (bits - 1))
        near = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5) < 1e-5
        assert np.array_equal(q[~near], q64[~near])
        assert np.mean(near) < 1e-3


def _decode_fp8(codes_row, scale_bytes, row_scale, cols, bits, block):
    """Element-by-element decoder of the fp8-scale format, written apart from
    the oracle's: the E4M3 byte read field by field."""
    out = []
    for j in range(cols):
        pos = j * bits
        code = (int(codes_row[pos // 8]) >> (pos % 8)) & ((1 << bits) - 1)
        b = int(scale_bytes[j // block])
        expo, man = (b >> 3) & 15, b & 7
        sv = (man * 2.0 ** -9) if expo == 0 else (8 + man) * 2.0 ** (expo - 10)
        sv = -sv if b & 0x80 else sv
        out.append((code - (1 << (bits - 1))) * sv * float(row_scale))
    return out


def test_one_expert_fp8_layer_is_dense_swiglu():
    shape = mi.MoeShape(experts=1, hidden=64, inter=32, top_k=1, shared=False, bits=4, block=32, fp8_scales=True)
    pool, _ = mi.layer_packed_pool(shape, 5, 0)
    lay = orc.OracleLayer(experts=1, hidden=64, inter=32, top_k=1, bits=4, block=32,
                          router_w_bits=mi.router_weight_bf16(shape, 5, 0), router_bias=None,
                          expert=lambda e: tuple(a[e] for a in pool), shared=lambda: None)
    x = mi.hidden_states_bf16(3, 64, seed=5)
    r = orc.layer_forward(lay, x)
    gc_, gs, dc, ds, grs, drs = lay.expert(0)
    H, I = 64, 32
    w13 = [_decode_fp8(gc_[i], gs[i], grs[i], H, 4, 32) for i in range(2 * I)]
    wd = [_decode_fp8(dc[i], ds[i], drs[i], I, 4, 32) for i in range(H)]
    xf = mi.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        hv = []
        for i in range(I):
            g = math.fsum(w13[2 * i][c] * xf[t, c] for c in range(H))
            u = math.fsum(w13[2 * i + 1][c] * xf[t, c] for c in range(H))
            hv.append(g / (1 + math.exp(-g)) * u)
        y = [math.fsum(wd[rr][i] * hv[i] for i in range(I)) for rr in range(H)]
        np.testing.assert_allclose(r["out"][t], y, rtol=1e-12, atol=1e-15)
