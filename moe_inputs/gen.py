"""Counter-based synthetic input generator (numpy side).

Recipe (identical on the CUDA side, ``csrc/gen_device.cu``):

* Hash: the SplitMix64 output function (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014), ``mix64``.
* Stream key for (seed, layer, role, expert):
  ``k = mix64(mix64(mix64(mix64(seed) + layer) + role) + expert)``
  (all arithmetic modulo 2**64).
* Element ``i`` of a stream: ``z = mix64(k + (i + 1) * GOLDEN)``.
* Approximate normal deviate: the Irwin-Hall sum of the four 16-bit fields
  of ``z``; ``D = 2 * (u0 + u1 + u2 + u3) - 262140`` is an even integer with
  mean 0 and standard deviation 75674.45, so ``D * (sigma / 75674.45)`` has
  standard deviation ``sigma`` (bounded at 3.46 sigma, kurtosis 2.7).  The
  product is one correctly rounded fp32 multiply by a fixed fp32 constant.
* bf16 tensors (hidden states, router weights): round-to-nearest-even of
  that fp32 value.
* Packed expert weights: fp32 masters of N(0, 0.02), encoded per block of
  ``block`` elements along the reduction axis by the symmetric absmax
  quantiser: ``s = fp16(fp32(absmax / qmax))``, ``q = clamp(rint(w / s),
  -qmax, qmax)`` (``q = 0`` where ``s == 0``), ``qmax = 2**(bits-1) - 1``,
  stored code ``c = q + 2**(bits-1)``, lower element index in the lower bits
  of each byte.  Half-integer levels (the format variant with 2**bits levels
  +-1/2 ... +-(2**(bits-1) - 1/2), e.g. four for 2-bit):
  ``s = fp16(fp32(absmax / L))`` with ``L = 2**(bits-1) - 1/2``, ``c =
  clamp(floor(fp32(w / s)) + 2**(bits-1), 0, 2**bits - 1)`` (the level just
  above w / s, so a value exactly on a boundary takes the upper level;
  ``c = 2**(bits-1)`` where ``s == 0``), decoded as ``q = c - (2**bits - 1)/2``.

Element indices: gate / up masters are ``[I, H]`` (index ``i*H + h``), down
masters ``[H, I]`` (index ``r*I + i``).  The packed gate/up matrix
interleaves rows: packed row ``2i`` is gate row ``i``, packed row ``2i + 1``
is up row ``i``.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "GOLDEN", "ROLE_ROUTER", "ROLE_GATE", "ROLE_UP", "ROLE_DOWN", "ROLE_SH_GATE",
    "ROLE_SH_UP", "ROLE_SH_DOWN", "ROLE_X", "ROLE_PERM", "ROLE_SH_GATE_W", "C_SIGMA1", "C_SIGMA002",
    "ZIPF_ALPHA", "MoeShape", "TINY", "FULL4", "FULL2", "mix64", "stream_key",
    "normal_f32", "bf16_bits_from_f32", "bf16_bits_to_f32", "quantize_blocks",
    "masters", "expert_packed", "shared_packed", "router_weight_bf16", "shared_gate_weight_bf16",
    "hidden_states_bf16", "zipf_router_bias", "layer_packed_pool",
    "packed_row_bytes", "scales_per_row",
]

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

ROLE_ROUTER, ROLE_GATE, ROLE_UP, ROLE_DOWN = 0, 1, 2, 3
ROLE_SH_GATE, ROLE_SH_UP, ROLE_SH_DOWN = 4, 5, 6
ROLE_X, ROLE_PERM = 7, 8
ROLE_SH_GATE_W = 9          # the shared expert's gate vector (format variant)

# sigma / std(D) rounded to fp32 once; both sides receive these exact bits.
_STD_D = math.sqrt(4.0 / 3.0 * (65536.0 ** 2 - 1.0))
C_SIGMA1 = np.float32(1.0 / _STD_D)        # 0x375db3d7
C_SIGMA002 = np.float32(0.02 / _STD_D)     # 0x348de3bd

# Router-bias strength of the skewed (Zipf-ranked) workload.  Found by
# bisection with the oracle's router (tests/golden/make_zipf_alpha.py) so that
# 95% of top-10 picks of an 8192-token batch land on the top 20% (102) of the
# 512 experts; the stored value is tests/golden/zipf_alpha.json.
ZIPF_ALPHA = 0.7175


@dataclasses.dataclass(frozen=True)
class MoeShape:
    """Shape and format of one MoE layer."""
    experts: int
    hidden: int
    inter: int
    top_k: int
    shared: bool
    bits: int
    block: int
    half: bool = False          # half-integer levels (2**bits levels, no zero)
    fp8_scales: bool = False    # E4M3 block scales under one fp32 scale per row

    @property
    def qmax(self) -> int:
        return (1 << (self.bits - 1)) - 1


TINY = MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=4, block=32)
FULL4 = MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=32)
FULL2 = MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=2, block=16)


def _u64(v) -> np.uint64:
    return np.uint64(int(v) & MASK64)


def mix64(z):
    """SplitMix64 output function on a uint64 scalar or array (wrapping)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z ^ (z >> np.uint64(30))
        z = z * np.uint64(_M1)
        z = z ^ (z >> np.uint64(27))
        z = z * np.uint64(_M2)
        z = z ^ (z >> np.uint64(31))
    return z


def _mix64_int(z: int) -> int:
    z &= MASK64
    z ^= z >> 30
    z = (z * _M1) & MASK64
    z ^= z >> 27
    z = (z * _M2) & MASK64
    z ^= z >> 31
    return z


def stream_key(seed: int, layer: int, role: int, expert: int) -> int:
    k = _mix64_int(seed)
    k = _mix64_int(k + layer)
    k = _mix64_int(k + role)
    k = _mix64_int(k + expert)
    return k


def _irwin_hall_d(key: int, start: int, count: int) -> np.ndarray:
    """Even integers D (int32) of elements start .. start+count-1."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = mix64(_u64(key) + idx * np.uint64(GOLDEN))
    m = np.uint64(0xFFFF)
    s = (z & m) + ((z >> np.uint64(16)) & m) + ((z >> np.uint64(32)) & m) + (z >> np.uint64(48))
    return (2 * s.astype(np.int64) - 262140).astype(np.int32)


def normal_f32(key: int, start: int, count: int, c: np.float32) -> np.ndarray:
    """fp32 deviates of standard deviation c * 75674.45 (c = C_SIGMA1 or C_SIGMA002)."""
    d = _irwin_hall_d(key, start, count).astype(np.float32)  # |D| < 2**18: exact
    return d * np.float32(c)


def bf16_bits_from_f32(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    return (b >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def packed_row_bytes(cols: int, bits: int) -> int:
    return cols * bits // 8


def scales_per_row(cols: int, block: int) -> int:
    return cols // block


def quantize_blocks(w: np.ndarray, bits: int, block: int, half: bool = False):
    """Encode fp32 masters [rows, cols] into (codes uint8 [rows, cols*bits/8],
    scales uint16 fp16-bits [rows, cols/block]).  Input preparation only."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % block == 0 and bits in (2, 4)
    qmax = (1 << (bits - 1)) - 1
    wb = w.reshape(rows, cols // block, block)
    amax = np.max(np.abs(wb), axis=-1)
    top = np.float32(qmax + 0.5) if half else np.float32(qmax)
    s16 = (amax / top).astype(np.float32).astype(np.float16)
    sf = s16.astype(np.float32)
    safe = np.where(sf == 0, np.float32(1), sf)
    with np.errstate(invalid="ignore", divide="ignore"):
        ratio = (wb / safe[..., None]).astype(np.float32)
    if half:
        c = np.clip(np.floor(ratio) + (1 << (bits - 1)), 0, (1 << bits) - 1)
        c[sf == 0] = 1 << (bits - 1)
        c = c.astype(np.uint8).reshape(rows, cols)
    else:
        q = np.clip(np.rint(ratio), -qmax, qmax)
        q[sf == 0] = 0
        c = (q.astype(np.int32) + (1 << (bits - 1))).astype(np.uint8).reshape(rows, cols)
    if bits == 4:
        codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    else:
        codes = (c[:, 0::4] | (c[:, 1::4] << 2) | (c[:, 2::4] << 4) | (c[:, 3::4] << 6)).astype(np.uint8)
    return np.ascontiguousarray(codes), np.ascontiguousarray(s16.view(np.uint16))


E4M3_MAX = 448.0


def e4m3_encode(t: np.ndarray) -> np.ndarray:
    """Nearest E4M3 byte (ties to even, saturating at 448) of non-negative
    fp32 values: 4 exponent bits with bias 7, 3 mantissa bits, exponent field
    0 for the subnormals m * 2**-9.  Input preparation only."""
    t = np.asarray(t, dtype=np.float32)
    out = np.zeros(t.shape, dtype=np.uint8)
    sub = t < np.float32(2.0 ** -6)
    m_sub = np.rint(t[sub] * np.float32(512.0)).astype(np.int32)     # exact scaling; 8 -> 2**-6, code 8
    out[sub] = m_sub.astype(np.uint8)
    nt = t[~sub]
    mant, ex = np.frexp(nt)                                            # nt = mant * 2**ex, mant in [0.5, 1)
    e = ex.astype(np.int32) - 1
    m = np.rint((mant * np.float32(2.0) - np.float32(1.0)) * np.float32(8.0)).astype(np.int32)
    carry = m == 8
    e = e + carry
    m = np.where(carry, 0, m)
    code = ((e + 7) << 3) | m
    out[~sub] = np.minimum(code, 0x7E).astype(np.uint8)
    return out


def _e4m3_f32(code: np.ndarray) -> np.ndarray:
    """fp32 value of non-negative E4M3 codes (the encoder's own view of what it
    chose)."""
    code = np.asarray(code, dtype=np.int32)
    e, m = (code >> 3) & 15, code & 7
    val = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e.astype(np.float64) - 10))
    return val.astype(np.float32)


def quantize_blocks_e4m3(w: np.ndarray, bits: int, block: int):
    """Encode fp32 masters [rows, cols] with integer levels, one E4M3 scale
    byte per block and one fp32 scale per row: S = rowmax|w| / (qmax * 448),
    scale byte = e4m3(blockmax|w| / (qmax * S)), q = clamp(rint(w / (e4m3 * S))).
    Returns (codes uint8 [rows, cols*bits/8], scale bytes uint8
    [rows, cols/block], row scales float32 [rows]).  Input preparation only."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % block == 0 and bits in (2, 4)
    qmax = (1 << (bits - 1)) - 1
    wb = w.reshape(rows, cols // block, block)
    amax = np.max(np.abs(wb), axis=-1)                                  # [rows, nb]
    rmax = np.max(amax, axis=-1)                                        # [rows]
    S = (rmax / np.float32(qmax * E4M3_MAX)).astype(np.float32)
    den = (S * np.float32(qmax)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = np.where(den[:, None] > 0, amax / np.where(den > 0, den, np.float32(1))[:, None], 0).astype(np.float32)
    s8 = e4m3_encode(t)
    sf = (_e4m3_f32(s8) * S[:, None]).astype(np.float32)
    safe = np.where(sf == 0, np.float32(1), sf)
    ratio = (wb / safe[..., None]).astype(np.float32)
    q = np.clip(np.rint(ratio), -qmax, qmax)
    q[sf == 0] = 0
    c = (q.astype(np.int32) + (1 << (bits - 1))).astype(np.uint8).reshape(rows, cols)
    if bits == 4:
        codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    else:
        codes = (c[:, 0::4] | (c[:, 1::4] << 2) | (c[:, 2::4] << 4) | (c[:, 3::4] << 6)).astype(np.uint8)
    return np.ascontiguousarray(codes), np.ascontiguousarray(s8), np.ascontiguousarray(S)


def masters(shape: MoeShape, seed: int, layer: int, expert: int):
    """fp32 masters (gate [I,H], up [I,H], down [H,I]) of routed expert
    ``expert`` (0 <= expert < E) or of the shared expert (expert == -1)."""
    H, I = shape.hidden, shape.inter
    if expert < 0:
        roles, ex = (ROLE_SH_GATE, ROLE_SH_UP, ROLE_SH_DOWN), 0
    else:
        roles, ex = (ROLE_GATE, ROLE_UP, ROLE_DOWN), expert
    g = normal_f32(stream_key(seed, layer, roles[0], ex), 0, I * H, C_SIGMA002).reshape(I, H)
    u = normal_f32(stream_key(seed, layer, roles[1], ex), 0, I * H, C_SIGMA002).reshape(I, H)
    d = normal_f32(stream_key(seed, layer, roles[2], ex), 0, H * I, C_SIGMA002).reshape(H, I)
    return g, u, d


def expert_packed(shape: MoeShape, seed: int, layer: int, expert: int):
    """Packed (gu_codes, gu_scales, d_codes, d_scales) of one expert.

    gu_codes [2I, H*bits/8] uint8, gu_scales [2I, H/block] fp16 bits,
    d_codes [H, I*bits/8] uint8, d_scales [H, I/block] fp16 bits.  With
    fp8 scales: gu_scales / d_scales are E4M3 bytes and two more arrays
    follow, the fp32 row scales gu_rs [2I] and d_rs [H]."""
    g, u, d = masters(shape, seed, layer, expert)
    w13 = np.empty((2 * shape.inter, shape.hidden), dtype=np.float32)
    w13[0::2] = g
    w13[1::2] = u
    if shape.fp8_scales:
        assert not shape.half, "fp8 block scales come with the integer levels"
        gc, gs, grs = quantize_blocks_e4m3(w13, shape.bits, shape.block)
        dc, ds, drs = quantize_blocks_e4m3(d, shape.bits, shape.block)
        return gc, gs, dc, ds, grs, drs
    gc, gs = quantize_blocks(w13, shape.bits, shape.block, shape.half)
    dc, ds = quantize_blocks(d, shape.bits, shape.block, shape.half)
    return gc, gs, dc, ds


def shared_packed(shape: MoeShape, seed: int, layer: int):
    return expert_packed(shape, seed, layer, -1)


def router_weight_bf16(shape: MoeShape, seed: int, layer: int) -> np.ndarray:
    """Router weight [E, H] as bf16 bits, N(0, 0.02)."""
    n = shape.experts * shape.hidden
    f = normal_f32(stream_key(seed, layer, ROLE_ROUTER, 0), 0, n, C_SIGMA002)
    return bf16_bits_from_f32(f).reshape(shape.experts, shape.hidden)


def shared_gate_weight_bf16(shape: MoeShape, seed: int, layer: int) -> np.ndarray:
    """The shared expert's gate vector [H] as bf16 bits, N(0, 0.02)."""
    f = normal_f32(stream_key(seed, layer, ROLE_SH_GATE_W, 0), 0, shape.hidden, C_SIGMA002)
    return bf16_bits_from_f32(f)


def hidden_states_bf16(tokens: int, hidden: int, seed: int, batch: int = 0) -> np.ndarray:
    """Hidden states [T, H] as bf16 bits, N(0, 1); token t of a batch does not
    depend on T."""
    f = normal_f32(stream_key(seed, 0, ROLE_X, batch), 0, tokens * hidden, C_SIGMA1)
    return bf16_bits_from_f32(f).reshape(tokens, hidden)


def zipf_router_bias(shape: MoeShape, seed: int, layer: int, alpha: float = ZIPF_ALPHA) -> np.ndarray:
    """fp32 router bias b_e = -alpha * ln(rank_e), rank_e in 1..E from a seeded
    permutation of the experts (host-only input)."""
    key = stream_key(seed, layer, ROLE_PERM, 0)
    h = mix64(_u64(key) + np.arange(1, shape.experts + 1, dtype=np.uint64) * np.uint64(GOLDEN))
    order = np.argsort(h, kind="stable")          # order[r-1] = expert of rank r
    rank = np.empty(shape.experts, dtype=np.float64)
    rank[order] = np.arange(1, shape.experts + 1, dtype=np.float64)
    return (-alpha * np.log(rank)).astype(np.float32)


def layer_packed_pool(shape: MoeShape, seed: int, layer: int):
    """Whole-layer packed pool on the host (small shapes only): arrays with a
    leading expert axis, plus the shared expert's arrays (or None)."""
    parts = [expert_packed(shape, seed, layer, e) for e in range(shape.experts)]
    pool = tuple(np.stack([p[i] for p in parts]) for i in range(len(parts[0])))
    sh = shared_packed(shape, seed, layer) if shape.shared else None
    return pool, sh
