"""Float64 CPU oracle of the quantized-expert MoE FFN layer (test infrastructure).

What the layer computes, per token (pages cited by title and section):

* The FFN of the transformer block is replaced by many parallel expert
  sub-networks and a light gating network (the router) picks the Top-K of
  them for each token ("Running a 125B Model on a Single RTX 5090: Strata
  Benchmarks Qwen3.8 Flash Next", section "Layer 1: On-Demand MoE Expert
  Scheduling"; "Strata Open Source Project: Run a 125B Model Locally on a
  Home PC", section "How Strata Makes Your Entire PC Work Together": 512
  experts per layer, 10 selected per token, 24,576 experts in all).
* Besides the 10 routed experts one shared expert is active for every token
  ("How a 125B Model Reaches 100 Tok/s on an RTX 4090", section "The model is
  large on paper, sparse in practice").
* Expert weights are stored as symmetric, group-wise quantised low-bit
  integers, 4-bit or 2-bit ("Running Massive Language Models on Consumer
  Hardware Without Breaking the Bank", sections "How Strata Makes the
  Impossible Possible" and "Quantization Techniques That Actually Work":
  bits=4, sym=True, grouped; "Strata Open Source Project...", section "A Few
  Things to Keep in Perspective": a 2-bit model).

Readings where the pages are silent (each one is listed with its reason in
the design notes): the router is a softmax over fp32 logits renormalised over
the selected experts; selection is by logit with ties going to the smaller
expert index, slots ordered by descending logit; the expert FFN is SwiGLU,
``W_down (silu(W_gate x) * (W_up x))``; the shared expert is added with
weight 1; packed codes are offset binary ``c = q + 2**(bits-1)`` with one
fp16 scale per block of ``block`` elements along the reduction axis, the lower
element in the lower bits of each byte; packed gate/up rows interleave (row
2i gate i, row 2i+1 up i); in the 48-layer stack each layer is
``x <- bf16(x + moe(bf16(rmsnorm(x))))`` with RMSNorm weight 1, eps 1e-6.

Format variants (readings of the pages' grouped symmetric quantiser): codes
read as half-integer levels ``q = c - (2**bits - 1)/2``; one E4M3 (fp8) scale
byte per block under one fp32 scale per weight row.

Precision: everything is float64 except what the interface fixes: bf16 at the
hidden states, the RMSNorm output and the stack's residual stream, fp16 (or
E4M3 times fp32) scales.

Pins (tests/test_oracle_*.py): hand-decoded bytes of the format
(tests/golden/format_blocks.txt), the round-trip bound of the block encoder,
brute-force top-k over all ordered k-tuples with constructed ties, closed-form
gate weights, brute-force stable grouping, the dense-SwiGLU identity of an
E=1, k=1 layer against an independent element-by-element evaluation, a hand
computed SwiGLU example (tests/golden/swiglu_tiny.txt), linearity in the down
weights, permutation invariance of expert storage, the RMSNorm closed form on
constant vectors and exact bf16 rounding cases; the stack against an
element-by-element restatement; the half-integer levels and the E4M3 scales
against hand-decoded bytes (tests/golden/format_blocks_half.txt,
tests/golden/format_blocks_fp8.txt) and the format's printed values.
"""

from __future__ import annotations

import dataclasses
from typing import Callable, Optional

import math

import numpy as np

__all__ = [
    "bf16_to_f64", "round_bf16", "unpack_codes", "e4m3_value", "dequantize", "router_logits",
    "select_topk", "gate_weights", "group_by_expert", "silu", "swiglu_ffn",
    "rmsnorm_bf16", "OracleLayer", "layer_forward", "layer_forward_ep", "stack_forward",
    "tie_band_ok", "RMS_EPS",
]

RMS_EPS = 1e-6


# ---------------------------------------------------------------- numbers ---

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned
    as float64.  bf16 keeps 8 significant bits; no value here reaches the
    overflow or subnormal range."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                       # v = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


# ------------------------------------------------------- packed weights ---

def unpack_codes(codes: np.ndarray, bits: int, n: int) -> np.ndarray:
    """Stored codes (0 .. 2**bits - 1) of the first n elements of a packed row
    vector: element j sits in byte j*bits//8 at bit offset (j*bits) % 8."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    j = np.arange(n)
    byte = codes[(j * bits) // 8].astype(np.int64)
    return (byte >> ((j * bits) % 8)) & ((1 << bits) - 1)


def e4m3_value(code) -> np.ndarray:
    """float64 value of E4M3 bytes (the OCP 8-bit floating-point format with
    4 exponent bits and 3 mantissa bits): sign s = bit 7, exponent field
    e = bits 3..6 with bias 7, mantissa m = bits 0..2; e = 0 encodes the
    subnormals (-1)**s * m/8 * 2**-6, otherwise (-1)**s * (1 + m/8) * 2**(e-7);
    the pattern e = 15, m = 7 is NaN (there are no infinities), so the largest
    finite value is 1.75 * 2**8 = 448."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequantize(codes: np.ndarray, scales_bits: np.ndarray, rows: int, cols: int,
               bits: int, block: int, half: bool = False, row_scale: Optional[np.ndarray] = None) -> np.ndarray:
    """Weights w[r, c] = q * scale[r, c // block] in float64, q = code -
    2**(bits-1) (integer levels), or q = code - (2**bits - 1) / 2 for the
    half-integer levels (2**bits levels symmetric about zero, e.g. +-1/2,
    +-3/2 for 2 bits).  Exact: a small integer or half-integer times an fp16
    value.  With ``row_scale`` (fp32 [rows]) the block scales are E4M3 bytes
    and scale[r, b] = e4m3(byte) * row_scale[r] (fp8 block scales under one
    fp32 scale per row), again exact in float64."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(rows, cols * bits // 8)
    if row_scale is None:
        scales = np.asarray(scales_bits, dtype=np.uint16).view(np.float16)
        scales = scales.reshape(rows, cols // block).astype(np.float64)
    else:
        sb = np.asarray(scales_bits, dtype=np.uint8).reshape(rows, cols // block)
        rsf = np.asarray(row_scale, dtype=np.float32).reshape(rows).astype(np.float64)
        scales = e4m3_value(sb) * rsf[:, None]
    offset = ((1 << bits) - 1) / 2.0 if half else float(1 << (bits - 1))
    w = np.empty((rows, cols), dtype=np.float64)
    for r in range(rows):
        q = unpack_codes(codes[r], bits, cols) - offset
        w[r] = q * np.repeat(scales[r], block)
    return w


# --------------------------------------------------------------- router ---

def router_logits(xhat: np.ndarray, router_w_bits: np.ndarray,
                  bias: Optional[np.ndarray]) -> np.ndarray:
    """l[t, e] = sum_h xhat[t, h] * Wr[e, h] (+ b[e]), float64."""
    wr = bf16_to_f64(router_w_bits)
    l = np.asarray(xhat, dtype=np.float64) @ wr.T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per token, by descending logit, ties to
    the smaller expert index."""
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    experts = np.arange(E)
    for t in range(T):
        order = np.lexsort((experts, -logits[t]))   # primary -logit, then index
        idx[t] = order[:k]
    return idx


def gate_weights(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """p = softmax over all E logits; w_j = p[idx_j] / sum_i p[idx_i]."""
    T, k = idx.shape
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        z = np.exp(logits[t] - np.max(logits[t]))
        p = z / np.sum(z)
        sel = p[idx[t]]
        w[t] = sel / np.sum(sel)
    return w


def tie_band_ok(logits_row: np.ndarray, chosen: np.ndarray, k: int, band: float) -> bool:
    """True when ``chosen`` (k expert ids) is a valid top-k of ``logits_row`` up
    to a tie band: every chosen logit is >= the oracle's k-th logit - band and
    every unchosen logit is <= the oracle's k-th logit + band, no repeats."""
    chosen = np.asarray(chosen, dtype=np.int64)
    if len(set(chosen.tolist())) != k or chosen.min() < 0 or chosen.max() >= logits_row.size:
        return False
    kth = np.sort(logits_row)[::-1][k - 1]
    mask = np.zeros(logits_row.size, dtype=bool)
    mask[chosen] = True
    return bool(np.all(logits_row[mask] >= kth - band) and np.all(logits_row[~mask] <= kth + band))


def group_by_expert(idx: np.ndarray, experts: int):
    """Per-expert token lists: counts[E], offsets[E+1] (exclusive prefix sum)
    and pairs[T*k], the pair ids t*k + j stably sorted by expert."""
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=experts).astype(np.int32)
    offsets = np.zeros(experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    pairs = np.argsort(flat, kind="stable").astype(np.int32)
    return counts, offsets, pairs


# ------------------------------------------------------------ expert FFN ---

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray,
               x: np.ndarray) -> np.ndarray:
    """W_down (silu(W_gate x) * (W_up x)) for one token, float64."""
    g = w_gate @ x
    u = w_up @ x
    return w_down @ (silu(g) * u)


def rmsnorm_bf16(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """bf16(x / sqrt(mean(x**2) + eps)) per token (weight 1)."""
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return round_bf16(x * r)


# ----------------------------------------------------------------- layer ---

@dataclasses.dataclass
class OracleLayer:
    """One layer's inputs as packed host arrays.

    ``expert(e)`` returns (gu_codes [2I, H*b/8], gu_scales [2I, H/bs] fp16
    bits, d_codes [H, I*b/8], d_scales [H, I/bs]); ``shared()`` the same for
    the shared expert or None.  With fp8 block scales the scales are E4M3
    bytes and the tuples carry two more arrays, the fp32 row scales
    (gu_row_scale [2I], d_row_scale [H])."""
    experts: int
    hidden: int
    inter: int
    top_k: int
    bits: int
    block: int
    router_w_bits: np.ndarray
    router_bias: Optional[np.ndarray]
    expert: Callable[[int], tuple]
    shared: Callable[[], Optional[tuple]]
    cache_size: int = 48
    shared_gate_w_bits: Optional[np.ndarray] = None   # [H] bf16 bits, or None (shared weight 1)
    half_levels: bool = False                         # codes are the half-integer levels

    def __post_init__(self):
        self._cache: dict = {}

    def _dense(self, key, packed):
        if key in self._cache:
            return self._cache[key]
        arrays = packed()
        gc, gs, dc, ds = arrays[:4]
        grs, drs = arrays[4:6] if len(arrays) == 6 else (None, None)
        H, I = self.hidden, self.inter
        w13 = dequantize(gc, gs, 2 * I, H, self.bits, self.block, self.half_levels, row_scale=grs)
        wd = dequantize(dc, ds, H, I, self.bits, self.block, self.half_levels, row_scale=drs)
        dense = (w13[0::2], w13[1::2], wd)
        if len(self._cache) >= self.cache_size:
            self._cache.pop(next(iter(self._cache)))
        self._cache[key] = dense
        return dense

    def expert_dense(self, e: int):
        return self._dense(("e", e), lambda: self.expert(e))

    def shared_dense(self):
        if self.shared() is None:
            return None
        return self._dense(("s",), self.shared)

    def shared_weight(self, xhat_t: np.ndarray) -> float:
        """Weight of the shared expert for one token: 1, or, for the gated
        variant, the logistic function of the dot product of the token with
        the gate vector (float64)."""
        if self.shared_gate_w_bits is None:
            return 1.0
        z = float(np.dot(xhat_t, bf16_to_f64(self.shared_gate_w_bits)))
        return 1.0 / (1.0 + math.exp(-z))


def layer_forward(layer: OracleLayer, x_bits: np.ndarray, *, rmsnorm: bool = False,
                  topk_override: Optional[dict] = None) -> dict:
    """Oracle of one MoE layer on hidden states x (bf16 bits [T, H]).

    Returns float64 ``out`` [T, H] (the MoE output, before any residual) and
    the intermediates ``xhat``, ``logits``, ``idx``, ``w``.  ``topk_override``
    maps a token to an index set that replaces the oracle's own selection (used
    only after that set has been checked with ``tie_band_ok``)."""
    x = bf16_to_f64(x_bits)
    xhat = rmsnorm_bf16(x) if rmsnorm else x
    logits = router_logits(xhat, layer.router_w_bits, layer.router_bias)
    idx = select_topk(logits, layer.top_k)
    if topk_override:
        for t, sel in topk_override.items():
            idx[t] = np.asarray(sel, dtype=np.int32)
    w = gate_weights(logits, idx)
    T = x.shape[0]
    out = np.zeros((T, layer.hidden), dtype=np.float64)
    shared = layer.shared_dense()
    for t in range(T):
        acc = np.zeros(layer.hidden, dtype=np.float64)
        if shared is not None:
            acc += layer.shared_weight(xhat[t]) * swiglu_ffn(*shared, xhat[t])
        for j in range(layer.top_k):
            acc += w[t, j] * swiglu_ffn(*layer.expert_dense(int(idx[t, j])), xhat[t])
        out[t] = acc
    return {"xhat": xhat, "logits": logits, "idx": idx, "w": w, "out": out}


def layer_forward_ep(layer: OracleLayer, x_bits: np.ndarray, ep_rank: int, ep_size: int, *,
                     topk_override: Optional[dict] = None) -> dict:
    """One rank's share of the layer when its experts are split over ep_size
    ranks by e % ep_size (expert parallelism; the pages run all experts of a
    layer on one machine, so this split is a reading of how the layer shards).

    Every rank routes all tokens over all experts exactly as layer_forward
    does; rank r then adds only the pairs (t, j) whose expert idx[t, j]
    satisfies idx % ep_size == r, weighted by w[t, j], and rank 0 alone adds
    the shared expert.  Returns float64 ``partial`` [T, H] and the routing;
    the sum of the partials over the ranks is layer_forward's ``out``.
    ``topk_override`` replaces selections as in layer_forward."""
    if not (1 <= ep_size <= layer.experts and 0 <= ep_rank < ep_size):
        raise ValueError("need 1 <= ep_size <= experts and 0 <= ep_rank < ep_size")
    x = bf16_to_f64(x_bits)
    logits = router_logits(x, layer.router_w_bits, layer.router_bias)
    idx = select_topk(logits, layer.top_k)
    if topk_override:
        for t, sel in topk_override.items():
            idx[t] = np.asarray(sel, dtype=np.int32)
    w = gate_weights(logits, idx)
    T = x.shape[0]
    partial = np.zeros((T, layer.hidden), dtype=np.float64)
    shared = layer.shared_dense() if ep_rank == 0 else None
    for t in range(T):
        if shared is not None:
            partial[t] += layer.shared_weight(x[t]) * swiglu_ffn(*shared, x[t])
        for j in range(layer.top_k):
            e = int(idx[t, j])
            if e % ep_size == ep_rank:
                partial[t] += w[t, j] * swiglu_ffn(*layer.expert_dense(e), x[t])
    return {"partial": partial, "idx": idx, "w": w}


def stack_forward(layers, x_bits: np.ndarray, *, choose_topk=None) -> dict:
    """Oracle of the stack: for each layer ``x <- bf16(x + moe(rmsnorm(x)))``.

    ``choose_topk(l, logits, idx)`` may return a {token: index set} override
    for layer l (a tie-band substitution validated by the caller)."""
    x = bf16_to_f64(x_bits)
    trace = []
    for l, layer in enumerate(layers):
        xb = _f64_to_bf16_bits(x)
        override = None
        if choose_topk is not None:
            probe = layer_forward_route_only(layer, xb)
            override = choose_topk(l, probe["logits"], probe["idx"])
        r = layer_forward(layer, xb, rmsnorm=True, topk_override=override)
        x = round_bf16(x + r["out"])
        trace.append({"idx": r["idx"], "logits": r["logits"], "x": x.copy()})
    return {"x": x, "trace": trace}


def layer_forward_route_only(layer: OracleLayer, x_bits: np.ndarray) -> dict:
    x = bf16_to_f64(x_bits)
    xhat = rmsnorm_bf16(x)
    logits = router_logits(xhat, layer.router_w_bits, layer.router_bias)
    return {"logits": logits, "idx": select_topk(logits, layer.top_k)}


def _f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """bf16-valued float64 -> uint16 bit patterns (exact)."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
