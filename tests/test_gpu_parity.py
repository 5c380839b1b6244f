"""GPU parity of the CUDA path against the float64 oracle, through the C ABI.

Tolerances: integer work (grouping, decoded codes) is bit-exact; expert ids are
bit-exact except inside the oracle's tie band (k-th and (k+1)-th logits within
1e-5, where both choices are correct); gate weights within 1e-5 (fp32 logits
and exp); layer outputs within max |err| <= 2e-2 * RMS(oracle output).
"""

import numpy as np
import pytest

import gpu_cases as gc
import moe_inputs as mi
import oracle as orc
import quantized_expert_ffn_moe_b200 as q

pytestmark = pytest.mark.gpu

SHAPE_2BIT_TINY = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=2, block=16)
# 4-bit with one scale per 128 elements (the GPTQ-style group size)
TINY_G128 = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=4, block=128)
FULL4_G128 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=128)
# half-integer levels (2-bit: the four levels +-1/2, +-3/2; 4-bit: sixteen)
TINY2H = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=2, block=16, half=True)
TINY4H = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=4, block=32, half=True)
FULL2H = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=2, block=16, half=True)
# one E4M3 scale byte per block under one fp32 scale per row
TINY4F8 = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=4, block=32, fp8_scales=True)
TINY2F8 = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=True, bits=2, block=16, fp8_scales=True)
FULL4F8 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=32, fp8_scales=True)
FULL2F8 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=2, block=16, fp8_scales=True)


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


# ------------------------------------------------------------ input bytes ---

@pytest.mark.parametrize("shape", [mi.TINY, SHAPE_2BIT_TINY, mi.FULL4, mi.FULL2, TINY_G128, TINY2H, TINY4H, FULL2H,
                                   TINY4F8, TINY2F8, FULL4F8, FULL2F8],
                         ids=["tiny4", "tiny2", "full4", "full2", "tiny4g128", "tiny2h", "tiny4h", "full2h",
                              "tiny4f8", "tiny2f8", "full4f8", "full2f8"])
def test_device_generator_matches_host(shape):
    """The device generator writes the same bytes as the numpy generator."""
    w = gc.device_layer(shape, seed=3, layer=5)
    f8 = shape.fp8_scales
    for e in (0, 1, shape.experts - 1):
        ref = mi.expert_packed(shape, 3, 5, e)
        got = (w.gate_up_codes[e], w.gate_up_scales[e], w.down_codes[e], w.down_scales[e])
        if f8:
            got += (w.gate_up_row_scales[e], w.down_row_scales[e])
        assert len(got) == len(ref)
        for r, g in zip(ref, got):
            np.testing.assert_array_equal(g.cpu().numpy().view(r.dtype).reshape(r.shape), r)
    ref = mi.shared_packed(shape, 3, 5)
    got = (w.shared_gate_up_codes, w.shared_gate_up_scales, w.shared_down_codes, w.shared_down_scales)
    if f8:
        got += (w.shared_gate_up_row_scales, w.shared_down_row_scales)
    for r, g in zip(ref, got):
        np.testing.assert_array_equal(g.cpu().numpy().view(r.dtype).reshape(r.shape), r)
    np.testing.assert_array_equal(gc.bits_to_np(w.router_w), mi.router_weight_bf16(shape, 3, 5))


# ----------------------------------------------------------- dequant hook ---

@pytest.mark.parametrize("shape", [mi.TINY, SHAPE_2BIT_TINY, mi.FULL4, mi.FULL2, FULL4_G128, TINY4H, FULL2H],
                         ids=["tiny4", "tiny2", "full4", "full2", "full4g128", "tiny4h", "full2h"])
def test_device_decoder_bit_exact(shape):
    torch = gc.torch()
    w = gc.device_layer(shape, seed=1, layer=0)
    cfg = gc.cfg_of(shape)
    e = shape.experts // 2
    gcodes, gsc, dcodes, dsc = mi.expert_packed(shape, 1, 0, e)
    H, I = shape.hidden, shape.inter
    out = torch.empty((2 * I, H), dtype=torch.float32, device="cuda")
    q.moe_dequant_rows(cfg, w.gate_up_codes[e], w.gate_up_scales[e], 0, 2 * I, H, out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64),
                                  orc.dequantize(gcodes, gsc, 2 * I, H, shape.bits, shape.block, shape.half))
    out = torch.empty((H - 3, I), dtype=torch.float32, device="cuda")
    q.moe_dequant_rows(cfg, w.down_codes[e], w.down_scales[e], 3, H - 3, I, out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64),
                                  orc.dequantize(dcodes, dsc, H, I, shape.bits, shape.block, shape.half)[3:])


@pytest.mark.parametrize("shape", [TINY4F8, TINY2F8, FULL4F8, FULL2F8], ids=["tiny4f8", "tiny2f8", "full4f8", "full2f8"])
def test_device_decoder_bit_exact_fp8_scales(shape):
    """E4M3 block scales times the fp32 row scale: q * e4m3 is exact, so the
    GEMV's decoder must give the float64 weight rounded once to fp32."""
    torch = gc.torch()
    w = gc.device_layer(shape, seed=1, layer=0)
    cfg = gc.cfg_of(shape)
    e = shape.experts // 2 + 1
    gcodes, gsc, dcodes, dsc, grs, drs = mi.expert_packed(shape, 1, 0, e)
    H, I = shape.hidden, shape.inter
    out = torch.empty((2 * I, H), dtype=torch.float32, device="cuda")
    q.moe_dequant_rows_scaled(cfg, w.gate_up_codes[e], w.gate_up_scales[e], w.gate_up_row_scales[e], 0, 2 * I, H, out)
    torch.cuda.synchronize()
    ref = orc.dequantize(gcodes, gsc, 2 * I, H, shape.bits, shape.block, row_scale=grs)
    np.testing.assert_array_equal(out.cpu().numpy(), ref.astype(np.float32))
    out = torch.empty((H - 5, I), dtype=torch.float32, device="cuda")
    q.moe_dequant_rows_scaled(cfg, w.down_codes[e], w.down_scales[e], w.down_row_scales[e], 5, H - 5, I, out)
    torch.cuda.synchronize()
    ref = orc.dequantize(dcodes, dsc, H, I, shape.bits, shape.block, row_scale=drs)[5:]
    np.testing.assert_array_equal(out.cpu().numpy(), ref.astype(np.float32))
    # the plain hook refuses fp8 scales
    assert q.moe_dequant_rows(cfg, w.down_codes[e], w.down_scales[e], 0, 4, I, out, check=False) == -2


# ----------------------------------------------------------------- router ---

def _check_route(shape, seed, layer, x_bits, zipf=False):
    w = gc.device_layer(shape, seed, layer, zipf=zipf)
    idx, wt, counts, offsets, pairs = gc.run_route(shape, w, x_bits)
    lay = gc.host_oracle_layer(shape, seed, layer, zipf=zipf)
    logits = orc.router_logits(orc.bf16_to_f64(x_bits), lay.router_w_bits, lay.router_bias)
    oidx = orc.select_topk(logits, shape.top_k)
    gc.check_selection(logits, oidx, idx, shape.top_k)
    # gate weights: the oracle's definition evaluated on the GPU's selection
    np.testing.assert_allclose(wt, orc.gate_weights(logits, idx), atol=1e-5, rtol=0)
    np.testing.assert_allclose(wt.sum(1), 1.0, atol=1e-5)
    c, o, p = orc.group_by_expert(idx, shape.experts)
    np.testing.assert_array_equal(counts, c)
    np.testing.assert_array_equal(offsets, o)
    np.testing.assert_array_equal(pairs, p)
    return idx


@pytest.mark.parametrize("T", [1, 3, 8, 64, 65, 300])
def test_route_tiny(T):
    _check_route(mi.TINY, 0, 0, mi.hidden_states_bf16(T, mi.TINY.hidden, 0, 7))


@pytest.mark.parametrize("T", [1, 16, 64, 4096])
def test_route_full(T):
    _check_route(mi.FULL4, 0, 0, mi.hidden_states_bf16(T, mi.FULL4.hidden, 0, 9))


def test_route_zipf_skew():
    idx = _check_route(mi.FULL2, 0, 0, mi.hidden_states_bf16(64, 2048, 0, 4), zipf=True)
    rank = np.rint(np.exp(mi.zipf_router_bias(mi.FULL2, 0, 0).astype(np.float64) / -mi.ZIPF_ALPHA))
    assert np.mean(rank[idx] <= 102) > 0.85


def test_route_exact_ties_go_to_smaller_index():
    """All router rows equal: every logit ties, so the selection is experts
    0..k-1 in order with equal gates."""
    torch = gc.torch()
    shape = mi.TINY
    w = gc.device_layer(shape, 0, 0)
    w.router_w = w.router_w[:1].repeat(shape.experts, 1).contiguous()
    x = mi.hidden_states_bf16(5, shape.hidden, 0, 1)
    idx, wt, counts, _, _ = gc.run_route(shape, w, x)
    np.testing.assert_array_equal(idx, np.tile(np.arange(shape.top_k), (5, 1)))
    np.testing.assert_allclose(wt, 1.0 / shape.top_k, atol=1e-7)
    assert counts[: shape.top_k].tolist() == [5] * shape.top_k
    del torch


# ------------------------------------------------------------------ layer ---

def _oracle_given(lay, x_bits, gpu_idx, differ):
    over = {t: gpu_idx[t] for t in differ}
    return orc.layer_forward(lay, x_bits, topk_override=over)


@pytest.mark.parametrize("shape", [mi.TINY, SHAPE_2BIT_TINY, TINY_G128, TINY2H, TINY4H, TINY4F8, TINY2F8],
                         ids=["tiny4", "tiny2", "tiny4g128", "tiny2h", "tiny4h", "tiny4f8", "tiny2f8"])
@pytest.mark.parametrize("T", [1, 2, 7, 8, 17, 64, 100])
def test_layer_tiny_live_oracle(shape, T):
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 0)
    w = gc.device_layer(shape, 0, 0)
    y = gc.run_layer(shape, w, x)
    lay = gc.host_oracle_layer(shape, 0, 0, cache_size=shape.experts + 1)
    idx = gc.run_route(shape, w, x)[0]
    r = orc.layer_forward(lay, x)
    differ = gc.check_selection(r["logits"], r["idx"], idx, shape.top_k)
    if differ:
        r = _oracle_given(lay, x, idx, differ)
    gc.assert_close(y, r["out"])


def test_layer_without_shared_expert():
    shape = mi.MoeShape(experts=64, hidden=256, inter=128, top_k=4, shared=False, bits=4, block=32)
    x = mi.hidden_states_bf16(9, shape.hidden, 0, 3)
    w = gc.device_layer(shape, 2, 0)
    y = gc.run_layer(shape, w, x)
    r = orc.layer_forward(gc.host_oracle_layer(shape, 2, 0, cache_size=70), x)
    gc.assert_close(y, r["out"])


def _stored_layer_case(name, T_list):
    case = gc.load_case(name)
    E, H, I, k, sh, bits, bs = case["shape"].tolist()
    shape = mi.MoeShape(E, H, I, k, bool(sh), bits, bs)
    zipf = bool(case["zipf"])
    w = gc.device_layer(shape, int(case["seed"]), 0, zipf=zipf)
    xall = mi.hidden_states_bf16(int(case["T"]), H, int(case["seed"]), int(case["batch"]))
    toks = case["tokens"]
    for T in T_list:
        x = xall[:T]
        y = gc.run_layer(shape, w, x)
        idx = gc.run_route(shape, w, x)[0]
        sel = toks[toks < T]
        rows = np.searchsorted(toks, sel)
        ref = case["out_"][rows].astype(np.float64)
        differ = gc.check_selection(case["logits"][rows], case["idx"][rows], idx[sel], k)
        if differ:   # re-run the oracle on the GPU's (valid) selection for those tokens
            lay = gc.host_oracle_layer(shape, int(case["seed"]), 0, zipf=zipf)
            for i in differ:
                r = orc.layer_forward(lay, x[sel[i]:sel[i] + 1], topk_override={0: idx[sel[i]]})
                ref[i] = r["out"][0]
        gc.assert_close(y[sel], ref)


def test_layer_full4_decode_stored_oracle():
    # 1-3 tokens: the routing lists built by one warp; 4 and 16: by the block scans
    _stored_layer_case("full4_decode", [1, 2, 3, 4, 16])


def test_layer_full2_zipf_decode_stored_oracle():
    _stored_layer_case("full2_zipf_decode", [1, 2, 8, 33, 64])


def test_layer_full4_prefill_stored_oracle():
    _stored_layer_case("full4_prefill", [4096])


def test_layer_is_deterministic():
    torch = gc.torch()
    shape = mi.FULL4
    w = gc.device_layer(shape, 0, 0)
    cfg = gc.cfg_of(shape)
    x = gc.to_dev_bits(mi.hidden_states_bf16(16, shape.hidden, 0, 5))
    ws = gc.workspace(cfg, 16)
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    q.moe_layer_forward(cfg, w, x, y1, ws)
    q.moe_layer_forward(cfg, w, x, y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_empty_batch_and_small_workspace():
    torch = gc.torch()
    shape = mi.TINY
    w = gc.device_layer(shape, 0, 0)
    cfg = gc.cfg_of(shape)
    x = gc.to_dev_bits(mi.hidden_states_bf16(4, shape.hidden, 0, 0))
    y = torch.full_like(x, 7)
    ws = gc.workspace(cfg, 4)
    assert q.moe_layer_forward(cfg, w, x, y, ws, tokens=0) == 0
    torch.cuda.synchronize()
    assert bool((y == 7).all())
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    assert q.moe_layer_forward(cfg, w, x, y, small, check=False) == -3


# --------------------------------------------------- tensor-core prefill ---
# Shapes small enough for the live oracle that still take the tcgen05 path
# (H and I multiples of 256): several expert groups per tile row, ragged tiles.
MID4 = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=4, shared=True, bits=4, block=32)
MID2 = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=4, shared=True, bits=2, block=16)
MID2H = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=4, shared=True, bits=2, block=16, half=True)
MID4H = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=4, shared=True, bits=4, block=32, half=True)


@pytest.mark.parametrize("shape", [MID4, MID2, MID2H, MID4H], ids=["mid4", "mid2", "mid2h", "mid4h"])
@pytest.mark.parametrize("T", [65, 129, 300])
def test_prefill_path_live_oracle(shape, T):
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 21)
    w = gc.device_layer(shape, 4, 0)
    y = gc.run_layer(shape, w, x)
    lay = gc.host_oracle_layer(shape, 4, 0, cache_size=shape.experts + 1)
    idx = gc.run_route(shape, w, x)[0]
    r = orc.layer_forward(lay, x)
    differ = gc.check_selection(r["logits"], r["idx"], idx, shape.top_k)
    if differ:
        r = _oracle_given(lay, x, idx, differ)
    gc.assert_close(y, r["out"])


def test_prefill_path_without_shared_expert():
    shape = mi.MoeShape(experts=32, hidden=512, inter=256, top_k=2, shared=False, bits=4, block=32)
    x = mi.hidden_states_bf16(200, shape.hidden, 0, 8)
    w = gc.device_layer(shape, 6, 0)
    y = gc.run_layer(shape, w, x)
    r = orc.layer_forward(gc.host_oracle_layer(shape, 6, 0, cache_size=40), x)
    idx = gc.run_route(shape, w, x)[0]
    differ = gc.check_selection(r["logits"], r["idx"], idx, shape.top_k)
    if differ:
        r = _oracle_given(gc.host_oracle_layer(shape, 6, 0, cache_size=40), x, idx, differ)
    gc.assert_close(y, r["out"])


def _sampled_full_case(shape, T, batch, seed, n_sample, sample_seed):
    """Full-shape layer at T tokens, checked on a seeded sample of tokens
    against the live oracle (tokens are independent in one layer)."""
    x = mi.hidden_states_bf16(T, shape.hidden, seed, batch)
    w = gc.device_layer(shape, seed, 0)
    y = gc.run_layer(shape, w, x)
    idx = gc.run_route(shape, w, x)[0]
    sel = np.sort(np.random.default_rng(sample_seed).choice(T, size=n_sample, replace=False))
    lay = gc.host_oracle_layer(shape, seed, 0, cache_size=8)
    r = orc.layer_forward(lay, x[sel])
    differ = gc.check_selection(r["logits"], r["idx"], idx[sel], shape.top_k)
    ref = r["out"].copy()
    for i in differ:
        ref[i] = orc.layer_forward(lay, x[sel[i]:sel[i] + 1], topk_override={0: idx[sel[i]]})["out"][0]
    gc.assert_close(y[sel], ref)


def _with_path(mode, fn):
    """Runs fn with the 32..64-token decode path fixed (1 CUDA cores, 2 tensor
    cores, 0 the cost model's choice)."""
    lib = q.load_library()
    lib.moe_debug_decode_path(mode)
    try:
        fn()
    finally:
        lib.moe_debug_decode_path(0)


def test_layer_full4_decode_unstaged_chunks():
    # 40 tokens do not fit the fused decode kernel's once-per-layer token
    # staging, so gate/up stages its tokens per slot chunk and per consumer group
    _with_path(1, lambda: _sampled_full_case(mi.FULL4, 40, 3, 0, 4, 40))


@pytest.mark.parametrize("mode", [1, 2, 0], ids=["cuda_cores", "tensor_cores", "cost_model"])
def test_decode_handover_full2_zipf(mode):
    """Skewed 2-bit batches of 33 and 64 tokens on each decode path: after the
    fused kernel's routing, the grouped tcgen05 kernels read its exported
    routing and finish the layer."""
    _with_path(mode, lambda: _stored_layer_case("full2_zipf_decode", [33, 64]))


def test_decode_handover_full4():
    _with_path(2, lambda: _sampled_full_case(mi.FULL4, 48, 5, 0, 4, 48))


def test_prefill_full4_large_batch_tile_lookup():
    # 60,000 tokens: more tiles per CTA than the per-CTA tile table holds (the
    # down pass falls back to the per-tile lookup) and the chunked grouping at scale
    _sampled_full_case(mi.FULL4, 60000, 4, 0, 4, 60000)


# ------------------------------------------------------- expert parallel ---

def _ep_partials(shape, w, x_bits, ep_size):
    """Every rank's fp32 partial, computed one rank after the other on this GPU
    (the ranks share nothing but the inputs)."""
    t = gc.torch()
    cfg = gc.cfg_of(shape)
    T = x_bits.shape[0]
    x = gc.to_dev_bits(x_bits)
    ws = gc.workspace(cfg, T)
    parts = []
    for r in range(ep_size):
        yp = t.full((T, shape.hidden), float("nan"), dtype=t.float32, device="cuda")
        q.moe_layer_forward_ep(cfg, w, x, yp, ws, r, ep_size)
        t.cuda.synchronize()
        assert q.moe_device_status(ws) == 0
        parts.append(yp.cpu().numpy().astype(np.float64))
    return parts


@pytest.mark.parametrize("shape,T", [(mi.TINY, 8), (mi.TINY, 100), (SHAPE_2BIT_TINY, 17), (MID4, 300)],
                         ids=["tiny4_t8", "tiny4_t100", "tiny2_t17", "mid4_t300"])
@pytest.mark.parametrize("ep_size", [1, 2, 3])
def test_expert_parallel_partials_live_oracle(shape, T, ep_size):
    """Each rank's partial against the oracle's share of that rank, and their
    sum against the whole layer (decode GEMV, and for mid4_t300 the chunked
    grouping and the tcgen05 path)."""
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 31)
    w = gc.device_layer(shape, 0, 0)
    lay = gc.host_oracle_layer(shape, 0, 0, cache_size=shape.experts + 1)
    idx = gc.run_route(shape, w, x)[0]
    full = orc.layer_forward(lay, x)
    differ = gc.check_selection(full["logits"], full["idx"], idx, shape.top_k)
    # a tie-band token's valid GPU selection replaces the oracle's (same rule
    # as the layer tests), so every token is compared
    over = {int(t): idx[t] for t in differ}
    if over:
        full = orc.layer_forward(lay, x, topk_override=over)
    parts = _ep_partials(shape, w, x, ep_size)
    scale = float(np.sqrt(np.mean(full["out"] ** 2)))
    for r, p in enumerate(parts):
        ref = orc.layer_forward_ep(lay, x, r, ep_size, topk_override=over)["partial"]
        err = float(np.abs(p - ref).max())
        assert err <= gc.REL_TOL * scale, (r, err / scale)
    err = float(np.abs(sum(parts) - full["out"]).max())
    assert err <= gc.REL_TOL * scale, err / scale


def test_expert_parallel_full4_decode_stored_oracle():
    """Full shape, 16 tokens, 2 and 4 ranks: the partials' sum against the
    stored oracle output."""
    case = gc.load_case("full4_decode")
    E, H, I, k, sh, bits, bs = case["shape"].tolist()
    shape = mi.MoeShape(E, H, I, k, bool(sh), bits, bs)
    w = gc.device_layer(shape, int(case["seed"]), 0)
    x = mi.hidden_states_bf16(int(case["T"]), H, int(case["seed"]), int(case["batch"]))[:16]
    idx = gc.run_route(shape, w, x)[0]
    toks = case["tokens"]
    sel = toks[toks < 16]
    rows = np.searchsorted(toks, sel)
    differ = gc.check_selection(case["logits"][rows], case["idx"][rows], idx[sel], k)
    ref = case["out_"][rows].astype(np.float64)
    if len(differ):
        # a tie-band token is compared against the oracle re-run on the GPU's
        # (validated) selection, as in the layer tests
        lay = gc.host_oracle_layer(shape, int(case["seed"]), 0, cache_size=24)
        for i in differ:
            t = int(sel[i])
            ref[i] = orc.layer_forward(lay, x[t:t + 1], topk_override={0: idx[t]})["out"][0]
    for ep_size in (2, 4):
        tot = sum(_ep_partials(shape, w, x, ep_size))
        gc.assert_close(tot[sel], ref)


# ------------------------------------------------- 4-bit, 128-element groups ---

@pytest.mark.parametrize("T", [16, 48, 100])
def test_layer_full4_g128_sampled(T):
    """Full shape with one scale per 128 elements: the fused decode kernel at
    16 and 48 tokens, the stand-alone GEMV kernels at 100 (no tensor-core path
    for this group size)."""
    _sampled_full_case(FULL4_G128, T, 7, 0, 4, 128 + T)


# --------------------------------------------------- half-integer levels ---

@pytest.mark.parametrize("T,path", [(1, 0), (16, 0), (48, 1), (48, 2), (300, 0)],
                         ids=["t1", "t16", "t48_cuda_cores", "t48_tensor_cores", "t300_prefill"])
def test_layer_full2_half_levels_sampled(T, path):
    """Full shape, 2-bit codes read as the four half-integer levels: the
    single-launch decode kernel (1, 16 tokens; 48 tokens on each side of the
    hand-over) and the tensor-core prefill (300 tokens)."""
    _with_path(path, lambda: _sampled_full_case(FULL2H, T, 13, 0, min(3, T), 900 + T))


# ------------------------------------------------------- fp8 block scales ---

@pytest.mark.parametrize("shape,T", [(FULL4F8, 1), (FULL4F8, 3), (FULL4F8, 16), (FULL4F8, 48), (FULL4F8, 100),
                                     (FULL2F8, 16), (FULL2F8, 64)],
                         ids=["full4_t1", "full4_t3", "full4_t16", "full4_t48", "full4_t100", "full2_t16", "full2_t64"])
def test_layer_full_fp8_scales_sampled(shape, T):
    """Full shape with E4M3 block scales and fp32 row scales: the
    single-launch decode kernel up to 64 tokens (3 tokens: the one-warp
    routing lists; 48: no tensor-core hand-over for this format) and the
    stand-alone GEMV kernels for the 100-token batch."""
    _sampled_full_case(shape, T, 17, 0, min(3, T), 700 + T)


def test_fp8_scales_stack_and_expert_parallel():
    """Two layers of fp8-scaled weights through moe_stack_forward (the
    separate kernels with the residual and the next layer's RMSNorm), and
    the expert-parallel partials of one of them."""
    torch = gc.torch()
    shape = TINY4F8
    T = 12
    x = mi.hidden_states_bf16(T, shape.hidden, 0, 41)
    ws_l = [gc.device_layer(shape, 0, l) for l in range(2)]
    cfg = gc.cfg_of(shape)
    xd = gc.to_dev_bits(x)
    ws = gc.workspace(cfg, T)
    q.moe_stack_forward(cfg, ws_l, xd, ws)
    torch.cuda.synchronize()
    got_stack = gc.bits_to_np(xd)
    # one layer at a time through the same entry point composes bitwise
    xs = gc.to_dev_bits(x)
    for l in range(2):
        q.moe_stack_forward(cfg, ws_l[l:l + 1], xs, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(gc.bits_to_np(xs), got_stack)
    # first step against the oracle at the layer tolerance
    lay = gc.host_oracle_layer(shape, 0, 0, cache_size=shape.experts + 1)
    xs = gc.to_dev_bits(x)
    tr = torch.empty((1, T, shape.top_k), dtype=torch.int32, device="cuda")
    q.moe_stack_forward(cfg, ws_l[:1], xs, ws, topk_trace=tr)
    torch.cuda.synchronize()
    idx = tr[0].cpu().numpy()
    r = orc.layer_forward(lay, x, rmsnorm=True)
    differ = gc.check_selection(r["logits"], r["idx"], idx, shape.top_k)
    if differ:
        r = orc.layer_forward(lay, x, rmsnorm=True, topk_override={t: idx[t] for t in differ})
    xf = orc.bf16_to_f64(x)
    eps = gc.REL_TOL * float(np.sqrt(np.mean(r["out"] ** 2)))
    got = orc.bf16_to_f64(gc.bits_to_np(xs))
    lo, hi = orc.round_bf16(xf + r["out"] - eps), orc.round_bf16(xf + r["out"] + eps)
    assert np.all(got >= lo) and np.all(got <= hi)
    # expert-parallel partials sum to the layer
    parts = _ep_partials(shape, ws_l[0], x, 2)
    full = orc.layer_forward(lay, x)
    idx0 = gc.run_route(shape, ws_l[0], x)[0]
    d0 = gc.check_selection(full["logits"], full["idx"], idx0, shape.top_k)
    if d0:
        full = orc.layer_forward(lay, x, topk_override={t: idx0[t] for t in d0})
    scale = float(np.sqrt(np.mean(full["out"] ** 2)))
    assert float(np.abs(sum(parts) - full["out"]).max()) <= gc.REL_TOL * scale


# ----------------------------------------------------- gated shared expert ---

def _gated_case(shape, T, seed, batch, sample=None):
    x = mi.hidden_states_bf16(T, shape.hidden, seed, batch)
    w = gc.device_layer(shape, seed, 0, shared_gate=True)
    y = gc.run_layer(shape, w, x)
    idx = gc.run_route(shape, w, x)[0]
    sel = np.arange(T) if sample is None else np.sort(np.random.default_rng(batch).choice(T, sample, replace=False))
    lay = gc.host_oracle_layer(shape, seed, 0, cache_size=min(shape.experts + 1, 24), shared_gate=True)
    r = orc.layer_forward(lay, x[sel])
    differ = gc.check_selection(r["logits"], r["idx"], idx[sel], shape.top_k)
    if differ:
        r = orc.layer_forward(lay, x[sel], topk_override={i: idx[sel[i]] for i in differ})
    gc.assert_close(y[sel], r["out"])


def test_device_generator_gate_vector():
    w = gc.device_layer(mi.TINY, 3, 2, shared_gate=True)
    np.testing.assert_array_equal(gc.bits_to_np(w.shared_gate_w), mi.shared_gate_weight_bf16(mi.TINY, 3, 2))


@pytest.mark.parametrize("T", [8, 100])
def test_gated_shared_expert_tiny(T):
    _gated_case(mi.TINY, T, 0, 41)


def test_gated_shared_expert_prefill_mid():
    _gated_case(MID4, 129, 4, 42)


def test_gated_shared_expert_full4_sampled():
    # the gated layer leaves the single-launch decode kernel for the separate kernels
    _gated_case(mi.FULL4, 16, 0, 43, sample=4)


def test_gated_shared_expert_expert_parallel():
    shape = mi.TINY
    x = mi.hidden_states_bf16(8, shape.hidden, 0, 44)
    w = gc.device_layer(shape, 0, 0, shared_gate=True)
    lay = gc.host_oracle_layer(shape, 0, 0, cache_size=shape.experts + 1, shared_gate=True)
    idx = gc.run_route(shape, w, x)[0]
    full = orc.layer_forward(lay, x)
    differ = gc.check_selection(full["logits"], full["idx"], idx, shape.top_k)
    if differ:     # the oracle on the GPU's (valid) selection for tokens in the tie band
        full = orc.layer_forward(lay, x, topk_override={t: idx[t] for t in differ})
    parts = _ep_partials(shape, w, x, 2)
    gc.assert_close(sum(parts), full["out"])


@pytest.mark.parametrize("T", [8, 100])
def test_gated_shared_expert_fp8_scales_tiny(T):
    # both variants at once: E4M3 block scales with row scales, and the gate
    _gated_case(TINY4F8, T, 0, 45)


# ------------------------------------------------------------ failure path ---

def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier that never completes gives up after its limit,
    records MOE_ERR_TIMEOUT in the status word, and the GPU keeps working."""
    torch = gc.torch()
    lib = q.load_library()
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    assert lib.moe_debug_wait_probe(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert q.moe_device_status(ws) == -6                      # MOE_ERR_TIMEOUT
    # the context is intact: a layer still runs and matches the oracle
    test_layer_without_shared_expert()
