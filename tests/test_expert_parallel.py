"""Expert-parallel layer: the oracle's per-rank share and the exchange step.

CPU only (no GPU): the oracle's partials are pinned to its full layer (their
sum over ranks is the layer output) and to the ownership rule (a rank
dequantizes only its own experts), and the exchange is run as a world_size-2
gloo process group through the package's ``ep_all_reduce`` -- the same call
that sums the GPU partials over NCCL.  The rank-timing reductions of
``bench.py`` run on the same gloo group."""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
import oracle as orc  # noqa: E402


def _tiny_layer(record=None, shared=True):
    shape = mi.TINY
    pool, sh = mi.layer_packed_pool(shape, 0, 0)

    def expert(e):
        if record is not None:
            record.append(e)
        return tuple(a[e] for a in pool)

    def shared_fn():
        if record is not None:
            record.append("shared")
        return sh if shared else None

    return orc.OracleLayer(
        experts=shape.experts, hidden=shape.hidden, inter=shape.inter, top_k=shape.top_k,
        bits=shape.bits, block=shape.block, router_w_bits=mi.router_weight_bf16(shape, 0, 0),
        router_bias=None, expert=expert, shared=shared_fn)


@pytest.mark.parametrize("ep_size", [1, 2, 3, 5])
def test_partials_sum_to_the_layer(ep_size):
    lay = _tiny_layer()
    x = mi.hidden_states_bf16(8, mi.TINY.hidden, seed=3)
    full = orc.layer_forward(lay, x)["out"]
    parts = [orc.layer_forward_ep(lay, x, r, ep_size)["partial"] for r in range(ep_size)]
    scale = np.abs(full).max()
    np.testing.assert_allclose(sum(parts), full, rtol=0, atol=1e-12 * scale)
    if ep_size > 1:
        # every rank carries a real share (no rank silently computes everything)
        for p in parts:
            assert np.abs(p - full).max() > 1e-6 * scale


def test_partials_follow_a_substituted_selection():
    """A replaced selection (the tie-band substitution the GPU tests use) moves
    the token's work to the new experts' owners: the partials still sum to the
    layer computed with the same replacement, and differ from the original."""
    lay = _tiny_layer()
    x = mi.hidden_states_bf16(6, mi.TINY.hidden, seed=9)
    base = orc.layer_forward(lay, x)
    alt = base["idx"][2].copy()
    alt[-1] = next(e for e in range(mi.TINY.experts) if e not in alt)   # swap the last pick
    over = {2: alt}
    full = orc.layer_forward(lay, x, topk_override=over)
    parts = [orc.layer_forward_ep(lay, x, r, 3, topk_override=over)["partial"] for r in range(3)]
    scale = np.abs(full["out"]).max()
    np.testing.assert_allclose(sum(parts), full["out"], rtol=0, atol=1e-12 * scale)
    assert np.abs(full["out"][2] - base["out"][2]).max() > 1e-6 * scale
    np.testing.assert_array_equal(full["out"][[0, 1, 3, 4, 5]], base["out"][[0, 1, 3, 4, 5]])


def test_rank_reads_only_its_experts():
    for ep_size in (2, 4):
        for r in range(ep_size):
            rec = []
            lay = _tiny_layer(record=rec)
            x = mi.hidden_states_bf16(8, mi.TINY.hidden, seed=5)
            res = orc.layer_forward_ep(lay, x, r, ep_size)
            experts = [e for e in rec if e != "shared"]
            assert all(e % ep_size == r for e in experts)
            owned = {int(e) for e in res["idx"].ravel() if e % ep_size == r}
            assert set(experts) == owned
            assert ("shared" in rec) == (r == 0)


def test_invalid_rank_is_rejected():
    lay = _tiny_layer()
    x = mi.hidden_states_bf16(2, mi.TINY.hidden, seed=1)
    for r, n in ((0, 0), (2, 2), (-1, 2), (0, mi.TINY.experts + 1)):
        with pytest.raises(ValueError):
            orc.layer_forward_ep(lay, x, r, n)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import quantized_expert_ffn_moe_b200 as q_pkg
        import bench
        lay = _tiny_layer()
        x = mi.hidden_states_bf16(8, mi.TINY.hidden, seed=11)
        part = torch.from_numpy(orc.layer_forward_ep(lay, x, rank, world)["partial"].copy())
        q_pkg.ep_all_reduce(part)
        full = orc.layer_forward(lay, x)["out"]
        err = float(np.abs(part.numpy() - full).max() / np.abs(full).max())
        tmax = bench.max_over_ranks(dist, world, 1.0 + rank)
        tsum = bench.sum_over_ranks(dist, world, 1.0 + rank)
        bench.barrier(dist, world)
        q.put((rank, err, tmax, tsum))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_exchange_and_timing():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, err, tmax, tsum in res:
        assert err < 1e-12
        assert tmax == 2.0 and tsum == 3.0
