"""Stored oracle results for the full-size parity cases.

The float64 oracle needs seconds per token at the full shape (each selected
expert is regenerated and dequantised on the host), so the expected values of
the large cases are computed once here and stored as oracle_<case>.npz next to
this file.  Only ``oracle`` and the host input generator ``moe_inputs`` are
used; nothing comes from the CUDA path.

    python tests/golden/make_oracle_cases.py [case ...]     # default: all

Tokens are independent in the layer (and in the stack, which has no
attention), so a case may store a seeded subset of the batch's tokens.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
import oracle as orc  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))

# name -> spec.  shape: MoeShape name; T: batch size; batch: x stream id;
# tokens: which tokens of the batch are stored (None = all); zipf: router bias;
# layers: number of stacked layers (0 = a single layer, no norm / residual);
# steps: stack layers evaluated one at a time (RMSNorm, MoE, residual), layer l
# on the seeded input of x stream batch + l.
CASES = {
    "full4_decode": dict(shape="FULL4", T=16, batch=0, tokens=None, zipf=False, layers=0),
    "full2_zipf_decode": dict(shape="FULL2", T=64, batch=0, tokens=None, zipf=True, layers=0),
    "full4_prefill": dict(shape="FULL4", T=4096, batch=1, tokens=("sample", 24, 11), zipf=False, layers=0),
    "full4_stack48_decode": dict(shape="FULL4", T=32, batch=2, tokens=(0, 1, 2, 3), zipf=False, layers=48),
    # one stack layer (RMSNorm, MoE, residual) at sampled depths of the
    # 48-layer stack, each on its own seeded input (x stream id batch + l)
    "full4_stack_step_t1": dict(shape="FULL4", T=1, batch=300, tokens=None, zipf=False, steps=(0, 1, 7, 23, 47)),
    "full4_stack_step_t32": dict(shape="FULL4", T=32, batch=400, tokens=(0, 9, 31), zipf=False,
                                 steps=(0, 1, 23, 47)),
    "full4_stack_step_t2048": dict(shape="FULL4", T=2048, batch=500, tokens=("sample", 6, 2048), zipf=False,
                                   steps=(0, 1, 23, 47)),
}
SEED = 0


def case_tokens(spec) -> np.ndarray:
    t = spec["tokens"]
    if t is None:
        return np.arange(spec["T"])
    if isinstance(t, tuple) and t and t[0] == "sample":
        rng = np.random.default_rng(t[2])
        return np.sort(rng.choice(spec["T"], size=t[1], replace=False))
    return np.asarray(t)


def oracle_layer(shape: mi.MoeShape, layer: int, zipf: bool) -> orc.OracleLayer:
    return orc.OracleLayer(
        experts=shape.experts, hidden=shape.hidden, inter=shape.inter, top_k=shape.top_k,
        bits=shape.bits, block=shape.block,
        router_w_bits=mi.router_weight_bf16(shape, SEED, layer),
        router_bias=mi.zipf_router_bias(shape, SEED, layer) if zipf else None,
        expert=lambda e: mi.expert_packed(shape, SEED, layer, e),
        shared=(lambda: mi.shared_packed(shape, SEED, layer)) if shape.shared else (lambda: None),
        cache_size=4)


def _layer_job(args):
    name, rows = args
    spec = CASES[name]
    shape = getattr(mi, spec["shape"])
    x = mi.hidden_states_bf16(spec["T"], shape.hidden, SEED, spec["batch"])[rows]
    r = orc.layer_forward(oracle_layer(shape, 0, spec["zipf"]), x)
    return rows, r


def _stack_job(args):
    name, rows = args
    spec = CASES[name]
    shape = getattr(mi, spec["shape"])
    x = mi.hidden_states_bf16(spec["T"], shape.hidden, SEED, spec["batch"])[rows]
    layers = [oracle_layer(shape, l, spec["zipf"]) for l in range(spec["layers"])]
    r = orc.stack_forward(layers, x)
    return rows, r


def _step_job(args):
    name, l, rows = args
    spec = CASES[name]
    shape = getattr(mi, spec["shape"])
    x = mi.hidden_states_bf16(spec["T"], shape.hidden, SEED, spec["batch"] + l)[rows]
    r = orc.layer_forward(oracle_layer(shape, l, spec["zipf"]), x, rmsnorm=True)
    return l, rows, r


def compute_steps(name: str, procs: int):
    """Stack layers one at a time: for each sampled layer l the MoE output
    (before the residual add), the routing, and the next residual stream."""
    spec = CASES[name]
    shape = getattr(mi, spec["shape"])
    toks = case_tokens(spec)
    steps = list(spec["steps"])
    jobs = [(name, l, toks[i::procs]) for l in steps for i in range(procs) if len(toks[i::procs])]
    ctx = mp.get_context("spawn")
    t0 = time.time()
    with ctx.Pool(min(len(jobs), procs)) as pool:
        res = pool.map(_step_job, jobs)
    out = dict(tokens=toks, shape=np.array([shape.experts, shape.hidden, shape.inter, shape.top_k,
                                            int(shape.shared), shape.bits, shape.block]),
               T=np.array(spec["T"]), batch=np.array(spec["batch"]), seed=np.array(SEED),
               zipf=np.array(int(spec["zipf"])), steps=np.array(steps))
    L, n, H = len(steps), len(toks), shape.hidden
    out_ = np.zeros((L, n, H), np.float64)
    logits = np.zeros((L, n, shape.experts), np.float64)
    idx = np.zeros((L, n, shape.top_k), np.int32)
    pos = {int(t): i for i, t in enumerate(toks)}
    for l, rows, r in res:
        li = steps.index(l)
        for j, t in enumerate(rows):
            out_[li, pos[int(t)]] = r["out"][j]
            logits[li, pos[int(t)]] = r["logits"][j]
            idx[li, pos[int(t)]] = r["idx"][j]
    out.update(out_=out_.astype(np.float32), logits=logits, idx=idx)
    path = os.path.join(HERE, f"oracle_{name}.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: {n} tokens x {L} layers in {time.time() - t0:.1f} s -> {path}", flush=True)


def compute(name: str, procs: int):
    spec = CASES[name]
    if "steps" in spec:
        return compute_steps(name, procs)
    shape = getattr(mi, spec["shape"])
    toks = case_tokens(spec)
    chunks = [toks[i::procs] for i in range(procs) if len(toks[i::procs])]
    ctx = mp.get_context("spawn")
    t0 = time.time()
    with ctx.Pool(len(chunks)) as pool:
        if spec["layers"] == 0:
            res = pool.map(_layer_job, [(name, c) for c in chunks])
        else:
            res = pool.map(_stack_job, [(name, c) for c in chunks])
    order = np.argsort(np.concatenate([r[0] for r in res]))
    cat = lambda key: np.concatenate([r[1][key] for r in res])[order]   # noqa: E731
    out = dict(tokens=toks, shape=np.array([shape.experts, shape.hidden, shape.inter, shape.top_k,
                                            int(shape.shared), shape.bits, shape.block]),
               T=np.array(spec["T"]), batch=np.array(spec["batch"]), seed=np.array(SEED),
               zipf=np.array(int(spec["zipf"])), layers=np.array(spec["layers"]))
    if spec["layers"] == 0:
        out.update(out_=cat("out").astype(np.float32), logits=cat("logits"), idx=cat("idx"), w=cat("w"))
    else:
        out["x_final"] = cat("x").astype(np.float32)
        L = spec["layers"]
        out["trace_idx"] = np.stack([np.concatenate([r[1]["trace"][l]["idx"] for r in res])[order]
                                     for l in range(L)])
        out["trace_logits"] = np.stack([np.concatenate([r[1]["trace"][l]["logits"] for r in res])[order]
                                        for l in range(L)])
        # residual stream after each layer (bf16 values, stored exactly as fp32)
        out["trace_x"] = np.stack([np.concatenate([r[1]["trace"][l]["x"] for r in res])[order]
                                   for l in range(L)]).astype(np.float32)
    path = os.path.join(HERE, f"oracle_{name}.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: {len(toks)} tokens in {time.time() - t0:.1f} s -> {path}", flush=True)


if __name__ == "__main__":
    names = sys.argv[1:] or list(CASES)
    procs = max(1, min(os.cpu_count() or 1, 16))
    for n in names:
        compute(n, procs)
