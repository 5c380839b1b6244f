"""Recompute the router-bias strength of the skewed 2-bit workload.

The workload asks for expert popularity that follows a Zipf law over a seeded
permutation of the 512 experts, with about 95% of picks on the top 20% of
experts.  A literal Zipf(1.1) marginal is not reachable under top-10 without
replacement (the top expert would need 19% of picks, but one token can pick it
only once, i.e. at most 10%), so the bias is read as b_e = -alpha * ln(rank_e)
and alpha is chosen by bisection so that 95% of the top-10 picks of an
8192-token batch (seed 0) land on the 102 highest-ranked experts.

Uses only the oracle's router; writes zipf_alpha.json next to this file.
Run:  python tests/golden/make_zipf_alpha.py
"""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import moe_inputs as mi  # noqa: E402
import oracle as orc  # noqa: E402

TOKENS, TARGET, HOT = 8192, 0.95, 102


def hot_share(logits0, bias, k, rank):
    idx = orc.select_topk(logits0 + bias[None, :].astype(np.float64), k)
    return float(np.mean(rank[idx] <= HOT))


def main():
    shape = mi.FULL2
    x = mi.hidden_states_bf16(TOKENS, shape.hidden, seed=0, batch=1000)
    logits0 = orc.router_logits(orc.bf16_to_f64(x), mi.router_weight_bf16(shape, 0, 0), None)
    unit = mi.zipf_router_bias(shape, 0, 0, alpha=1.0)          # = -ln(rank)
    rank = np.rint(np.exp(-unit.astype(np.float64))).astype(np.int64)
    lo, hi = 0.0, 4.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if hot_share(logits0, mi.zipf_router_bias(shape, 0, 0, alpha=mid), shape.top_k, rank) < TARGET:
            lo = mid
        else:
            hi = mid
    alpha = round(hi, 4)
    share = hot_share(logits0, mi.zipf_router_bias(shape, 0, 0, alpha=alpha), shape.top_k, rank)
    out = {"alpha": alpha, "hot_share": share, "tokens": TOKENS, "hot_experts": HOT,
           "target": TARGET, "seed": 0}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_alpha.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
