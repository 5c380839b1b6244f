#!/usr/bin/env python
"""Benchmark of the routed quantized-expert MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one full MoE layer forward (router -> top-10 -> grouping -> fused
dequant gate/up + SwiGLU -> down -> gate-weighted combine with the shared
expert) over one batch of decode tokens, through the C ABI.  Headline
workload: 512 experts, hidden 2048, expert intermediate 768, top-10 + 1 shared,
4-bit blocks of 32 with fp16 scales, 16 decode tokens.  Steps rotate over
distinct seeded layer instances (and 16 distinct token batches), so the
expert bytes a step touches are never still in the 126 MB L2 from an earlier
step.  Prints one JSON line (rank 0).  Under torchrun every rank runs its own
replica (no data-path collective: the path shards by independent batches).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

EXPERT_BYTES = {4: 2654208, 2: 1769472,     # packed gate/up + down of one expert (H=2048, I=768)
                "4g128": 2433024,            # 4-bit with one fp16 scale per 128 elements
                "4f8": 2521088}              # 4-bit, one E4M3 byte per 32 elements + an fp32 scale per row
GU_BYTES = {4: 1769472, 2: 1179648}
ROUTER_BYTES = 512 * 2048 * 2
METRIC = "MoE-layer decode tokens/s (512 experts, top-10 + shared, H=2048, I=768, 4-bit/32, 16 tokens)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=16)
    ap.add_argument("--instances", type=int, default=48, help="distinct layer instances rotated over")
    ap.add_argument("--no-detail", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--quick", action="store_true",
                    help="headline loop only (no e2e, detail or CPU baseline): the small case used for ncu")
    return ap.parse_args()


# ------------------------------------------------------------------ utils ---

def profiled_fields(profile: str, sources, profiles_dir: str | None = None, csrc_dir: str | None = None):
    """The `key: value` lines of a committed ncu summary under profiles/, or
    None when the kernel's sources changed since that capture (the summary
    records the sha256 of the sources it was taken with)."""
    import hashlib
    path = os.path.join(profiles_dir or os.path.join(ROOT, "profiles"), profile)
    if not os.path.exists(path):
        return None
    fields = {}
    for ln in open(path):
        if ":" in ln and not ln.startswith(" "):
            k, v = ln.split(":", 1)
            fields[k.strip()] = v.strip().split()[0] if v.strip() else ""
    h = hashlib.sha256()
    for f in sources:
        h.update(open(os.path.join(csrc_dir or os.path.join(ROOT, "quantized_expert_ffn_moe_b200", "csrc"), f),
                      "rb").read())
    if fields.get("source_sha256") != h.hexdigest():
        return None
    return fields


def profiled_traffic(profile: str, sources) -> float | None:
    """DRAM bytes per launch from a committed ncu summary (None if stale)."""
    fields = profiled_fields(profile, sources)
    if not fields or "traffic_bytes_per_launch" not in fields:
        return None
    return float(fields["traffic_bytes_per_launch"])


# Lane operations per weight of the integer GEMV's inner loop, counted from its
# source: decoding a 32-bit word of codes into signed bytes (4-bit: one shift
# and two lop3 per 8 weights; 2-bit: three shifts and four lop3 per 16), and
# per token the dp2a dot products (two products each) plus the fold of each
# block's integer sum (I2F + FFMA per 32 / 16 weights).
ALU_OPS = {4: (3 / 8, 0.5 + 2 / 32), 2: (7 / 16, 0.5 + 2 / 16), "4g128": (3 / 8, 0.5 + 2 / 128),
           "4f8": (3 / 8, 0.5 + 2 / 32)}
WEIGHTS_PER_EXPERT = 3 * 2048 * 768
ST_PATH = 3        # status word of the workspace: 1 when the tensor-core kernels ran the call


def alu_ceiling(bits, distinct: float, T: int, us_step: float, sm_mhz: float | None, sms: int = 148) -> dict:
    """The CUDA-core decode's compute ceiling: lane-ops = dequant ops x (U+1)
    x weights per expert + per-token ops x (T k + T) x weights per expert,
    over 148 SMs x 128 lanes at the sampled SM clock."""
    dq, per_tok = ALU_OPS[bits]
    lane_ops = dq * (distinct + 1) * WEIGHTS_PER_EXPERT + per_tok * (T * 10 + T) * WEIGHTS_PER_EXPERT
    mhz = sm_mhz or 1965.0
    min_us = 1e6 * lane_ops / (sms * 128 * mhz * 1e6)
    return {"lane_ops_per_step": lane_ops, "min_us": min_us, "frac": min_us / us_step, "sm_mhz": mhz,
            "ops_per_weight": {"dequant": dq, "per_token": per_tok},
            "source": "ops counted from the integer GEMV inner loop; the path the kernel ran is the other keys'"}


def issue_ceiling(instructions: float, launch_s: float, sms: int, sm_mhz: float = 1965.0) -> dict:
    """Warp instructions per launch (ncu smsp__inst_executed.sum) against the
    issue capacity of the GPU: one warp instruction per cycle per scheduler,
    4 schedulers per SM, at the given SM clock."""
    peak = sms * 4 * sm_mhz * 1e6
    achieved = instructions / launch_s
    return {"instructions_per_launch": instructions, "achieved_inst_per_s": achieved, "peak_inst_per_s": peak,
            "peak_source": f"{sms} SMs x 4 schedulers x 1 warp instruction/cycle x {sm_mhz:.0f} MHz",
            "frac": achieved / peak, "min_launch_us": 1e6 * instructions / peak}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- oracle ---
# The CPU baseline runs the float64 oracle as it stands, one process per host
# core (spawned, one BLAS thread each), each process taking its share of the
# batch's tokens (tokens are independent in the layer).  The packed experts a
# process needs are generated before the clock starts; a timed step is the
# wall time of all processes running their tokens once.

def _ref_env():
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"


_REF = {}


def _ref_prepare(tokens):
    import moe_inputs as mi
    import oracle as orc
    shape = mi.FULL4
    x = mi.hidden_states_bf16(16, shape.hidden, 0, 0)[tokens]
    rw = mi.router_weight_bf16(shape, 0, 0)
    logits = orc.router_logits(orc.bf16_to_f64(x), rw, None)
    need = sorted(set(orc.select_topk(logits, shape.top_k).reshape(-1).tolist()))
    packed = {e: mi.expert_packed(shape, 0, 0, e) for e in need}
    sh = mi.shared_packed(shape, 0, 0)
    _REF["x"] = x
    _REF["layer"] = orc.OracleLayer(experts=shape.experts, hidden=shape.hidden, inter=shape.inter,
                                    top_k=shape.top_k, bits=shape.bits, block=shape.block, router_w_bits=rw,
                                    router_bias=None, expert=lambda e: packed[e], shared=lambda: sh, cache_size=4)
    return len(need)


def _ref_run(_):
    import oracle as orc
    t0 = time.perf_counter()
    orc.layer_forward(_REF["layer"], _REF["x"])
    return time.perf_counter() - t0


def _mask(cpus) -> str:
    m = 0
    for c in cpus:
        m |= 1 << c
    return hex(m)


class OraclePool:
    """The oracle on the 16-token headline batch, spread over the host cores."""

    def __init__(self, tokens: int = 16):
        import multiprocessing as mp
        try:
            self.affinity = sorted(os.sched_getaffinity(0))
        except AttributeError:
            self.affinity = list(range(os.cpu_count() or 1))
        self.procs = max(1, min(tokens, len(self.affinity)))
        self.tokens = tokens
        chunks = [list(range(i, tokens, self.procs)) for i in range(self.procs)]
        _ref_env()
        self.pool = mp.get_context("spawn").Pool(self.procs)
        self.pool.map(_ref_prepare, chunks, chunksize=1)      # untimed: inputs and packed experts

    def step(self) -> float:
        t0 = time.perf_counter()
        self.pool.map(_ref_run, range(self.procs), chunksize=1)
        return time.perf_counter() - t0

    def describe(self, value: float, steps: int, seconds: float) -> dict:
        return {"value": value, "unit": "tokens/s", "cores": self.procs, "kind": "oracle",
                "nproc": os.cpu_count(), "affinity": _mask(self.affinity),
                "sample": f"the whole {self.tokens}-token headline batch (layer 0, seed 0) per step, float64 numpy, "
                          f"tokens split over {self.procs} spawned processes with one BLAS thread each; "
                          f"{steps} step(s), {seconds:.1f} s wall"}

    def close(self):
        self.pool.close()
        self.pool.join()


def oracle_sample(steps: int = 1, warm: int = 1):
    op = OraclePool()
    try:
        for _ in range(warm):
            op.step()
        tot = sum(op.step() for _ in range(steps))
        return op.describe(steps * op.tokens / tot, steps, tot), tot
    finally:
        op.close()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # every one of the K steps runs the oracle on the whole batch; more than
    # 60 steps would not finish within a few minutes, so K is capped there
    steps = max(1, min(args.steps, 60))
    warm = min(max(args.warmup, 0), 3)
    cb, tot = oracle_sample(steps, warm)
    v = cb["value"]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": 1000.0 * tot / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "full-shape MoE layer decode, 16 tokens, 4-bit/32 (CPU oracle)",
                       "experts": 512, "hidden": 2048, "inter": 768, "top_k": 10, "shared": 1, "bits": 4,
                       "block": 32, "tokens": 16},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU ---

class Runner:
    def __init__(self, torch, q, mi, md):
        self.torch, self.q, self.mi, self.md = torch, q, mi, md

    def layers(self, shape, n, zipf=False, seed=0):
        return [self.q.LayerWeights(**self.md.device_layer_tensors(shape, seed, l, zipf=zipf)) for l in range(n)]

    def xbatches(self, shape, T, n, seed=0, base=100):
        return [self.torch.from_numpy(self.mi.hidden_states_bf16(T, shape.hidden, seed, base + b).view(np.int16))
                .to("cuda") for b in range(n)]

    def touched(self, shape, cfg, layers, xs, steps):
        """Distinct routed experts each step selects (from the routing itself)."""
        torch, q = self.torch, self.q
        T = xs[0].shape[0]
        ws = torch.empty(q.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        wt = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
        cnt = torch.empty(shape.experts, dtype=torch.int32, device="cuda")
        us = []
        for i in range(steps):
            w = layers[i % len(layers)]
            q.moe_route(cfg, w.router_w, w.router_bias, xs[i % len(xs)], idx, wt, ws, counts=cnt)
            us.append(int((cnt > 0).sum().item()))
        return us

    def timed_graph(self, fn, K, W, chunk=32):
        """Warm-up W steps, then exactly K steps replayed from CUDA graphs of
        `chunk` steps (remainder in a second graph); returns elapsed ms."""
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(max(W, 1)):
                fn(i)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graphs = []
        full, rem = divmod(K, chunk)
        for n, offset in ((chunk if full else 0, 0), (rem, full * chunk)):
            if n == 0:
                graphs.append(None)
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for i in range(n):
                    fn(offset + i)
            graphs.append(g)
        torch.cuda.synchronize()
        return graphs, full

    def timed_graph_runs(self, run, K, W, chunk=32):
        """Like timed_graph for a function that issues a run of n steps
        itself: run(offset, n) on the current stream."""
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run(0, max(W, 2))
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graphs = []
        full, rem = divmod(K, chunk)
        for n, offset in ((chunk if full else 0, 0), (rem, full * chunk)):
            if n == 0:
                graphs.append(None)
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                run(offset, n)
            graphs.append(g)
        torch.cuda.synchronize()
        return graphs, full

    def replay(self, graphs, full):
        torch = self.torch
        st = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(st)
        for _ in range(full):
            graphs[0].replay()
        if graphs[1] is not None:
            graphs[1].replay()
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b)


def barrier(dist, world):
    if world > 1:
        dist.barrier()


def _reduce_scalar(dist, v: float, op) -> float:
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(dist, world, v: float) -> float:
    """Step time of the whole job: the slowest rank's."""
    return v if world <= 1 else _reduce_scalar(dist, v, dist.ReduceOp.MAX)


def sum_over_ranks(dist, world, v: float) -> float:
    return v if world <= 1 else _reduce_scalar(dist, v, dist.ReduceOp.SUM)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    import moe_inputs as mi
    import moe_inputs.device as md
    import quantized_expert_ffn_moe_b200 as q
    q.load_library()          # fails loudly if the CUDA library is missing
    md.load()
    R = Runner(torch, q, mi, md)
    hbm_peak, tf_peak, tf_sust, peak_src = measured_peaks()
    shape = mi.FULL4
    cfg = q.config_of(shape.experts, shape.hidden, shape.inter, shape.top_k, True, shape.bits, shape.block)
    T, K, W = args.tokens, args.steps, max(3, args.warmup)
    NI = args.instances
    pool = R.layers(shape, NI)
    NX = 16
    xs = R.xbatches(shape, T, NX)
    ys = [torch.empty_like(xs[0]) for _ in range(4)]
    ws = torch.empty(q.moe_workspace_bytes(cfg, max(T, 4096)), dtype=torch.uint8, device="cuda")

    def step(i):
        q.moe_layer_forward(cfg, pool[i % NI], xs[i % NX], ys[i % 4], ws)

    # ---- headline: exactly K steps, device-timed, max over ranks
    graphs, full = R.timed_graph(step, K, W)
    barrier(dist, world)
    clk = Clocks(local)
    clk.start()
    ms = R.replay(graphs, full)
    clocks = clk.stop()
    del graphs
    ms = max_over_ranks(dist, world, ms)
    tokens_all = sum_over_ranks(dist, world, float(T * K))
    value = tokens_all / (ms / 1000.0)
    ms_step = ms / K
    assert q.moe_device_status(ws) == 0, "device-side check failed"

    # ---- bytes the steps touch, and per-phase times (events on the launch stream)
    us = R.touched(shape, cfg, pool, xs, NI * 2)
    mean_u = float(np.mean(us))
    touched_bytes = (mean_u + 1) * EXPERT_BYTES[4] + ROUTER_BYTES + 2 * T * 2048 * 2
    n_prof = min(256, K)
    torch.cuda.synchronize()
    q.moe_profile_begin(n_prof)
    for i in range(n_prof):
        step(i)
    phase_ms, calls = q.moe_profile_end()
    fused = phase_ms[4] > 0
    if fused:
        # one cooperative kernel per layer is the step's only launch: its mean
        # duration is the graph-replayed step time of the timed region above
        # (CUDA events on the launching stream; it includes the gaps between
        # launches), and it moves all the touched bytes of those K steps
        k_ms = ms_step
        k_bytes = float(np.mean([(us[i % len(us)] + 1) for i in range(K)])) * EXPERT_BYTES[4] + ROUTER_BYTES
        kname = "fused_decode_kernel (whole layer, one launch)"
        timing = ("CUDA events around the K graph-replayed steps on the launching stream; one launch of this "
                  "kernel per step")
    else:
        k_ms = phase_ms[1] / calls
        k_bytes = float(np.mean([(us[i % len(us)] + 1) for i in range(calls)])) * GU_BYTES[4]
        kname = "ffn_tma_kernel<gate/up>"
        timing = "CUDA events around each launch of this kernel (eager loop of the same steps)"
    pf = profiled_fields("fused_decode_kernel_decode4_t16.txt",
                         ["fused.cu", "decode_common.cuh", "moe_internal.cuh"]) if fused else None
    traffic = float(pf["traffic_bytes_per_launch"]) if pf and "traffic_bytes_per_launch" in pf else None
    roofline = {"bound": "hbm", "kernel": kname, "achieved": k_bytes / (k_ms * 1e-3) / 1e9,
                "peak": hbm_peak, "unit": "GB/s", "frac": None, "traffic": traffic,
                "traffic_source": "profiles/fused_decode_kernel_decode4_t16.txt (ncu dram__bytes_read.sum + "
                                  "dram__bytes_write.sum, one launch of the same workload)" if traffic else None,
                "peak_source": f"{peak_src} (copy bandwidth)",
                "algorithmic_bytes_per_launch": k_bytes, "launch_us": 1000 * k_ms, "timing": timing,
                "launch_us_eager": 1000 * (phase_ms[4] if fused else phase_ms[1]) / calls,
                "phase_us_eager": {"route": 1000 * phase_ms[0] / calls, "gate_up": 1000 * phase_ms[1] / calls,
                                   "down": 1000 * phase_ms[2] / calls, "combine": 1000 * phase_ms[3] / calls,
                                   "fused": 1000 * phase_ms[4] / calls}}
    roofline["frac"] = roofline["achieved"] / hbm_peak
    try:
        # the decode kernel's second ceiling: instruction issue at the SM
        # clock sampled during the timed region
        if pf and "instructions_per_launch" in pf:
            sms = torch.cuda.get_device_properties(0).multi_processor_count
            mhz = clocks.get("sm_mhz") or 1965.0
            roofline["issue"] = issue_ceiling(float(pf["instructions_per_launch"]), k_ms * 1e-3, sms, mhz)
            roofline["issue"]["clock_source"] = ("median SM clock sampled during the timed region"
                                                 if clocks.get("sm_mhz") else "nominal maximum (no clock samples)")
    except Exception:
        pass
    # single launch path: the one-block status reset, then the decode kernel
    launches_per_step = 2 if fused else 5

    if args.quick:
        print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "steps": K, "ms_per_step": ms_step,
                          "roofline": roofline, "quick": True}), flush=True)
        return
    # ---- end to end: pinned host x -> device -> layer -> host y, every step.
    # The copies run on a second stream, double-buffered, so step i's result
    # copy-out and step i+2's input copy-in overlap the layer of step i+1 (the
    # way a serving loop feeds the library); every copy is inside the timed
    # region and ordered by events.
    x_host = [xs[i].cpu().pin_memory() for i in range(NX)]
    y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(xs[0]) for _ in range(2)]
    yd = [torch.empty_like(xs[0]) for _ in range(2)]
    cs = torch.cuda.Stream()

    def e2e_run(offset, n):
        main = torch.cuda.current_stream()
        cs.wait_stream(main)                                     # fork
        ev_in = [torch.cuda.Event(), torch.cuda.Event()]
        with torch.cuda.stream(cs):
            for j in range(min(2, n)):
                xd[j].copy_(x_host[(offset + j) % NX], non_blocking=True)
                ev_in[j].record(cs)
        for j in range(n):
            b = j % 2
            main.wait_event(ev_in[b])
            q.moe_layer_forward(cfg, pool[(offset + j) % NI], xd[b], yd[b], ws, stream=main)
            done = torch.cuda.Event()
            done.record(main)
            cs.wait_event(done)
            with torch.cuda.stream(cs):
                y_host[b].copy_(yd[b], non_blocking=True)
                if j + 2 < n:
                    xd[b].copy_(x_host[(offset + j + 2) % NX], non_blocking=True)
                    ev_in[b].record(cs)
        main.wait_stream(cs)                                     # join

    Ke = min(K, 4000)
    graphs, full = R.timed_graph_runs(e2e_run, Ke, W)
    barrier(dist, world)
    ems = max_over_ranks(dist, world, R.replay(graphs, full))
    del graphs
    e2e = {"value": sum_over_ranks(dist, world, float(T * Ke)) / (ems / 1000.0), "unit": "tokens/s",
           "h2d_bytes_per_step": T * 2048 * 2, "d2h_bytes_per_step": T * 2048 * 2,
           "path": "pinned host x -> device, moe_layer_forward, device y -> pinned host, per step; "
                   "copies on a second stream, double-buffered, overlapping the next step's layer"}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8 x int16 dp2a dot products (4-bit codes as signed bytes, int16 activations with a power-of-two scale per token), one fp32 fold per 32-element block, bf16 in/out", "data": "synthetic",
            "config": {"workload": "full-shape MoE layer decode (512 experts, H 2048, I 768, top-10 + shared, "
                                   "4-bit/32 fp16 scales), 16 tokens per step",
                       "tokens": T, "experts": 512, "hidden": 2048, "inter": 768, "top_k": 10, "shared": 1,
                       "bits": 4, "block": 32, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: steps rotate over {NI} distinct layer instances "
                             f"({NI * (512 * EXPERT_BYTES[4] + EXPERT_BYTES[4] + ROUTER_BYTES) / 1e9:.1f} GB) "
                             f"and {NX} token batches"},
            "hbm": {"touched_bytes_per_step": touched_bytes, "distinct_experts_per_step": mean_u,
                    "achieved_gbs": touched_bytes / (ms_step * 1e-3) / 1e9,
                    "frac_of_measured": touched_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak,
                    "frac_of_8tbs": touched_bytes / (ms_step * 1e-3) / 8e12},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches_per_step * K, "clocks": clocks}

    # ---- secondary workloads of the same layer family
    if not args.no_detail:
        line["detail"] = detail(R, args, pool, ws, W, hbm_peak, tf_peak, dist, world, clocks.get("sm_mhz"), tf_sust)

    # ---- CPU oracle baseline (rank 0, one GPU only)
    if world == 1:
        line["cpu_baseline"] = oracle_sample(1, 1)[0]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def detail(R, args, pool4, ws, W, hbm_peak, tf_peak, dist, world, clock_mhz=None, tf_sust=None):
    torch, q, mi = R.torch, R.q, R.mi
    out = {}
    shape = mi.FULL4
    cfg = q.config_of(512, 2048, 768, 10, True, 4, 32)
    NI = len(pool4)

    def layer_rate(cfg, shape, pool, T, K, bits, name, zipf=False):
        xs = R.xbatches(shape, T, 8, base=300 + T)
        ys = [torch.empty_like(xs[0]) for _ in range(2)]

        def step(i):
            q.moe_layer_forward(cfg, pool[i % len(pool)], xs[i % len(xs)], ys[i % 2], ws)
        graphs, full = R.timed_graph(step, K, 3, chunk=min(32, K))
        barrier(dist, world)
        ms = max_over_ranks(dist, world, R.replay(graphs, full))
        us = R.touched(shape, cfg, pool, xs, min(K, 2 * len(pool)))
        mb = (np.mean(us) + 1) * EXPERT_BYTES[bits] + ROUTER_BYTES
        r = {"tokens": T, "steps": K, "us_per_step": 1000 * ms / K, "tokens_per_s": T * K / (ms / 1000),
             "distinct_experts": float(np.mean(us)), "touched_mb": mb / 1e6,
             "achieved_gbs": mb / (ms / K * 1e-3) / 1e9}
        r["frac_of_measured_hbm"] = r["achieved_gbs"] / hbm_peak
        tc_share = 1.0 if T > 64 else 0.0
        if 32 <= T <= 64:
            # which side of the hand-over the calls took (the decode kernel
            # records its choice in the workspace's status words)
            picks = []
            for i in range(8):
                step(i)
                torch.cuda.synchronize()
                picks.append(int(ws[4 * ST_PATH:4 * ST_PATH + 4].view(torch.int32).item()))
            tc_share = float(np.mean(picks))
            r["tensor_core_share_of_calls"] = tc_share
        if tc_share > 0:
            flops = 9437184.0 * (T * 10 + T)
            r["tflops"] = flops / (ms / K * 1e-3) / 1e12
            r["frac_of_measured_bf16"] = r["tflops"] / tf_peak
            if tf_sust:
                # the tensor cores hold the part at its power cap for the whole
                # loop: the sustained figure is the matching ceiling
                r["frac_of_measured_bf16_sustained"] = r["tflops"] / tf_sust
            r["tensor_operands"] = ("fp16 x fp16 -> fp32: weights dequantized to q*s (one rounding), token rows "
                                    "scaled by a power of two per row (exact), compared against the bf16 dense "
                                    "peak (fp16 has the same dense rate)")
        if T <= 64:
            r["alu"] = alu_ceiling(bits, float(np.mean(us)), T, 1000 * ms / K, clock_mhz)
        out[name] = r

    for T in (1, 4):
        layer_rate(cfg, shape, pool4, T, 4000, 4, f"decode4_t{T}")
    # 4-bit with GPTQ-style 128-element groups, 16 tokens (4 layer instances:
    # 9.7 GB, far above L2)
    sg = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=128)
    cfg_g = q.config_of(512, 2048, 768, 10, True, 4, 128)
    poolg = R.layers(sg, 4)
    layer_rate(cfg_g, sg, poolg, 16, 2000, "4g128", "decode4g128_t16")
    del poolg
    # 2-bit codes read as the four half-integer levels (+-1/2, +-3/2), 16
    # tokens, near-uniform routing (8 layer instances: 7.3 GB, far above L2)
    sh2 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=2, block=16, half=True)
    cfg_h = q.config_of(512, 2048, 768, 10, True, 2, 16, half_levels=True)
    poolh = R.layers(sh2, 8)
    layer_rate(cfg_h, sh2, poolh, 16, 2000, 2, "decode2h_t16")
    del poolh
    # 4-bit with one E4M3 scale byte per 32 elements and an fp32 scale per row
    # (the single-launch decode kernel; 8 layer instances: 10.4 GB, far above L2)
    sf8 = mi.MoeShape(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=32, fp8_scales=True)
    cfg_f8 = q.config_of(512, 2048, 768, 10, True, 4, 32, fp8_scales=True)
    poolf8 = R.layers(sf8, 8)
    layer_rate(cfg_f8, sf8, poolf8, 16, 2000, "4f8", "decode4f8_t16")
    del poolf8
    layer_rate(cfg, shape, pool4, 4096, 8, 4, "prefill4_t4096")

    # expert-parallel share: one rank's partial of the 4096-token layer when
    # the experts are split over n ranks (computed on this one GPU; the
    # all-reduce of the fp32 partials is not included)
    xs = R.xbatches(shape, 4096, 2, base=900)
    yp = torch.empty((4096, shape.hidden), dtype=torch.float32, device="cuda")
    ep = {}
    for n in (1, 2, 4, 8):
        def estep(i, n=n):
            q.moe_layer_forward_ep(cfg, pool4[i % NI], xs[i % 2], yp, ws, 0, n)
        graphs, full = R.timed_graph(estep, 4, 2, chunk=4)
        barrier(dist, world)
        ms = max_over_ranks(dist, world, R.replay(graphs, full))
        ep[f"ep{n}_rank0_us"] = 1000 * ms / 4
    out["expert_parallel_share_t4096"] = ep
    # 2-bit skewed routing
    s2 = mi.FULL2
    cfg2 = q.config_of(512, 2048, 768, 10, True, 2, 16)
    pool2 = R.layers(s2, 16, zipf=True)
    for T in (1, 8, 64):
        layer_rate(cfg2, s2, pool2, T, 2000, 2, f"zipf2_t{T}", zipf=True)
    del pool2
    torch.cuda.empty_cache()
    # 48-layer stack: residual stream through all layers resident in HBM
    if NI >= 48:
        for T in (1, 32):
            xs = R.xbatches(shape, T, 4, base=500 + T)
            xw = torch.empty_like(xs[0])

            def sstep(i):
                xw.copy_(xs[i % 4])
                q.moe_stack_forward(cfg, pool4[:48], xw, ws)
            K = 20 if T == 1 else 10
            graphs, full = R.timed_graph(sstep, K, 2, chunk=K)
            barrier(dist, world)
            ms = max_over_ranks(dist, world, R.replay(graphs, full))
            r = {"tokens": T, "steps": K, "ms_per_step": ms / K, "tokens_per_s": T * K / (ms / 1000)}
            # decode T = 1 touches 10 routed + the shared expert per layer; at
            # T = 32 the distinct experts are counted from the routing of layer 0
            # of each batch (near-uniform routing makes the layers alike)
            if T == 1:
                bytes_step = 48 * (11 * EXPERT_BYTES[4] + ROUTER_BYTES)
                r["touched_gb_per_step"] = bytes_step / 1e9
                r["frac_of_measured_hbm"] = bytes_step / (ms / K * 1e-3) / 1e9 / hbm_peak
            out[f"stack48_t{T}"] = r
        # 2048-token prefill through the 48-layer stack: every layer touches
        # all 512 experts (2048 x 10 picks), 1.364 GB, and does 212.6 GFLOP of
        # expert FFN (+ 4.3 GFLOP router); HBM-bound (about 142 FLOP/B)
        xs = R.xbatches(shape, 2048, 2, base=650)
        xw = torch.empty_like(xs[0])

        def pstep(i):
            xw.copy_(xs[i % 2])
            q.moe_stack_forward(cfg, pool4[:48], xw, ws)
        K = 3
        graphs, full = R.timed_graph(pstep, K, 1, chunk=K)
        barrier(dist, world)
        ms = max_over_ranks(dist, world, R.replay(graphs, full))
        del graphs
        T = 2048
        bytes_step = 48 * (513 * EXPERT_BYTES[4] + ROUTER_BYTES) + 2 * 2 * T * 2048 * 2
        flops_step = 48 * (9437184.0 * (T * 10 + T) + 2.0 * T * 512 * 2048)
        sec = ms / K * 1e-3
        out["stack48_prefill_t2048"] = {
            "tokens": T, "steps": K, "ms_per_step": ms / K, "tokens_per_s": T / sec,
            "gb_per_step": bytes_step / 1e9, "achieved_gbs": bytes_step / sec / 1e9,
            "frac_of_measured_hbm": bytes_step / sec / 1e9 / hbm_peak,
            "tflops": flops_step / sec / 1e12, "frac_of_measured_bf16": flops_step / sec / 1e12 / tf_peak,
            "frac_of_measured_bf16_sustained": flops_step / sec / 1e12 / tf_sust if tf_sust else None,
            "bound": "hbm (about 142 FLOP per byte of expert weights, below the ridge)"}
    return out


if __name__ == "__main__":
    main()
