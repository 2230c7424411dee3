#!/usr/bin/env python
"""Benchmark of the decode-time MXFP4 MoE expert layer (one verify block per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--tokens T]

A step is one pass of the whole hot path -- router, permutation, gate/up
projection + SwiGLU, down projection, weighted combine -- over one token block
(one ``moe_forward`` call, a single engine launch).  Default workload: the
single-sequence decode verify step, T=9 tokens, H=4096, I=1536, E=128, top-8,
MXFP4 expert weights drawn N(0, 0.02) and quantised on the device, activations
N(0, 1).  Each step routes a different seeded token block (8 blocks in
rotation), and the ~0.5 GB of expert weights one step streams exceeds the
126 MB L2, so no L2 flush is inserted between steps.  The K timed calls are
captured once into a CUDA graph and replayed (``--no-graph``: K stream
launches); either way every step is a full engine launch on its own inputs.
At verify-block sizes the line also carries ``ops_baseline``: the same calls as
six launches per layer (``moe_forward_ops``: stream launches, a CUDA graph,
and a CUDA graph of programmatic dependent launches) next to the engine's own
launch, in µs per step.

Under torchrun each rank runs the same layer on its own token blocks (independent
verify steps: weak scaling, no collective on the data path); the timed region is
bracketed by a barrier and device synchronisation, and the slowest rank's time
is reported.  ``--impl reference`` times the fp64 CPU oracle on a bounded sample
of the same workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from synth.spec import VERIFY_WORKLOADS  # noqa: E402

METRIC = "MoE layer µs + MXFP4 weight-stream HBM GB/s (% of peak) at T=9; tokens/s"
VERIFY_METRIC = "speculative-verify acceptance step: verify blocks/s (G=8 drafts, V=152064)"
PROFILE = os.path.join(ROOT, "profiles", "engine_decode_t9_h4096_e128.md")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="decode_t9_h4096_e128",
                    choices=sorted(synth.WORKLOADS) + sorted(VERIFY_WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None, help="override T (default: the workload's own; 9 for the sweep)")
    ap.add_argument("--batches", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--large-kind", choices=("f16", "mxf4", "mxf8"), default="mxf4",
                    help="weight stream for many positions per expert: bf16 tiles, E2M1 term tiles or "
                         "E4M3 term tiles")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying them as one CUDA graph")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--shard-i", action="store_true",
                    help="I-sharded layer across the ranks (the default with more than one rank): every rank "
                         "streams its I-slice of the same token block; the partials are summed by the engine's "
                         "fused all-reduce (peer loads) and rounded to bf16")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one rank: independent replicas (each rank its own token blocks, no "
                         "collective on the data path) instead of the I-sharded layer")
    ap.add_argument("--nccl-allreduce", action="store_true",
                    help="I-sharded layer: sum the partials with an NCCL all-reduce between launches instead of "
                         "the fused all-reduce")
    ap.add_argument("--no-ops-baseline", action="store_true",
                    help="skip timing the operator-by-operator launches (moe_forward_ops)")
    return ap.parse_args()


ENGINE_SOURCES = ("engine.cu", "engine.cuh", "ptx.cuh")


def source_digest() -> str:
    """Digest of the sources engine_kernel's code is compiled from."""
    h = hashlib.sha256()
    for f in ENGINE_SOURCES:
        with open(os.path.join(ROOT, "mxfp4_moe_expert_router_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


PROFILED_WORKLOAD = "decode_t9_h4096_e128"


def traffic_for(name: str, T: int):
    """The committed capture's DRAM bytes per launch, for the launch it was taken of:
    the decode workload at its own token count (another token count takes another
    kernel instance and other bytes), else None."""
    if name != PROFILED_WORKLOAD or T != synth.WORKLOADS[PROFILED_WORKLOAD].tokens:
        return None
    return profile_traffic()


def profile_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    try:
        txt = open(PROFILE).read()
    except OSError:
        return None
    kv = {}
    for ln in txt.splitlines():
        if ln.startswith("- ") and ":" in ln:
            k, v = ln[2:].split(":", 1)
            kv[k.strip()] = v.strip().strip("`")
    if kv.get("source_sha256_16") != source_digest():
        return None
    try:
        return float(kv["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def upload_graph(graph, stream):
    """Upload an instantiated CUDA graph to the device before its first replay,
    so the timed replay carries no upload (driver entry point cuGraphUpload)."""
    import ctypes
    import torch
    cuda = ctypes.CDLL("libcuda.so.1")
    cuda.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rc = cuda.cuGraphUpload(ctypes.c_void_p(graph.raw_cuda_graph_exec()), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cuGraphUpload failed: {rc}")
    torch.cuda.synchronize()


def time_calls(mx, stream, n: int, launch, use_graph: bool) -> float:
    """Device time per call (us) of n calls launch(i, stream_handle): stream
    launches, or the n calls captured into one CUDA graph and replayed."""
    import torch
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = mx._stream()
            for i in range(n):
                launch(i, cap)
        upload_graph(graph, stream)
    sp = mx._stream(stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(n):
            launch(i, sp)
    e1.record(stream)
    torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) * 1e3 / n


def per_call_times(m, mx, stream, step, n: int) -> dict:
    """Device time of each of n stream-launched calls, an event pair around each:
    median / p10 / p90 in us (the graph replay gives only the mean)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(ev):
        a.record(stream)
        step(i)
        b.record(stream)
    torch.cuda.synchronize()
    m.moe_status()
    us = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
    q = lambda f: us[min(len(us) - 1, int(f * (len(us) - 1) + 0.5))]
    return {"median_us": q(0.5), "p10_us": q(0.1), "p90_us": q(0.9), "n": n,
            "launch": "stream launches, an event pair around each call"}


def ops_baseline(mx, m, stream, xptr, yptr, T: int, steps: int) -> dict:
    """The same layer(s) as six launches per layer (moe_forward_ops) against the
    single engine launch, each as stream launches and as a CUDA graph; the ops
    also as a graph of programmatic dependent launches."""
    def ops(flags):
        def launch(i, sp):
            st = mx.lib.moe_forward_ops(m.handle, xptr[i % len(xptr)], T, yptr, None, flags, sp)
            if st != 0:
                raise mx.MoeError(st, "moe_forward_ops")
        return launch

    def engine(i, sp):
        st = mx.lib.moe_forward(m.handle, xptr[i % len(xptr)], T, yptr, None, sp)
        if st != 0:
            raise mx.MoeError(st, "moe_forward")

    for i in range(3):
        ops(mx.MOE_OPS_PDL)(i, mx._stream(stream))
        ops(0)(i, mx._stream(stream))
    m.moe_status()
    res = {"engine_stream": time_calls(mx, stream, steps, engine, False),
           "engine_graph": time_calls(mx, stream, steps, engine, True),
           "ops_stream": time_calls(mx, stream, steps, ops(0), False),
           "ops_graph": time_calls(mx, stream, steps, ops(0), True),
           "ops_graph_pdl": time_calls(mx, stream, steps, ops(mx.MOE_OPS_PDL), True)}
    m.moe_status()
    return {"us_per_step": {k: round(v, 2) for k, v in res.items()},
            "launches_per_step": {"engine": 1, "ops": 6 * m.cfg.num_layers}, "steps": steps,
            "ops": "router partial logits; routing (1 CTA); x term images; gate/up + SwiGLU; down; combine"}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak (burst: the engine is timed alone), measured, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


# Tensor-core kinds of the large-T weight stream: nominal dense rate relative to
# bf16 (B200: fp4 9, fp8 4.5, bf16 2.25 PFLOP/s) and the MMA columns each
# activation value occupies in the gate/up and down projections.
LARGE_KINDS = {
    "mxf4": {"mma": "tcgen05.mma kind::mxf4 (E2M1 x E2M1, E8M0 scales)", "ratio_to_bf16": 4.0,
             "terms_gate_up": 5, "terms_down": 5},
    "f16": {"mma": "tcgen05.mma kind::f16 (bf16 x bf16, weights dequantised)", "ratio_to_bf16": 1.0,
            "terms_gate_up": 1, "terms_down": 2},
    "mxf8": {"mma": "tcgen05.mma kind::mxf8f6f4 (E2M1 x E4M3, E8M0 scales)", "ratio_to_bf16": 2.0,
             "terms_gate_up": 2, "terms_down": 3},
}


def layer_flops(w: synth.Workload, T: int) -> float:
    """Algorithmic FLOP of one call: 6 T k H I (gate, up, down) + 2 T H E (router), per layer."""
    return (6.0 * T * w.top_k * w.hidden * w.inter + 2.0 * T * w.hidden * w.experts) * w.layers


def roofline(w: synth.Workload, T: int, alg_bytes: float, ms_step: float, large_kind: str, traffic) -> dict:
    """HBM roofline of the weight stream, or the tensor roofline where the tile stream's
    arithmetic intensity exceeds the ridge of its kind (the FP4 peak divided by the term
    expansion of the activations, over the HBM peak)."""
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (ms_step * 1e-3) / 1e9
    hbm = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
           "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg_bytes, "traffic": traffic,
           "kernel": "engine_kernel"}
    TK = T * w.top_k
    if not (TK > 256 and TK >= 8 * w.experts):
        return hbm
    k = LARGE_KINDS[large_kind]
    bf16, bf16_kind = measured_bf16_tflops()
    kind_peak = bf16 * k["ratio_to_bf16"]
    flops = layer_flops(w, T)
    terms = (2 * k["terms_gate_up"] + k["terms_down"]) / 3.0  # gate and up carry 2/3 of the FLOP
    intensity = flops / alg_bytes
    ridge = kind_peak / terms * 1e12 / (peak * 1e9)
    if intensity <= ridge:
        hbm["intensity_flop_per_byte"] = intensity
        hbm["ridge_flop_per_byte"] = ridge
        return hbm
    tf = flops / (ms_step * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": tf, "peak": kind_peak, "unit": "TFLOP/s", "frac": tf / kind_peak,
            "peak_source": f"{bf16_kind} bf16 {bf16:.1f} TFLOP/s x {k['ratio_to_bf16']:g} (nominal ratio of "
                           f"{k['mma']} to bf16 on B200)",
            "algorithmic_flop_per_launch": flops, "mma_columns_per_value": terms,
            "frac_of_term_adjusted_peak": tf / (kind_peak / terms),
            "intensity_flop_per_byte": intensity, "ridge_flop_per_byte": ridge,
            "traffic": None, "kernel": "engine_kernel", "hbm": hbm}


class ClockSampler:
    """nvidia-smi clocks/throttle sampling of one GPU while the timed region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")
        if uuid is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in open(self.path):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---- workload construction ---------------------------------------------------------------------

def build_layer(mx, w: synth.Workload, layer: int, seed: int):
    """Draw and quantise one layer on the device with the library's own quantiser."""
    import torch
    H, I, E = w.hidden, w.inter, w.experts
    u8 = dict(dtype=torch.uint8, device="cuda")
    gc, uc = torch.empty((E, I, H // 2), **u8), torch.empty((E, I, H // 2), **u8)
    gs, us = torch.empty((E, I, H // 32), **u8), torch.empty((E, I, H // 32), **u8)
    dc, ds = torch.empty((E, H, I // 2), **u8), torch.empty((E, H, I // 32), **u8)
    stream = mx._stream()
    for e in range(E):
        for kind, c, s in (("gate", gc, gs), ("up", uc, us), ("down", dc, ds)):
            wt = synth.expert_torch(w, layer, e, kind, seed=seed)
            st = mx.lib.mxfp4_quantize(mx._ptr(wt), wt.shape[0], wt.shape[1], mx._ptr(c[e]),
                                       mx._ptr(s[e]), stream)
            if st != 0:
                raise mx.MoeError(st, "mxfp4_quantize")
    dense = synth.layer_inputs_torch(w, layer=layer, seed=seed)
    return mx.LayerMX(gc, gs, uc, us, dc, ds, dense["router_w"].contiguous(), dense["router_b"])


def token_block_ids(rank: int, n: int) -> list:
    """Stream ids of the n token blocks rank `rank` runs: 64 ids per rank, disjoint across ranks
    (every rank verifies its own blocks; nothing is exchanged on the data path)."""
    if not 0 < n <= 64:
        raise ValueError("1..64 token blocks per rank")
    return [1000 + rank * 64 + b for b in range(n)]


def token_blocks(w: synth.Workload, T: int, n: int, rank: int):
    return [synth.draw_torch(i, 0, "x", -1, (T, w.hidden), 1.0) for i in token_block_ids(rank, n)]


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's time (identity with one rank or no process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, T: int, steps: int, seconds: float) -> float:
    """Whole-job throughput: every rank verifies T tokens per step."""
    return world * T * steps / seconds


def algorithmic_bytes(w: synth.Workload, T: int, hit: int) -> float:
    """MXFP4 bytes of the hit experts + fp32 router weights + bf16 x and y, per layer."""
    return hit * 3 * w.hidden * w.inter * 0.53125 + 4.0 * w.experts * w.hidden + 4.0 * T * w.hidden


# ---- the CPU oracle as baseline / reference arm --------------------------------------------------

def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_prepare(w: synth.Workload, layer_dev, x_dev, n_experts: int):
    """Untimed set-up of the oracle baseline: the block's fp64 inputs, its routing, and the
    oracle's own MXFP4 codes of the first n hit experts (quantised from the same seeded bf16
    weights as the GPU's)."""
    import torch
    from oracle import moe, mxfp4
    xb = x_dev.view(torch.int16).cpu().numpy().view(np.uint16)
    x = mxfp4.bf16_to_f64(xb)
    rw = layer_dev.router_w.cpu().numpy()
    rb = None if layer_dev.router_b is None else layer_dev.router_b.cpu().numpy()
    idx, wts, _ = moe.route(x, rw, rb, w.top_k)
    counts, offsets, perm, inv = moe.permute(idx, w.experts)
    hit = [int(e) for e in np.nonzero(counts)[0]]
    q = {}
    dev = x_dev.device
    for e in hit[:n_experts]:
        q[e] = {kind: mxfp4.quantize(synth.expert_torch(w, 0, e, kind, device=dev)
                                     .view(torch.int16).cpu().numpy().view(np.uint16))
                for kind in ("gate", "up", "down")}
    return {"x": x, "rw": rw, "rb": rb, "hit": hit, "q": q, "offsets": offsets, "perm": perm,
            "flat_w": wts.reshape(-1)}


def oracle_step(w: synth.Workload, prep, e: int):
    """One timed sample of the oracle: the routing of the whole block, then one hit expert
    (dequantise + SwiGLU FFN + routing weight).  Returns (route s, expert s)."""
    from oracle import moe, mxfp4
    t0 = time.perf_counter()
    moe.permute(moe.route(prep["x"], prep["rw"], prep["rb"], w.top_k)[0], w.experts)
    t1 = time.perf_counter()
    q = prep["q"][e]
    seg = prep["perm"][prep["offsets"][e]:prep["offsets"][e + 1]]
    wg, wu, wd = (mxfp4.dequantize(*q[k]) for k in ("gate", "up", "down"))
    _ = moe.expert_ffn(prep["x"][seg // w.top_k], wg, wu, wd) * prep["flat_w"][seg][:, None]
    return t1 - t0, time.perf_counter() - t1


def oracle_baseline(w: synth.Workload, T: int, layer_dev, x_dev, n_experts: int = 4, reps: int = 3):
    """The oracle on this host's cores, BLAS on all threads and on one: per setting, `reps`
    repetitions of (routing of the block + n hit experts), median taken; the layer time is
    routing + (hit experts) x (median time of one expert)."""
    from threadpoolctl import threadpool_limits
    prep = oracle_prepare(w, layer_dev, x_dev, n_experts)
    out = {}
    for label, limit in (("all", None), ("one", 1)):
        with threadpool_limits(limits=limit, user_api="blas"):
            threads = blas_threads()
            routes, experts = [], []
            for _ in range(reps):
                for i, e in enumerate(prep["q"]):
                    r, x = oracle_step(w, prep, e)
                    experts.append(x)
                    if i == 0:
                        routes.append(r)
            t_route, t_exp = statistics.median(routes), statistics.median(experts)
            out[label] = {"threads": threads, "route_s": t_route, "expert_s": t_exp,
                          "layer_s": t_route + t_exp * len(prep["hit"])}
    out["hit"] = len(prep["hit"])
    out["experts_timed"] = len(prep["q"])
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ---- main ------------------------------------------------------------------------------------------

PHASES = ("router_logits", "x_images", "route_wait", "topk_or_tables", "permute", "stream", "combine")


def main():
    args = parse_args()
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in VERIFY_WORKLOADS:
        return run_verify(args, VERIFY_WORKLOADS[args.workload], rank, world)
    w = synth.WORKLOADS[args.workload]
    sweep = args.workload.startswith("sweep")
    T = args.tokens or (9 if sweep else w.tokens)
    if sweep:
        w = w.with_tokens(max(T, w.tokens))
    elif args.tokens:  # another token count on this workload's shapes
        w = w.with_tokens(T)

    if args.impl == "reference":
        return run_reference(args, w, T, rank, world)

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import mxfp4_moe_expert_router_b200 as mx

    layers = [build_layer(mx, w, l, seed=0) for l in range(w.layers)]
    if args.shard_i or (world > 1 and not args.replicas and w.layers == 1):
        return run_shard_i(args, mx, w, T, layers, rank, world)
    m = mx.Moe(w.hidden, w.inter, w.experts, w.top_k, T, layers)
    m.moe_set_large_kind({"f16": m.LARGE_F16, "mxf4": m.LARGE_MXF4, "mxf8": m.LARGE_MXF8}[args.large_kind])
    xs = token_blocks(w, T, args.batches, rank)
    hits = []
    for x in xs:
        r = m.moe_route(x, layer=0)
        hits.append(int((r["counts"] > 0).sum().item()))
    m.moe_status()
    y = torch.empty((T, w.hidden), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    sp = mx._stream(stream)
    xptr = [mx._ptr(x) for x in xs]
    yptr = mx._ptr(y)

    def step(i):
        st = mx.lib.moe_forward(m.handle, xptr[i % len(xptr)], T, yptr, None, sp)
        if st != 0:
            raise mx.MoeError(st, "moe_forward")

    for i in range(args.warmup):
        step(i)
    m.moe_status()
    # The timed steps are the same moe_forward calls captured into one CUDA
    # graph (a stream launch leaves the GPU idle ~3.4 us between calls, a graph
    # replay ~1.5 us); --no-graph times them as individual stream launches.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = mx._stream()
            for i in range(args.steps):
                st = mx.lib.moe_forward(m.handle, xptr[i % len(xptr)], T, yptr, None, cap)
                if st != 0:
                    raise mx.MoeError(st, "moe_forward (capture)")
        upload_graph(graph, stream)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid if rank == 0 else None)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    m.moe_status()
    phases = m.moe_phase_ns()  # the last timed step, CTA 0's view
    per_call = per_call_times(m, mx, stream, step, min(args.steps, 200))
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), dist if world > 1 else None, "cuda")
    ms_step = ms_total / args.steps
    tokens_per_s = job_tokens_per_s(world, T, args.steps, ms_total / 1e3)
    mean_hit = float(np.mean([hits[i % len(hits)] for i in range(args.steps)]))
    alg_bytes = algorithmic_bytes(w, T, mean_hit) * w.layers if w.layers == 1 else None
    # the chain workload's later layers route on the previous layer's output: count them
    if alg_bytes is None:
        alg_bytes = float(np.mean([sum(algorithmic_bytes(w, T, h) for h in chain_hits(m, mx, w, T, x))
                                   for x in xs[:2]]))
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (ms_step * 1e-3) / 1e9
    # the committed capture is of the decode workload's engine launch
    traffic = traffic_for(w.name, T)

    # the pages' baseline execution model: one launch per operator
    ops = None
    if world == 1 and not args.no_ops_baseline and T * w.top_k <= 256:
        ops = ops_baseline(mx, m, stream, xptr, yptr, T, max(1, min(args.steps, 500)))

    # end-to-end: the same metric through the public host-buffer entry point
    e2e = None
    if not args.no_e2e:
        xh = [x.cpu().pin_memory() for x in xs]
        yh = torch.empty((T, w.hidden), dtype=torch.bfloat16).pin_memory()
        n_e2e = args.e2e_steps or 500
        for i in range(min(3, n_e2e)):
            m.moe_forward_host(xh[i % len(xh)], yh)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # pipelined: moe_forward_host_async enqueues each call's H2D (copy
        # stream), layers (this stream) and D2H (second copy stream); the
        # timed region ends once every output copy has landed
        yh2 = [yh, torch.empty_like(yh).pin_memory()]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n_e2e):
            m.moe_forward_host_async(xh[i % len(xh)], yh2[i % 2], stream=stream)
        m.moe_host_join(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        m.moe_status(stream)
        el = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, "cuda")
        # per call synchronous (each call's result on the host before the next call)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(n_e2e):
            m.moe_forward_host(xh[i % len(xh)], yh, stream=stream)
        s1.record(stream)
        torch.cuda.synchronize()
        el_sync = max_over_ranks(s0.elapsed_time(s1) / 1e3, dist if world > 1 else None, "cuda")
        e2e = {"value": job_tokens_per_s(world, T, n_e2e, el), "unit": "tokens/s", "steps": n_e2e,
               "h2d_bytes_per_step": T * w.hidden * 2, "d2h_bytes_per_step": T * w.hidden * 2,
               "api": "moe_forward_host_async (copies overlap the neighbouring calls)",
               "per_call_sync_value": job_tokens_per_s(world, T, n_e2e, el_sync)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ob = oracle_baseline(w, T, layers[0], xs[0])
        layers_n = w.layers
        cpu = {"value": T / (ob["all"]["layer_s"] * layers_n), "unit": "tokens/s",
               "cores": ob["all"]["threads"], "kind": "oracle",
               "sample": f"fp64 numpy oracle, layer 0, token block 0, median of 3: routing of all {T} tokens "
                         f"+ each of {ob['experts_timed']} hit experts (dequantise + SwiGLU FFN); layer time = "
                         f"routing + {ob['hit']} hit experts x median expert time"
                         + (f", x {layers_n} layers" if layers_n > 1 else ""),
               "cpu_model": cpu_model(), "cpu_count": os.cpu_count(),
               "layer_s_estimate": ob["all"]["layer_s"] * layers_n,
               "blas_one_thread": {"value": T / (ob["one"]["layer_s"] * layers_n), "unit": "tokens/s",
                                   "threads": ob["one"]["threads"],
                                   "layer_s_estimate": ob["one"]["layer_s"] * layers_n},
               "timed_s": {k: {"route": ob[k]["route_s"], "expert": ob[k]["expert_s"]} for k in ("all", "one")}}

    if rank == 0:
        out = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "mxfp4-w/fp32-acc",
            "data": "synthetic (seeded N(0,0.02) expert weights quantised to MXFP4, N(0,1) bf16 tokens)",
            "config": {"workload": w.name if not (sweep or args.tokens) else f"{w.name}_t{T}",
                       "hidden": w.hidden, "inter": w.inter, "experts": w.experts, "top_k": w.top_k,
                       "tokens_per_gpu": T, "layers": w.layers, "token_blocks": len(xs),
                       "mean_experts_hit": mean_hit,
                       "l2": "no flush: ~%.0f MB of expert weights streamed per step > 126 MB L2"
                             % (alg_bytes / 1e6),
                       "parallelism": f"replicas x{world} (independent verify blocks)",
                       "large_kind": args.large_kind,
                       "launch": "stream launches" if graph is None else
                                 "the timed moe_forward calls replayed as one CUDA graph"},
            "layer_us": ms_step * 1e3 / w.layers,
            "weight_stream_gbs": achieved,
            "roofline": roofline(w, T, alg_bytes, ms_step, args.large_kind, traffic),
            "per_call": per_call,
            "gpu_launches": args.steps,
            "phase_us_last_step": {k: round(v / 1e3, 2) for k, v in
                                   zip(PHASES, phases[:7])},
            "phase_us_mean_over_layers": None if w.layers == 1 else
                {k: round(float(np.mean(phases[i::7][:w.layers])) / 1e3, 2) for i, k in enumerate(PHASES)},
            "e2e": e2e,
            "ops_baseline": ops,
            "cpu_baseline": cpu,
            "clocks": clk,
        }
        print(json.dumps(out), flush=True)
    m.close()
    if world > 1:
        dist.destroy_process_group()


def chain_hits(m, mx, w, T, x):
    """Experts hit per layer of the chain on token block x (routes each layer's real input)."""
    import torch
    io = torch.empty((w.layers + 1, T, w.hidden), dtype=torch.bfloat16, device="cuda")
    m.moe_forward(x, layer_io=io)
    hits = []
    for l in range(w.layers):
        r = m.moe_route(io[l].contiguous(), layer=l)
        hits.append(int((r["counts"] > 0).sum().item()))
    return hits


def run_reference(args, w, T, rank, world):
    """The fp64 CPU oracle on this host's cores as the reference arm, rank 0 only.

    Each timed step is a measured, bounded sample of the layer: the oracle's
    routing of the whole token block, then one whole hit expert (dequantise +
    SwiGLU FFN + routing weight), the experts taken in turn from the first few
    hit ones.  ``ms_per_step`` is that step's measured time.  ``value`` is the
    layer's tokens/s extrapolated from the medians (routing + hit experts x
    one expert), reported with the extrapolation's inputs."""
    if rank != 0:
        return
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.draw_torch(1000, 0, "x", -1, (T, w.hidden), 1.0, device=dev)
    dense = synth.layer_inputs_torch(w, 0, 0, tokens=T, device=dev)

    class _L:  # the two dense router tensors oracle_prepare reads
        router_w, router_b = dense["router_w"], dense["router_b"]

    prep = oracle_prepare(w, _L, x, n_experts=min(4, max(1, args.steps + args.warmup)))
    experts = list(prep["q"])
    for i in range(args.warmup):
        oracle_step(w, prep, experts[i % len(experts)])
    routes, times, steps_s = [], [], []
    t_all = time.perf_counter()
    for i in range(args.steps):
        t0 = time.perf_counter()
        r, e = oracle_step(w, prep, experts[i % len(experts)])
        steps_s.append(time.perf_counter() - t0)
        routes.append(r)
        times.append(e)
    wall = time.perf_counter() - t_all
    hit = len(prep["hit"])
    layer_s = (statistics.median(routes) + statistics.median(times) * hit) * w.layers
    value = T / layer_s
    ms_step = wall * 1e3 / max(1, args.steps)
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": {"workload": w.name, "hidden": w.hidden, "inter": w.inter, "experts": w.experts,
                      "top_k": w.top_k, "tokens_per_gpu": T, "layers": w.layers},
           "step": "measured: oracle routing of all %d tokens + one whole hit expert (of %d hit)" % (T, hit),
           "value_basis": {"layer_s_extrapolated": layer_s, "route_s_median": statistics.median(routes),
                           "expert_s_median": statistics.median(times), "hit_experts": hit,
                           "layers": w.layers},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                            "cpu_model": cpu_model(), "cpu_count": os.cpu_count(),
                            "sample": f"each step: the oracle's routing of the block + one of the first "
                                      f"{len(experts)} hit experts in turn (measured); layer time = routing "
                                      f"+ {hit} hit experts x the median expert time"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def ishard_groups(inter: int, world: int):
    """(group size g, groups): the largest g dividing `world` whose I-slices are multiples
    of 128 (the engine's tiling); the world is then world / g groups of g ranks, each an
    I-sharded layer on its own token blocks."""
    for g in range(min(world, 8), 0, -1):
        if world % g == 0 and inter % g == 0 and (inter // g) % 128 == 0:
            return g, world // g
    return 1, world


def run_shard_i(args, mx, w, T, layers, rank, world):
    """The I-sharded layer: each rank of a group of g holds rows [r*I/g, (r+1)*I/g) of
    every expert's gate/up matrices and the same down columns, and streams them for the
    group's token block; the engine's last combine sums the g fp32 partials over NVLink
    peer loads (moe_forward_ishard, one launch per step) and rounds to bf16.  With
    --nccl-allreduce the partials are summed by an NCCL all-reduce between launches
    (moe_forward_partial, all-reduce, moe_round_bf16).  Strong scaling within a group."""
    import torch
    import torch.distributed as dist
    if w.layers != 1:
        raise SystemExit("--shard-i: one layer per call")
    g, groups = ishard_groups(w.inter, world)
    my_group, grank = rank // g, rank % g
    pgs = [dist.new_group(list(range(k * g, (k + 1) * g))) for k in range(groups)] if world > 1 else [None]
    pg = pgs[my_group]
    shard = mx.shard_layer_i(layers[0], grank, g)
    m = mx.Moe(w.hidden, w.inter // g, w.experts, w.top_k, T, [shard])
    xs = token_blocks(w, T, args.batches, my_group)  # the same token blocks within a group
    hits = [int((m.moe_route(x, layer=0)["counts"] > 0).sum().item()) for x in xs]
    part = torch.empty((T, w.hidden), dtype=torch.float32, device="cuda")
    y = torch.empty((T, w.hidden), dtype=torch.bfloat16, device="cuda")
    fused = not args.nccl_allreduce
    opened = []
    if fused:
        if g > 1:
            opened = mx.connect_ishard(m, pg)
        else:
            m.moe_ishard_attach(0, 1, [m.moe_ishard_region()[0]])

    def step(i):
        if fused:
            m.moe_forward_ishard(xs[i % len(xs)], y)
        else:
            m.moe_forward_partial(xs[i % len(xs)], part)
            if g > 1:
                dist.all_reduce(part, group=pg)
            mx.round_bf16(part, y)

    for i in range(args.warmup):
        step(i)
    m.moe_status()
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(("GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid))
                          if rank == 0 else None)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    m.moe_status()
    ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, "cuda")
    us_step = ms * 1e3 / args.steps
    mean_hit = float(np.mean([hits[i % len(hits)] for i in range(args.steps)]))
    shard_w = synth.Workload(w.name, w.hidden, w.inter // g, w.experts, w.top_k, T)
    alg = algorithmic_bytes(shard_w, T, mean_hit)
    peak, peak_kind = measured_peaks()
    achieved = alg / (us_step * 1e-6) / 1e9
    # end to end: every step copies its token block from pinned host memory and its
    # output back (the group's rank 0 would hand y on; every rank copies it here)
    e2e = None
    if not args.no_e2e:
        xh = [x.cpu().pin_memory() for x in xs]
        yh = torch.empty((T, w.hidden), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(xs[0])
        n_e2e = args.e2e_steps or max(args.steps, 100)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(n_e2e):
            xd.copy_(xh[i % len(xh)], non_blocking=True)
            if fused:
                m.moe_forward_ishard(xd, y)
            else:
                m.moe_forward_partial(xd, part)
                if g > 1:
                    dist.all_reduce(part, group=pg)
                mx.round_bf16(part, y)
            yh.copy_(y, non_blocking=True)
        a1.record(stream)
        torch.cuda.synchronize()
        m.moe_status()
        el = max_over_ranks(a0.elapsed_time(a1) / 1e3, dist if world > 1 else None, "cuda")
        e2e = {"value": groups * T * n_e2e / el, "unit": "tokens/s", "steps": n_e2e,
               "h2d_bytes_per_step": T * w.hidden * 2, "d2h_bytes_per_step": T * w.hidden * 2,
               "api": "moe_forward_ishard on a device copy of pinned host tokens, output copied back"
                      if fused else "moe_forward_partial + all-reduce + moe_round_bf16, host copies each step"}
    if world > 1:
        dist.barrier()
    for b in opened:
        mx.moe_ishard_ipc_close(b)
    if rank == 0:
        how = ("one launch per step: moe_forward_ishard (engine + fused all-reduce over peer loads)" if fused else
               "stream launches: moe_forward_partial, NCCL all-reduce, moe_round_bf16")
        print(json.dumps({
            "metric": METRIC, "value": groups * T / (us_step * 1e-6), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us_step / 1e3, "higher_is_better": True,
            "scaling": "strong" if groups == 1 else "weak", "vs_baseline": None, "dtype": "mxfp4-w/fp32-acc",
            "data": "synthetic (seeded N(0,0.02) expert weights quantised to MXFP4, N(0,1) bf16 tokens)",
            "config": {"workload": w.name if not args.tokens else f"{w.name}_t{T}", "hidden": w.hidden,
                       "inter": w.inter, "inter_per_rank": w.inter // g, "experts": w.experts,
                       "top_k": w.top_k, "tokens": T, "ishard_group": g, "groups": groups,
                       "parallelism": f"I-sharded x{g}" + (f", {groups} groups on their own token blocks"
                                                            if groups > 1 else ""),
                       "allreduce": "fused (peer loads in the engine's last combine)" if fused else "NCCL",
                       "launch": how},
            "layer_us": us_step,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "algorithmic_bytes_per_launch": alg, "traffic": None, "kernel": "engine_kernel",
                         "per": "rank (its I-slice of the hit experts)"},
            "gpu_launches": (1 if fused else 3) * args.steps, "e2e": e2e, "cpu_baseline": None,
            "clocks": clk}), flush=True)
    m.close()
    if world > 1:
        dist.destroy_process_group()


def run_verify(args, w, rank, world):
    """The speculative-verify acceptance step: one spec_verify launch per step over
    the workload's verify blocks.  Enough distinct input sets are cycled that one
    pass over them exceeds the L2 (no flush needed)."""
    import torch
    import torch.distributed as dist
    from synth.spec import verify_inputs

    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            verify_reference(args, w)
        return
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import mxfp4_moe_expert_router_b200 as mx
    B, G, V = w.blocks, w.gamma, w.vocab
    step_bytes = B * (2 * G + 1) * V * 4
    nsets = max(2, min(16, -(-160 * 2 ** 20 // step_bytes)))
    host = [verify_inputs(w, seed=1000 * rank + i) for i in range(nsets)]
    dev = [{k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in h.items()} for h in host]
    sv = mx.SpecVerify(B, G, V)
    n_out = torch.empty((B,), dtype=torch.int32, device="cuda")
    t_out = torch.empty((B, G + 1), dtype=torch.int32, device="cuda")
    accepted = []
    for t in dev[:4]:
        n, _ = sv(t["lt"], t["ld"], t["d"], t["r"], t["u"])
        accepted.append(n.float().mean().item())
    sv.status()
    stream = torch.cuda.current_stream()
    ptrs = [[mx._ptr(t[k]) for k in ("lt", "ld", "d", "r", "u")] for t in dev]
    wsp, wsn = mx._ptr(sv.workspace), sv.workspace.numel()
    np_, tp_ = mx._ptr(n_out), mx._ptr(t_out)

    def launch(i, sp):
        st = mx.lib.spec_verify(*ptrs[i % nsets], B, G, V, np_, tp_, wsp, wsn, sp)
        if st != 0:
            raise mx.MoeError(st, "spec_verify")

    for i in range(args.warmup):
        launch(i, mx._stream(stream))
    sv.status()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid if rank == 0 else None)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    us = time_calls(mx, stream, args.steps, launch, not args.no_graph)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    sv.status()
    us = max_over_ranks(us, dist if world > 1 else None, "cuda")
    blocks_per_s = world * B / (us * 1e-6)
    peak, peak_kind = measured_peaks()
    achieved = step_bytes / (us * 1e-6) / 1e9

    e2e = None
    if not args.no_e2e:
        # host buffers: every step copies its pinned inputs in and n, tokens out
        hp = [{k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in h.items()} for h in host]
        nh = torch.empty((B,), dtype=torch.int32).pin_memory()
        th = torch.empty((B, G + 1), dtype=torch.int32).pin_memory()
        stage = {k: torch.empty_like(v) for k, v in dev[0].items()}
        n_e2e = max(1, min(args.steps, 200))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n_e2e):
            for k in stage:
                stage[k].copy_(hp[i % nsets][k], non_blocking=True)
            sv(stage["lt"], stage["ld"], stage["d"], stage["r"], stage["u"], n_out=n_out, tokens_out=t_out)
            nh.copy_(n_out, non_blocking=True)
            th.copy_(t_out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        sv.status()
        el = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, "cuda")
        e2e = {"value": world * B * n_e2e / el, "unit": "blocks/s", "steps": n_e2e,
               "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in hp[0].values()),
               "d2h_bytes_per_step": nh.numel() * 4 + th.numel() * 4,
               "api": "SpecVerify (spec_verify) on device copies of pinned host inputs"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import spec as ospec  # the CPU-baseline leg only
        t0 = time.perf_counter()
        nb = 0
        while time.perf_counter() - t0 < 5.0 and nb < 64:
            h = host[nb % nsets]
            bi = nb % B
            ospec.verify_block(h["lt"][bi], h["ld"][bi], h["d"][bi], h["r"][bi], float(h["u"][bi]))
            nb += 1
        el = time.perf_counter() - t0
        cpu = {"value": nb / el, "unit": "blocks/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"fp64 numpy oracle, {nb} verify blocks of this workload"}
    if rank == 0:
        out = {
            "metric": VERIFY_METRIC, "value": blocks_per_s, "unit": "blocks/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded logits: N(0, 2) plus one boosted token per row; draft = target "
                    "+ N(0, 0.25); draft tokens drawn from the draft by Gumbel-max)",
            "config": {"workload": w.name, "blocks_per_gpu": B, "gamma": G, "vocab": V,
                       "input_sets": nsets,
                       "l2": "no flush: %d input sets of %.0f MB cycled (> 126 MB L2)" % (nsets, step_bytes / 1e6),
                       "mean_accepted": float(np.mean(accepted)),
                       "launch": "stream launches" if args.no_graph else
                                 "the timed calls replayed as one CUDA graph"},
            "us_per_step": us,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "algorithmic_bytes_per_launch": step_bytes, "traffic": None,
                         "kernel": "spec_verify_kernel"},
            "gpu_launches": args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def verify_reference(args, w):
    """The fp64 oracle on this host's cores as the reference arm of the verify step."""
    from oracle import spec as ospec
    from synth.spec import verify_inputs
    B = min(w.blocks, 4)
    h = verify_inputs(w.with_blocks(B), seed=0)
    for i in range(args.warmup):
        ospec.verify_block(h["lt"][0], h["ld"][0], h["d"][0], h["r"][0], float(h["u"][0]))
    t0 = time.perf_counter()
    for i in range(args.steps):
        bi = i % B
        ospec.verify_block(h["lt"][bi], h["ld"][bi], h["d"][bi], h["r"][bi], float(h["u"][bi]))
    el = time.perf_counter() - t0
    v = args.steps / el
    print(json.dumps({"impl": "reference", "metric": VERIFY_METRIC, "value": v, "unit": "blocks/s",
                      "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
                      "config": {"workload": w.name, "blocks_per_gpu": w.blocks, "gamma": w.gamma,
                                 "vocab": w.vocab},
                      "cpu_baseline": {"value": v, "unit": "blocks/s", "cores": blas_threads(), "kind": "oracle",
                                       "sample": f"one verify block per step, {B} distinct blocks cycled"},
                      "e2e": {"value": v, "unit": "blocks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


if __name__ == "__main__":
    main()
