"""Shared test helpers: build MXFP4 layers from seeded draws through the oracle quantiser."""
from __future__ import annotations

import importlib.util
import os

import numpy as np

import synth
from oracle import moe, mxfp4


def quantized_layer_np(w: synth.Workload, layer: int = 0, seed: int = 0, tokens=None):
    """Host draw of one layer, quantised by the oracle.  Returns (x_bits or None, LayerWeights, raw)."""
    raw = synth.layer_inputs_np(w, layer=layer, seed=seed, tokens=tokens)
    q = {k: [mxfp4.quantize(a) for a in raw[k]] for k in ("gate", "up", "down")}
    lw = moe.LayerWeights(
        gate_codes=[c for c, _ in q["gate"]], gate_scales=[s for _, s in q["gate"]],
        up_codes=[c for c, _ in q["up"]], up_scales=[s for _, s in q["up"]],
        down_codes=[c for c, _ in q["down"]], down_scales=[s for _, s in q["down"]],
        router_w=raw["router_w"], router_b=raw["router_b"])
    return raw.get("x"), lw, raw


def x_values(bits: np.ndarray) -> np.ndarray:
    return mxfp4.bf16_to_f64(bits)


def tolerance_ok(got: np.ndarray, ref: np.ndarray, rel=8e-3, rms_frac=1e-3):
    """Elementwise |got-ref| <= rel*|ref| + rms_frac*rms(ref); returns (ok, worst ratio)."""
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = rel * np.abs(ref) + rms_frac * rms
    err = np.abs(got - ref)
    ratio = float((err / np.maximum(bound, 1e-300)).max()) if ref.size else 0.0
    return bool((err <= bound).all()), ratio


def build_library():
    """Compile libmoe_mxfp4.so if stale, without importing the binding package."""
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "mxfp4_moe_expert_router_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_moe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def shard_layer_np(lw, rank: int, world: int):
    """Rank `rank` of `world`'s I-slice of an oracle layer (gate/up rows, down columns,
    their block scales; the router replicated)."""
    from oracle import moe as omoe
    I = lw.gate_codes[0].shape[0]
    i0, i1 = rank * I // world, (rank + 1) * I // world
    rows = lambda a: [x[i0:i1].copy() for x in a]
    return omoe.LayerWeights(
        gate_codes=rows(lw.gate_codes), gate_scales=rows(lw.gate_scales),
        up_codes=rows(lw.up_codes), up_scales=rows(lw.up_scales),
        down_codes=[x[:, i0 // 2:i1 // 2].copy() for x in lw.down_codes],
        down_scales=[x[:, i0 // 32:i1 // 32].copy() for x in lw.down_scales],
        router_w=lw.router_w, router_b=lw.router_b)
