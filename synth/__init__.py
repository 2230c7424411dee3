"""Seeded synthetic inputs for the MXFP4 MoE expert feed-forward.

This module only draws random numbers and rounds them to the storage dtypes of
the workload (fp32 -> bf16, round-to-nearest-even).  It holds none of the
method's arithmetic: no quantisation, routing, projection or normalisation.
Both the CPU oracle (``oracle/``) and the CUDA path consume what it produces.

Recipe (one independent stream per tensor, so any expert can be regenerated on
its own):

* stream id = (seed, layer, kind, expert); kind is one of ``x``, ``router``,
  ``gate``, ``up``, ``down``.  The stream seed is the first 8 bytes of the
  SHA-256 of the id written as text.
* activations ``x``  ~ N(0, 1)    drawn fp32, rounded to bf16 (RNE);
* router weight ``Wr`` ~ N(0, 0.02) drawn fp32 and kept fp32, shape [E][H];
* expert weights ``Wg``, ``Wu`` [I][H] and ``Wd`` [H][I] ~ N(0, 0.02) drawn
  fp32, rounded to bf16; the caller quantises them to MXFP4;
* router bias: zero, except for the skewed-popularity chain workload, where
  ``b_e = -alpha * ln(e + 1)`` (a Zipf(alpha) log-prior, expert 0 the most
  popular), identical for every layer.

Host draws use numpy's PCG64; device draws (for the multi-GB workloads, whose
10^10 normals per layer are too slow on a host) use torch's CUDA Philox
generator.  The two give different numbers for the same id; every workload
states which one it uses, and the oracle always receives the very bytes the
CUDA path received.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "stream_seed", "bf16_bits_from_f32", "f32_from_bf16_bits",
    "draw_np", "layer_inputs_np", "router_bias", "draw_torch", "layer_inputs_torch",
]

EXPERT_SIGMA = 0.02
ROUTER_SIGMA = 0.02


@dataclass(frozen=True)
class Workload:
    """One synthetic MoE workload: layer shapes, token count and bias recipe."""
    name: str
    hidden: int
    inter: int
    experts: int
    top_k: int
    tokens: int
    layers: int = 1
    zipf_alpha: float | None = None
    device_draw: bool = True  # True: torch CUDA Philox; False: numpy PCG64
    tokens_sweep: tuple = field(default_factory=tuple)

    def with_tokens(self, t: int) -> "Workload":
        return Workload(self.name, self.hidden, self.inter, self.experts, self.top_k, t,
                        self.layers, self.zipf_alpha, self.device_draw, self.tokens_sweep)


# The five workloads: a tiny layer, the single-sequence decode verify step, a
# 16-sequence batched verify step, an 8-layer chain with skewed routing, and a
# token-count sweep into the compute-bound regime.
WORKLOADS = {
    "tiny_h256_e8": Workload("tiny_h256_e8", 256, 128, 8, 2, 9, device_draw=False),
    "decode_t9_h4096_e128": Workload("decode_t9_h4096_e128", 4096, 1536, 128, 8, 9),
    "batched_t144_h6144_e256": Workload("batched_t144_h6144_e256", 6144, 2048, 256, 8, 144),
    "chain8_t9_h6144_e256_zipf": Workload("chain8_t9_h6144_e256_zipf", 6144, 2048, 256, 8, 9,
                                          layers=8, zipf_alpha=1.2),
    "sweep_h7168_e256": Workload("sweep_h7168_e256", 7168, 2048, 256, 8, 4608,
                                 tokens_sweep=(1, 9, 72, 576, 4608)),
}


def stream_seed(seed: int, layer: int, kind: str, expert: int = -1) -> int:
    """63-bit seed of the stream named (seed, layer, kind, expert)."""
    tag = f"mxfp4-moe/{seed}/{layer}/{kind}/{expert}".encode()
    return int.from_bytes(hashlib.sha256(tag).digest()[:8], "little") & ((1 << 63) - 1)


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_np(seed: int, layer: int, kind: str, expert: int, shape, sigma: float) -> np.ndarray:
    """fp32 N(0, sigma) draw from the host stream (PCG64) of the given id."""
    rng = np.random.Generator(np.random.PCG64(stream_seed(seed, layer, kind, expert)))
    return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(sigma)


def router_bias(w: Workload) -> np.ndarray | None:
    """Router bias b_e = -alpha*ln(e+1) for skewed workloads, else None (no bias)."""
    if w.zipf_alpha is None:
        return None
    e = np.arange(w.experts, dtype=np.float64)
    return (-w.zipf_alpha * np.log(e + 1.0)).astype(np.float32)


def layer_inputs_np(w: Workload, layer: int = 0, seed: int = 0, tokens: int | None = None,
                    experts=None) -> dict:
    """Host draw of one layer's inputs.

    Returns a dict with ``x`` (uint16 bf16 bits [T][H], layer 0 only), ``router_w``
    (fp32 [E][H]), ``router_b`` (fp32 [E] or None) and ``gate``/``up``/``down``:
    lists over experts of uint16 bf16 bits ([I][H], [I][H], [H][I]).  ``experts``
    restricts which experts are drawn (others are None).
    """
    T = w.tokens if tokens is None else tokens
    out = {"router_w": draw_np(seed, layer, "router", -1, (w.experts, w.hidden), ROUTER_SIGMA),
           "router_b": router_bias(w)}
    if layer == 0:
        out["x"] = bf16_bits_from_f32(draw_np(seed, 0, "x", -1, (T, w.hidden), 1.0))
    sel = range(w.experts) if experts is None else set(int(e) for e in experts)
    for kind, shp in (("gate", (w.inter, w.hidden)), ("up", (w.inter, w.hidden)),
                      ("down", (w.hidden, w.inter))):
        out[kind] = [bf16_bits_from_f32(draw_np(seed, layer, kind, e, shp, EXPERT_SIGMA))
                     if e in sel else None for e in range(w.experts)]
    return out


# ---- device draws (torch CUDA Philox) for the multi-GB workloads -------------

def draw_torch(seed: int, layer: int, kind: str, expert: int, shape, sigma: float,
               device="cuda", dtype=None):
    """N(0, sigma) draw on ``device`` from torch's generator seeded by the stream id.

    Drawn in fp32 and rounded to ``dtype`` (bf16 by default, RNE); fp32 when
    ``dtype`` is ``torch.float32``.
    """
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, layer, kind, expert))
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    t.mul_(sigma)
    return t.to(torch.bfloat16 if dtype is None else dtype)


def layer_inputs_torch(w: Workload, layer: int = 0, seed: int = 0, tokens: int | None = None,
                       device="cuda"):
    """Device draw of one layer's dense inputs; expert weights come from ``expert_torch``.

    ``x`` is drawn as the full [w.tokens][H] block and sliced to its first
    ``tokens`` rows, so every token count of a sweep sees a prefix of one draw.
    """
    import torch
    T = w.tokens if tokens is None else tokens
    out = {"router_w": draw_torch(seed, layer, "router", -1, (w.experts, w.hidden), ROUTER_SIGMA,
                                  device, torch.float32)}
    b = router_bias(w)
    out["router_b"] = None if b is None else torch.from_numpy(b).to(device)
    if layer == 0:
        full = draw_torch(seed, 0, "x", -1, (max(T, w.tokens), w.hidden), 1.0, device)
        out["x"] = full[:T].contiguous()
    return out


def expert_torch(w: Workload, layer: int, expert: int, kind: str, seed: int = 0, device="cuda"):
    """bf16 device draw of one expert projection: gate/up [I][H], down [H][I]."""
    shp = (w.inter, w.hidden) if kind in ("gate", "up") else (w.hidden, w.inter)
    return draw_torch(seed, layer, kind, expert, shp, EXPERT_SIGMA, device)
