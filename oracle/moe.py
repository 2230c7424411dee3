"""fp64 MoE expert feed-forward: router, permutation, SwiGLU experts, combine, RMSNorm.

What it follows.  The pages describe the decode step only as design prose: MoE
routing is the runtime dynamism the engine must absorb (HyperAI salon
transcript on TileRT, section "Achieving maximum speed improvement through the
collaborative approach of algorithms, systems, and hardware"), routing stays
at original precision while the experts are MXFP4 (sandbot blog "1000 TPS
paradigm", section "三、技术拆解：怎么做到的？"), and small ops such as RMSNorm
sit on the critical path between layers (TileRT blog "Breaking 1000 TPS",
section "第二次跃迁").  They define neither the router nor the expert
function; this module takes the plainest MoE reading:

* router: logits = x Wr^T + b; p = softmax over all E experts; the k experts
  with the largest logits (ties: lower expert index first), in that order;
  weights w = p_sel / sum(p_sel);
* permutation: pairs p = t*k + slot grouped by expert; inside an expert's
  segment pairs are in ascending p; ``perm[pos] = p``, ``inv[p] = pos``;
* expert e on token row x: g = Wg x, u = Wu x, a = silu(g) * u, out = Wd a,
  silu(g) = g / (1 + exp(-g)); each pair's output is scaled by its weight;
* combine: y_t = sum over slots, in slot order, of the pair outputs;
* chain: layer i's bf16 output goes through RMSNorm (unit gamma, eps 1e-6,
  no residual) and is rounded to bf16 to become layer i+1's input.

No capacity limit, token dropping or shared expert: the pages never mention one.
All arithmetic is fp64 on exactly decoded MXFP4 weights and exactly widened
bf16 activations.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import mxfp4

RMS_EPS = 1e-6


@dataclass
class LayerWeights:
    """One MoE layer in the canonical MXFP4 layout.

    gate_codes/up_codes ``[E][I][H/2]``, gate_scales/up_scales ``[E][I][H/32]``,
    down_codes ``[E][H][I/2]``, down_scales ``[E][H][I/32]`` (uint8);
    router_w ``[E][H]`` fp32; router_b ``[E]`` fp32 or None.
    Entries of the per-expert lists may be None for experts never used.
    """
    gate_codes: list
    gate_scales: list
    up_codes: list
    up_scales: list
    down_codes: list
    down_scales: list
    router_w: np.ndarray
    router_b: np.ndarray | None

    @property
    def experts(self) -> int:
        return self.router_w.shape[0]

    def dense(self, e: int):
        """Exactly decoded (Wg, Wu, Wd) of expert e in fp64."""
        return (mxfp4.dequantize(self.gate_codes[e], self.gate_scales[e]),
                mxfp4.dequantize(self.up_codes[e], self.up_scales[e]),
                mxfp4.dequantize(self.down_codes[e], self.down_scales[e]))


def router_logits(x: np.ndarray, router_w: np.ndarray, router_b=None) -> np.ndarray:
    """fp64 logits ``[T][E]`` = x Wr^T (+ b)."""
    lg = np.asarray(x, np.float64) @ np.asarray(router_w, np.float64).T
    if router_b is not None:
        lg = lg + np.asarray(router_b, np.float64)[None, :]
    return lg


def softmax(v: np.ndarray) -> np.ndarray:
    m = v.max(axis=-1, keepdims=True)
    ex = np.exp(v - m)
    return ex / ex.sum(axis=-1, keepdims=True)


def route(x, router_w, router_b, top_k: int):
    """Top-k routing in fp64.

    Returns (idx ``[T][k]`` int32 in descending-logit order with ties to the lower
    expert, weights ``[T][k]`` fp64 renormalised over the k, logits ``[T][E]``).
    Selecting on logits equals selecting on softmax probabilities (softmax is
    monotone), so no probability is compared.
    """
    lg = router_logits(x, router_w, router_b)
    order = np.argsort(-lg, axis=-1, kind="stable")  # stable: equal logits keep ascending e
    idx = order[:, :top_k].astype(np.int32)
    p = softmax(lg)
    psel = np.take_along_axis(p, idx.astype(np.int64), axis=-1)
    return idx, psel / psel.sum(axis=-1, keepdims=True), lg


def logit_error_bound(x, router_w, router_b=None, unit_roundoff: float = 2.0 ** -53) -> np.ndarray:
    """Bound on |computed logit - exact logit| for any summation order.

    A length-H dot product accumulated with fused multiply-adds at unit
    roundoff u, plus one bias add, differs from the exact value by at most
    gamma_(H+1) times the sum of the absolute terms, gamma_n = n u / (1 - n u)
    (standard rounding-error analysis of recursive summation).  The default u
    is fp64's: products of a bf16 and an fp32 value are exact in fp64, and the
    sums are fp64, both in this oracle and in a router that accumulates in fp64.
    """
    xa = np.abs(np.asarray(x, np.float64))
    wa = np.abs(np.asarray(router_w, np.float64))
    s = xa @ wa.T
    if router_b is not None:
        s = s + np.abs(np.asarray(router_b, np.float64))[None, :]
    n = xa.shape[-1] + 1
    u = unit_roundoff
    return s * (n * u / (1 - n * u))


def unpinned_tokens(logits: np.ndarray, bound: np.ndarray, top_k: int) -> np.ndarray:
    """Tokens whose top-k set or order two correctly rounded evaluations may disagree on.

    Both this oracle's logits and the checked ones are within ``bound`` of the
    exact logits, so two experts among a token's first k+1 (in descending
    order) are undecided when their computed gap is at most twice the sum of
    their bounds.
    """
    order = np.argsort(-logits, axis=-1, kind="stable")[:, : top_k + 1]
    lg = np.take_along_axis(logits, order, axis=-1)
    bd = np.take_along_axis(bound, order, axis=-1)
    gap = lg[:, :-1] - lg[:, 1:]
    return np.nonzero((gap <= 2 * (bd[:, :-1] + bd[:, 1:])).any(axis=-1))[0]


def permute(idx: np.ndarray, num_experts: int):
    """Per-expert segments of the flat pairs p = t*k + slot.

    Returns (counts ``[E]``, offsets ``[E+1]``, perm ``[T*k]``, inv ``[T*k]``), int32.
    A stable sort by expert keeps each segment in ascending pair id.
    """
    flat = np.asarray(idx, np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    perm = np.argsort(flat, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return (counts.astype(np.int32), offsets.astype(np.int32), perm.astype(np.int32),
            inv.astype(np.int32))


def silu(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def expert_ffn(xr: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """SwiGLU expert on token rows ``[n][H]``: Wd (silu(Wg x) * (Wu x)) -> ``[n][H]``."""
    g = xr @ wg.T
    u = xr @ wu.T
    return (silu(g) * u) @ wd.T


def moe_layer(x: np.ndarray, lw: LayerWeights, top_k: int, idx=None):
    """One MoE layer in fp64.

    ``x`` ``[T][H]`` (exact values of the bf16 activations).  ``idx`` optionally
    overrides the routing (to evaluate the layer at another selection, e.g. the
    one an fp32 router took on a near tie); weights are then the renormalised
    fp64 probabilities of that selection.
    Returns a dict: y ``[T][H]``, idx, w, logits, counts, offsets, perm, inv,
    and pair_out ``[T*k][H]`` (weighted expert outputs in permuted order).
    """
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    r_idx, r_w, lg = route(x, lw.router_w, lw.router_b, top_k)
    if idx is not None:
        r_idx = np.asarray(idx, np.int32)
        p = softmax(lg)
        ps = np.take_along_axis(p, r_idx.astype(np.int64), axis=-1)
        r_w = ps / ps.sum(axis=-1, keepdims=True)
    counts, offsets, perm, inv = permute(r_idx, lw.experts)
    flat_w = r_w.reshape(-1)
    pair_out = np.zeros((T * top_k, x.shape[1]), dtype=np.float64)
    for e in np.nonzero(counts)[0]:
        seg = perm[offsets[e]:offsets[e + 1]]
        wg, wu, wd = lw.dense(int(e))
        out = expert_ffn(x[seg // top_k], wg, wu, wd)
        pair_out[offsets[e]:offsets[e + 1]] = out * flat_w[seg][:, None]
    y = combine(pair_out, inv, T, top_k)
    return dict(y=y, idx=r_idx, w=r_w, logits=lg, counts=counts, offsets=offsets,
                perm=perm, inv=inv, pair_out=pair_out)


def combine(pair_out: np.ndarray, inv: np.ndarray, T: int, top_k: int) -> np.ndarray:
    """y_t = sum over slots 0..k-1 (in order) of the weighted pair outputs."""
    y = np.zeros((T, pair_out.shape[1]), dtype=np.float64)
    for slot in range(top_k):
        y += pair_out[inv[np.arange(T) * top_k + slot]]
    return y


def rmsnorm(v: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """v / sqrt(mean(v^2) + eps) over the last axis; unit gamma."""
    v = np.asarray(v, np.float64)
    return v / np.sqrt((v * v).mean(axis=-1, keepdims=True) + eps)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), as float64.

    bf16 keeps 8 significant bits; below 2^-126 the spacing is fixed at 2^-133;
    values beyond the largest finite bf16 after rounding become infinite.
    """
    v = np.asarray(v, np.float64)
    _, p = np.frexp(v)
    q = np.ldexp(1.0, np.maximum(p.astype(np.int64) - 8, -133).astype(np.int32))
    r = np.rint(v / q) * q
    big = np.ldexp(1.0, 128) * (1 - 2.0 ** -9)  # rounding threshold above bf16 max
    return np.where(np.abs(r) >= big, np.copysign(np.inf, v), r)


def chain(x0: np.ndarray, layers, top_k: int):
    """Free-running stack: y_i = layer_i(x_i) rounded to bf16; x_{i+1} = bf16(rmsnorm(y_i)).

    Returns (xs, ys): the fp64 values of every layer input and bf16-rounded output.
    """
    xs, ys = [np.asarray(x0, np.float64)], []
    for i, lw in enumerate(layers):
        y = round_bf16(moe_layer(xs[-1], lw, top_k)["y"])
        ys.append(y)
        if i + 1 < len(layers):
            xs.append(round_bf16(rmsnorm(y)))
    return xs, ys
