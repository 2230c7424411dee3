"""Parity at the full workload sizes.

The GPU runs whole layers at the bench and parity sizes, then:
- the routing of EVERY token is compared with the oracle's fp64 routing
  (indices bit-exact except near ties, which are counted and must stay rare;
  counts, offsets, perm and inv bit-exact; weights within 1e-5);
- the output rows of sampled tokens are recomputed by the oracle one by one.
  The oracle quantises the same seeded bf16 expert weights itself (nothing it
  uses comes from the CUDA path), checks that the GPU's codes and scales of
  those experts are bit-identical, and evaluates the sampled tokens' SwiGLU
  experts expert by expert (a few experts in memory at a time).  Each row is
  compared within the tolerance, the rms term over the sampled rows.
Sampling: every token of the verify-block workloads (T = 9, every layer of
the chain teacher-forced), and 16 tokens spread over the block for T >= 72,
which puts sampled pairs in interior tiles and in both epilogue sets of the
tile stream (checked).

The oracle's quantiser runs in a spawn process pool.
"""
import multiprocessing as mproc
import os

import numpy as np
import pytest

import synth
from oracle import moe, mxfp4
from tests.helpers import tolerance_ok, x_values

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

LT_MAX = 38  # positions per tile of the tile stream (engine.cuh)


def _quantize_bits(bits):
    from oracle import mxfp4 as q
    return q.quantize(bits)


@pytest.fixture(scope="module")
def pool():
    ctx = mproc.get_context("spawn")
    p = ctx.Pool(processes=max(2, min(16, (os.cpu_count() or 4))))
    yield p
    p.terminate()
    p.join()


@pytest.fixture(scope="module")
def mx():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mxfp4_moe_expert_router_b200 as m
    return m


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sample_tokens(T: int, n: int = 16) -> list:
    """Every token up to n, else n tokens spread evenly over [0, T) (first and last included)."""
    if T <= n:
        return list(range(T))
    return sorted({int(v) for v in np.linspace(0, T - 1, n)})


def oracle_rows(pool, w, layer, gpu_layer, xv, tokens, idx, wts, chunk=8):
    """fp64 layer output rows of the sampled tokens (their routing idx/wts given).

    Expert by expert, `chunk` experts at a time: the oracle quantises the
    seeded bf16 weights, checks the GPU's codes and scales bit for bit,
    dequantises, and adds each routed pair's weighted SwiGLU output; the k
    contributions of a row are summed in slot order."""
    users = {}
    for j in range(len(tokens)):
        for slot, e in enumerate(idx[j]):
            users.setdefault(int(e), []).append((j, slot))
    contrib = np.zeros((len(tokens), w.top_k, w.hidden))
    gpu = {"gate": (gpu_layer.gate_codes, gpu_layer.gate_scales), "up": (gpu_layer.up_codes, gpu_layer.up_scales),
           "down": (gpu_layer.down_codes, gpu_layer.down_scales)}
    experts = sorted(users)
    for c0 in range(0, len(experts), chunk):
        part = experts[c0:c0 + chunk]
        jobs = [(e, kind) for e in part for kind in ("gate", "up", "down")]
        bits = [_bits(synth.expert_torch(w, layer, e, kind, seed=0)) for e, kind in jobs]
        res = pool.map(_quantize_bits, bits)
        mats = {}
        for (e, kind), (c, s) in zip(jobs, res):
            gc, gs = gpu[kind]
            assert (gc[e].cpu().numpy() == c).all(), f"codes of expert {e} {kind}"
            assert (gs[e].cpu().numpy() == s).all(), f"scales of expert {e} {kind}"
            mats[(e, kind)] = mxfp4.dequantize(c, s)
        for e in part:
            rows = users[e]
            xr = np.stack([xv[tokens[j]] for j, _ in rows])
            out = moe.expert_ffn(xr, mats[(e, "gate")], mats[(e, "up")], mats[(e, "down")])
            for (j, slot), o in zip(rows, out):
                contrib[j, slot] = wts[j][slot] * o
        del mats
    y = np.zeros((len(tokens), w.hidden))
    for slot in range(w.top_k):  # slot order
        y += contrib[:, slot]
    return y


def _route_all(route, xv, rw, rb, k, T):
    """Every token's routing against the oracle; returns (oracle idx, oracle-side weights of
    the GPU's selection, unpinned count).  Near ties are counted and evaluated at the GPU's
    own selection; everything else is bit-exact."""
    idx, w, lg = moe.route(xv, rw, rb, k)
    bound = moe.logit_error_bound(xv, rw, rb)
    loose = set(moe.unpinned_tokens(lg, bound, k).tolist())
    g_idx = route["topk_idx"].cpu().numpy()
    for t in range(T):
        if t not in loose:
            assert g_idx[t].tolist() == idx[t].tolist(), (t, g_idx[t], idx[t])
    counts, offsets, perm, inv = moe.permute(g_idx, rw.shape[0])
    assert (route["counts"].cpu().numpy() == counts).all()
    assert (route["offsets"].cpu().numpy() == offsets).all()
    assert (route["perm"].cpu().numpy() == perm).all()
    assert (route["inv_perm"].cpu().numpy() == inv).all()
    p = moe.softmax(lg)
    ps = np.take_along_axis(p, g_idx.astype(np.int64), axis=-1)
    ws = ps / ps.sum(-1, keepdims=True)
    assert np.abs(route["topk_w"].cpu().numpy() - ws).max() <= 1e-5
    # rare: a near tie needs a logit gap below ~1e-13 relative
    assert len(loose) <= max(1, T // 500), f"{len(loose)} unpinned tokens of {T}"
    return g_idx, ws, len(loose)


def _tile_coverage(route, tokens, k, E):
    """(tile index within the expert's segment, epilogue set) of every sampled pair."""
    inv = route["inv_perm"].cpu().numpy()
    offsets = route["offsets"].cpu().numpy()
    idx = route["topk_idx"].cpu().numpy()
    cov = set()
    for t in tokens:
        for slot in range(k):
            e = int(idx[t, slot])
            p = int(inv[t * k + slot]) - int(offsets[e])
            cov.add((p // LT_MAX, (p % LT_MAX) % 2))
    return cov


def _run(mx, w, T, layer_io=False):
    import torch
    import bench
    layers = [bench.build_layer(mx, w, l, seed=0) for l in range(w.layers)]
    m = mx.Moe(w.hidden, w.inter, w.experts, w.top_k, T, layers)
    x = synth.draw_torch(1000, 0, "x", -1, (T, w.hidden), 1.0)
    io = torch.empty((w.layers + 1, T, w.hidden), dtype=torch.bfloat16, device="cuda") if layer_io else None
    y = m.moe_forward(x, layer_io=io)
    m.moe_status()
    dense = [synth.layer_inputs_torch(w, l, 0, tokens=T) for l in range(w.layers)]
    return m, layers, x, y, io, dense


def _check_layer(m, pool, w, layer, gpu_layer, dense_l, x_dev, out_dev, tokens, normalise):
    """Route every token of x_dev on the GPU and in the oracle, then the sampled rows of out_dev."""
    import torch
    T = x_dev.shape[0]
    route = m.moe_route(x_dev.contiguous(), layer=layer)
    m.moe_status()
    xv = mxfp4.bf16_to_f64(_bits(x_dev))
    rw = dense_l["router_w"].cpu().numpy().astype(np.float64)
    rb = None if dense_l["router_b"] is None else dense_l["router_b"].cpu().numpy().astype(np.float64)
    g_idx, ws, loose = _route_all(route, xv, rw, rb, w.top_k, T)
    ref = oracle_rows(pool, w, layer, gpu_layer, xv, tokens, g_idx[tokens], ws[tokens])
    if normalise:
        ref = moe.round_bf16(moe.rmsnorm(ref))
    got = x_values(out_dev[tokens].contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    ok, ratio = tolerance_ok(got, ref)
    assert ok, f"layer {layer}: worst |err|/bound = {ratio:.3f}"
    return route, ratio, loose


@pytest.mark.parametrize("name", ["decode_t9_h4096_e128", "batched_t144_h6144_e256"])
def test_single_layer_full_size(mx, pool, name):
    w = synth.WORKLOADS[name]
    m, layers, x, y, _, dense = _run(mx, w, w.tokens)
    tokens = sample_tokens(w.tokens)
    _check_layer(m, pool, w, 0, layers[0], dense[0], x, y, tokens, False)
    m.close()


def test_chain_full_size_teacher_forced(mx, pool):
    """8-layer chain (Zipf-biased router): every layer, every token, on the GPU's own bf16 inputs."""
    w = synth.WORKLOADS["chain8_t9_h6144_e256_zipf"]
    m, layers, x, y, io, dense = _run(mx, w, w.tokens, layer_io=True)
    assert (io[w.layers] == y).all()
    tokens = sample_tokens(w.tokens)
    for l in range(w.layers):
        last = l == w.layers - 1
        _check_layer(m, pool, w, l, layers[l], dense[l], io[l], io[l + 1], tokens, normalise=not last)
    m.close()


@pytest.mark.parametrize("T", [1, 9, 72, 576, 4608])
def test_sweep_full_size(mx, pool, T):
    """H = 7168, E = 256 over the token sweep: decode (1, 9), the pipeline stream with
    grid-wide routing (72), the tile stream (576, 4608)."""
    w = synth.WORKLOADS["sweep_h7168_e256"].with_tokens(T)
    m, layers, x, y, _, dense = _run(mx, w, T)
    tokens = sample_tokens(T)
    route, _, _ = _check_layer(m, pool, w, 0, layers[0], dense[0], x, y, tokens, False)
    if T * w.top_k >= 8 * w.experts:  # tile stream: both epilogue sets, interior tiles at 4608
        cov = _tile_coverage(route, tokens, w.top_k, w.experts)
        assert {s for _, s in cov} == {0, 1}, cov
        if T >= 4608:
            assert max(t for t, _ in cov) >= 2, cov
    m.close()
