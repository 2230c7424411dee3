"""Parity at the full workload sizes, on sampled tokens.

The GPU runs whole layers at the bench and parity sizes.
- The oracle recomputes a few sampled tokens one by one.
- It quantises the same seeded bf16 expert weights itself (nothing it uses comes
  from the CUDA path), and checks that the GPU's codes and scales for those
  experts are bit-identical.
- It routes the sampled tokens in fp64 and evaluates their SwiGLU experts.
- It compares each token's y row within the tolerance (the rms term over the
  sampled rows).

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


class ExpertCache:
    """Oracle MXFP4 weights of one layer, quantised on demand and checked against the GPU's."""

    def __init__(self, w, layer, gpu_layer, pool):
        self.w, self.layer, self.g, self.pool, self.dense = w, layer, gpu_layer, pool, {}

    def need(self, experts):
        todo = [e for e in experts if e not in self.dense]
        jobs = [(e, kind) for e in todo for kind in ("gate", "up", "down")]
        bits = [_bits(synth.expert_torch(self.w, self.layer, e, kind, seed=0)) for e, kind in jobs]
        res = self.pool.map(_quantize_bits, bits)
        gpu = {"gate": (self.g.gate_codes, self.g.gate_scales), "up": (self.g.up_codes, self.g.up_scales),
               "down": (self.g.down_codes, self.g.down_scales)}
        mats = {}
        for (e, kind), (c, s) in zip(jobs, res):
            gc, gs = gpu[kind]
            assert (gc[e].cpu().numpy() == c).all(), f"codes of expert {e} {kind}"
            assert (gs[e].cpu().numpy() == s).all(), f"scales of expert {e} {kind}"
            mats[(e, kind)] = mxfp4.dequantize(c, s)
        for e in todo:
            self.dense[e] = (mats[(e, "gate")], mats[(e, "up")], mats[(e, "down")])

    def token_y(self, x_row, idx_row, w_row):
        y = np.zeros(self.w.hidden)
        for e, wt in zip(idx_row, w_row):  # slot order
            wg, wu, wd = self.dense[int(e)]
            y += wt * moe.expert_ffn(x_row[None, :], wg, wu, wd)[0]
        return y


def _route_and_check(x, router_w, router_b, k, gpu_idx, tokens):
    idx, w, lg = moe.route(x[tokens], router_w, router_b, k)
    bound = moe.logit_error_bound(x[tokens], router_w, router_b)
    loose = set(moe.unpinned_tokens(lg, bound, k).tolist())
    for j, t in enumerate(tokens):
        if j not in loose:
            assert gpu_idx[t].tolist() == idx[j].tolist(), (t, gpu_idx[t], idx[j])
        else:  # near tie: evaluate the layer at the GPU's own selection
            p = moe.softmax(lg[j])
            ps = p[gpu_idx[t]]
            idx[j], w[j] = gpu_idx[t], ps / ps.sum()
    return idx, w


def _run(mx, pool, w, T, tokens, layer_io=False):
    import torch
    import bench
    layers = [bench.build_layer(mx, w, l, seed=0) for l in range(w.layers)]
    m = mx.Moe(w.hidden, w.inter, w.experts, w.top_k, T, layers)
    x = synth.draw_torch(1000, 0, "x", -1, (T, w.hidden), 1.0)
    route = m.moe_route(x, layer=0)
    io = torch.empty((w.layers + 1, T, w.hidden), dtype=torch.bfloat16, device="cuda") if layer_io else None
    y = m.moe_forward(x, layer_io=io)
    m.moe_status()
    dense = [synth.layer_inputs_torch(w, l, 0, tokens=T) for l in range(w.layers)]
    return m, layers, x, route, y, io, dense


def _check_layer(pool, w, layer, gpu_layer, dense_l, x_bits, gpu_idx, got_rows, tokens, normalise):
    xv = mxfp4.bf16_to_f64(x_bits)
    rw = dense_l["router_w"].cpu().numpy().astype(np.float64)
    rb = None if dense_l["router_b"] is None else dense_l["router_b"].cpu().numpy().astype(np.float64)
    idx, wts = _route_and_check(xv, rw, rb, w.top_k, gpu_idx, tokens)
    cache = ExpertCache(w, layer, gpu_layer, pool)
    cache.need(sorted({int(e) for row in idx for e in row}))
    ref = np.stack([cache.token_y(xv[t], idx[j], wts[j]) for j, t in enumerate(tokens)])
    if normalise:
        ref = moe.round_bf16(moe.rmsnorm(ref))
    ok, ratio = tolerance_ok(got_rows, ref)
    assert ok, f"layer {layer}: worst |err|/bound = {ratio:.3f}"
    return ratio


def _gpu_rows(t, tokens):
    import torch
    return x_values(t[tokens].contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("name,tokens", [("decode_t9_h4096_e128", [0, 8]),
                                         ("batched_t144_h6144_e256", [5, 143])])
def test_single_layer_full_size(mx, pool, name, tokens):
    w = synth.WORKLOADS[name]
    m, layers, x, route, y, _, dense = _run(mx, pool, w, w.tokens, tokens)
    gpu_idx = route["topk_idx"].cpu().numpy()
    _check_layer(pool, w, 0, layers[0], dense[0], _bits(x), gpu_idx, _gpu_rows(y, tokens), tokens, False)
    m.close()


def test_chain_full_size_teacher_forced(mx, pool):
    """8-layer chain (Zipf-biased router): layers 0 and 7 on the GPU's own bf16 inputs."""
    w = synth.WORKLOADS["chain8_t9_h6144_e256_zipf"]
    tokens = [3]
    m, layers, x, route, y, io, dense = _run(mx, pool, w, w.tokens, tokens, layer_io=True)
    for l in (0, w.layers - 1):
        xl = io[l]
        r = m.moe_route(xl.contiguous(), layer=l)
        gpu_idx = r["topk_idx"].cpu().numpy()
        last = l == w.layers - 1
        out = io[l + 1]
        _check_layer(pool, w, l, layers[l], dense[l], _bits(xl), gpu_idx, _gpu_rows(out, tokens), tokens,
                     normalise=not last)
    m.close()


@pytest.mark.parametrize("T", [1, 72, 4608])
def test_sweep_full_size(mx, pool, T):
    """H = 7168, E = 256: T = 1 (decode), 72 and 4608 (the large-T routing path)."""
    w = synth.WORKLOADS["sweep_h7168_e256"].with_tokens(T)
    tokens = [0] if T == 1 else [1, T - 1]
    m, layers, x, route, y, _, dense = _run(mx, pool, w, T, tokens)
    gpu_idx = route["topk_idx"].cpu().numpy()
    _check_layer(pool, w, 0, layers[0], dense[0], _bits(x), gpu_idx, _gpu_rows(y, tokens), tokens, False)
    m.close()
