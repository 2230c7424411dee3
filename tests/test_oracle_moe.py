"""Pins for the oracle's router, permutation, SwiGLU experts, combine and RMSNorm (CPU only).

Expected values come from closed forms, pure-Python brute force written
independently of ``oracle.moe``, and exact invariants.
"""
import math

import numpy as np
import pytest

import synth
from oracle import moe, mxfp4
from tests.helpers import quantized_layer_np, x_values

TINY = synth.Workload("t", hidden=64, inter=32, experts=6, top_k=2, tokens=5, device_draw=False)


def _layer(w=TINY, seed=0):
    xb, lw, _ = quantized_layer_np(w, seed=seed)
    return x_values(xb), lw


def test_route_weights_sum_to_one():
    x, lw = _layer()
    idx, w, _ = moe.route(x, lw.router_w, lw.router_b, 2)
    assert np.allclose(w.sum(-1), 1.0, atol=1e-15, rtol=0)
    assert (w > 0).all()


def test_topk_is_prefix_of_full_stable_sort():
    x, lw = _layer(synth.Workload("t", 96, 32, 16, 5, 11, device_draw=False))
    idx, _, lg = moe.route(x, lw.router_w, lw.router_b, 5)
    for t in range(x.shape[0]):
        want = [e for _, e in sorted((-float(lg[t, e]), e) for e in range(16))][:5]
        assert idx[t].tolist() == want


def test_route_invariant_to_logit_shift():
    x, lw = _layer()
    idx0, w0, _ = moe.route(x, lw.router_w, None, 2)
    idx1, w1, _ = moe.route(x, lw.router_w, np.full(lw.experts, 3.25), 2)
    assert (idx0 == idx1).all()
    assert np.allclose(w0, w1, rtol=0, atol=1e-14)


def test_zero_input_routes_by_bias_alone():
    b = synth.router_bias(synth.Workload("z", 32, 32, 10, 3, 2, zipf_alpha=1.2))
    x = np.zeros((2, 32))
    idx, w, lg = moe.route(x, np.ones((10, 32), np.float32), b, 3)
    assert (lg == b.astype(np.float64)).all()
    assert idx.tolist() == [[0, 1, 2]] * 2
    ex = [math.exp(float(b[e])) for e in range(3)]
    assert np.allclose(w[0], [v / sum(ex) for v in ex], rtol=0, atol=1e-15)


def test_constant_logits_tie_break_lower_expert():
    idx, w, _ = moe.route(np.ones((3, 8)), np.zeros((7, 8), np.float32), None, 4)
    assert idx.tolist() == [[0, 1, 2, 3]] * 3
    assert np.allclose(w, 0.25, rtol=0, atol=1e-16)


def test_permutation_against_dict_rebuild():
    rng = np.random.default_rng(3)
    T, k, E = 13, 3, 7
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = moe.permute(idx, E)
    seg = {e: [] for e in range(E)}
    for p in range(T * k):  # ascending pair id
        seg[int(idx[p // k, p % k])].append(p)
    flat = [p for e in range(E) for p in seg[e]]
    assert perm.tolist() == flat
    assert counts.tolist() == [len(seg[e]) for e in range(E)]
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert (inv[perm] == np.arange(T * k)).all()
    for e in range(E):
        s = perm[offsets[e]:offsets[e + 1]]
        assert (np.diff(s) > 0).all()


def _constant_layer(E, H, I, cg, cu, cd, sg, su, sd):
    def mk(c, s, rows, K):
        return np.full((rows, K // 2), c | (c << 4), np.uint8), np.full((rows, K // 32), s, np.uint8)
    g = [mk(cg, sg, I, H) for _ in range(E)]
    u = [mk(cu, su, I, H) for _ in range(E)]
    d = [mk(cd, sd, H, I) for _ in range(E)]
    rng = np.random.default_rng(5)
    return moe.LayerWeights([a for a, _ in g], [b for _, b in g], [a for a, _ in u],
                            [b for _, b in u], [a for a, _ in d], [b for _, b in d],
                            rng.standard_normal((E, H)).astype(np.float32), None)


@pytest.mark.parametrize("codes", [(3, 13, 5), (7, 2, 9), (1, 1, 1)])
def test_constant_code_experts_closed_form(codes):
    """All codes of Wg/Wu/Wd equal: y_h = dv * I * silu(gv*S) * uv * S with S = sum_h x_h."""
    E, H, I = 5, 64, 32
    cg, cu, cd = codes
    sg, su, sd = 120, 121, 125
    lw = _constant_layer(E, H, I, cg, cu, cd, sg, su, sd)
    table = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}
    val = lambda c, s: (-1 if c & 8 else 1) * table[c & 7] * 2.0 ** (s - 127)
    gv, uv, dv = val(cg, sg), val(cu, su), val(cd, sd)
    x = np.random.default_rng(6).standard_normal((4, H))
    y = moe.moe_layer(x, lw, 2)["y"]
    for t in range(4):
        S = math.fsum(x[t])
        g = gv * S
        want = dv * I * (g / (1 + math.exp(-g))) * uv * S
        assert np.allclose(y[t], want, rtol=1e-12, atol=1e-300)


def _decode_loop(codes, scales, rows, K):
    """Dequantise with plain integer bit logic, one element at a time."""
    out = [[0.0] * K for _ in range(rows)]
    for r in range(rows):
        for k in range(K):
            byte = int(codes[r][k // 2])
            c = byte & 15 if k % 2 == 0 else byte >> 4
            e, m = (c >> 1) & 3, c & 1
            mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1 + m / 2)
            out[r][k] = (-mag if c & 8 else mag) * 2.0 ** (int(scales[r][k // 32]) - 127)
    return out


def test_brute_force_scalar_moe():
    """T=2, H=I=32, E=4, k=2 entirely in Python scalar loops."""
    w = synth.Workload("bf", 32, 32, 4, 2, 2, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=7)
    x = x_values(xb)
    H = I = 32
    ref = moe.moe_layer(x, lw, 2)
    for t in range(2):
        lg = [math.fsum(x[t][h] * float(lw.router_w[e][h]) for h in range(H)) for e in range(4)]
        sel = sorted(range(4), key=lambda e: (-lg[e], e))[:2]
        m = max(lg)
        ps = [math.exp(lg[e] - m) for e in sel]
        wts = [p / sum(ps) for p in ps]
        y = [0.0] * H
        for e, wt in zip(sel, wts):
            wg = _decode_loop(lw.gate_codes[e], lw.gate_scales[e], I, H)
            wu = _decode_loop(lw.up_codes[e], lw.up_scales[e], I, H)
            wd = _decode_loop(lw.down_codes[e], lw.down_scales[e], H, I)
            a = []
            for i in range(I):
                g = math.fsum(wg[i][h] * x[t][h] for h in range(H))
                u = math.fsum(wu[i][h] * x[t][h] for h in range(H))
                a.append(g / (1 + math.exp(-g)) * u)
            for h in range(H):
                y[h] += wt * math.fsum(wd[h][i] * a[i] for i in range(I))
        assert ref["idx"][t].tolist() == sel
        assert np.allclose(ref["y"][t], y, rtol=1e-11, atol=1e-14)


def test_single_expert_is_dense_swiglu():
    w = synth.Workload("d", 64, 32, 1, 1, 3, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=8)
    x = x_values(xb)
    wg, wu, wd = (mxfp4.dequantize(lw.gate_codes[0], lw.gate_scales[0]),
                  mxfp4.dequantize(lw.up_codes[0], lw.up_scales[0]),
                  mxfp4.dequantize(lw.down_codes[0], lw.down_scales[0]))
    out = moe.moe_layer(x, lw, 1)
    assert (out["w"] == 1.0).all()
    for t in range(3):
        g = [sum(wg[i, h] * x[t, h] for h in range(64)) for i in range(32)]
        u = [sum(wu[i, h] * x[t, h] for h in range(64)) for i in range(32)]
        a = [gi / (1 + math.exp(-gi)) * ui for gi, ui in zip(g, u)]
        y = [sum(wd[h, i] * a[i] for i in range(32)) for h in range(64)]
        assert np.allclose(out["y"][t], y, rtol=1e-11, atol=1e-15)


def test_zero_input_zero_output():
    _, lw = _layer()
    y = moe.moe_layer(np.zeros((4, TINY.hidden)), lw, 2)["y"]
    assert (y == 0).all()


def test_token_permutation_equivariance():
    x, lw = _layer()
    p = np.array([3, 0, 4, 1, 2])
    y = moe.moe_layer(x, lw, 2)["y"]
    yp = moe.moe_layer(x[p], lw, 2)["y"]
    assert (yp == y[p]).all()


def test_down_scale_increment_doubles_output():
    x, lw = _layer()
    y = moe.moe_layer(x, lw, 2)["y"]
    lw2 = moe.LayerWeights(lw.gate_codes, lw.gate_scales, lw.up_codes, lw.up_scales,
                           lw.down_codes, [s + 1 for s in lw.down_scales], lw.router_w, lw.router_b)
    assert (moe.moe_layer(x, lw2, 2)["y"] == 2 * y).all()


def test_rmsnorm_unit_mean_square():
    v = np.random.default_rng(9).standard_normal((5, 6144)) * 37.0
    r = moe.rmsnorm(v, eps=0.0)
    assert np.allclose((r * r).mean(-1), 1.0, rtol=0, atol=4e-16)
    assert np.allclose(moe.rmsnorm(v) * np.sqrt((v * v).mean(-1, keepdims=True) + 1e-6), v,
                       rtol=1e-15, atol=0)


def test_round_bf16_matches_integer_rne():
    rng = np.random.default_rng(10)
    f = (rng.standard_normal(200000) * np.exp(rng.uniform(-80, 80, 200000))).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    rb = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint32) << 16
    want = rb.astype(np.uint32).view(np.float32).astype(np.float64)
    assert (moe.round_bf16(f.astype(np.float64)) == want).all()
    assert moe.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0  # tie to even
    assert moe.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6


def test_logit_bound_covers_fp32_dot_products():
    x, lw = _layer(synth.Workload("b", 4096, 32, 8, 2, 4, device_draw=False))
    exact = moe.router_logits(x, lw.router_w)
    bound = moe.logit_error_bound(x, lw.router_w, unit_roundoff=2.0 ** -24)
    xf = x.astype(np.float32)
    for t in range(4):
        for e in range(8):
            acc = np.float32(0)
            for h in range(0, 4096, 7):  # a sequential fp32 order over a subset
                acc = np.float32(acc + xf[t, h] * lw.router_w[e, h])
            sub = math.fsum(float(xf[t, h]) * float(lw.router_w[e, h]) for h in range(0, 4096, 7))
            assert abs(float(acc) - sub) <= bound[t, e]
    assert (bound > 0).all() and (bound < 2e-2).all()
    b64 = moe.logit_error_bound(x, lw.router_w)
    assert (b64 < 1e-10).all()
    # fp64 accumulation of exact bf16*fp32 products stays within the fp64 bound
    for t in range(2):
        for e in range(3):
            acc = 0.0
            for h in range(4096):
                acc += float(xf[t, h]) * float(lw.router_w[e, h])
            assert abs(acc - math.fsum(float(xf[t, h]) * float(lw.router_w[e, h])
                                       for h in range(4096))) <= b64[t, e]


def test_chain_rmsnorm_inputs():
    w = synth.Workload("c", 64, 32, 6, 2, 3, layers=2, device_draw=False)
    xb, lw0, _ = quantized_layer_np(w, layer=0)
    _, lw1, _ = quantized_layer_np(w, layer=1)
    xs, ys = moe.chain(x_values(xb), [lw0, lw1], 2)
    assert len(xs) == 2 and len(ys) == 2
    assert (moe.round_bf16(xs[1]) == xs[1]).all()
    m = (ys[0] ** 2).mean(-1)
    ms = (moe.rmsnorm(ys[0]) ** 2).mean(-1)
    assert np.allclose(ms, m / (m + moe.RMS_EPS), rtol=1e-14, atol=0)  # closed form with eps
    assert np.allclose((xs[1] ** 2).mean(-1), ms, rtol=2 ** -7, atol=0)  # after bf16 rounding


@pytest.mark.parametrize("world", [2, 4])
def test_i_sharded_partials_sum_to_the_layer(world):
    """SwiGLU acts per intermediate row, so splitting I across ranks (gate/up rows, down
    columns) and summing the ranks' outputs gives the layer.  The routing depends only on
    the router and is the same on every rank."""
    from tests.helpers import quantized_layer_np, shard_layer_np, x_values
    w = synth.Workload("shard", 256, 512, 8, 2, 9, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=31)
    x = x_values(xb)
    full = moe.moe_layer(x, lw, w.top_k)
    parts = [moe.moe_layer(x, shard_layer_np(lw, r, world), w.top_k) for r in range(world)]
    for part in parts:
        assert (part["idx"] == full["idx"]).all() and (part["perm"] == full["perm"]).all()
    total = sum(part["y"] for part in parts)
    assert np.allclose(total, full["y"], rtol=1e-12, atol=1e-12 * np.abs(full["y"]).max())
    # a single rank is not the layer: every slice carries a share
    assert not np.allclose(parts[0]["y"], full["y"], rtol=1e-3)
