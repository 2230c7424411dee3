"""Helpers for the GPU parity tests: upload oracle-side layers, run the C ABI, compare."""
from __future__ import annotations

import numpy as np

import synth
from oracle import moe, mxfp4
from tests.helpers import build_library, quantized_layer_np, tolerance_ok, x_values


def mx():
    build_library()
    import mxfp4_moe_expert_router_b200 as m
    return m


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits: np.ndarray):
    import torch
    return to_dev(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_host_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def layer_dev(lw: moe.LayerWeights):
    m = mx()
    st = lambda arrs: to_dev(np.stack(arrs))
    return m.LayerMX(st(lw.gate_codes), st(lw.gate_scales), st(lw.up_codes), st(lw.up_scales),
                     st(lw.down_codes), st(lw.down_scales), to_dev(lw.router_w.astype(np.float32)),
                     None if lw.router_b is None else to_dev(lw.router_b.astype(np.float32)))


def make_moe(w: synth.Workload, lws, max_tokens=None, rms_eps=1e-6):
    m = mx()
    return m.Moe(w.hidden, w.inter, w.experts, w.top_k, max_tokens or w.tokens,
                 [layer_dev(lw) for lw in lws], rms_eps=rms_eps)


def check_route(out, x, lw, k):
    """Compare moe_route outputs with the oracle; returns the number of unpinned tokens."""
    idx, w, lg = moe.route(x, lw.router_w, lw.router_b, k)
    bound = moe.logit_error_bound(x, lw.router_w, lw.router_b)
    loose = set(moe.unpinned_tokens(lg, bound, k).tolist())
    g_idx = out["topk_idx"].cpu().numpy()
    g_w = out["topk_w"].cpu().numpy()
    for t in range(x.shape[0]):
        if t not in loose:
            assert g_idx[t].tolist() == idx[t].tolist(), (t, g_idx[t], idx[t])
    # the rest is a function of the GPU's own selection
    E = lw.experts
    counts, offsets, perm, inv = moe.permute(g_idx, E)
    assert (out["counts"].cpu().numpy() == counts).all()
    assert (out["offsets"].cpu().numpy() == offsets).all()
    assert (out["perm"].cpu().numpy() == perm).all()
    assert (out["inv_perm"].cpu().numpy() == inv).all()
    p = moe.softmax(lg)
    ps = np.take_along_axis(p, g_idx.astype(np.int64), axis=-1)
    assert np.abs(g_w - ps / ps.sum(-1, keepdims=True)).max() <= 1e-5
    return len(loose)


def check_forward(y_dev, x, lw, k, idx_gpu=None):
    ref = moe.moe_layer(x, lw, k, idx=idx_gpu)["y"]
    got = x_values(bf16_host_bits(y_dev))
    ok, ratio = tolerance_ok(got, ref)
    assert ok, f"worst |err|/bound = {ratio:.3f}"
    return ratio


def check_verify(inp, n_gpu, tok_gpu):
    """spec_verify outputs against the oracle, block by block; returns the number of
    unpinned blocks (a decision or draw within the oracle's rounding bound)."""
    from oracle import spec
    lt, ld, d, r, u = inp["lt"], inp["ld"], inp["d"], inp["r"], inp["u"]
    B, G = d.shape
    V = lt.shape[2]
    loose = 0
    for b in range(B):
        res = spec.verify_block(lt[b], ld[b], d[b], r[b], float(u[b]))
        n = int(n_gpu[b])
        assert 0 <= n <= G
        assert (tok_gpu[b, :n] == d[b, :n]).all() and (tok_gpu[b, n + 1:] == -1).all()
        assert 0 <= tok_gpu[b, n] < V
        if any(spec.decision_unpinned(rr, pp, qq, V) for rr, pp, qq in res["tested"]):
            loose += 1
            continue
        assert n == res["n"], (b, n, res["n"])
        unp, cands = spec.sample_unpinned(res["weights"], float(u[b]), V, res["kind"])
        if unp:
            loose += 1
            assert int(tok_gpu[b, n]) in cands, (b, tok_gpu[b, n], cands)
        else:
            assert int(tok_gpu[b, n]) == res["tokens"][-1], (b, tok_gpu[b, n], res["tokens"][-1], res["kind"])
    return loose
