"""The operator-by-operator path (moe_forward_ops) against the engine and the oracle.

moe_forward_ops runs the engine's phases as six launches per layer. The
arithmetic of every phase is the same and so is its order. Its outputs must
equal the single launch's bit for bit, and they must pass the oracle's
tolerance on their own. This holds with and without programmatic dependent
launch, in a CUDA graph, and over a chain of layers.
"""
import numpy as np
import pytest

import synth
from oracle import moe
from tests.helpers import quantized_layer_np, x_values

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": (256, 128, 8, 2, 9),
    "ragged_small": (512, 256, 16, 4, 37),
    "one_token": (256, 128, 8, 2, 1),
    "all_experts": (256, 128, 4, 4, 9),
    "top1": (256, 256, 8, 1, 17),
    "many_tokens_one_expert": (256, 128, 2, 1, 40),
}


@pytest.fixture(scope="module")
def m():
    from tests.gpu_helpers import mx
    return mx()


def _workload(name, layers=1, zipf=None):
    H, I, E, k, T = SHAPES[name]
    return synth.Workload(name, H, I, E, k, T, layers=layers, zipf_alpha=zipf, device_draw=False)


@pytest.mark.parametrize("pdl", [False, True])
@pytest.mark.parametrize("name", list(SHAPES))
def test_ops_match_engine_and_oracle(m, name, pdl):
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, check_forward, make_moe
    w = _workload(name)
    xb, lw, _ = quantized_layer_np(w, seed=41)
    mo = make_moe(w, [lw])
    x = bf16_dev(xb)
    y_engine = bf16_host_bits(mo.moe_forward(x))
    y = mo.moe_forward_ops(x, pdl=pdl)
    mo.moe_status()
    assert (bf16_host_bits(y) == y_engine).all()
    check_forward(y, x_values(xb), lw, w.top_k)


@pytest.mark.parametrize("pdl", [False, True])
def test_ops_chain_matches_engine(m, pdl):
    """Three layers with RMSNorm between them: every layer's bf16 input and the
    output equal the single launch's; the last layer passes the oracle on the
    GPU's own input."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    from tests.helpers import tolerance_ok
    w = synth.Workload("chain", 512, 256, 16, 4, 9, layers=3, zipf_alpha=1.2, device_draw=False)
    lws = [quantized_layer_np(w, layer=l, seed=43)[1] for l in range(3)]
    xb = quantized_layer_np(w, layer=0, seed=43)[0]
    mo = make_moe(w, lws)
    x = bf16_dev(xb)
    io_e = torch.empty((4, w.tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    io_o = torch.empty_like(io_e)
    y_e = mo.moe_forward(x, layer_io=io_e)
    y_o = mo.moe_forward_ops(x, layer_io=io_o, pdl=pdl)
    mo.moe_status()
    assert (bf16_host_bits(io_o) == bf16_host_bits(io_e)).all()
    assert (bf16_host_bits(y_o) == bf16_host_bits(y_e)).all()
    io_h = x_values(bf16_host_bits(io_o))
    ok, ratio = tolerance_ok(io_h[3], moe.moe_layer(io_h[2], lws[2], w.top_k)["y"])
    assert ok, ratio


def test_ops_with_pdl_in_cuda_graph(m):
    """Two calls captured with programmatic dependent launches, replayed."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_small")
    xa, lw, _ = quantized_layer_np(w, seed=45)
    xb = quantized_layer_np(w, seed=46)[0]
    mo = make_moe(w, [lw])
    xs = [bf16_dev(xa), bf16_dev(xb)]
    ref = [bf16_host_bits(mo.moe_forward(x)) for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for x, y in zip(xs, ys):
            mo.moe_forward_ops(x, y, pdl=True)
    for y in ys:
        y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    mo.moe_status()
    for y, r in zip(ys, ref):
        assert (bf16_host_bits(y) == r).all()


def test_ops_refuse_large_t_and_bad_flags(m):
    import torch
    from tests.gpu_helpers import bf16_dev, make_moe
    w = synth.Workload("large", 384, 256, 16, 4, 80, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=47)
    mo = make_moe(w, [lw])
    x = bf16_dev(xb)
    with pytest.raises(m.MoeError) as ei:
        mo.moe_forward_ops(x)
    assert ei.value.status == m.MOE_ERR_UNSUPPORTED_SHAPE
    y = torch.empty_like(x)
    st = m.lib.moe_forward_ops(mo.handle, x.data_ptr(), w.tokens, y.data_ptr(), None, 2, None)
    assert st == m.MOE_ERR_INVALID_ARG
    mo.moe_status()


def test_ops_full_size_decode_matches_engine(m):
    """The decode workload's shapes (H 4096, I 1536, E 128, top-8, T 9),
    device-drawn weights: ops with PDL equal the single launch bit for bit."""
    import bench
    from tests.gpu_helpers import bf16_host_bits
    w = synth.WORKLOADS["decode_t9_h4096_e128"]
    layers = [bench.build_layer(m, w, 0, seed=0)]
    mo = m.Moe(w.hidden, w.inter, w.experts, w.top_k, w.tokens, layers)
    for blk in range(2):
        x = synth.draw_torch(1000 + blk, 0, "x", -1, (w.tokens, w.hidden), 1.0)
        y_e = bf16_host_bits(mo.moe_forward(x))
        y_o = bf16_host_bits(mo.moe_forward_ops(x, pdl=True))
        mo.moe_status()
        assert (y_o == y_e).all(), blk
    mo.close()
