"""GPU path vs the fp64 oracle through the C ABI: quantiser, routing, forward.

Bit-exact: MXFP4 codes/scales, top-k indices (outside counted near ties),
counts/offsets/perm/inv.  Routing weights within 1e-5.  bf16 outputs within
|err| <= 8e-3*|ref| + 1e-3*rms(ref): bf16 output rounding alone is up to
2^-8 = 3.9e-3 relative (half an ulp at the bottom of a binade), fp32
accumulation over K <= 8192 terms adds ~1e-6 relative, and the 1e-3*rms
floor absorbs absolute error on outputs near zero.
"""
import numpy as np
import pytest

import synth
from oracle import moe, mxfp4
from tests.helpers import quantized_layer_np, x_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from tests.gpu_helpers import mx
    return mx()


def _q_gpu(m, bits):
    from tests.gpu_helpers import bf16_dev
    c, s = m.mxfp4_quantize(bf16_dev(bits))
    return c.cpu().numpy(), s.cpu().numpy()


def test_quantize_every_bf16_pattern(m):
    bits = np.zeros((65536, 32), np.uint16)
    bits[:, 0] = np.arange(65536)
    bits[:, 1] = np.arange(65536)[::-1]
    c, s = _q_gpu(m, bits)
    rc, rs = mxfp4.quantize(bits)
    assert (s == rs).all() and (c == rc).all()


@pytest.mark.parametrize("amax", [1.0, 6.0 * 2.0 ** 10, 1.5 * 2.0 ** -120, 2.0 ** -125, 3.0e38])
def test_quantize_all_patterns_under_fixed_max(m, amax):
    ab = int(np.array([amax], np.float32).view(np.uint32)[0] >> 16)
    bits = np.zeros((65536, 32), np.uint16)
    bits[:, 5] = ab
    bits[:, 6] = np.arange(65536)
    fin = ((bits[:, 6] >> 7) & 0xFF) != 0xFF
    vals = np.abs(mxfp4.bf16_to_f64(bits[:, 6]))
    keep = fin & (vals <= mxfp4.bf16_to_f64(np.array([ab], np.uint16))[0])
    bits = bits[keep]
    c, s = _q_gpu(m, bits)
    rc, rs = mxfp4.quantize(bits)
    assert (s == rs).all() and (c == rc).all()


@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (256, 7168), (2048, 128)])
def test_quantize_random_weights(m, shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    w.reshape(-1)[:: max(1, w.size // 7)] *= 1e-30  # a few subnormal-range elements
    bits = synth.bf16_bits_from_f32(w)
    if shape[0] > 2:
        bits[1, :32] = 0x7F80  # +inf block
        bits[2, :32] = 0x8000  # all -0 block
    c, s = _q_gpu(m, bits)
    rc, rs = mxfp4.quantize(bits)
    assert (s == rs).all() and (c == rc).all()


SHAPES = {
    # name: (H, I, E, k, T) -- several tiles and ragged segments; small (T*k<=256) and large paths
    "tiny": (256, 128, 8, 2, 9),
    "ragged_small": (512, 256, 16, 4, 37),
    "ragged_large": (384, 256, 16, 4, 80),
    "one_token": (256, 128, 8, 2, 1),
    "all_experts": (256, 128, 4, 4, 9),
    "top1": (256, 256, 8, 1, 17),
    "many_tokens_one_expert": (256, 128, 2, 1, 40),
    # H % 256 == 0 and T*k / E <= 24: tile pairs (two row blocks per job)
    "pairs": (512, 256, 16, 4, 80),
    # grid-wide routing without tiles, >= 4 positions per expert: units of up
    # to 8 positions (5 and 4.4 per expert on average; ragged units)
    "big_units": (384, 256, 64, 4, 80),
    "big_units_ragged": (256, 128, 64, 4, 70),
    # grid-wide routing without tiles, < 4 positions per expert: units of <= 4
    "grid_routed": (256, 128, 128, 4, 80),
}


def _workload(name, zipf=None):
    H, I, E, k, T = SHAPES[name]
    return synth.Workload(name, H, I, E, k, T, zipf_alpha=zipf, device_draw=False)


@pytest.mark.parametrize("name", list(SHAPES))
def test_route_matches_oracle(m, name):
    from tests.gpu_helpers import bf16_dev, check_route, make_moe
    w = _workload(name, zipf=1.2 if name == "ragged_small" else None)
    xb, lw, _ = quantized_layer_np(w, seed=11)
    mo = make_moe(w, [lw])
    out = mo.moe_route(bf16_dev(xb))
    mo.moe_status()
    assert check_route(out, x_values(xb), lw, w.top_k) == 0


@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_matches_oracle(m, name):
    from tests.gpu_helpers import bf16_dev, check_forward, make_moe
    w = _workload(name)
    xb, lw, _ = quantized_layer_np(w, seed=12)
    mo = make_moe(w, [lw])
    y = mo.moe_forward(bf16_dev(xb))
    mo.moe_status()
    check_forward(y, x_values(xb), lw, w.top_k)


@pytest.mark.parametrize("kind", ["mxf4", "f16", "mxf8"])
@pytest.mark.parametrize("name,tokens", [("ragged_large", 80), ("ragged_large", 192), ("pairs", 80),
                                         ("pairs", 96), ("pairs", 101), ("pairs", 300)])
def test_large_t_kinds_match_oracle(m, kind, name, tokens):
    """The three weight streams for many positions per expert (E2M1 term tiles on
    the fp4 MMA, bf16 tiles on the bf16 MMA, E4M3 term tiles on the fp8/fp6/fp4
    MMA): ragged tiles, T*K = 320 and 768 with one row block per job, T*K = 320
    and 384 as tile pairs (segments split into tiles of at most 22), T*K = 404
    back on single row blocks, T*K = 1200 (75 positions per expert: several
    tiles of every kind per expert)."""
    from tests.gpu_helpers import bf16_dev, check_forward, make_moe
    H, I, E, k, _ = SHAPES[name]
    w = synth.Workload(name, H, I, E, k, tokens, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=23)
    mo = make_moe(w, [lw])
    mo.moe_set_large_kind({"mxf4": mo.LARGE_MXF4, "f16": mo.LARGE_F16, "mxf8": mo.LARGE_MXF8}[kind])
    y = mo.moe_forward(bf16_dev(xb))
    mo.moe_status()
    check_forward(y, x_values(xb), lw, w.top_k)


@pytest.mark.parametrize("name", ["ragged_large", "pairs", "big_units"])
def test_forward_with_router_bias(m, name):
    """Zipf-biased routing: a few experts hold many positions (several tiles or
    units of 8 each)."""
    from tests.gpu_helpers import bf16_dev, check_forward, make_moe
    w = _workload(name, zipf=1.2)
    xb, lw, _ = quantized_layer_np(w, seed=13)
    mo = make_moe(w, [lw])
    check_forward(mo.moe_forward(bf16_dev(xb)), x_values(xb), lw, w.top_k)


def test_tokens_fewer_than_max_and_empty(m):
    from tests.gpu_helpers import bf16_dev, check_forward, make_moe
    import torch
    w = _workload("ragged_small")
    xb, lw, _ = quantized_layer_np(w, seed=14)
    mo = make_moe(w, [lw], max_tokens=64)
    for T in (37, 5, 1):
        y = mo.moe_forward(bf16_dev(xb[:T]))
        check_forward(y, x_values(xb[:T]), lw, w.top_k)
    y0 = mo.moe_forward(torch.empty((0, w.hidden), dtype=torch.bfloat16, device="cuda"))
    assert y0.shape == (0, w.hidden)
    mo.moe_status()
    with pytest.raises(m.MoeError):
        mo.moe_forward(bf16_dev(np.zeros((65, w.hidden), np.uint16)))


def test_zero_input_gives_zero_output(m):
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_small")
    _, lw, _ = quantized_layer_np(w, seed=15)
    mo = make_moe(w, [lw])
    y = mo.moe_forward(bf16_dev(np.zeros((w.tokens, w.hidden), np.uint16)))
    assert (x_values(bf16_host_bits(y)) == 0).all()


def test_down_scale_increment_doubles_output_exactly(m):
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_small")
    xb, lw, _ = quantized_layer_np(w, seed=16)
    lw2 = moe.LayerWeights(lw.gate_codes, lw.gate_scales, lw.up_codes, lw.up_scales,
                           lw.down_codes, [s + 1 for s in lw.down_scales], lw.router_w, lw.router_b)
    y1 = x_values(bf16_host_bits(make_moe(w, [lw]).moe_forward(bf16_dev(xb))))
    y2 = x_values(bf16_host_bits(make_moe(w, [lw2]).moe_forward(bf16_dev(xb))))
    assert (y2 == 2 * y1).all()


def test_token_permutation_equivariance_and_determinism(m):
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_large")
    xb, lw, _ = quantized_layer_np(w, seed=17)
    mo = make_moe(w, [lw])
    perm = np.random.default_rng(0).permutation(w.tokens)
    y = bf16_host_bits(mo.moe_forward(bf16_dev(xb)))
    y_again = bf16_host_bits(mo.moe_forward(bf16_dev(xb)))
    yp = bf16_host_bits(mo.moe_forward(bf16_dev(xb[perm])))
    assert (y == y_again).all()
    assert (yp == y[perm]).all()


def test_forward_host_matches_device(m):
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("tiny")
    xb, lw, _ = quantized_layer_np(w, seed=18)
    mo = make_moe(w, [lw])
    y = bf16_host_bits(mo.moe_forward(bf16_dev(xb)))
    xh = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = mo.moe_forward_host(xh)
    assert (bf16_host_bits(yh) == y).all()


@pytest.mark.parametrize("shape", [(512, 256, 16, 4, 9, 3), (384, 256, 64, 4, 80, 2)])
def test_chain_teacher_forced(m, shape):
    """Chained layers in one launch; each layer checked on the GPU's own bf16
    input.  Per-CTA routing (T*k = 36), and grid-wide routing with units of up
    to 8 positions (T*k = 320, E = 64)."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    from tests.helpers import tolerance_ok
    H, I, E, k, T, L = shape
    w = synth.Workload("chain", H, I, E, k, T, layers=L, zipf_alpha=1.2, device_draw=False)
    lws, xb = [], None
    for l in range(L):
        xl, lw, _ = quantized_layer_np(w, layer=l, seed=19)
        lws.append(lw)
        xb = xl if l == 0 else xb
    mo = make_moe(w, lws)
    io = torch.empty((L + 1, w.tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    y = mo.moe_forward(bf16_dev(xb), layer_io=io)
    mo.moe_status()
    io_h = x_values(bf16_host_bits(io))
    assert (bf16_host_bits(io[0]) == xb).all()
    assert (bf16_host_bits(io[L]) == bf16_host_bits(y)).all()
    for l in range(L):
        ref_y = moe.moe_layer(io_h[l], lws[l], w.top_k)["y"]
        if l < L - 1:
            ok, ratio = tolerance_ok(io_h[l + 1], moe.rmsnorm(ref_y))
        else:
            ok, ratio = tolerance_ok(io_h[L], ref_y)
        assert ok, (l, ratio)


def test_status_reports_ok_and_handle_reusable(m):
    from tests.gpu_helpers import bf16_dev, make_moe
    w = _workload("tiny")
    xb, lw, _ = quantized_layer_np(w, seed=20)
    mo = make_moe(w, [lw])
    for _ in range(3):
        mo.moe_forward(bf16_dev(xb))
    mo.moe_status()
    assert mo.grid > 0


def test_forward_captured_in_cuda_graph_matches_stream_launch(m):
    """moe_forward is stream-capture safe: replaying a CUDA graph of calls on two
    token blocks gives the stream launches' outputs bit for bit."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_large")
    xa, lw, _ = quantized_layer_np(w, seed=21)
    xb = quantized_layer_np(w, seed=22)[0]
    mo = make_moe(w, [lw])
    xs = [bf16_dev(xa), bf16_dev(xb)]
    ref = [bf16_host_bits(mo.moe_forward(x)) for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for x, y in zip(xs, ys):
            mo.moe_forward(x, y)
    for y in ys:
        y.zero_()
    g.replay()
    torch.cuda.synchronize()
    mo.moe_status()
    for y, r in zip(ys, ref):
        assert (bf16_host_bits(y) == r).all()


def test_forward_host_async_matches_device(m):
    """Pipelined host entry point: five calls over three token blocks (both
    staging slots reused) give the device path's outputs bit for bit."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, make_moe
    w = _workload("ragged_small")
    lw = quantized_layer_np(w, seed=24)[1]
    xbs = [quantized_layer_np(w, seed=25 + i)[0] for i in range(3)]
    mo = make_moe(w, [lw])
    ref = [bf16_host_bits(mo.moe_forward(bf16_dev(xb))) for xb in xbs]
    xh = [torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory() for xb in xbs]
    yh = [torch.empty((w.tokens, w.hidden), dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    for i in range(5):
        mo.moe_forward_host_async(xh[i % 3], yh[i])
    mo.moe_host_join()
    mo.moe_status()
    for i in range(5):
        assert (bf16_host_bits(yh[i]) == ref[i % 3]).all(), i
