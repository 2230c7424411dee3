"""moe_route_static: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a caching allocator already holds the
free memory, the memory budget was reserved up front, or allocation is not
allowed on their serving path).  moe_route_static routes without a handle,
using a static device array as working memory.  These tests check, through the
C ABI:
- two calls in a row against the oracle (indices bit-exact, maps bit-exact,
  weights within 1e-5) and against the handle-based moe_route (everything bit
  for bit), on a shape routed per CTA and on one routed across the grid;
- the largest size the header's working-memory formula admits is accepted and
  routes correctly;
- a wait bound that runs out is reported by moe_route_static_status, which
  clears it, and the next call is correct again;
- sizes beyond the static array and bad arguments are refused.
The file is collected last, so that a failure here cannot hide the result of
any other test.
"""
import ctypes
import os

import numpy as np
import pytest

import synth
from tests.helpers import quantized_layer_np, x_values

pytestmark = pytest.mark.gpu

KEYS = ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")
SHAPES = [(512, 256, 16, 4, 37, None), (384, 256, 16, 4, 80, 1.2)]


def _inputs(shape, seed=31):
    from tests.gpu_helpers import bf16_dev, to_dev
    H, I, E, k, T, zipf = shape
    w = synth.Workload("static", H, I, E, k, T, zipf_alpha=zipf, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=seed)
    rw = to_dev(lw.router_w.astype(np.float32))
    rb = None if lw.router_b is None else to_dev(lw.router_b.astype(np.float32))
    return w, xb, lw, bf16_dev(xb), rw, rb


def static_bytes(T, E, k):
    """The header's working-memory formula of one moe_route_static call (without alignment)."""
    return 64 * T * E + 36 * min(E, T * k) + 17 * T * k


@pytest.mark.parametrize("shape", SHAPES)
def test_route_static_matches_oracle_and_handle_route_twice(shape):
    import torch
    from tests.gpu_helpers import check_route, make_moe, mx
    m = mx()
    w, xb, lw, x, rw, rb = _inputs(shape)
    handle = make_moe(w, [lw])
    ref = handle.moe_route(x)
    handle.moe_status()
    ref = {key: ref[key].cpu().numpy() for key in KEYS}
    for _ in range(2):
        got = m.moe_route_static(x, rw, rb, w.top_k)
        assert m.moe_route_static_status() == m.MOE_OK
        torch.cuda.synchronize()
        assert check_route(got, x_values(xb), lw, w.top_k) == 0  # no near ties at this seed
        for key in KEYS:
            a = got[key].cpu().numpy()
            assert a.tobytes() == ref[key].tobytes(), key  # the same kernel code: bit for bit
    handle.close()


def test_route_static_largest_admitted_size():
    """The largest T the header's formula admits (with its 2 KB alignment margin) is accepted."""
    import torch
    from tests.gpu_helpers import bf16_dev, check_route, mx, to_dev
    m = mx()
    H, E, k = 256, 16, 4
    limit = m.MOE_ROUTE_STATIC_SCRATCH_BYTES
    T = 1
    while static_bytes(T + 1, E, k) + 2048 <= limit:
        T += 1
    xb = synth.bf16_bits_from_f32(synth.draw_np(5, 0, "x", -1, (T, H), 1.0))
    rwf = synth.draw_np(5, 0, "router", -1, (E, H), 0.02)
    from oracle import moe
    lw = moe.LayerWeights(gate_codes=[], gate_scales=[], up_codes=[], up_scales=[], down_codes=[],
                          down_scales=[], router_w=rwf.astype(np.float64), router_b=None)
    got = m.moe_route_static(bf16_dev(xb), to_dev(rwf), None, k)
    assert m.moe_route_static_status() == m.MOE_OK
    torch.cuda.synchronize()
    loose = check_route(got, x_values(xb), lw, k)
    assert loose <= T // 1000, loose  # near ties are counted, not gated


def test_route_static_timeout_is_reported_and_cleared():
    """A 1 ns wait bound makes the routing barrier run out (the routing-only kernel
    holds no tensor memory and issues no bulk copies); the status query reports it
    once, and the next call with the default bound routes correctly."""
    import torch
    from tests.gpu_helpers import check_route, mx
    m = mx()
    for shape in SHAPES:
        w, xb, lw, x, rw, rb = _inputs(shape)
        os.environ["MOE_TIMEOUT_NS"] = "1"
        try:
            m.moe_route_static(x, rw, rb, w.top_k)
            assert m.moe_route_static_status() == m.MOE_ERR_TIMEOUT
        finally:
            del os.environ["MOE_TIMEOUT_NS"]
        assert m.moe_route_static_status() == m.MOE_OK  # cleared
        got = m.moe_route_static(x, rw, rb, w.top_k)
        assert m.moe_route_static_status() == m.MOE_OK
        torch.cuda.synchronize()
        assert check_route(got, x_values(xb), lw, w.top_k) == 0


def test_route_static_rejects_oversize_and_bad_args():
    from tests.gpu_helpers import mx
    m = mx()
    p = ctypes.c_void_p(1 << 20)
    # far more tokens than the static working memory holds
    assert m.lib.moe_route_static(p, 1 << 20, 8192, p, None, 512, 8, p, p, p, p, p, p, None) == \
        m.MOE_ERR_UNSUPPORTED_SHAPE
    assert m.lib.moe_route_static(p, 9, 100, p, None, 8, 2, p, p, p, p, p, p, None) == \
        m.MOE_ERR_UNSUPPORTED_SHAPE
    assert m.lib.moe_route_static(None, 9, 256, p, None, 8, 2, p, p, p, p, p, p, None) == \
        m.MOE_ERR_INVALID_ARG
    assert m.lib.moe_route_static(p, 0, 256, p, None, 8, 2, p, p, p, p, p, p, None) == m.MOE_OK
