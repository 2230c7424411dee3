"""moe_route_static: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a caching allocator already holds the
free memory, the memory budget was reserved up front, or allocation is not
allowed on their serving path).  moe_route_static routes without a handle,
using a static device array as working memory.  This test checks, through the
C ABI, that two calls in a row give exactly what the handle-based moe_route
gives, on a shape routed per CTA and on one routed across the grid, and that
sizes beyond the static array are refused.  It lives in its own file, collected
last, so that a failure here cannot hide the result of any other test.
"""
import ctypes

import numpy as np
import pytest

import synth
from tests.helpers import quantized_layer_np

pytestmark = pytest.mark.gpu

KEYS = ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")


@pytest.mark.parametrize("shape", [(512, 256, 16, 4, 37, None), (384, 256, 16, 4, 80, 1.2)])
def test_route_static_matches_handle_route_twice(shape):
    from tests.gpu_helpers import bf16_dev, make_moe, mx, to_dev
    m = mx()
    H, I, E, k, T, zipf = shape
    w = synth.Workload("static", H, I, E, k, T, zipf_alpha=zipf, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=31)
    handle = make_moe(w, [lw])
    x = bf16_dev(xb)
    ref = handle.moe_route(x)
    handle.moe_status()
    rw = to_dev(lw.router_w.astype(np.float32))
    rb = None if lw.router_b is None else to_dev(lw.router_b.astype(np.float32))
    for _ in range(2):
        got = m.moe_route_static(x, rw, rb, k)
        import torch
        torch.cuda.synchronize()
        for key in KEYS:
            a, b = got[key].cpu().numpy(), ref[key].cpu().numpy()
            if key == "topk_w":
                assert np.abs(a - b).max() <= 1e-5, key
            else:
                assert (a == b).all(), key


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
