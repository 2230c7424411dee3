"""Failure detection on the GPU without a fault: the engine's bounded waits.

Every wait inside the engine kernel (grid barriers, the routing barrier, ring
mbarriers, the job queue, per-unit readiness) gives up after the handle's wait
bound; the kernel then records a status code, stops issuing work, lets the
copies and MMAs it already issued complete (their drains have a fixed bound of
their own), frees its tensor memory and returns.  moe_status reports
MOE_ERR_TIMEOUT once and resets the handle's wait state.

These tests make the bound run out with a short moe_set_timeout_ns (nothing is
broken on purpose: every wait still ends, only sooner), check the status, then
restore the default bound and check that the same handle routes and runs the
layer exactly as before (against the oracle).
"""
import numpy as np
import pytest

import synth
from tests.helpers import quantized_layer_np, x_values

pytestmark = pytest.mark.gpu

DEFAULT_NS = 2_000_000_000
# (H, I, E, k, T): per-CTA routing (T*k <= 256), the grid-wide routing with the
# pipeline stream (units of up to 8 positions, then of up to 4), and the
# grid-wide routing with the tile stream (T*k >= 8 E): tile pairs (H % 256 ==
# 0, T*k <= 24 E) and single row blocks
SHAPES = [(512, 256, 16, 4, 37), (384, 256, 64, 4, 80), (256, 128, 128, 4, 80), (256, 256, 16, 4, 80),
          (384, 256, 16, 4, 80)]


def _case(shape, seed=41):
    from tests.gpu_helpers import bf16_dev, make_moe
    H, I, E, k, T = shape
    w = synth.Workload("timeout", H, I, E, k, T, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=seed)
    return w, xb, lw, make_moe(w, [lw]), bf16_dev(xb)


def _check_healthy(m, w, xb, lw, x):
    import torch
    from tests.gpu_helpers import check_forward, check_route
    m.moe_set_timeout_ns(DEFAULT_NS)
    r = m.moe_route(x)
    m.moe_status()
    torch.cuda.synchronize()
    assert check_route(r, x_values(xb), lw, w.top_k) == 0
    y = m.moe_forward(x)
    m.moe_status()
    check_forward(y, x_values(xb), lw, w.top_k)


def _status(mx, m):
    return mx.lib.moe_status(m.handle, mx._stream())


@pytest.mark.parametrize("shape", SHAPES)
def test_route_timeout_reported_and_handle_reusable(shape):
    """Routing alone (no tensor memory, no bulk copies) with a 1 ns bound."""
    from tests.gpu_helpers import mx
    m_ = mx()
    w, xb, lw, m, x = _case(shape)
    m.moe_set_timeout_ns(1)
    m.moe_route(x)
    assert _status(m_, m) == m_.MOE_ERR_TIMEOUT
    assert _status(m_, m) == m_.MOE_OK  # reported once, then cleared
    _check_healthy(m, w, xb, lw, x)
    m.close()


@pytest.mark.parametrize("shape", SHAPES)
def test_forward_timeout_reported_and_handle_reusable(shape):
    """A whole forward with a 1 ns bound: the CTAs give up at the routing barrier
    with tensor memory allocated; they must release it and leave the handle usable."""
    from tests.gpu_helpers import mx
    m_ = mx()
    w, xb, lw, m, x = _case(shape)
    m.moe_set_timeout_ns(1)
    m.moe_forward(x)
    assert _status(m_, m) == m_.MOE_ERR_TIMEOUT
    _check_healthy(m, w, xb, lw, x)
    m.close()


def test_forward_timeout_inside_the_stream():
    """Bounds of a few microseconds also run out inside the weight stream (ring,
    queue and readiness waits), with copies and MMAs in flight.  Each call either
    completes or reports MOE_ERR_TIMEOUT; a completed call is correct, and after
    each the handle runs the layer correctly with the default bound."""
    from tests.gpu_helpers import bf16_host_bits, mx
    from oracle import moe
    from tests.helpers import tolerance_ok
    m_ = mx()
    for shape in SHAPES[1:]:
        w, xb, lw, m, x = _case(shape)
        ref = moe.moe_layer(x_values(xb), lw, w.top_k)["y"]
        seen = set()
        for ns in (2_000, 5_000, 10_000, 20_000, 50_000):
            m.moe_set_timeout_ns(ns)
            y = m.moe_forward(x)
            st = _status(m_, m)
            assert st in (m_.MOE_OK, m_.MOE_ERR_TIMEOUT), st
            seen.add(st)
            if st == m_.MOE_OK:
                assert tolerance_ok(x_values(bf16_host_bits(y)), ref)[0]
            _check_healthy(m, w, xb, lw, x)
        assert m_.MOE_ERR_TIMEOUT in seen
        m.close()
