"""The I-sharded layer on one GPU: each rank's share (moe_forward_partial on a handle built
from its I-slice) run in turn, the partials summed in rank order, rounded by moe_round_bf16.

Checks: one rank reproduces moe_forward bit for bit; every shard routes exactly as the
whole layer; N shards give the oracle's layer within the bf16 tolerance, on the verify-block
path and on the large-T tile path.  The all-reduce across GPUs is not exercised here (one
GPU); its host side runs under gloo in tests/test_multirank_host.py.
"""
import numpy as np
import pytest

import synth
from oracle import moe
from tests.helpers import quantized_layer_np, tolerance_ok, x_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from tests.gpu_helpers import mx as load
    return load()


def _moe(mx, w, layer, inter):
    return mx.Moe(w.hidden, inter, w.experts, w.top_k, w.tokens, [layer])


def test_one_rank_is_moe_forward_bit_for_bit(mx):
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, layer_dev
    w = synth.Workload("s1", 512, 256, 16, 4, 37, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=51)
    m = _moe(mx, w, layer_dev(lw), w.inter)
    x = bf16_dev(xb)
    y = bf16_host_bits(m.moe_forward(x))
    yp = bf16_host_bits(mx.round_bf16(m.moe_forward_partial(x)))
    m.moe_status()
    assert (y == yp).all()
    m.close()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("T", [37, 80])  # T*k = 148 (verify-block path), 320 (tile path)
def test_shards_sum_to_the_layer(mx, world, T):
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits, layer_dev
    w = synth.Workload("s2", 512, 512, 16, 4, T, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=52 + T)
    full = layer_dev(lw)
    x = bf16_dev(xb)
    whole = _moe(mx, w, full, w.inter)
    ref_route = whole.moe_route(x)
    total = torch.zeros((T, w.hidden), dtype=torch.float32, device="cuda")
    for r in range(world):
        m = _moe(mx, w, mx.shard_layer_i(full, r, world), w.inter // world)
        route = m.moe_route(x)
        for k in ("topk_idx", "counts", "perm", "inv_perm"):
            assert torch.equal(route[k], ref_route[k]), (r, k)
        assert torch.equal(route["topk_w"], ref_route["topk_w"])
        total += m.moe_forward_partial(x)
        m.moe_status()
        m.close()
    y = x_values(bf16_host_bits(mx.round_bf16(total)))
    ok, ratio = tolerance_ok(y, moe.moe_layer(x_values(xb), lw, w.top_k)["y"])
    assert ok, ratio
    whole.close()


def test_partial_needs_a_single_layer_and_sharding_needs_multiples_of_128(mx):
    from tests.gpu_helpers import bf16_dev, layer_dev
    w = synth.Workload("s3", 256, 256, 8, 2, 9, layers=2, device_draw=False)
    lws = [quantized_layer_np(w, layer=l, seed=53)[1] for l in range(2)]
    m = mx.Moe(w.hidden, w.inter, w.experts, w.top_k, w.tokens, [layer_dev(lw) for lw in lws])
    with pytest.raises(mx.MoeError) as ei:
        m.moe_forward_partial(bf16_dev(quantized_layer_np(w, seed=53)[0]))
    assert ei.value.status == mx.MOE_ERR_UNSUPPORTED_SHAPE
    m.close()
    with pytest.raises(ValueError):
        mx.shard_layer_i(layer_dev(lws[0]), 0, 4)  # 256 / 4 = 64 rows
