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


def _virtual_ranks(mx, w, lw, world):
    """One handle per virtual rank on this GPU, each on its I-slice, all attached to every
    handle's region (plain device addresses: every region is on this GPU)."""
    from tests.gpu_helpers import layer_dev
    full = layer_dev(lw)
    ms = [_moe(mx, w, mx.shard_layer_i(full, r, world), w.inter // world) for r in range(world)]
    regions = [m.moe_ishard_region()[0] for m in ms]
    for r, m in enumerate(ms):
        m.moe_ishard_attach(r, world, regions)
    views = [mx.region_views(b, w.tokens, w.hidden) for b in regions]
    return ms, views


@pytest.mark.parametrize("world", [2, 4])
# T*k = 148 (per-CTA routing), 320 over 16 experts (tile path), 320 over 64
# experts (grid-wide routing with units of up to 8 positions)
@pytest.mark.parametrize("E,T", [(16, 37), (16, 80), (64, 80)])
def test_fused_allreduce_virtual_ranks(mx, world, E, T):
    """The fused all-reduce of moe_forward_ishard, one virtual rank at a time on one GPU.

    Before rank r's call of epoch e, every other rank's partial is put in its slot
    e % 2 and its epoch in rank r's region (what the peers' kernels would have done),
    so rank r's wait ends at once.  Checks: rank r's own partial is moe_forward_partial's
    bit for bit; every rank's y is the same bits; y is the rank-order fp32 sum of the
    partials rounded to bf16, bit for bit; y meets the oracle's tolerance; both slots
    (epochs 1 and 2)."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits
    w = synth.Workload("s4", 512, 512, E, 4, T, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=60 + T)
    x = bf16_dev(xb)
    ms, views = _virtual_ranks(mx, w, lw, world)
    parts = [m.moe_forward_partial(x).clone() for m in ms]
    for m in ms:
        m.moe_status()
    total = parts[0].clone()
    for p_ in parts[1:]:
        total += p_  # rank order
    ref_bits = bf16_host_bits(total.to(torch.bfloat16))
    oracle_y = moe.moe_layer(x_values(xb), lw, w.top_k)["y"]
    for epoch in (1, 2):
        slot = epoch % 2
        ys = []
        for r in range(world):
            for s in range(world):
                if s != r:
                    views[s][1][slot, :T].copy_(parts[s])
                    views[r][0][s] = epoch
            torch.cuda.synchronize()
            y = ms[r].moe_forward_ishard(x)
            ms[r].moe_status()
            assert torch.equal(views[r][1][slot, :T], parts[r]), (epoch, r)
            assert int(views[r][0][r].item()) == epoch
            ys.append(bf16_host_bits(y))
        for r in range(world):
            assert (ys[r] == ref_bits).all(), (epoch, r)
        ok, ratio = tolerance_ok(x_values(ys[0]), oracle_y)
        assert ok, ratio
    for m in ms:
        m.close()


def test_fused_allreduce_peer_timeout(mx):
    """A peer that never publishes its epoch: the bounded wait runs out, moe_status
    reports MOE_ERR_TIMEOUT, and after re-attaching the handle is correct again."""
    import torch
    from tests.gpu_helpers import bf16_dev, bf16_host_bits
    world, T = 2, 37
    w = synth.Workload("s5", 512, 512, 16, 4, T, device_draw=False)
    xb, lw, _ = quantized_layer_np(w, seed=71)
    x = bf16_dev(xb)
    ms, views = _virtual_ranks(mx, w, lw, world)
    parts = [m.moe_forward_partial(x).clone() for m in ms]
    ms[0].moe_set_timeout_ns(200_000)
    ms[0].moe_forward_ishard(x)  # rank 1 never publishes epoch 1
    assert mx.lib.moe_status(ms[0].handle, mx._stream()) == mx.MOE_ERR_TIMEOUT
    ms[0].moe_set_timeout_ns(2_000_000_000)
    regions = [m.moe_ishard_region()[0] for m in ms]
    for r, m in enumerate(ms):
        m.moe_ishard_attach(r, world, regions)
    views[1][1][1, :T].copy_(parts[1])
    views[0][0][1] = 1
    torch.cuda.synchronize()
    y = ms[0].moe_forward_ishard(x)
    ms[0].moe_status()
    ref = bf16_host_bits((parts[0] + parts[1]).to(torch.bfloat16))
    assert (bf16_host_bits(y) == ref).all()
    for m in ms:
        m.close()
