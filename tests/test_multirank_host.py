"""Host logic of the N > 1 bench path on CPU: two gloo ranks (no GPU).

Each rank verifies its own token blocks (weak scaling, no collective on the data
path); the only collective is the max over ranks of the timed region.
"""
import os
import socket

import pytest

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports a distinct elapsed time; every rank must see the slowest
        mine = 10.0 + 7.5 * rank
        slowest = bench.max_over_ranks(mine, dist, "cpu")
        ids = bench.token_block_ids(rank, 8)
        dist.barrier()
        out.put((rank, mine, slowest, ids))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_disjoint_blocks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[2] for r in res] == [17.5, 17.5]           # both ranks see the slowest rank
    ids0, ids1 = res[0][3], res[1][3]
    assert len(set(ids0)) == 8 and not set(ids0) & set(ids1)  # each rank its own blocks


def test_max_over_ranks_without_a_group_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_job_throughput_counts_every_rank():
    # 4 ranks x 9 tokens x 100 steps in 0.5 s
    assert bench.job_tokens_per_s(4, 9, 100, 0.5) == pytest.approx(7200.0)
    assert bench.job_tokens_per_s(1, 9, 100, 0.5) == pytest.approx(1800.0)


def test_token_block_ids_bounds():
    assert bench.token_block_ids(0, 1) == [1000]
    assert bench.token_block_ids(3, 2) == [1192, 1193]
    with pytest.raises(ValueError):
        bench.token_block_ids(0, 65)


def _shard_rank_main(rank, world, port, out):
    """Rank r: the oracle's partial output over its I-slice, summed across ranks by an
    all-reduce (gloo) -- the host composition of the I-sharded layer."""
    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    from oracle import moe
    from tests.helpers import quantized_layer_np, shard_layer_np, x_values
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.Workload("shard", 256, 256, 8, 2, 9, device_draw=False)
        xb, lw, _ = quantized_layer_np(w, seed=61)
        part = torch.from_numpy(moe.moe_layer(x_values(xb), shard_layer_np(lw, rank, world), w.top_k)["y"])
        dist.all_reduce(part)
        full = moe.moe_layer(x_values(xb), lw, w.top_k)["y"]
        out.put((rank, float(np.abs(part.numpy() - full).max() / np.abs(full).max())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_all_reduce_i_shards_to_the_layer():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _ in res] == [0, 1]
    assert all(err < 1e-12 for _, err in res), res


def test_shard_layer_i_slices_like_the_oracle_side():
    """The binding's I-slicer (torch, any device) against the oracle-side slicer."""
    import numpy as np
    import torch
    import synth
    from tests.helpers import build_library, quantized_layer_np, shard_layer_np
    build_library()
    import mxfp4_moe_expert_router_b200 as mx
    w = synth.Workload("shard", 256, 512, 4, 2, 9, device_draw=False)
    _, lw, _ = quantized_layer_np(w, seed=62)
    st = lambda a: torch.from_numpy(np.stack(a))
    layer = mx.LayerMX(st(lw.gate_codes), st(lw.gate_scales), st(lw.up_codes), st(lw.up_scales),
                       st(lw.down_codes), st(lw.down_scales), torch.from_numpy(lw.router_w), None)
    for world in (1, 2, 4):
        for r in range(world):
            a, b = mx.shard_layer_i(layer, r, world), shard_layer_np(lw, r, world)
            for k in ("gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales"):
                assert (getattr(a, k).numpy() == np.stack(getattr(b, k))).all(), (world, r, k)
    with pytest.raises(ValueError):
        mx.shard_layer_i(layer, 0, 8)  # 512 / 8 = 64 rows


class _FakeHandle:
    """Stands in for a Moe handle: a region address per rank, a recognisable IPC handle."""

    def __init__(self, rank):
        self.rank, self.attached = rank, None

    def moe_ishard_region(self):
        return 0x1000 * (self.rank + 1), 4096

    def moe_ishard_ipc_handle(self):
        return bytes([self.rank + 1]) * 64

    def moe_ishard_attach(self, rank, world, regions):
        self.attached = (rank, world, list(regions))


def _ipc_rank_main(rank, world, port, out):
    import torch.distributed as dist
    from tests.helpers import build_library
    build_library()
    import mxfp4_moe_expert_router_b200 as mx
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = mx.exchange_ipc_handles(bytes([rank + 1]) * 64)
        fake = _FakeHandle(rank)
        # a peer's region as this rank maps it: tagged with the handle it came from
        opened = mx.connect_ishard(fake, opener=lambda h: 0x100000 + h[0])
        out.put((rank, [g[0] for g in got], fake.attached, opened))
    finally:
        dist.destroy_process_group()


def test_ishard_handle_exchange_and_attach_order_under_gloo():
    """connect_ishard over 3 gloo ranks: every rank gets all IPC handles in rank order,
    maps each peer's, and attaches its own region at its rank and the mapped peers elsewhere."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_ipc_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tags, attached, opened in res:
        assert tags == [1, 2, 3]
        r, w, regions = attached
        assert (r, w) == (rank, world)
        expect = [0x1000 * (rank + 1) if s == rank else 0x100000 + s + 1 for s in range(world)]
        assert regions == expect
        assert opened == [0x100000 + s + 1 for s in range(world) if s != rank]
