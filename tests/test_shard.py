"""Column-parallel sharding of a layer over several GPUs (host logic, CPU):
the tile-row split balanced by stored bytes or by MMA work, and -- with two gloo ranks --
that the shards' outputs concatenate to the whole layer's output."""
import functools
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DENSE, SPARSE = 32768, 16384 + 2048


def _row_bytes(bm):
    return np.where(bm != 0, SPARSE, DENSE).sum(axis=1) + 16 * bm.shape[1]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("kind", ["exact", "clustered", "bernoulli"])
def test_shard_rows_definition_and_balance(n, kind):
    N, K = 128 * 43, 128 * 8
    bm = {"exact": si.tiles_exact, "clustered": si.tiles_clustered, "bernoulli": si.tiles_bernoulli}[kind](
        N, K, 0.5, 3, n)
    rows = tsg.shard_rows(bm, n)
    rb = _row_bytes(bm)
    prefix = np.concatenate([[0], np.cumsum(rb)])
    total = prefix[-1]
    assert rows[0][0] == 0 and rows[-1][1] == bm.shape[0]
    for (b0, e0), (b1, e1) in zip(rows, rows[1:]):
        assert e0 == b1  # contiguous
    for i, (b, e) in enumerate(rows):
        assert e > b  # never empty
        if i > 0:  # the first row whose prefix reaches i/n of the total (no clamp needed at these sizes)
            assert prefix[b] * n >= i * total and prefix[b - 1] * n < i * total
    # balance: no shard exceeds its fair share by more than one row
    worst = max(prefix[e] - prefix[b] for b, e in rows)
    assert worst <= total / n + rb.max()


@pytest.mark.parametrize("n", [2, 3, 8])
def test_shard_rows_by_flops_balances_the_mma_work(n):
    """by="flops": each tile row weighs 2 per dense tile and 1 per sparse tile
    (a sparse tile's MMAs multiply half of W); the same prefix rule as by bytes."""
    N, K = 128 * 43, 128 * 8
    bm = si.tiles_clustered(N, K, 0.5, 3, 7 + n)
    rows = tsg.shard_rows(bm, n, by="flops")
    rw = np.where(bm != 0, 1, 2).sum(axis=1)
    prefix = np.concatenate([[0], np.cumsum(rw)])
    total = prefix[-1]
    assert rows[0][0] == 0 and rows[-1][1] == bm.shape[0]
    for i, (b, e) in enumerate(rows):
        assert e > b
        if i > 0:
            assert prefix[b] * n >= i * total and prefix[b - 1] * n < i * total
    assert max(prefix[e] - prefix[b] for b, e in rows) <= total / n + rw.max()


def test_shard_balance_by_bytes_and_by_flops_differ_where_they_should():
    """A sparse row weighs ~0.56 of a dense one in bytes (18448 vs 32784 with
    its descriptor) but 0.5 in MMA work: 3 dense rows then 6 sparse ones split
    4 + 5 by bytes (the 3 dense rows hold 98352 B of 209040, under half, so
    the second shard starts after row 4) and 3 + 6 by work (6 of 12)."""
    bm = np.zeros((9, 1), np.uint8)
    bm[3:] = 1
    assert tsg.shard_rows(bm, 2, by="flops") == [(0, 3), (3, 9)]
    assert tsg.shard_rows(bm, 2, by="bytes") == [(0, 4), (4, 9)]
    assert tsg.shard_rows(bm, 2) == tsg.shard_rows(bm, 2, by="bytes")
    with pytest.raises(KeyError):
        tsg.shard_rows(bm, 2, by="rows")


def test_shard_rows_keeps_every_shard_non_empty():
    bm = np.zeros((5, 3), np.uint8)
    bm[0] = 1  # one light row, then heavy ones
    assert tsg.shard_rows(bm, 5) == [(0, 1), (1, 2), (2, 3), (3, 4), (4, 5)]
    with pytest.raises(tsg.PatchError):
        tsg.shard_rows(bm, 6)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as orc
        import synth_inputs as s
        import tile_sparse_gemm_b200 as t
        N, K, M = 128 * 7, 256, 5
        w, x = s.gen_w(N, K, 15, 0), s.gen_x(M, K, 15, 0)
        bm, ids = s.tiles_clustered(N, K, 0.5, 15, 0), s.patterns_top2(w)
        b, e = t.shard_rows(bm, world)[rank]
        # this rank's shard of Y (the oracle stands in for the GPU GEMM on CPU)
        y = orc.hybrid_gemm(x, w[b * 128:e * 128], bm[b:e], ids[b * 128:e * 128])
        parts = [None] * world
        dist.all_gather_object(parts, y)
        out[rank] = np.concatenate(parts, axis=1)
    finally:
        dist.destroy_process_group()


def test_two_ranks_concatenate_to_the_whole_layer():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork of this multi-threaded process
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    N, K, M = 128 * 7, 256, 5
    w, x = si.gen_w(N, K, 15, 0), si.gen_x(M, K, 15, 0)
    ref = oracle.hybrid_gemm(x, w, si.tiles_clustered(N, K, 0.5, 15, 0), si.patterns_top2(w))
    for r in range(world):
        assert np.array_equal(out[r], ref)


def _bench_rank(rank, world, port, out, by):
    """bench.py's sharded step on CPU: its shard plan (balanced by `by`), its
    gather layout and one all-gather (gloo), with the oracle standing in for each
    rank's GEMMs."""
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle as orc
        import synth_inputs as s
        import tile_sparse_gemm_b200 as t
        layers = []
        for i, (N, K) in enumerate([(128 * 7, 256), (128 * 3, 384), (128 * 10, 128)]):
            w = s.gen_w(N, K, 18, i)
            layers.append(dict(name=f"l{i}", N=N, K=K, w=w, bm=s.tiles_clustered(N, K, 0.5, 18, i),
                               ids=s.patterns_top2(w), xs={M: s.gen_x(M, K, 18, 10 * i + M) for M in (1, 5)}))
        calls = bench.calls_of(layers)
        split = functools.partial(t.shard_rows, by=by)
        mine = bench.shard_layers(layers, rank, world, split)
        offset, sizes, seg = bench.gather_layout(layers, calls, world, split)
        buf = torch.zeros(seg, dtype=torch.float64)
        for j, (li, M) in enumerate(calls):
            L = mine[li]
            y = orc.hybrid_gemm(L["xs"][M], L["w"], L["bm"], L["ids"])  # this rank's columns
            assert y.size == sizes[rank][j]
            buf[offset[rank][j]:offset[rank][j] + y.size] = torch.from_numpy(y.ravel())
        got = [torch.zeros(seg, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, buf)
        full = []
        for j, (li, M) in enumerate(calls):
            parts = [got[r][offset[r][j]:offset[r][j] + sizes[r][j]].numpy().reshape(M, -1) for r in range(world)]
            full.append(np.concatenate(parts, axis=1))
        out[rank] = full
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("by", ["bytes", "flops"])
def test_bench_shard_plan_and_gather_reassemble_every_call(by):
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_bench_rank, args=(world, _free_port(), out, by), nprocs=world, start_method="spawn")
    for i, (N, K) in enumerate([(128 * 7, 256), (128 * 3, 384), (128 * 10, 128)]):
        w = si.gen_w(N, K, 18, i)
        bm, ids = si.tiles_clustered(N, K, 0.5, 18, i), si.patterns_top2(w)
        for M in (1, 5):
            ref = oracle.hybrid_gemm(si.gen_x(M, K, 18, 10 * i + M), w, bm, ids)
            j = (0 if M == 1 else 3) + i  # calls: every layer at M = 1, then every layer at M = 5
            for r in range(world):
                assert np.array_equal(out[r][j], ref)
