"""Host logic of the data-parallel linear step on CPU, two gloo ranks on 127.0.0.1: the token
shard offsets of each rank, and the reduce-scatter of dW partial sums -- each rank keeps its rows
of the fp32 sum over ranks, which is what the whole batch's wgrad GEMM computes (the K sum over
all tokens split by rank)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nvfp4_bit_quantized_02_b200 import dp_dw_rows, dp_token_rows


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_token_shards_tile_the_batch():
    for world in (1, 2, 3, 8):
        spans = [dp_token_rows(64, r, world) for r in range(world)]
        assert all(total == 64 * world for _, total in spans)
        assert [off for off, _ in spans] == [64 * r for r in range(world)]


def test_dw_rows_partition_the_output():
    for world in (1, 2, 4, 8):
        rows = [dp_dw_rows(20480, r, world) for r in range(world)]
        assert rows[0][0] == 0 and rows[-1][1] == 20480
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        n, d, T = 12, 5, 16
        g = torch.Generator().manual_seed(0)
        dy = torch.randn(world * T, n, generator=g, dtype=torch.float64)
        x = torch.randn(world * T, d, generator=g, dtype=torch.float64)
        off, _ = dp_token_rows(T, rank, world)
        partial = (dy[off:off + T].t() @ x[off:off + T]).to(torch.float32)   # this rank's wgrad
        r0, r1 = dp_dw_rows(n, rank, world)
        mine = torch.empty((r1 - r0, d), dtype=torch.float32)
        _reduce_scatter_gloo(mine, partial, world)
        full = (dy.t() @ x)[r0:r1]
        out[rank] = float((mine.double() - full).abs().max() / full.abs().max())
    finally:
        dist.destroy_process_group()


def _reduce_scatter_gloo(out, inp, world):
    # the reduce-scatter's result on gloo (which has no reduce_scatter_tensor): the sum over ranks
    # of every partial, of which this rank keeps its rows
    t = inp.clone()
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    r0, r1 = dp_dw_rows(inp.shape[0], dist.get_rank(), world)
    out.copy_(t[r0:r1])


def test_reduce_scatter_of_partials_gives_each_rank_its_rows_of_the_batch_dw():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, _port(), out), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        assert out[r] < 1e-6
