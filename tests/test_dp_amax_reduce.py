"""The data-parallel amax exchange on CPU: two gloo ranks on 127.0.0.1 reduce the amax words of
their token shards with an integer MAX over the fp32 bit patterns, as nvfp4_quantize_dual_dp does
between the shards' two passes.  For non-negative floats (zero, subnormals, huge values) the bit
patterns order like the values, so the result is the float maximum exactly."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


VALUES = [
    [0.0, 0.0],
    [1.5e-40, 3.0e-39],            # subnormals
    [2.0 ** -126, 1.0],
    [3.3e38, 7.0],
    [0.125, 4096.0],
]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        res = []
        for pair in VALUES:
            mine = np.array([pair[rank], pair[1 - rank] * 0.5], np.float32)   # (plain, after RHT)
            words = torch.from_numpy(mine.view(np.int32).copy())
            dist.all_reduce(words, op=dist.ReduceOp.MAX)
            res.append(words.numpy().view(np.float32).tolist())
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_int32_max_of_amax_words_is_float_max():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, _port(), out), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        for pair, got in zip(VALUES, out[r]):
            a = np.float32(pair[0]), np.float32(pair[1])
            want_plain = max(a)
            want_rht = max(np.float32(pair[1] * 0.5), np.float32(pair[0] * 0.5))
            assert np.float32(got[0]) == want_plain and np.float32(got[1]) == want_rht
