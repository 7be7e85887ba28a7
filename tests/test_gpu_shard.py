"""Data-parallel token shards on the GPU: each shard's forms equal, bit for bit, its slice of the
oracle's forms of the whole tensor (the tensor scale from the whole tensor's amax, SR fields
indexed in the whole tensor's forms; gist.science "Pretraining Large Language Models with
NVFP4", 2.A and 2.B.4).  Two shards on one GPU stand in for two ranks; their amax words are
reduced with MAX between the passes, as the ranks' all-reduce does."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import assert_form_equal, check_gemm, make_form, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _row_slice(q, r0, r1):
    """Rows [r0, r1) of a form, as a form of its own (its scales re-laid out in MMA tiles)."""
    return make_form(r1 - r0, q.K, q.nibbles()[r0:r1], q.scales_rm[r0:r1], q.s_t)


def _k_slice(q, k0, k1):
    """K range [k0, k1) of a form (multiples of 64), as a form of its own."""
    return make_form(q.R, k1 - k0, q.nibbles()[:, k0:k1], q.scales_rm[:, k0 // 16:k1 // 16], q.s_t)


@pytest.mark.parametrize("mode,kind", [(1, "grad"), (0, "act")])
@pytest.mark.parametrize("T,n,shards", [(512, 768, 2), (384, 320, 3)])
def test_shards_equal_slices_of_the_whole(mode, kind, T, n, shards):
    m = nv()
    t = synth.grad_output(T, n, seed=2) if kind == "grad" else synth.activations(T, n, seed=0, outlier_frac=0.01)
    bits = synth.bf16_bits(t)
    rht_seed, sr_seed = 13, 21
    q_row = oracle.quantize(bits, along=0, mode=mode, sr_seed=sr_seed, stream_id=1)
    q_col = oracle.quantize(bits, along=1, mode=mode, rht=True, rht_seed=rht_seed, sr_seed=sr_seed, stream_id=2)
    rows = T // shards
    xs = [to_device_bf16(t[i * rows:(i + 1) * rows]) for i in range(shards)]
    wss = [m.Workspace() for _ in range(shards)]
    for x, ws in zip(xs, wss):
        m.nvfp4_amax(x, True, rht_seed, ws)
    words = torch.stack([ws.amax_words() for ws in wss]).max(dim=0).values   # the ranks' MAX all-reduce
    for ws in wss:
        ws.amax_words().copy_(words)
    for i, (x, ws) in enumerate(zip(xs, wss)):
        r, c = m.nvfp4_quantize_dual_shard(x, i * rows, T, mode, rht_seed, sr_seed, 1, 2, ws=ws)
        assert_form_equal(r, _row_slice(q_row, i * rows, (i + 1) * rows), f"shard {i} row form")
        assert_form_equal(c, _k_slice(q_col, i * rows, (i + 1) * rows), f"shard {i} column form")
        assert m.nvfp4_poll(ws) == 0


def test_dp_helper_on_one_rank_equals_whole_tensor_call():
    # nvfp4_quantize_dual_dp through a one-rank NCCL group: the all-reduce is the identity, so the
    # result is nvfp4_quantize_dual's
    import torch.distributed as dist
    m = nv()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        t = synth.grad_output(256, 384, seed=5)
        x = to_device_bf16(t)
        r1, c1 = m.nvfp4_quantize_dual_dp(x, None, 0, 256, mode=1, rht_seed=3, sr_seed=4, stream_row=1, stream_col=2)
        r2, c2 = m.nvfp4_quantize_dual(x, mode=1, rht_seed=3, sr_seed=4, stream_row=1, stream_col=2)
        torch.cuda.synchronize()
        for a, b in ((r1, r2), (c1, c2)):
            assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
            assert torch.equal(a.tensor_scale, b.tensor_scale)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,d,n,shards", [(1024, 256, 384, 2), (1024, 320, 256, 4)])
def test_shard_wgrad_partials_reduce_to_the_whole_batch_dw(T, d, n, shards):
    # Data-parallel wgrad: with the amax reduced across ranks and SR indexed in the whole batch's
    # forms, each rank's dW partial is GEMM(its K range of dY^T, its K range of X^T); the fp32 sum
    # of the partials (what the ranks' reduction computes) equals the whole batch's dW within the
    # GEMM bound |err| <= 1e-5 sum_k |a_k b_k|, the sum now running over all T tokens.
    m = nv()
    x = synth.activations(T, d, seed=0, outlier_frac=0.01)
    dy = synth.grad_output(T, n, seed=2)
    rht_seed, sr_seed = 3, 4
    q_x = oracle.quantize(synth.bf16_bits(x), along=1, rht=True, rht_seed=rht_seed)
    q_dy = oracle.quantize(synth.bf16_bits(dy), along=1, mode=oracle.SR, rht=True, rht_seed=rht_seed,
                           sr_seed=sr_seed, stream_id=2)
    ref, sabs = oracle.gemm_full(q_dy, q_x)
    rows = T // shards

    def shard_forms(t, mode):
        parts = [to_device_bf16(t[i * rows:(i + 1) * rows]) for i in range(shards)]
        wss = [m.Workspace() for _ in range(shards)]
        for p, ws in zip(parts, wss):
            m.nvfp4_amax(p, True, rht_seed, ws)
        words = torch.stack([ws.amax_words() for ws in wss]).max(dim=0).values   # the ranks' MAX all-reduce
        out = []
        for i, (p, ws) in enumerate(zip(parts, wss)):
            ws.amax_words().copy_(words)
            _, c = m.nvfp4_quantize_dual_shard(p, i * rows, T, mode, rht_seed, sr_seed, 1, 2, ws=ws)
            assert m.nvfp4_poll(ws) == 0
            out.append(c)
        return out

    xc, dyc = shard_forms(x, 0), shard_forms(dy, 1)
    total = torch.zeros((n, d), dtype=torch.float32, device="cuda")
    for a, b in zip(dyc, xc):
        total += m.nvfp4_gemm(a, b, out_dtype=torch.float32)
    check_gemm(total.cpu().numpy(), ref, sabs, False, f"sum of {shards} shard dW partials")


def test_dp_linear_on_one_rank_equals_the_linear_layer():
    # DPLinear through a one-rank NCCL group: the all-reduce is the identity and the reduce-scatter
    # keeps every row, so Y, dX and dW equal nvfp4_linear_fwd/bwd bit for bit
    import torch.distributed as dist
    m = nv()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        T, d, n = 256, 320, 512
        x, w, dy = (to_device_bf16(t) for t in (synth.activations(T, d, seed=0, outlier_frac=0.01),
                                                 synth.weights(n, d, seed=1), synth.grad_output(T, n, seed=2)))
        ctx = m.LinearContext(T, d, n, rht_seed=3)
        y1 = m.nvfp4_linear_fwd(ctx, x, w)
        dx1, dw1 = m.nvfp4_linear_bwd(ctx, dy, 4)
        dp = m.DPLinear(T, d, n, rht_seed=3)
        y2 = dp.fwd(x, w)
        dx2 = dp.bwd(dy, 4)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2) and torch.equal(dx1, dx2) and torch.equal(dw1, dp.dw)
    finally:
        dist.destroy_process_group()
