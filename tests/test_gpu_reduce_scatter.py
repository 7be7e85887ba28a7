"""The wgrad GEMM with its reduce-scatter fused into the epilogue (nvfp4_gemm_reduce_scatter):
each output tile is added (fp32, by the TMA engine) into the row shard of its owner.

Data-parallel weight gradient: dW is a sum over tokens (gist.science "Pretraining Large Language
Models with NVFP4", 2.B: the wgrad GEMM contracts over the token dimension), so each rank's GEMM
over its own tokens gives a K-partial and the ranks' partials are summed, each rank keeping a row
range.  On one GPU the ranks are emulated by several calls into the same local shard buffers, one
after the other on one stream (no kernel waits on another)."""
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_gemm, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _dp_wgrad_forms(m, x, dy, ranks, rht_seed, sr_seed):
    """Each emulated rank's wgrad forms (dY^T and X^T of its tokens), with the tensor scales of
    the whole batch (MAX of the ranks' amax words) and SR indexed in the whole batch's forms."""
    T = x.shape[0]
    rows = T // ranks

    def forms(t, mode):
        parts = [to_device_bf16(t[i * rows:(i + 1) * rows]) for i in range(ranks)]
        wss = [m.Workspace() for _ in range(ranks)]
        for p, ws in zip(parts, wss):
            m.nvfp4_amax(p, True, rht_seed, ws)
        words = torch.stack([ws.amax_words() for ws in wss]).max(dim=0).values
        out = []
        for i, (p, ws) in enumerate(zip(parts, wss)):
            ws.amax_words().copy_(words)
            _, c = m.nvfp4_quantize_dual_shard(p, i * rows, T, mode, rht_seed, sr_seed, 1, 2, ws=ws)
            assert m.nvfp4_poll(ws) == 0
            out.append(c)
        return out

    return forms(dy, 1), forms(x, 0)


# (T, d, n, ranks, owners): n = M rows of dW (the SM-pair kernel for n >= 256, the 1-SM kernel
# below), d = N columns (ragged against the 64-column store boxes in the last case), owner shares
# a multiple of 32 rows with a shorter last share where n is not a multiple of the share
@pytest.mark.parametrize("T,d,n,ranks,owners", [(1024, 256, 384, 2, 2), (1024, 320, 256, 4, 3),
                                                 (512, 208, 192, 2, 2), (768, 272, 640, 3, 8)])
def test_fused_reduce_scatter_equals_the_sum_of_partials(T, d, n, ranks, owners):
    m = nv()
    x = synth.activations(T, d, seed=0, outlier_frac=0.01)
    dy = synth.grad_output(T, n, seed=2)
    rht_seed, sr_seed = 3, 4
    dyc, xc = _dp_wgrad_forms(m, x, dy, ranks, rht_seed, sr_seed)
    share = -(-n // owners)
    share = -(-share // 32) * 32
    owners = -(-n // share)
    shards = [torch.zeros((min(share, n - o * share), d), dtype=torch.float32, device="cuda") for o in range(owners)]
    for a, b in zip(dyc, xc):
        m.nvfp4_gemm_reduce_scatter(a, b, shards, share)
    # the same partials stored by nvfp4_gemm and summed in rank order by fp32 adds: the fused adds
    # run in that order too (one stream), so the shards equal that sum bit for bit
    total = torch.zeros((n, d), dtype=torch.float32, device="cuda")
    for a, b in zip(dyc, xc):
        total += m.nvfp4_gemm(a, b, out_dtype=torch.float32)
    fused = torch.cat(shards, dim=0)
    torch.cuda.synchronize()
    assert torch.equal(fused, total), "fused reduce-scatter differs from the stored partials' sum"
    # and against the oracle's whole-batch dW within the GEMM bound
    q_x = oracle.quantize(synth.bf16_bits(x), along=1, rht=True, rht_seed=rht_seed)
    q_dy = oracle.quantize(synth.bf16_bits(dy), along=1, mode=oracle.SR, rht=True, rht_seed=rht_seed,
                           sr_seed=sr_seed, stream_id=2)
    ref, sabs = oracle.gemm_full(q_dy, q_x)
    check_gemm(fused.cpu().numpy(), ref, sabs, False, f"{ranks} ranks reduce-scattered to {owners} owners")


@pytest.mark.parametrize("M,N,K", [(512, 320, 256), (128, 200, 192)])
def test_one_owner_accumulates_into_a_strided_buffer(M, N, K):
    # one owner with owner_rows >= M: D is added into an existing fp32 buffer (gradient
    # accumulation); the buffer is a column window of a wider one, whose other columns stay as
    # they were
    m = nv()
    a = to_device_bf16(synth.activations(M, K, seed=7, outlier_frac=0.01))
    b = to_device_bf16(synth.weights(N, K, seed=8))
    qa, qb = m.nvfp4_quantize(a, along=0), m.nvfp4_quantize(b, along=0)
    g = torch.Generator(device="cpu").manual_seed(9)
    wide = torch.randn((M, N + 12), generator=g, dtype=torch.float32).cuda()
    before = wide.clone()
    acc = wide[:, 4:4 + N]
    m.nvfp4_gemm_reduce_scatter(qa, qb, [acc], -(-M // 32) * 32)
    d = m.nvfp4_gemm(qa, qb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(acc, before[:, 4:4 + N] + d)
    assert torch.equal(wide[:, :4], before[:, :4]) and torch.equal(wide[:, 4 + N:], before[:, 4 + N:])


def test_full_size_wgrad_into_zeroed_shards_equals_the_stored_gemm():
    # the 20480 x 5120 x 8192 wgrad GEMM of the 8192-token layer: adds into zeroed shards of
    # 8 owners (2560 rows each) give D bit for bit (0 + D = D; the same kernel and order)
    m = nv()
    T, d, n = 8192, 5120, 20480
    g = torch.Generator(device="cpu").manual_seed(11)
    x = (torch.randn((T, d), generator=g) * 2.0).to(torch.bfloat16).cuda()
    dy = (torch.randn((T, n), generator=g) * 1e-3).to(torch.bfloat16).cuda()
    _, xc = m.nvfp4_quantize_dual(x, mode=0, rht_seed=3)
    _, dyc = m.nvfp4_quantize_dual(dy, mode=1, rht_seed=3, sr_seed=4, stream_row=1, stream_col=2)
    del x, dy
    share = n // 8
    shards = [torch.zeros((share, d), dtype=torch.float32, device="cuda") for _ in range(8)]
    m.nvfp4_gemm_reduce_scatter(dyc, xc, shards, share)
    ref = m.nvfp4_gemm(dyc, xc, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for o in range(8):
        assert torch.equal(shards[o], ref[o * share:(o + 1) * share]), f"owner {o}"


def test_reduce_scatter_argument_errors():
    m = nv()
    a = m.nvfp4_quantize(to_device_bf16(synth.activations(256, 128, seed=1, outlier_frac=0.0)), along=0)
    b = m.nvfp4_quantize(to_device_bf16(synth.weights(64, 128, seed=2)), along=0)
    sh = [torch.zeros((128, 64), dtype=torch.float32, device="cuda") for _ in range(2)]
    bad = {
        "share not a multiple of 32": (sh, 120),
        "owner count not ceil(M / share)": (sh, 64),
        "more than 8 owners": ([torch.zeros((32, 64), dtype=torch.float32, device="cuda")] * 9, 32),
    }
    for what, (s, share) in bad.items():
        with pytest.raises(m.NVFP4Error) as e:
            m.nvfp4_gemm_reduce_scatter(a, b, s, share)
        assert e.value.status == 3, what
    with pytest.raises(ValueError):
        m.nvfp4_gemm_reduce_scatter(a, b, [t.to(torch.bfloat16) for t in sh], 128)
    with pytest.raises(ValueError):
        m.nvfp4_gemm_reduce_scatter(a, b, [sh[0], sh[1][:64]], 128)
    mis = torch.zeros((128 * 64 + 1,), dtype=torch.float32, device="cuda")[1:].view(128, 64)
    with pytest.raises(m.NVFP4Error) as e:
        m.nvfp4_gemm_reduce_scatter(a, b, [sh[0], mis], 128)
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert all(float(t.abs().max()) == 0.0 for t in sh), "a rejected call wrote a shard"


@pytest.mark.parametrize("with_group", [False, True])
def test_dp_linear_fused_reduce_on_one_rank_equals_the_linear_layer(with_group):
    # DPLinear with the reduce-scatter fused into the wgrad GEMM, over three steps (both shard
    # buffers, each reused after its zeroing): on one rank every row is its own, so dW equals
    # nvfp4_linear_bwd's bit for bit.  with_group: through a one-rank NCCL group, the shard in
    # symmetric memory and the barrier an all-reduce
    import datetime
    import socket
    import torch.distributed as dist
    m = nv()
    if with_group:
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        T, d, n = 256, 320, 512
        x, w = (to_device_bf16(t) for t in (synth.activations(T, d, seed=0, outlier_frac=0.01),
                                             synth.weights(n, d, seed=1)))
        ctx = m.LinearContext(T, d, n, rht_seed=3)
        dp = m.DPLinear(T, d, n, rht_seed=3, dw_reduce="fused")
        for step in range(3):
            dy = to_device_bf16(synth.grad_output(T, n, seed=20 + step))
            m.nvfp4_linear_fwd(ctx, x, w)
            dx1, dw1 = m.nvfp4_linear_bwd(ctx, dy, 4 + step)
            dp.fwd(x, w)
            dx2 = dp.bwd(dy, 4 + step)
            torch.cuda.synchronize()
            assert torch.equal(dx1, dx2) and torch.equal(dw1, dp.dw), f"step {step}"
    finally:
        if with_group:
            dist.destroy_process_group()
