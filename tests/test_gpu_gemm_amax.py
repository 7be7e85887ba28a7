"""The GEMM whose epilogue also produces its bf16 output's amax (nvfp4_gemm_amax): the plain amax
and the amax of the 16-point RHT along the rows, the two words the amax pass of the quantize call
that reads the output would compute (gist.science "Pretraining Large Language Models with NVFP4",
2.A: the FP32 tensor scale comes from the amax of the whole tensor).  The words must equal, bit for
bit, those of nvfp4_amax over the stored output, and the output must equal nvfp4_gemm's."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _operands(m, M, N, K, seed):
    x = to_device_bf16(synth.activations(M, K, seed=seed, outlier_frac=0.01))
    w = to_device_bf16(synth.weights(N, K, seed=seed + 1))
    return m.nvfp4_quantize(x, along=0), m.nvfp4_quantize(w, along=0, block=m.BLOCK_16x16 if N % 16 == 0 else m.BLOCK_1x16)


def _oracle_words(d: torch.Tensor, rht_seed: int) -> list:
    """The amax words of a quantize call over d: max |d| (its definition) and the oracle's amax of
    the RHT form (the transform along the rows)."""
    d = d.contiguous()
    bits = d.view(torch.int16).cpu().numpy().view(np.uint16)
    plain = np.abs(d.float().cpu().numpy()).max()
    rht = oracle.quantize(bits, along=1, rht=True, rht_seed=rht_seed).amax
    return [int(np.float32(plain).view(np.int32)), int(np.float32(rht).view(np.int32))]


# SM-pair tiles (M >= 256, ragged M and N), the 1-SM kernel (M < 256), an odd N (a column pair
# straddling the edge), and a K that is not a multiple of 256
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (528, 320, 192), (96, 200, 128), (160, 203, 96), (784, 1040, 320)])
@pytest.mark.parametrize("rht_seed", [0, 5])
def test_epilogue_amax_equals_the_amax_pass(M, N, K, rht_seed):
    m = nv()
    a, b = _operands(m, M, N, K, seed=M + N)
    ws_amax, ws = m.Workspace(), m.Workspace()
    ld = -(-N // 8) * 8   # rows of D 16-byte aligned
    d = m.nvfp4_gemm_amax(a, b, ws_amax, rht_seed=rht_seed, out=torch.empty((M, ld), dtype=torch.bfloat16,
                                                                                device="cuda")[:, :N], ws=ws)
    ref = m.nvfp4_gemm(a, b, out=torch.empty((M, ld), dtype=torch.bfloat16, device="cuda")[:, :N], ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(d, ref), "output differs from nvfp4_gemm"
    got = ws_amax.amax_words().cpu().tolist()
    assert got == _oracle_words(ref, rht_seed), f"amax words {got} vs the oracle {_oracle_words(ref, rht_seed)}"
    if N % 16 == 0:   # and the product's own amax pass over the stored output
        ws_ref = m.Workspace()
        m.nvfp4_amax(ref.contiguous(), True, rht_seed, ws_ref)
        assert ws_ref.amax_words().cpu().tolist() == got
        assert m.nvfp4_poll(ws_ref) == 0
    assert m.nvfp4_poll(ws) == 0


def test_quantize_from_the_epilogue_amax_equals_the_two_pass_quantize():
    # the words feed the quantize pass directly: both forms equal nvfp4_quantize_dual's
    m = nv()
    M, N, K = 512, 768, 256
    a, b = _operands(m, M, N, K, seed=3)
    ws_amax = m.Workspace()
    d = m.nvfp4_gemm_amax(a, b, ws_amax, rht_seed=9)
    for mode in (m.RNE, m.SR):
        r1, c1 = m.nvfp4_quantize_dual_shard(d, 0, M, mode, 9, 4, 1, 2, ws=ws_amax)
        r2, c2 = m.nvfp4_quantize_dual(d, mode=mode, rht_seed=9, sr_seed=4, stream_row=1, stream_col=2)
        torch.cuda.synchronize()
        for x, y in ((r1, r2), (c1, c2)):
            assert torch.equal(x.codes, y.codes) and torch.equal(x.scales, y.scales)
            assert torch.equal(x.tensor_scale, y.tensor_scale)


def test_full_size_fprop_epilogue_amax():
    # the 8192 x 20480 x 5120 fprop of the layer
    m = nv()
    g = torch.Generator(device="cpu").manual_seed(12)
    x = (torch.randn((8192, 5120), generator=g) * 2.0).to(torch.bfloat16).cuda()
    w = (torch.randn((20480, 5120), generator=g) * 0.02).to(torch.bfloat16).cuda()
    a = m.nvfp4_quantize(x, along=0)
    b = m.nvfp4_quantize(w, along=0, block=m.BLOCK_16x16)
    del x, w
    ws_amax, ws_ref = m.Workspace(), m.Workspace()
    d = m.nvfp4_gemm_amax(a, b, ws_amax, rht_seed=1)
    ref = m.nvfp4_gemm(a, b)
    m.nvfp4_amax(ref, True, 1, ws_ref)
    torch.cuda.synchronize()
    assert torch.equal(d, ref)
    assert torch.equal(ws_amax.amax_words().cpu(), ws_ref.amax_words().cpu())


def test_epilogue_amax_argument_errors():
    m = nv()
    a, b = _operands(m, 104, 64, 64, seed=1)   # M % 16 != 0
    with pytest.raises(m.NVFP4Error) as e:
        m.nvfp4_gemm_amax(a, b, m.Workspace())
    assert e.value.status == 3


def test_stacked_layers_with_fed_amax_equal_the_plain_stack():
    # two layers, the second reading the first's y: with feed() the first's fprop GEMM writes y's
    # amax words for the second's quantize and the second's dgrad GEMM writes dx's for the first's
    # backward, so both skip an amax pass; every output equals the stack without it, bit for bit
    m = nv()
    T, d, n = 256, 320, 512
    x = to_device_bf16(synth.activations(T, d, seed=0, outlier_frac=0.01))
    w1 = to_device_bf16(synth.weights(n, d, seed=1))
    w2 = to_device_bf16(synth.weights(d, n, seed=3))
    dy2 = to_device_bf16(synth.grad_output(T, d, seed=4))

    def run(fed):
        l1 = m.LinearContext(T, d, n, rht_seed=3)
        l2 = m.LinearContext(T, n, d, rht_seed=8)
        if fed:
            l1.feed(l2)
        y1 = m.nvfp4_linear_fwd(l1, x, w1)
        l2.amax_ready = fed
        y2 = m.nvfp4_linear_fwd(l2, y1, w2)
        dx2, dw2 = m.nvfp4_linear_bwd(l2, dy2, 5)
        l1.amax_ready = fed
        dx1, dw1 = m.nvfp4_linear_bwd(l1, dx2, 6)
        torch.cuda.synchronize()
        assert m.nvfp4_poll(l1.ws) == 0 and m.nvfp4_poll(l2.ws) == 0
        assert not l1.amax_ready and not l2.amax_ready
        return [y1, y2, dx2, dw2, dx1, dw1]

    for name, a, b in zip(("y1", "y2", "dx2", "dw2", "dx1", "dw1"), run(False), run(True)):
        assert torch.equal(a, b), name


def test_non_finite_output_raises_the_flag():
    # operands near the top of bf16's range overflow the fp32 accumulation to inf: the epilogue's
    # plain amax sees it and raises the non-finite flag in the call's workspace, as the amax pass
    # over the stored output does in its own
    m = nv()
    M, N, K = 256, 256, 256
    x = torch.full((M, K), 1e19, dtype=torch.bfloat16, device="cuda")
    w = torch.full((N, K), 1e19, dtype=torch.bfloat16, device="cuda")
    a, b = m.nvfp4_quantize(x, along=0), m.nvfp4_quantize(w, along=0, block=m.BLOCK_16x16)
    ws_amax, ws, ws_ref = m.Workspace(), m.Workspace(), m.Workspace()
    d = m.nvfp4_gemm_amax(a, b, ws_amax, ws=ws)
    m.nvfp4_amax(d, True, 0, ws_ref)
    torch.cuda.synchronize()
    assert torch.isinf(d.float()).all()
    assert m.nvfp4_poll(ws) == 7 and m.nvfp4_poll(ws_ref) == 7
    assert int(ws_amax.amax_words()[0]) == 0x7F800000
