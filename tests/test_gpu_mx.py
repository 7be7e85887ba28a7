"""MXFP4, the format the pages compare NVFP4 with (gist.science "Pretraining Large Language
Models with NVFP4", 2.A: blocks of 32 elements, UE8M0 power-of-two scales, no tensor scale).
The CUDA quantizer against the oracle bit for bit (codes and swizzled scales, padding included),
row and column forms, RNE and SR; the kind::mxf4 GEMM against the oracle's fp64 GEMM: exactly on
dyadic operands (which pins the scale-tile placement and the per-MMA scale selection) and within
|D - D_ref| <= 1e-5 sum_k |a_k b_k| (+ 2^-8 |D_ref| for bf16 output) on quantized data."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import bf16_to_f64, check_gemm, nv, to_device_bf16

pytestmark = pytest.mark.gpu


def _oracle_form(bits, along, mode, sr_seed, stream_id):
    src = np.ascontiguousarray(bits.T) if along else bits
    codes, scales = oracle.quantize_mx(src, mode=mode, sr_seed=sr_seed, stream_id=stream_id)
    return codes, scales, oracle.mx_scales_swizzled(scales, src.shape[1])


def _assert_mx_equal(g, codes, sw, what):
    torch.cuda.synchronize()
    got = g.codes[: codes.size].cpu().numpy().reshape(codes.shape)
    bad = np.argwhere(got != codes)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first {bad[0].tolist()}"
    gs = g.scales[: sw.size].cpu().numpy()
    bads = np.nonzero(gs != sw)[0]
    assert bads.size == 0, f"{what}: {bads.size} scale bytes differ, first at {bads[0]}: gpu {gs[bads[0]]} oracle {sw[bads[0]]}"


@pytest.mark.parametrize("rows,cols", [(256, 256), (112, 544), (64, 1056), (1040, 96), (300, 160)])
@pytest.mark.parametrize("mode", [0, 1])
def test_mx_row_form(rows, cols, mode):
    m = nv()
    t = synth.activations(rows, cols, seed=rows + cols, outlier_frac=0.02)
    g = m.nvfp4_mx_quantize(to_device_bf16(t), along=0, mode=mode, sr_seed=7, stream_id=1)
    codes, _, sw = _oracle_form(synth.bf16_bits(t), 0, mode, 7, 1)
    _assert_mx_equal(g, codes, sw, f"MX row form {rows}x{cols} mode {mode}")


@pytest.mark.parametrize("rows,cols", [(256, 256), (96, 160), (320, 48), (64, 1040), (160, 528)])
@pytest.mark.parametrize("mode", [0, 1])
def test_mx_column_form(rows, cols, mode):
    m = nv()
    t = synth.grad_output(rows, cols, seed=3) if mode else synth.activations(rows, cols, seed=3, outlier_frac=0.02)
    g = m.nvfp4_mx_quantize(to_device_bf16(t), along=1, mode=mode, sr_seed=9, stream_id=2)
    codes, _, sw = _oracle_form(synth.bf16_bits(t), 1, mode, 9, 2)
    _assert_mx_equal(g, codes, sw, f"MX column form {rows}x{cols} mode {mode}")


# both forms from one read: each against the oracle, bit for bit; shapes with ragged 64-row and
# 256-column tiles (multiples of 32 only, e.g. a last tile of 32 columns)
@pytest.mark.parametrize("rows,cols", [(256, 256), (96, 160), (320, 544), (64, 1056), (1056, 96)])
@pytest.mark.parametrize("mode", [0, 1])
def test_mx_dual_forms(rows, cols, mode):
    m = nv()
    t = synth.grad_output(rows, cols, seed=5) if mode else synth.activations(rows, cols, seed=5, outlier_frac=0.02)
    gr, gc = m.nvfp4_mx_quantize_dual(to_device_bf16(t), mode=mode, sr_seed=11, stream_row=1, stream_col=2)
    bits = synth.bf16_bits(t)
    codes, _, sw = _oracle_form(bits, 0, mode, 11, 1)
    _assert_mx_equal(gr, codes, sw, f"MX dual, row form {rows}x{cols} mode {mode}")
    codes, _, sw = _oracle_form(bits, 1, mode, 11, 2)
    _assert_mx_equal(gc, codes, sw, f"MX dual, column form {rows}x{cols} mode {mode}")


def test_mx_dual_full_size_equals_two_single_calls():
    # the 8192 x 20480 gradient of the layer, SR: both forms equal the one-form calls'
    m = nv()
    g = torch.Generator(device="cpu").manual_seed(21)
    x = (torch.randn((8192, 20480), generator=g) * 1e-2).to(torch.bfloat16).cuda()
    gr, gc = m.nvfp4_mx_quantize_dual(x, mode=1, sr_seed=3, stream_row=1, stream_col=2)
    r = m.nvfp4_mx_quantize(x, along=0, mode=1, sr_seed=3, stream_id=1)
    c = m.nvfp4_mx_quantize(x, along=1, mode=1, sr_seed=3, stream_id=2)
    torch.cuda.synchronize()
    for a, b in ((gr, r), (gc, c)):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


def test_mx_dual_shape_errors():
    m = nv()
    x = torch.zeros((48, 256), dtype=torch.bfloat16, device="cuda")   # rows % 32 != 0
    with pytest.raises(m.NVFP4Error) as e:
        m.nvfp4_mx_quantize_dual(x)
    assert e.value.status == 3


def test_mx_extreme_magnitudes():
    # scales at both ends of the UE8M0 range: huge, tiny (bf16 subnormal) and zero blocks
    m = nv()
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x[0:8] *= 1e37
    x[8:16] *= 1e-39
    x[16:24] = 0.0
    x[24, 5] = -0.0
    t = torch.from_numpy(x).to(torch.bfloat16)
    for along in (0, 1):
        g = m.nvfp4_mx_quantize(to_device_bf16(t), along=along)
        codes, _, sw = _oracle_form(synth.bf16_bits(t), along, 0, 0, 0)
        _assert_mx_equal(g, codes, sw, f"extremes along {along}")


def _upload(codes, sw, R, K):
    m = nv()
    t = m.MXTensor.empty(R, K)
    t.codes[: codes.size].copy_(torch.from_numpy(codes.reshape(-1)))
    t.scales.zero_()
    t.scales[: sw.size].copy_(torch.from_numpy(sw))
    return t


def _dyadic_operand(rng, R, K):
    nib = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.choice(np.array([125, 126, 127, 128, 129], np.uint8), size=(R, K // 32))
    return codes, scales


@pytest.fixture(params=["1sm", "2sm"])
def variant(request, monkeypatch):
    monkeypatch.setenv("NVFP4_GEMM_VARIANT", request.param)
    return request.param


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (128, 256, 512), (256, 512, 1024), (384, 256, 512),
                                   (200, 328, 96), (1, 8, 32), (300, 200, 160), (512, 384, 2048)])
def test_mx_gemm_exact_dyadic(M, N, K, variant):
    m = nv()
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    (ca, sa), (cb, sb) = _dyadic_operand(rng, M, K), _dyadic_operand(rng, N, K)
    d = m.nvfp4_mx_gemm(_upload(ca, oracle.mx_scales_swizzled(sa, K), M, K),
                        _upload(cb, oracle.mx_scales_swizzled(sb, K), N, K), out_dtype=torch.float32)
    ref, _ = oracle.gemm_mx(ca, sa, cb, sb)
    got = d.cpu().numpy().astype(np.float64)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} differ; first {bad[0].tolist()}: gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("M,N,K", [(512, 768, 1280), (256, 256, 256), (64, 1024, 2048)])
@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_mx_gemm_on_quantized_layer_data(M, N, K, out):
    # X N(0,1) with outlier channels and W N(0,0.02), both quantized to MXFP4 on the GPU (the
    # forms are checked against the oracle first), then the fprop GEMM
    m = nv()
    x = synth.activations(M, K, seed=M, outlier_frac=0.01)
    w = synth.weights(N, K, seed=N)
    xq = m.nvfp4_mx_quantize(to_device_bf16(x))
    wq = m.nvfp4_mx_quantize(to_device_bf16(w))
    (cx, sx, swx), (cw, sw_, sww) = (_oracle_form(synth.bf16_bits(t), 0, 0, 0, 0) for t in (x, w))
    _assert_mx_equal(xq, cx, swx, "X")
    _assert_mx_equal(wq, cw, sww, "W")
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    d = m.nvfp4_mx_gemm(xq, wq, out_dtype=dt)
    ref, sabs = oracle.gemm_mx(cx, sx, cw, sw_)
    check_gemm(bf16_to_f64(d) if out == "bf16" else d.cpu().numpy(), ref, sabs, out == "bf16", f"MX {M}x{N}x{K}")
