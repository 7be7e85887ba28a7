"""Helpers shared by the GPU parity tests: move seeded inputs to the device, read quantized
forms back, upload oracle forms, and the GEMM tolerance check."""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def nv():
    import nvfp4_bit_quantized_02_b200 as m
    return m


def to_device_bf16(t_cpu: torch.Tensor) -> torch.Tensor:
    return t_cpu.contiguous().cuda()


def form_np(t):
    """(codes [R][K/2], swizzled scales (padded), tile scales or None, s_t) of a device form."""
    torch.cuda.synchronize()
    R, K = t.rows, t.k
    codes = t.codes[: R * (K // 2)].cpu().numpy().reshape(R, K // 2)
    scales = t.scales[: oracle.scales_sw_bytes(R, K)].cpu().numpy()
    tiles = None
    if t.tile_scales is not None:
        tiles = t.tile_scales[: (R // 16) * (K // 16)].cpu().numpy().reshape(R // 16, K // 16)
    st = t.tensor_scale.cpu().numpy()[0]
    return codes, scales, tiles, st


def assert_form_equal(gpu_form, q: "oracle.QForm", what=""):
    codes, scales, tiles, st = form_np(gpu_form)
    assert gpu_form.rows == q.R and gpu_form.k == q.K, what
    bad = np.argwhere(codes != q.codes)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first at {bad[0].tolist()}: gpu {codes[tuple(bad[0])]:#04x} oracle {q.codes[tuple(bad[0])]:#04x}"
    badsc = np.nonzero(scales != q.scales_sw)[0]
    assert badsc.size == 0, f"{what}: {badsc.size} scale bytes differ, first at {badsc[0]}"
    if q.tile_scales is not None and tiles is not None:
        assert np.array_equal(tiles, q.tile_scales), f"{what}: tile scales differ"
    assert np.float32(st).view(np.uint32) == np.float32(q.s_t).view(np.uint32), f"{what}: s_t {st!r} vs {q.s_t!r}"


def upload_form(q: "oracle.QForm", block: int = 0):
    """An oracle form as a device NVFP4Tensor (the GEMM's inputs taken from the oracle)."""
    m = nv()
    t = m.NVFP4Tensor.empty(q.R, q.K, block)
    t.codes[: q.codes.size].copy_(torch.from_numpy(q.codes.reshape(-1)))
    t.scales[: q.scales_sw.size].copy_(torch.from_numpy(q.scales_sw))
    if block == 1 and q.tile_scales is not None:
        t.tile_scales[: q.tile_scales.size].copy_(torch.from_numpy(q.tile_scales.reshape(-1)))
    t.tensor_scale.fill_(float(q.s_t))
    return t


def make_form(R: int, K: int, codes_nib: np.ndarray, scales_rm: np.ndarray, s_t: float) -> "oracle.QForm":
    """A QForm built directly from nibbles [R][K] and row-major scales [R][K/16]."""
    codes = (codes_nib[:, 0::2] | (codes_nib[:, 1::2] << 4)).astype(np.uint8)
    sw = np.zeros(oracle.scales_sw_bytes(R, K), np.uint8)
    rr, kk = np.meshgrid(np.arange(R), np.arange(K // 16), indexing="ij")
    nkt = (K // 16 + 3) // 4
    off = ((rr // 128) * nkt + kk // 4) * 512 + (rr % 32) * 16 + ((rr // 32) % 4) * 4 + kk % 4
    sw[off.reshape(-1)] = scales_rm.reshape(-1)
    return oracle.QForm(R, K, np.ascontiguousarray(codes), np.ascontiguousarray(scales_rm.astype(np.uint8)), sw, None,
                        1.0, float(np.float32(s_t)))


def check_gemm(d_gpu: np.ndarray, d_ref: np.ndarray, sabs: np.ndarray, bf16_out: bool, what=""):
    """|D - D_ref| <= 1e-5 * sum_k |a_k b_k| (fp32 out); bf16 out adds 2^-8 |D_ref| for the
    final rounding of the fp32 accumulator to bf16."""
    d_gpu = d_gpu.astype(np.float64)
    tol = 1e-5 * sabs + (2.0 ** -8 * np.abs(d_ref) if bf16_out else 0.0) + 1e-30
    err = np.abs(d_gpu - d_ref)
    bad = err > tol
    if bad.any():
        i = int(np.argmax(err / tol))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at flat {i}: "
                             f"gpu {d_gpu.reshape(-1)[i]!r} ref {d_ref.reshape(-1)[i]!r} tol {np.reshape(tol, -1)[i]!r}")


def sample_positions(Mo: int, No: int, seed: int):
    """Output positions checked at full size: every element of 8 full 128 x 128 tiles (the four
    corners, the centre and three seeded random tiles) plus 65536 seeded random elements."""
    tiles = [(0, 0), (0, No // 128 - 1), (Mo // 128 - 1, 0), (Mo // 128 - 1, No // 128 - 1),
             (Mo // 256, No // 256)]
    rng = np.random.default_rng(seed)
    tiles += [(int(rng.integers(0, Mo // 128)), int(rng.integers(0, No // 128))) for _ in range(3)]
    ii, jj = [], []
    for ti, tj in tiles:
        a, b = np.meshgrid(np.arange(128) + 128 * ti, np.arange(128) + 128 * tj, indexing="ij")
        ii.append(a.reshape(-1))
        jj.append(b.reshape(-1))
    ri, rj = synth.sample_indices(Mo, No, 65536, seed)
    return np.concatenate(ii + [ri]), np.concatenate(jj + [rj])


def check_gemm_sampled(out: torch.Tensor, a: "oracle.QForm", b: "oracle.QForm", bf16_out: bool, what: str, seed: int):
    """A GEMM output checked on sample_positions against the oracle's fp64 GEMM."""
    Mo, No = out.shape
    ii, jj = sample_positions(Mo, No, seed)
    ref, s = oracle.gemm_sampled(a, b, ii, jj)
    got = out[torch.from_numpy(ii).to(out.device), torch.from_numpy(jj).to(out.device)]
    check_gemm(bf16_to_f64(got) if bf16_out else got.cpu().numpy().astype(np.float64), ref, s, bf16_out, what)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


# ---------------------------------------------------------------------------------------
# test-only device-check library
# ---------------------------------------------------------------------------------------
_CHK = None


def checks():
    global _CHK
    if _CHK is None:
        import importlib.util
        spec = importlib.util.spec_from_file_location("cuda_helpers_build", os.path.join(HERE, "cuda_helpers", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        L = ctypes.CDLL(mod.build())
        vp, i64, u32, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
        L.chk_e2m1_rne.argtypes = [u32, i64, vp]
        L.chk_e2m1x8.argtypes = [vp, i64, vp]
        L.chk_e2m1_sr_threshold.argtypes = [u32, i64, vp]
        L.chk_e2m1_sr.argtypes = [vp, vp, i64, vp]
        L.chk_e4m3.argtypes = [u32, i64, vp]
        L.chk_e4m3_decode.argtypes = [vp]
        L.chk_philox.argtypes = [u64, u32, u64, i64, vp]
        L.chk_curand_philox.argtypes = [u64, u32, u64, i64, vp]
        L.chk_rht16.argtypes = [vp, i64, u32, vp]
        _CHK = L
    return _CHK


def parallel_map(fn, items, workers=None):
    workers = workers or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(workers) as ex:
        return list(ex.map(fn, items))
