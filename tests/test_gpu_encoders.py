"""The device encoders of the CUDA path against the CPU oracle, exhaustively over their input
ranges, and the device Philox4x32-10 against the oracle and against cuRAND's independent
Philox4_32_10 (which pins the oracle's generator to a third implementation)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import checks, parallel_map

pytestmark = pytest.mark.gpu

CHUNK = 1 << 26


def _oracle_chunked(fn, x: np.ndarray, out_dtype):
    out = np.empty(x.shape, out_dtype)
    step = 1 << 21
    def work(i):
        out[i:i + step] = fn(x[i:i + step])
    parallel_map(work, range(0, x.size, step))
    return out


def _sweep(lo_bits: int, hi_bits: int, gpu_fn, ora_fn, out_dtype, torch_dtype, transform=None):
    for start in range(lo_bits, hi_bits, CHUNK):
        n = min(CHUNK, hi_bits - start)
        dev = torch.empty(n, dtype=torch_dtype, device="cuda")
        assert gpu_fn(start, n, ctypes.c_void_p(dev.data_ptr())) == 0
        got = dev.cpu().numpy()
        x = (np.arange(n, dtype=np.uint64) + np.uint64(start)).astype(np.uint32).view(np.float32)
        want = _oracle_chunked(ora_fn, x, out_dtype)
        if transform is not None:
            got = transform(got)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, f"bits {start + int(bad[0]):#010x}: gpu {got[bad[0]]} oracle {want[bad[0]]}"


def test_e2m1_rne_all_finite_fp32():
    L = checks()
    both = lambda b: np.where((b & 15) == (b >> 4), b & 15, 255).astype(np.uint8)   # both nibbles must agree
    for lo, hi in ((0x00000000, 0x7F800000), (0x80000000, 0xFF800000)):
        _sweep(lo, hi, L.chk_e2m1_rne, oracle.e2m1_rne, np.uint8, torch.uint8, transform=both)


def test_e2m1_eight_per_word_packing():
    # the quantize kernels convert eight values into one code word (byte q = pair q, first value
    # in the low nibble): every nibble position against the oracle's RNE code of its value, over
    # random fp32 bit patterns and the grid's ties, values and neighbours in every position
    L = checks()
    rng = np.random.default_rng(8)
    grid = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7, 1e30, np.inf, np.nan], np.float32)
    near = np.concatenate([np.nextafter(grid, np.float32(np.inf)), np.nextafter(grid, np.float32(-np.inf))])
    special = np.concatenate([grid, -grid, near, -near])
    special = np.concatenate([np.roll(special, k) for k in range(8)])   # each value in every nibble position
    x = np.concatenate([rng.integers(0, 1 << 32, 1 << 22, dtype=np.uint64).astype(np.uint32).view(np.float32),
                        special])
    x = np.concatenate([x, np.zeros(-x.size % 8, np.float32)])
    xd = torch.from_numpy(x).cuda()
    out = torch.empty(x.size // 8, dtype=torch.int32, device="cuda")
    assert L.chk_e2m1x8(ctypes.c_void_p(xd.data_ptr()), x.size // 8, ctypes.c_void_p(out.data_ptr())) == 0
    b = out.cpu().numpy().view(np.uint8)                         # little-endian: byte q of word i at 4i + q
    got = np.stack([b & 15, b >> 4], axis=1).reshape(-1)         # low nibble first
    finite = np.isfinite(x)
    want = np.zeros(x.size, np.uint8)
    want[finite] = oracle.e2m1_rne(x[finite])
    assert np.array_equal(got[finite], want[finite])


def test_e2m1_sr_threshold_all_below_six():
    L = checks()
    _sweep(0x00000000, 0x40C00000, L.chk_e2m1_sr_threshold, oracle.e2m1_sr_threshold, np.uint32, torch.int32,
           transform=lambda a: a.view(np.uint32))


def test_e2m1_sr_codes_random():
    L = checks()
    rng = np.random.default_rng(3)
    n = 1 << 22
    x = (rng.standard_normal(n) * rng.choice([0.1, 1, 3, 10], n)).astype(np.float32)
    r = rng.integers(0, 1 << 16, n, dtype=np.uint32)
    xd, rd = torch.from_numpy(x).cuda(), torch.from_numpy(r.view(np.int32)).cuda()
    out = torch.empty(n, dtype=torch.uint8, device="cuda")
    assert L.chk_e2m1_sr(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(rd.data_ptr()), n, ctypes.c_void_p(out.data_ptr())) == 0
    assert np.array_equal(out.cpu().numpy(), oracle.e2m1_sr(x, r))


def test_e4m3_all_nonnegative_fp32():
    L = checks()
    _sweep(0x00000000, 0x7F800001, L.chk_e4m3, oracle.e4m3_rne_sat, np.uint8, torch.uint8)


def test_e4m3_decode_all_codes():
    L = checks()
    out = torch.empty(128, dtype=torch.float32, device="cuda")
    assert L.chk_e4m3_decode(ctypes.c_void_p(out.data_ptr())) == 0
    got = out.cpu().numpy()[:127].astype(np.float64)
    want = np.array([oracle.e4m3_value(c) for c in range(127)])
    assert np.array_equal(got, want)


@pytest.mark.parametrize("seed,stream", [(0, 1), (0x123456789ABCDEF, 2), (2 ** 64 - 1, 3), (42, 0)])
def test_philox_matches_oracle_and_curand(seed, stream):
    L = checks()
    n = 1 << 16
    for g0 in (0, (1 << 32) - 5, 123456789012):
        dev = torch.empty(4 * n, dtype=torch.int32, device="cuda")
        cur = torch.empty(4 * n, dtype=torch.int32, device="cuda")
        assert L.chk_philox(seed, stream, g0, n, ctypes.c_void_p(dev.data_ptr())) == 0
        assert L.chk_curand_philox(seed, stream, g0, n, ctypes.c_void_p(cur.data_ptr())) == 0
        ours = dev.cpu().numpy().view(np.uint32).reshape(n, 4)
        theirs = cur.cpu().numpy().view(np.uint32).reshape(n, 4)
        want = oracle.philox_blocks(seed, stream, g0, n)
        assert np.array_equal(theirs, want), "oracle Philox disagrees with cuRAND"
        assert np.array_equal(ours, want), "device Philox disagrees with the oracle"


def test_rht16_matches_oracle_bit_exact():
    L = checks()
    rng = np.random.default_rng(8)
    n = 4096
    x = (rng.standard_normal((n, 16)) * rng.choice([1e-30, 1e-3, 1, 1e4], (n, 1))).astype(np.float32)
    for seed in (0, 7, 99):
        signs = oracle.rht_signs(seed)
        xd = torch.from_numpy(x).cuda()
        out = torch.empty_like(xd)
        assert L.chk_rht16(ctypes.c_void_p(xd.data_ptr()), n, signs, ctypes.c_void_p(out.data_ptr())) == 0
        got = out.cpu().numpy()
        want = np.stack([oracle.rht16(r, signs) for r in x])
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_e2m1_sr_codes_at_every_threshold():
    # for every fp32 |u| in [0, 6) (and its negative), the device SR encode at the two 16-bit
    # random values around the oracle's threshold t(u): r = t - 1 must round up (when t > 0),
    # r = t must not; a monotone decision in r is then pinned completely
    L = checks()
    for lo, hi in ((0x00000000, 0x40C00000),):
        for start in range(lo, hi, CHUNK):
            n = min(CHUNK, hi - start)
            x = (np.arange(n, dtype=np.uint64) + np.uint64(start)).astype(np.uint32).view(np.float32)
            t = _oracle_chunked(oracle.e2m1_sr_threshold, x, np.uint32)
            for sign in (1.0, -1.0):
                xs = (x * np.float32(sign)).astype(np.float32)
                for r in (np.clip(t.astype(np.int64) - 1, 0, 65535).astype(np.uint32), np.minimum(t, 65535).astype(np.uint32)):
                    xd = torch.from_numpy(xs).cuda()
                    rd = torch.from_numpy(r.view(np.int32)).cuda()
                    out = torch.empty(n, dtype=torch.uint8, device="cuda")
                    assert L.chk_e2m1_sr(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(rd.data_ptr()), n,
                                         ctypes.c_void_p(out.data_ptr())) == 0
                    got = out.cpu().numpy()
                    want = np.empty(n, np.uint8)
                    step = 1 << 21
                    def work(i):
                        want[i:i + step] = oracle.e2m1_sr(xs[i:i + step], r[i:i + step])
                    parallel_map(work, range(0, n, step))
                    bad = np.nonzero(got != want)[0]
                    assert bad.size == 0, f"u={xs[bad[0]]!r} r={r[bad[0]]}: gpu {got[bad[0]]} oracle {want[bad[0]]}"


@pytest.mark.parametrize("seed", [0, 7, 0x123456789ABCDEF, 2 ** 64 - 1])
def test_rht_signs_are_the_low_half_of_curands_block_at_stream_3(seed):
    # The RHT sign word is the low 16 bits of word 0 of the Philox4x32-10 block at counter
    # (0, 0, 3, 0) under the seed: computed here by cuRAND's own Philox4_32_10 (subsequence 3,
    # offset 0), an implementation the oracle shares nothing with.
    L = checks()
    cur = torch.empty(4, dtype=torch.int32, device="cuda")
    assert L.chk_curand_philox(seed, 3, 0, 1, ctypes.c_void_p(cur.data_ptr())) == 0
    word0 = int(cur.cpu().numpy().view(np.uint32)[0])
    assert oracle.rht_signs(seed) == word0 & 0xFFFF
