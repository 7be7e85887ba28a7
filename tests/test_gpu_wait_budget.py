"""The GEMM's device-side waits are bounded: a wait that runs out of its budget raises the
timeout flag, the kernel drains its own copies and MMAs on a fixed internal budget, frees its
tensor memory and returns, and the context stays usable.

The budget is set to 1 ns for one long-K GEMM on the 1-SM kernel (M = 128).  Its epilogue warps
wait for an accumulator that needs ~1 ms of MMAs, far longer than their first polls, so their wait
runs out for certain; nvfp4_poll must report NVFP4_ERR_TIMEOUT (8).  With the default budget
restored, the next GEMMs (both kernels) are exact again."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import make_form, nv, upload_form

pytestmark = pytest.mark.gpu

POW2_SCALES = np.array([0x30, 0x38, 0x40], np.uint8)


def _exact_operand(rng, R, K):
    nib = rng.integers(0, 16, size=(R, K), dtype=np.uint8)
    sc = rng.choice(POW2_SCALES, size=(R, K // 16))
    return make_form(R, K, nib, sc, 0.125)


def _long_k_operand(m, R, K, seed):
    t = m.NVFP4Tensor.empty(R, K)
    g = torch.Generator(device="cuda").manual_seed(seed)
    t.codes.copy_(torch.randint(0, 256, t.codes.shape, generator=g, device="cuda", dtype=torch.int32).to(torch.uint8))
    t.scales.fill_(0x38)     # 1.0
    t.tensor_scale.fill_(1.0)
    return t


def _exact_gemm_ok(m, M, N, K, seed):
    rng = np.random.default_rng(seed)
    a, b = _exact_operand(rng, M, K), _exact_operand(rng, N, K)
    ws = m.Workspace()
    d = m.nvfp4_gemm(upload_form(a), upload_form(b), out_dtype=torch.float32, ws=ws)
    assert m.nvfp4_poll(ws) == 0
    ref, _ = oracle.gemm_full(a, b)
    return np.array_equal(d.cpu().numpy().astype(np.float64), ref)


def test_budget_expiry_is_reported_and_the_next_gemm_is_exact():
    m = nv()
    assert _exact_gemm_ok(m, 128, 256, 256, 1)
    M, N, K = 128, 256, 1 << 19
    a, b = _long_k_operand(m, M, K, 1), _long_k_operand(m, N, K, 2)
    ws = m.Workspace()
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    m.nvfp4_set_wait_budget_ns(1)
    try:
        m.nvfp4_gemm(a, b, out=out, ws=ws)
        status = m.nvfp4_poll(ws)
    finally:
        m.nvfp4_set_wait_budget_ns(0)     # back to the default
    assert status == 8, f"expected NVFP4_ERR_TIMEOUT, got {status}"
    assert m.nvfp4_poll(ws) == 0          # the flag was cleared by the poll
    # the same long GEMM with the default budget completes without a flag
    m.nvfp4_gemm(a, b, out=out, ws=ws)
    assert m.nvfp4_poll(ws) == 0
    assert _exact_gemm_ok(m, 128, 256, 256, 2)      # 1-SM kernel
    assert _exact_gemm_ok(m, 256, 512, 1024, 3)     # SM-pair kernel
