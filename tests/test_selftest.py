"""Self-test entry points: the device polynomial exp2 and the bounded-wait failure path."""
import os
import re
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_attention_forward_03_b200", "csrc")


def test_header_polynomial_is_the_remez_fit():
    """The constants compiled into the kernel are the fp32-rounded Remez fit of 2^f."""
    sys.path.insert(0, CSRC)
    try:
        import fit_exp2_poly as fit
    finally:
        sys.path.remove(CSRC)
    coeffs, err = fit.remez_relative(3)
    c32 = coeffs.astype(np.float32)
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = text[text.index("ATTN_DEV float2 exp2_poly2"):]
    body = body[: body.index("return r;")]
    consts = [float(x) for x in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    # Horner order in the kernel: c3, c2, c1, c0
    assert np.array_equal(np.float32(consts[:4]), np.float32([c32[3], c32[2], c32[1], c32[0]]))
    assert err < 8e-5
    assert fit.fp32_horner_error(c32) < 8e-5


@pytest.fixture(scope="module")
def attn():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


@pytest.mark.gpu
def test_device_exp2_poly_error_bound(attn):
    import torch
    x = np.concatenate([np.linspace(-125.0, 9.0, 1_000_001), np.random.default_rng(0).uniform(-30, 8.5, 100_000)])
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    st = attn.attn_selftest_exp2_poly(xd.data_ptr(), yd.data_ptr(), xd.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == attn.ATTN_OK
    torch.cuda.synchronize()
    xf = xd.cpu().numpy().astype(np.float64)
    y = yd.cpu().numpy().astype(np.float64)
    rel = np.abs(y / np.exp2(xf) - 1.0)
    assert rel.max() < 1e-4, rel.max()
    # below the clamp the result is a tiny positive number (about 2^-125)
    xl = torch.tensor([-126.0, -200.0, -1e30], dtype=torch.float32, device="cuda")
    yl = torch.empty_like(xl)
    assert attn.attn_selftest_exp2_poly(xl.data_ptr(), yl.data_ptr(), 3, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    v = yl.cpu().numpy()
    assert np.all(v > 0) and np.all(v < 2.0 ** -124)


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(attn):
    import torch
    from attn_inputs import make_qkv
    s = torch.cuda.current_stream().cuda_stream
    assert attn.attn_device_status(s) == (attn.ATTN_OK, 0)
    assert attn.attn_selftest_wait_timeout(20000, s) == attn.ATTN_OK      # 20 ms limit
    st, site = attn.attn_device_status(s)
    assert st == attn.ATTN_ERR_TIMEOUT and site == 10
    assert attn.attn_device_status(s) == (attn.ATTN_OK, 0)                 # record cleared
    # the context is still usable: a forward pass runs and reports no timeout
    q, k, v = (x.cuda() for x in make_qkv(1, 2, 2, 256, 64, seed=5))
    o, lse = attn.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and attn.attn_device_status(s) == (attn.ATTN_OK, 0)


@pytest.mark.gpu
def test_selftest_argument_checks(attn):
    assert attn.attn_selftest_exp2_poly(None, None, -1, None) == attn.ATTN_ERR_INVALID_ARG
    assert attn.attn_selftest_exp2_poly(None, None, 0, None) == attn.ATTN_OK
    assert attn.attn_selftest_wait_timeout(0, None) == attn.ATTN_ERR_INVALID_ARG
    assert attn.attn_selftest_wait_timeout(2_000_000, None) == attn.ATTN_ERR_INVALID_ARG
