"""attn_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Such callers (code whose device memory belongs to another allocator, or that must not
risk the synchronisation an allocation can cause) cannot hand attn_fwd_ws a workspace.
attn_fwd_noalloc runs the same kernel with its workspace in a static device array of the
library.  These tests call it through the C ABI and compare it with the existing entry
points, twice in a row (the array keeps the previous call's contents).  The file is
named to be collected last.
"""
import math

import numpy as np
import pytest
import torch

from tiled_attention_forward_03_b200.synth import make_qkv

pytestmark = pytest.mark.gpu

TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


def _noalloc(attn, q, k, v, causal, scale):
    B, Hq, N, D = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=q.device)
    st = attn.attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               B, Hq, k.shape[1], N, D, causal, scale, torch.cuda.current_stream().cuda_stream)
    assert st == attn.ATTN_OK, attn.attn_status_string(st) + " " + attn.attn_last_cuda_error()
    return o, lse


def _close(o, lse, o_ref, lse_ref):
    d = (o.float() - o_ref.float()).abs()
    dl = (lse - lse_ref).abs()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert d.max().item() <= TOL_O_MAX and d.mean().item() <= TOL_O_MEAN and dl.max().item() <= TOL_LSE


@pytest.mark.parametrize("shape", [
    (4, 16, 16, 2048, 128, False),   # last wave split: the static array holds the partial rows
    (1, 4, 2, 1100, 64, False),      # split, GQA, empty second tile in the last pair
    (2, 8, 2, 1000, 128, True),      # causal: no split, no scratch use
    (1, 4, 2, 700, 256, False),      # wide head dim: the one-tile kernel, no scratch use
])
def test_noalloc_matches_existing_entry_points_twice(attn, shape):
    B, Hq, Hkv, N, D, causal = shape
    need = attn.attn_fwd_workspace_bytes(B, Hq, N, D, causal)
    assert 0 <= need <= attn.attn_fwd_noalloc_scratch_bytes()
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hkv, N, D, seed=6000 + N))
    scale = 1.0 / math.sqrt(D)
    o_ref, lse_ref = attn.forward(q, k, v, causal=causal, scale=scale)           # attn_fwd_ws / attn_fwd
    for _ in range(2):                                                            # two calls in a row
        o, lse = _noalloc(attn, q, k, v, causal, scale)
        torch.cuda.synchronize()
        assert attn.device_status() == (attn.ATTN_OK, 0)
        _close(o, lse, o_ref, lse_ref)


def test_noalloc_rejects_bad_arguments_before_touching_the_gpu(attn):
    P = 0x10000
    s = torch.cuda.current_stream().cuda_stream
    assert attn.attn_fwd_noalloc(P, P, P, P, P, 1, 2, 1, 128, 80, 0, 0.1, s) == attn.ATTN_ERR_UNSUPPORTED
    assert attn.attn_fwd_noalloc(None, P, P, P, P, 1, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_ERR_INVALID_ARG
    assert attn.attn_fwd_noalloc(P + 2, P, P, P, P, 1, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_ERR_MISALIGNED
    assert attn.attn_fwd_noalloc(None, None, None, None, None, 0, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_OK
