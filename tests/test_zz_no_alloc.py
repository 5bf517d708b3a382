"""attn_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Such callers (code whose device memory belongs to another allocator, or that must not
risk the synchronisation an allocation can cause) cannot hand attn_fwd_ws a workspace.
attn_fwd_noalloc runs the same kernel with the same schedule, its workspace a static
device array of the library.  These tests call it through the C ABI and require it to
equal attn_fwd_ws (given a workspace of its own of the size the schedule needs) bit for
bit, twice in a row (the array keeps the previous call's contents), with the first call of
the process on a side stream; one shape is also compared with the fp64 oracle.  The file
is named to be collected last.
"""
import math

import numpy as np
import pytest
import torch

from attn_inputs import make_qkv
from oracle import attention_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


def _outputs(q):
    B, Hq, N, D = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=q.device)
    return o, lse


def _noalloc(attn, q, k, v, causal, scale, stream):
    B, Hq, N, D = q.shape
    o, lse = _outputs(q)
    st = attn.attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               B, Hq, k.shape[1], N, D, causal, scale, stream.cuda_stream)
    assert st == attn.ATTN_OK, attn.attn_status_string(st) + " " + attn.attn_last_cuda_error()
    return o, lse


def _with_workspace(attn, q, k, v, causal, scale, stream):
    """attn_fwd_ws with a workspace of exactly the size the split schedule needs (or none)."""
    B, Hq, N, D = q.shape
    need = attn.attn_fwd_workspace_bytes(B, Hq, N, D, causal)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    o, lse = _outputs(q)
    st = attn.attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
                          k.shape[1], N, D, causal, scale, ws.data_ptr() if need > 0 else None, need,
                          stream.cuda_stream)
    assert st == attn.ATTN_OK, attn.attn_status_string(st)
    return o, lse


SHAPES = [
    (4, 16, 16, 2048, 128, False),   # last wave split: the static array holds the partial rows
    (1, 4, 2, 1100, 64, False),      # split, GQA, empty second tile in the last pair
    (2, 8, 2, 1000, 128, True),      # causal: no split, no scratch use
    (1, 4, 2, 700, 256, False),      # wide head dim: the one-tile kernel, no scratch use
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_noalloc_equals_workspace_entry_point_bitwise_twice(attn, shape):
    B, Hq, Hkv, N, D, causal = shape
    need = attn.attn_fwd_workspace_bytes(B, Hq, N, D, causal)
    assert 0 <= need <= attn.attn_fwd_noalloc_scratch_bytes()
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hkv, N, D, seed=6000 + N))
    scale = 1.0 / math.sqrt(D)
    side = torch.cuda.Stream()          # a non-blocking stream: the first call must not need the legacy one
    with torch.cuda.stream(side):
        for _ in range(2):              # two calls in a row share the array
            o, lse = _noalloc(attn, q, k, v, causal, scale, side)
            o_ref, lse_ref = _with_workspace(attn, q, k, v, causal, scale, side)
            side.synchronize()
            assert attn.device_status(side) == (attn.ATTN_OK, 0)
            assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
            assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_noalloc_split_shape_against_the_oracle(attn):
    """The split last wave through the static array, against the fp64 definition."""
    B, Hq, Hkv, N, D = 1, 4, 2, 1100, 64
    assert attn.attn_fwd_workspace_bytes(B, Hq, N, D, False) > 0
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=6100)
    scale = 1.0 / math.sqrt(D)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        o, lse = _noalloc(attn, q.cuda(), k.cuda(), v.cuda(), False, scale, side)
        side.synchronize()
    o_ref, lse_ref = attention_forward(q, k, v, False, scale)
    d = np.abs(o.float().cpu().numpy() - o_ref)
    dl = np.abs(lse.cpu().numpy() - lse_ref)
    assert d.max() <= 2e-2 and d.mean() <= 2e-3 and dl.max() <= 1e-3, (d.max(), d.mean(), dl.max())


def test_noalloc_rejects_bad_arguments_before_touching_the_gpu(attn):
    P = 0x10000
    s = torch.cuda.current_stream().cuda_stream
    assert attn.attn_fwd_noalloc(P, P, P, P, P, 1, 2, 1, 128, 80, 0, 0.1, s) == attn.ATTN_ERR_UNSUPPORTED
    assert attn.attn_fwd_noalloc(None, P, P, P, P, 1, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_ERR_INVALID_ARG
    assert attn.attn_fwd_noalloc(P + 2, P, P, P, P, 1, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_ERR_MISALIGNED
    assert attn.attn_fwd_noalloc(None, None, None, None, None, 0, 2, 1, 128, 128, 0, 0.1, s) == attn.ATTN_OK
