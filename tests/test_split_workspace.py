"""The split-tail workspace of attn_fwd_ws under reuse (GPU).

When the last wave of a non-causal launch is partial, each of its units is split into two KV
ranges on two CTAs, which merge through the caller's workspace: a per-tile counter word
tagged with the launch's epoch, and a ready flag.  The library numbers its launches itself,
so two copies of it loaded in one process (or one copy after its 24-bit epoch wraps round)
can issue the same epoch.  The merging range therefore zeroes the words it used once it has
read them.  These tests load two fresh copies of the library, whose first launches carry the
same epoch, run them on one workspace in turn, and require every result to equal the
installed library's bit for bit and to match the oracle.
"""
import ctypes
import math
import shutil

import numpy as np
import pytest
import torch

from oracle import attention_forward
from attn_inputs import make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


def _copy_of_library(attn, tmp_path, name):
    path = tmp_path / name
    shutil.copyfile(attn.lib_path, path)
    L = ctypes.CDLL(str(path))
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.attn_fwd_ws.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    L.attn_fwd_ws.restype = i
    return L


def _run(L, q, k, v, causal, scale, ws):
    B, Hq, N, D = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=q.device)
    st = L.attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
                       k.shape[1], N, D, int(causal), scale, ws.data_ptr(), ws.numel(),
                       torch.cuda.current_stream().cuda_stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("shape", [
    (2, 4, 2, 1000, 64, False),     # 32 units: every unit split, ragged tail
    (4, 16, 16, 2048, 128, False),  # 512 units: 3 whole waves, the rest split
])
def test_two_library_copies_share_a_workspace(attn, tmp_path, shape):
    B, Hq, Hkv, N, D, causal = shape
    need = attn.attn_fwd_workspace_bytes(B, Hq, N, D, causal)
    assert need > 0, "the shape must split its last wave"
    scale = 1.0 / math.sqrt(D)
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hkv, N, D, seed=7000 + N))
    o_ref, lse_ref = attn.forward(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()

    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    first, second = (_copy_of_library(attn, tmp_path, f"libattn_copy{i}.so") for i in (1, 2))
    runs = [first, second, first, second]   # the copies' first and second launches share epochs
    for L in runs:
        o, lse = _run(L, q, k, v, causal, scale, ws)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)

    # the installed library's result against the fp64 oracle, on whole heads
    heads = [(0, 0), (B - 1, Hq - 1)]
    for b, h in heads:
        kh = h // (Hq // Hkv)
        O, L = attention_forward(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, kh:kh + 1].cpu(),
                                 v[b:b + 1, kh:kh + 1].cpu(), causal, scale)
        d = np.abs(o_ref[b, h].float().cpu().numpy() - O[0, 0])
        dl = np.abs(lse_ref[b, h].cpu().numpy() - L[0, 0])
        assert d.max() <= 2e-2 and d.mean() <= 2e-3 and dl.max() <= 1e-3, (d.max(), d.mean(), dl.max())
