"""GPU parity: the CUDA attention backward against the fp64 backward oracle (needs a B200).

Tolerance (the spec states none for the backward; derived from its arithmetic): the
kernel rounds P and dS to bf16 before the gradient matmuls and rounds dQ, dK, dV to
bf16, and delta uses the forward's bf16 O.  Emulating exactly those roundings on the
CPU against the fp64 oracle gives, at N = 384..1024 and D = 64/128, a mean error of
about 2.3e-3 x mean|ref| (mostly the final bf16 rounding) and a max error of at most
4.3e-3 x max|ref|.  The bar is about 2-3.5x above that, per gradient tensor:

    max |d - ref|  <= 1.5e-2 * max |ref|       mean |d - ref| <= 5e-3 * mean |ref|

plus an absolute floor of 1e-4 (max) and 1e-5 (mean) for gradients that are exactly 0
in the definition (N = 1, identical rows): there the kernel's dP - delta cancels in fp32
to a residual of about 1e-7 instead of 0.  Gradient entries elsewhere are 0.3-6 in size.

A kernel slip of one key or query tile, or one masked element on the diagonal, moves
some entries by a good fraction of their size and fails the max bound.

The forward used to produce o and lse is the library's own (parity-tested on its own);
the oracle computes the gradients from q, k, v and dO alone.
"""
import numpy as np
import pytest
import torch

from oracle import attention_backward, head_backward
from attn_inputs import Workload, CFG2, CFG3, CFG4, make_dout, make_qkv

pytestmark = pytest.mark.gpu

TOL_MAX = 1.5e-2
TOL_MEAN = 5e-3
ABS_MAX = 1e-4
ABS_MEAN = 1e-5


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


def gpu_backward(attn, q, k, v, do, causal, scale):
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = attn.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    return tuple(x.float().cpu().numpy().astype(np.float64) for x in (dq, dk, dv))


def assert_grad_close(got, ref, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    d = np.abs(got - ref)
    scale_max = max(float(np.abs(ref).max()), 1e-30)
    scale_mean = max(float(np.abs(ref).mean()), 1e-30)
    bar_max = TOL_MAX * scale_max + ABS_MAX
    bar_mean = TOL_MEAN * scale_mean + ABS_MEAN
    msg = f"{what}: max|d|={d.max():.3e} (bar {bar_max:.3e}) mean|d|={d.mean():.3e} (bar {bar_mean:.3e})"
    assert d.max() <= bar_max, msg
    assert d.mean() <= bar_mean, msg


def check_full(attn, B, Hq, Hkv, N, D, causal, scale=None, seed=0, what=""):
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed)
    do = make_dout(B, Hq, N, D, seed + 500)
    scale = D ** -0.5 if scale is None else scale
    got = gpu_backward(attn, q, k, v, do, causal, scale)
    ref = attention_backward(q, k, v, do, causal, scale)
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        if name == "dq" and scale == 0.0 or name == "dk" and scale == 0.0:
            assert np.all(a == 0.0), f"{what} {name}: scale 0 must give exact zeros"
            continue
        assert_grad_close(a, r, f"{what} {name}")
    return got


# ------------------------------------------------------------------ small shapes, all elements

SHAPES = [
    # B, Hq, Hkv, N, D, causal
    (1, 2, 2, 256, 128, False),
    (1, 2, 2, 256, 128, True),
    (1, 2, 2, 384, 64, False),
    (2, 4, 1, 384, 64, True),      # GQA 4:1
    (1, 4, 2, 513, 128, False),    # ragged tail of one row
    (1, 2, 1, 200, 128, True),     # ragged, GQA 2:1
    (1, 2, 2, 130, 96, False),
    (1, 2, 2, 300, 96, True),
    (1, 2, 1, 300, 32, True),
    (1, 2, 2, 129, 32, False),
    (1, 1, 1, 1, 64, False),       # one key, one query
    (1, 1, 1, 1, 128, True),
    (1, 1, 1, 127, 128, True),     # one partial tile
    (3, 2, 2, 640, 128, True),     # several batches and tiles
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", SHAPES)
def test_backward_small_shapes(attn, B, Hq, Hkv, N, D, causal):
    check_full(attn, B, Hq, Hkv, N, D, causal, seed=3000 + N + D, what=f"B{B} Hq{Hq} Hkv{Hkv} N{N} D{D} c{causal}")


@pytest.mark.parametrize("scale", [0.0, -0.09, 0.3])
def test_backward_scales(attn, scale):
    check_full(attn, 1, 2, 1, 320, 128, True, scale=scale, seed=3100, what=f"scale {scale}")


def test_backward_is_deterministic(attn):
    q, k, v = make_qkv(1, 4, 2, 640, 128, 3200)
    do = make_dout(1, 4, 640, 128, 3201)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward(qd, kd, vd, causal=True)
    a = attn.backward(qd, kd, vd, o, lse, dod, causal=True)
    b = attn.backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_invariants_full_size(attn):
    """At a size too large for a full oracle run: dV rows of a KV head sum to the dO rows
    of its query heads, and dK rows sum to zero.  With the kernel's roundings emulated on
    the CPU (one KV head, 4 query heads, N = 4096, causal) both residuals come to 0.056;
    the bound is 0.25.  One missing 128-row tile would move them by about 10."""
    B, Hq, Hkv, N, D = 2, 8, 2, 4096, 128
    q, k, v = make_qkv(B, Hq, Hkv, N, D, 3300)
    do = make_dout(B, Hq, N, D, 3301)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward(qd, kd, vd, causal=True)
    dq, dk, dv = attn.backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    want = dod.double().reshape(B, Hkv, Hq // Hkv, N, D).sum(dim=(2, 3))
    assert torch.max(torch.abs(dv.double().sum(dim=2) - want)).item() <= 0.25
    assert torch.max(torch.abs(dk.double().sum(dim=2))).item() <= 0.25
    assert torch.isfinite(dq.float()).all()


# ------------------------------------------------------------------ the benchmark shapes, sampled heads

def check_heads(attn, w, heads):
    """The backward at a workload's full size; the oracle recomputes the listed KV heads
    (their dk, dv need every query head of the group; dq is checked on those heads)."""
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, w.seed)
    do = make_dout(w.B, w.Hq, w.N, w.D, w.seed + 500)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward(qd, kd, vd, causal=w.causal, scale=w.softmax_scale)
    dq, dk, dv = attn.backward(qd, kd, vd, o, lse, dod, causal=w.causal, scale=w.softmax_scale)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    for x in (dq, dk, dv):
        assert torch.isfinite(x.float()).all()
    g = w.Hq // w.Hkv
    host = lambda t: t.float().cpu().numpy().astype(np.float64)
    for (b, hkv) in heads:
        gk = np.zeros((w.N, w.D))
        gv = np.zeros((w.N, w.D))
        for h in range(hkv * g, (hkv + 1) * g):
            a, c, e = head_backward(q[b, h], k[b, hkv], v[b, hkv], do[b, h], w.causal, w.softmax_scale)
            assert_grad_close(host(dq[b, h]), a, f"{w.name} dq head {(b, h)}")
            gk += c
            gv += e
        assert_grad_close(host(dk[b, hkv]), gk, f"{w.name} dk kv head {(b, hkv)}")
        assert_grad_close(host(dv[b, hkv]), gv, f"{w.name} dv kv head {(b, hkv)}")


def test_backward_cfg2_sampled_heads(attn):
    check_heads(attn, CFG2, [(0, 0), (CFG2.B - 1, CFG2.Hkv - 1)])


def test_backward_cfg3_sampled_head(attn):
    check_heads(attn, CFG3, [(CFG3.B - 1, 5)])


def test_backward_cfg4_sampled_kv_head(attn):
    # one KV head of the GQA workload: its 4 query heads at N = 8192
    check_heads(attn, CFG4, [(3, 6)])


@pytest.mark.parametrize("name,heads", [("sweep_D128_N8192_noncausal", [(1, 15)]),
                                        ("sweep_D64_N4096_causal", [(0, 0), (3, 9)])])
def test_backward_sweep_benchmark_shapes_sampled_heads(attn, name, heads):
    """The other workloads the backward is benchmarked on, at full size: whole KV heads."""
    from attn_inputs import get_workload
    check_heads(attn, get_workload(name), heads)


BWD_PERSISTENT = [
    # (B, Hq, Hkv, N, D, causal): the persistent schedule's item kinds at sizes where CTAs take
    # many units: causal block pairs with 17 blocks per head (a lone middle block); GQA group 5
    # with the dK/dV pass unpaired (fewer pairs than SMs) and the dQ pass paired; non-causal with
    # ~13 units per CTA
    (8, 16, 16, 2176, 128, True),
    (4, 20, 4, 2048, 64, True),
    (8, 16, 16, 1920, 96, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", BWD_PERSISTENT)
def test_backward_persistent_items_sampled_heads(attn, B, Hq, Hkv, N, D, causal):
    w = Workload(f"bwdp_B{B}_Hq{Hq}_Hkv{Hkv}_N{N}_D{D}", B, Hq, Hkv, N, D, causal, 4700 + N + D)
    check_heads(attn, w, [(0, 0), (B - 1, Hkv - 1)])


@pytest.mark.parametrize("B,Hq,Hkv", [(3, 4, 2), (1, 8, 2)])
def test_backward_host_path_in_pieces_equals_device_call(attn, B, Hq, Hkv):
    """backward_from_host pipelines batch rows (or whole KV-head groups when B == 1); the
    gradients equal one device call bit for bit."""
    q, k, v = make_qkv(B, Hq, Hkv, 384, 128, 3400 + B)
    do = make_dout(B, Hq, 384, 128, 3401 + B)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward(qd, kd, vd, causal=True)
    ref = attn.backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    got = attn.backward_from_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), o.cpu().pin_memory(),
                                  lse.cpu().pin_memory(), do.pin_memory(), causal=True)
    for g, r in zip(got, ref):
        assert torch.equal(g, r.cpu())
