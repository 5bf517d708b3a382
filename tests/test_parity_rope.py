"""GPU parity: RoPE of Q and K, the attention forward of the rotated tensors and the backward
through both, against the fp64 oracle (needs a B200).

The rotation alone: the kernel works in fp32 on the bf16 inputs and fp32 tables and rounds to
bf16 (nearest even), so each element is within half a bf16 step of the exact rotation plus
fp32 rounding: |x' - ref| <= 2^-8 |ref| + 1e-6 (2^-8 = one bf16 step, twice the rounding bound).
The rotated Q and K are bf16 tensors (the tensor core's operand type and attn_rope_qk's
output type), so the attention is held to the forward's own tolerances (max |dO| <= 2e-2,
mean |dO| <= 2e-3, max |dLSE| <= 1e-3) against the oracle's fp64 rotation rounded to bf16
(nearest even, by the test) and then fp64 attention.  Against the unrounded fp64 rotation the
LSE moves by the rounding of the rotated operands, up to ~2e-3 at D = 128 (measured 1.6e-3 at
N = 256); that comparison is kept with LSE bound 5e-3.
"""
import numpy as np
import pytest
import torch

from oracle import attention_backward, attention_forward, attention_forward_rope, attention_rows, rope_angles
from oracle import rope_rotate, rope_rotate_transpose
from attn_inputs import CFG2, make_dout, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


@pytest.mark.parametrize("B,Hq,Hkv,N,D,base", [
    (1, 2, 1, 300, 128, 10000.0), (2, 4, 4, 129, 64, 10000.0), (1, 3, 1, 77, 96, 500.0), (1, 2, 2, 1, 32, 10000.0),
    (1, 2, 1, 16384, 128, 10000.0), (1, 2, 1, 300, 192, 10000.0), (2, 2, 2, 129, 256, 500.0),
])
def test_rope_rotation(attn, B, Hq, Hkv, N, D, base):
    q, k, _ = make_qkv(B, Hq, Hkv, N, D, 4000 + N)
    cos_t, sin_t = attn.rope_tables(N, D, base, device="cuda")
    qo, ko = attn.rope(q.cuda(), k.cuda(), cos_t, sin_t)
    torch.cuda.synchronize()
    for got, x in ((qo, q), (ko, k)):
        ref = rope_rotate(x, base)
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6), float(np.max(np.abs(g - ref)))


@pytest.mark.parametrize("N,D,base", [(1, 2, 10000.0), (7, 8, 100.0), (300, 64, 10000.0), (4096, 128, 500000.0),
                                      (16384, 128, 10000.0)])
def test_rope_tables_hold_the_oracle_angles(attn, N, D, base):
    """attn_rope_tables fills cos / sin of the oracle's angles p * base^(-2d/D): fp32 rounding
    of values in [-1, 1] (<= 2^-25) plus the fp64 evaluation of angles up to ~16384 rad."""
    cos_t, sin_t = attn.rope_tables(N, D, base)
    torch.cuda.synchronize()
    assert tuple(cos_t.shape) == (N, D // 2) and tuple(sin_t.shape) == (N, D // 2)
    assert cos_t.dtype == torch.float32 and cos_t.is_cuda and cos_t.is_contiguous() and sin_t.is_contiguous()
    th = rope_angles(N, D, base)
    assert np.abs(cos_t.cpu().numpy().astype(np.float64) - np.cos(th)).max() <= 1e-7
    assert np.abs(sin_t.cpu().numpy().astype(np.float64) - np.sin(th)).max() <= 1e-7


def test_rope_in_place(attn):
    q, k, _ = make_qkv(1, 2, 2, 256, 128, 4100)
    cos_t, sin_t = attn.rope_tables(256, 128, device="cuda")
    a = attn.rope(q.cuda(), k.cuda(), cos_t, sin_t)
    qd, kd = q.cuda(), k.cuda()
    attn.rope(qd, kd, cos_t, sin_t, q_out=qd, k_out=kd)
    torch.cuda.synchronize()
    assert torch.equal(a[0], qd) and torch.equal(a[1], kd)


def check_forward_rope(attn, q, k, v, causal, scale, base=10000.0):
    N, D = q.shape[2], q.shape[3]
    cos_t, sin_t = attn.rope_tables(N, D, base, device="cuda")
    o, lse = attn.forward_rope(q.cuda(), k.cuda(), v.cuda(), cos_t, sin_t, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_fwd_close(o, lse, o_ref, lse_ref, what, lse_tol=1e-3):
    d, dl = np.abs(o - o_ref), np.abs(lse - lse_ref)
    msg = f"{what}: max|dO|={d.max():.3e} mean|dO|={d.mean():.3e} max|dLSE|={dl.max():.3e}"
    assert d.max() <= 2e-2 and d.mean() <= 2e-3 and dl.max() <= lse_tol, msg


def rot_bf16(x, base=10000.0):
    """The oracle's fp64 rotation, rounded to bf16 (nearest even) as the kernel's operands are."""
    return torch.from_numpy(rope_rotate(x, base)).to(torch.bfloat16)


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [
    (1, 2, 2, 256, 128, False), (1, 4, 2, 513, 128, True), (2, 2, 1, 300, 64, True), (1, 2, 2, 1000, 64, False),
    (1, 2, 2, 200, 96, True), (1, 2, 1, 129, 32, False), (1, 2, 1, 300, 256, True), (1, 2, 2, 257, 192, False),
])
def test_forward_rope_small(attn, B, Hq, Hkv, N, D, causal):
    q, k, v = make_qkv(B, Hq, Hkv, N, D, 4200 + N)
    scale = D ** -0.5
    o, lse = check_forward_rope(attn, q, k, v, causal, scale)
    what = f"rope B{B} Hq{Hq} Hkv{Hkv} N{N} D{D} c{causal}"
    o_ref, lse_ref = attention_forward(rot_bf16(q), rot_bf16(k), v, causal, scale)
    assert_fwd_close(o, lse, o_ref, lse_ref, what)
    o_ref, lse_ref = attention_forward_rope(q, k, v, causal, scale)
    assert_fwd_close(o, lse, o_ref, lse_ref, what + " (unrounded rotation)", lse_tol=5e-3)


def test_forward_rope_cfg2_sampled(attn):
    """cfg2 size (B4 H16 N2048 D128): sampled rows against the oracle's rotation of the sampled heads."""
    w = CFG2
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, w.seed)
    o, lse = check_forward_rope(attn, q, k, v, w.causal, w.softmax_scale)
    rng = np.random.default_rng(17)
    for (b, h) in [(0, 0), (w.B - 1, w.Hq - 1)]:
        qr = rot_bf16(q[b:b + 1, h:h + 1])
        kr = rot_bf16(k[b:b + 1, h:h + 1])
        rows = [(0, 0, int(i)) for i in sorted(set(rng.integers(0, w.N, 64)) | {0, 127, 128, w.N - 1})]
        o_ref, l_ref = attention_rows(qr, kr, v[b:b + 1, h:h + 1], rows, w.causal, w.softmax_scale)
        idx = [r[2] for r in rows]
        assert_fwd_close(o[b, h, idx], lse[b, h, idx], o_ref, l_ref, f"cfg2 rope head {(b, h)}")


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [
    (1, 1, 1, 2048, 128, False),    # the split last wave
    (1, 4, 4, 1500, 96, False),
    (2, 4, 2, 700, 64, True),
    (1, 8, 2, 1025, 32, True),
])
def test_forward_rope_matches_rotate_then_forward(attn, B, Hq, Hkv, N, D, causal):
    """attn_fwd_rope (the rotary kernel into the workspace, then the forward, the split last wave
    included) against rotating both tensors with attn_rope_qk and running the plain forward
    without a split, and against the oracle."""
    q, k, v = make_qkv(B, Hq, Hkv, N, D, 4300 + N + D)
    scale = D ** -0.5
    if not causal and B * Hq * N == 2048:
        assert attn.attn_fwd_workspace_bytes(B, Hq, N, D, False) > 0
    o, lse = check_forward_rope(attn, q, k, v, causal, scale)
    cos_t, sin_t = attn.rope_tables(N, D)
    qr, kr = attn.rope(q.cuda(), k.cuda(), cos_t, sin_t)
    o2, l2 = attn.forward(qr, kr, v.cuda(), causal=causal, scale=scale, split=False)
    torch.cuda.synchronize()
    o2 = o2.float().cpu().numpy().astype(np.float64)
    l2 = l2.cpu().numpy().astype(np.float64)
    # the same rotated operands, two schedules: fp32 summation order only
    assert np.abs(o - o2).max() <= 2e-2 and np.abs(lse - l2).max() <= 1e-4
    o_ref, lse_ref = attention_forward(rot_bf16(q), rot_bf16(k), v, causal, scale)
    assert_fwd_close(o, lse, o_ref, lse_ref, f"fused rope B{B} Hq{Hq} Hkv{Hkv} N{N} D{D} c{causal}")


def test_forward_rope_long_sequence_sampled(attn):
    """N = 8192 (angles up to ~8200 rad), causal GQA: sampled rows of two heads."""
    B, Hq, Hkv, N, D = 1, 4, 2, 8192, 128
    q, k, v = make_qkv(B, Hq, Hkv, N, D, 4400)
    o, lse = check_forward_rope(attn, q, k, v, True, D ** -0.5)
    rng = np.random.default_rng(19)
    for h in (0, Hq - 1):
        qr = rot_bf16(q[:, h:h + 1])
        kr = rot_bf16(k[:, h // 2:h // 2 + 1])
        rows = [(0, 0, int(i)) for i in sorted(set(rng.integers(0, N, 48)) | {0, 1, 4095, N - 1})]
        o_ref, l_ref = attention_rows(qr, kr, v[:, h // 2:h // 2 + 1], rows, True, D ** -0.5)
        idx = [r[2] for r in rows]
        assert_fwd_close(o[0, h, idx], lse[0, h, idx], o_ref, l_ref, f"long rope head {h}")


# ------------------------------------------------------------------ the backward of the rotation

def _pair_norm(x):
    """Per element, the norm of its rotation pair (x_d, x_{d+D/2})."""
    h = x.shape[-1] // 2
    n = np.sqrt(x[..., :h] ** 2 + x[..., h:] ** 2)
    return np.concatenate([n, n], axis=-1)


@pytest.mark.parametrize("B,Hq,Hkv,N,D,base", [
    (1, 2, 1, 300, 128, 10000.0), (2, 4, 4, 129, 64, 10000.0), (1, 3, 1, 77, 96, 500.0), (1, 2, 2, 1, 32, 10000.0),
])
def test_rope_inverse(attn, B, Hq, Hkv, N, D, base):
    """attn_rope_qk_inverse against the oracle's transpose R^T (the same one-rounding bound as the
    rotation), and rope followed by rope_inverse returning the inputs within the two roundings
    (each at most half a bf16 step of its pair's norm)."""
    q, k, _ = make_qkv(B, Hq, Hkv, N, D, 4100 + N)
    cos_t, sin_t = attn.rope_tables(N, D, base, device="cuda")
    gq, gk = attn.rope_inverse(q.cuda(), k.cuda(), cos_t, sin_t)
    qr, kr = attn.rope(q.cuda(), k.cuda(), cos_t, sin_t)
    q2, k2 = attn.rope_inverse(qr, kr, cos_t, sin_t)
    torch.cuda.synchronize()
    for got, back, x in ((gq, q2, q), (gk, k2, k)):
        ref = rope_rotate_transpose(x, base)
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6), float(np.max(np.abs(g - ref)))
        xf = x.float().numpy().astype(np.float64)
        b = back.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(b - xf) <= 2.0 ** -7 * _pair_norm(xf) + 1e-6), float(np.max(np.abs(b - xf)))


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [
    (1, 2, 2, 256, 128, False), (1, 2, 1, 200, 128, True), (2, 4, 1, 384, 64, True), (1, 2, 2, 130, 96, False),
    (1, 2, 1, 300, 32, True), (1, 1, 1, 1, 64, False),
])
def test_backward_rope(attn, B, Hq, Hkv, N, D, causal):
    """backward_rope (attn_bwd_rope) against the oracle: the rotation in fp64 rounded to bf16
    (the operand type the backward kernels read), the fp64 attention backward, then R^T; held to
    the backward's tolerance bars."""
    from test_parity_bwd import assert_grad_close

    q, k, v = make_qkv(B, Hq, Hkv, N, D, 4200 + N + D)
    do = make_dout(B, Hq, N, D, 4300 + N + D)
    scale = D ** -0.5
    cos_t, sin_t = attn.rope_tables(N, D, device="cuda")
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.forward_rope(qd, kd, vd, cos_t, sin_t, causal=causal)
    dq, dk, dv = attn.backward_rope(qd, kd, vd, cos_t, sin_t, o, lse, dod, causal=causal)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    qr, kr = _bf16(rope_rotate(q)), _bf16(rope_rotate(k))
    rq, rk, rv = attention_backward(qr, kr, v, do, causal, scale)
    ref = (rope_rotate_transpose(rq), rope_rotate_transpose(rk), rv)
    for name, a, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_grad_close(a.float().cpu().numpy().astype(np.float64), r, f"rope backward {name}")


@pytest.mark.parametrize("shape", [(2, 4, 2, 700, 128, True), "cfg2", "cfg3"], ids=str)
def test_backward_rope_is_rotate_backward_then_inverse(attn, shape):
    """attn_bwd_rope equals its three steps called one by one (bit for bit), also at the sizes
    the backward through RoPE is benchmarked on (cfg2, cfg3), where the plain backward's own
    parity is checked on sampled heads."""
    from attn_inputs import get_workload

    if isinstance(shape, str):
        w = get_workload(shape)
        B, Hq, Hkv, N, D, causal = w.B, w.Hq, w.Hkv, w.N, w.D, w.causal
    else:
        B, Hq, Hkv, N, D, causal = shape
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hkv, N, D, 4400))
    do = make_dout(B, Hq, N, D, 4401).cuda()
    cos_t, sin_t = attn.rope_tables(N, D, device="cuda")
    o, lse = attn.forward_rope(q, k, v, cos_t, sin_t, causal=causal)
    got = attn.backward_rope(q, k, v, cos_t, sin_t, o, lse, do, causal=causal)
    qr, kr = attn.rope(q, k, cos_t, sin_t)
    dqr, dkr, dv = attn.backward(qr, kr, v, o, lse, do, causal=causal)
    dq, dk = attn.rope_inverse(dqr, dkr, cos_t, sin_t)
    torch.cuda.synchronize()
    for a, b in zip(got, (dq, dk, dv)):
        assert torch.equal(a, b)
