"""GPU parity: the E4M3 (FP8) attention forward against the fp64 oracle (needs a B200).

The oracle is the plain definition (attention_forward) on the dequantized inputs
descale * stored value, which are exact in fp64.  The kernel's scores are exact fp32 sums of
E4M3 products, so LSE keeps the forward's bound (max |dLSE| <= 1e-3); the probabilities are
rounded to E4M3 (3 mantissa bits) before P V.  Tolerance (derived): emulating that rounding
on the CPU (fp32 row sums, bf16 output) gives max |dO| up to 4e-2 (causal rows with few
keys) and mean |dO| up to 2.2e-3 at N = 512..2048, D = 32..256; the bar is

    max |dO| <= 1e-1,   mean |dO| <= 6e-3,   max |dLSE| <= 1e-3.
"""
import numpy as np
import pytest
import torch

from oracle import attention_forward, attention_rows
from attn_inputs import CFG2, make_qkv_e4m3

pytestmark = pytest.mark.gpu

TOL_O_MAX = 1e-1
TOL_O_MEAN = 6e-3
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_attention_forward_03_b200 as mod
    return mod


def deq(x, s):
    return x.float().numpy().astype(np.float64) * s


def run(attn, q8, k8, v8, ds, causal, scale, descales=None):
    qd_, kd_, vd_ = descales if descales is not None else (ds, ds, ds)
    o, lse = attn.forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), qd_, kd_, vd_, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_close(o, lse, o_ref, lse_ref, what):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), f"{what}: non-finite output"
    d, dl = np.abs(o - o_ref), np.abs(lse - lse_ref)
    msg = f"{what}: max|dO|={d.max():.3e} mean|dO|={d.mean():.3e} max|dLSE|={dl.max():.3e}"
    assert d.max() <= TOL_O_MAX and d.mean() <= TOL_O_MEAN and dl.max() <= TOL_LSE, msg


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [
    (1, 2, 2, 256, 128, False), (1, 2, 2, 256, 128, True), (1, 4, 1, 513, 128, True), (2, 2, 2, 384, 64, False),
    (1, 4, 2, 300, 64, True), (1, 2, 2, 1, 128, False), (1, 2, 1, 1000, 128, False), (1, 2, 2, 2048, 128, True),
    # head dims 32 and 96 (one 128-byte row chunk, partly used and zero-filled by TMA)
    (1, 2, 2, 512, 32, True), (2, 4, 2, 1000, 32, False), (1, 2, 2, 1, 32, True),
    (1, 2, 2, 1024, 96, True), (1, 4, 1, 777, 96, False), (2, 2, 2, 2048, 96, False),
    # head dims 192 and 256 on the wide-head kernel (192: a second 128-byte chunk, half zero-filled)
    (1, 2, 2, 256, 192, True), (1, 4, 1, 513, 192, False), (1, 2, 2, 1, 192, False), (2, 2, 2, 1000, 192, True),
    (1, 2, 2, 384, 256, False), (1, 4, 2, 777, 256, True), (1, 2, 2, 1, 256, True), (1, 2, 2, 2048, 256, False),
])
def test_fp8_small_shapes(attn, B, Hq, Hkv, N, D, causal):
    q8, k8, v8, ds = make_qkv_e4m3(B, Hq, Hkv, N, D, 5000 + N + D)
    scale = D ** -0.5
    o, lse = run(attn, q8, k8, v8, ds, causal, scale)
    o_ref, lse_ref = attention_forward(deq(q8, ds), deq(k8, ds), deq(v8, ds), causal, scale)
    assert_close(o, lse, o_ref, lse_ref, f"fp8 B{B} Hq{Hq} Hkv{Hkv} N{N} D{D} c{causal}")


@pytest.mark.parametrize("descales,scale", [((0.05, 0.1, 0.2), 0.08838834764831843), ((0.0625, 0.0625, 0.0625), -0.05),
                                            ((0.1, 0.02, 1.0), 0.0)])
def test_fp8_descales_and_scales(attn, descales, scale):
    q8, k8, v8, _ = make_qkv_e4m3(1, 2, 1, 384, 128, 5100)
    o, lse = run(attn, q8, k8, v8, None, True, scale, descales)
    o_ref, lse_ref = attention_forward(deq(q8, descales[0]), deq(k8, descales[1]), deq(v8, descales[2]), True, scale)
    # O scales with the V descale: compare relative to it
    assert_close(o / descales[2] * 0.0625, lse, o_ref / descales[2] * 0.0625, lse_ref, f"fp8 descales {descales}")


def test_fp8_deterministic(attn):
    q8, k8, v8, ds = make_qkv_e4m3(1, 4, 2, 640, 128, 5200)
    a = attn.forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds, ds, ds, causal=True)
    b = attn.forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds, ds, ds, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8_cfg2_sampled(attn):
    """cfg2 size (B4 H16 N2048 D128, split tail on): sampled rows of every 16th head."""
    w = CFG2
    q8, k8, v8, ds = make_qkv_e4m3(w.B, w.Hq, w.Hkv, w.N, w.D, w.seed)
    o, lse = run(attn, q8, k8, v8, ds, w.causal, w.softmax_scale)
    rng = np.random.default_rng(23)
    rows = [(int(b), int(h), int(i)) for b, h, i in zip(rng.integers(0, w.B, 200), rng.integers(0, w.Hq, 200),
                                                      rng.integers(0, w.N, 200))]
    q, k, v = (x.float() * ds for x in (q8, k8, v8))
    o_ref, lse_ref = attention_rows(q, k, v, rows, w.causal, w.softmax_scale)
    idx = tuple(np.array(x) for x in zip(*rows))
    assert_close(o[idx], lse[idx], o_ref, lse_ref, "fp8 cfg2 sampled rows")


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [(8, 16, 16, 2176, 256, True), (10, 16, 16, 1920, 192, False)])
def test_fp8_wide_persistent_items_sampled(attn, B, Hq, Hkv, N, D, causal):
    """The wide-head kernel's persistent schedule with E4M3 inputs (causal tile pairs with a
    lone middle tile; non-causal, many tiles per CTA): seeded sampled rows."""
    from attn_inputs import sample_rows

    q8, k8, v8, ds = make_qkv_e4m3(B, Hq, Hkv, N, D, 5300 + N + D)
    scale = D ** -0.5
    o, lse = run(attn, q8, k8, v8, ds, causal, scale)
    rows = sample_rows(B, Hq, N, 96, seed=5301 + N)
    q, k, v = (x.float() * ds for x in (q8, k8, v8))
    o_ref, lse_ref = attention_rows(q, k, v, rows, causal, scale)
    idx = tuple(np.array(x) for x in zip(*rows))
    assert_close(o[idx], lse[idx], o_ref, lse_ref, f"fp8 wide persistent B{B} N{N} D{D}")


@pytest.mark.parametrize("name", ["cfg3", "cfg4", "sweep_D128_N8192_noncausal", "sweep_D64_N4096_noncausal",
                                  "sweep_D64_N4096_causal", "wide_D192_N8192_noncausal", "wide_D256_N8192_noncausal",
                                  "wide_D256_N8192_causal", "wide_D192_N2048_causal"])
def test_fp8_benchmark_workloads_sampled(attn, name):
    """Every workload the E4M3 pass is benchmarked on, at full size: seeded sampled rows (every
    128-row tile edge of one head plus uniform draws), each computed by the oracle on its own
    from the dequantized inputs."""
    from attn_inputs import get_workload, sample_rows

    w = get_workload(name)
    q8, k8, v8, ds = make_qkv_e4m3(w.B, w.Hq, w.Hkv, w.N, w.D, w.seed)
    o, lse = run(attn, q8, k8, v8, ds, w.causal, w.softmax_scale)
    rows = sample_rows(w.B, w.Hq, w.N, 96, seed=w.seed + 11)
    q, k, v = (x.float() * ds for x in (q8, k8, v8))
    o_ref, lse_ref = attention_rows(q, k, v, rows, w.causal, w.softmax_scale)
    idx = tuple(np.array(x) for x in zip(*rows))
    assert_close(o[idx], lse[idx], o_ref, lse_ref, f"fp8 {w.name} sampled rows")
