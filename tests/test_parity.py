"""GPU parity: the CUDA attention forward against the fp64 oracle (needs a B200).

Tolerances (stated for this path): over all compared O elements, max |dO| <= 2e-2
and mean |dO| <= 2e-3; over all compared rows, max |dLSE| <= 1e-3.  Small cases
are compared element by element in full; the full-size workloads are compared on
seeded sampled rows (plus one whole head), each row computed by the oracle on its own.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention_forward, attention_rows, head_forward
from attn_inputs import (
    CFG1, CFG2, CFG3, CFG4, Workload, make_qkv, make_workload_inputs, sample_rows, sweep_points, wide_points)

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


def gpu_forward(attn, q, k, v, causal, scale):
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = attn.forward(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, f"kernel wait gave up at site {site}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_close(o, lse, o_ref, lse_ref, what=""):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), f"{what}: non-finite output"
    d = np.abs(o - o_ref)
    dl = np.abs(lse - lse_ref)
    msg = f"{what}: max|dO|={d.max():.3e} mean|dO|={d.mean():.3e} max|dLSE|={dl.max():.3e}"
    assert d.max() <= TOL_O_MAX, msg
    assert d.mean() <= TOL_O_MEAN, msg
    assert dl.max() <= TOL_LSE, msg


def check_full(attn, q, k, v, causal, scale, what=""):
    o, lse = gpu_forward(attn, q, k, v, causal, scale)
    o_ref, lse_ref = attention_forward(q, k, v, causal, scale)
    assert_close(o, lse, o_ref, lse_ref, what)
    return o, lse


def check_sampled(attn, w, q, k, v, count=256, full_heads=((0, 0),), rows=None):
    o, lse = gpu_forward(attn, q, k, v, w.causal, w.softmax_scale)
    if rows is None:
        rows = sample_rows(w.B, w.Hq, w.N, count, seed=w.seed + 7)
    o_ref, lse_ref = attention_rows(q, k, v, rows, w.causal, w.softmax_scale)
    idx = tuple(np.array(x) for x in zip(*rows))
    assert_close(o[idx], lse[idx], o_ref, lse_ref, w.name + " sampled rows")
    g = w.Hq // w.Hkv
    for (b, h) in full_heads:
        oh, lh = head_forward(q[b, h], k[b, h // g], v[b, h // g], w.causal, w.softmax_scale)
        assert_close(o[b, h], lse[b, h], oh, lh, f"{w.name} head {(b, h)}")
    # properties at any size: finite everywhere; on the sampled rows, the row's largest allowed
    # score m_i <= LSE_i <= m_i + ln(number of allowed keys) (bounds of a log-sum-exp)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    check_lse_bounds(lse, q, k, rows, w.causal, w.softmax_scale, g)


def check_lse_bounds(lse, q, k, rows, causal, scale, g):
    for (b, h, i) in rows:
        qi = q[b, h, i].double()
        kk = k[b, h // g].double()
        n = (i + 1) if causal else kk.shape[0]
        m = float((scale * (kk[:n] @ qi)).max())
        assert m - TOL_LSE <= lse[b, h, i] <= m + math.log(n) + TOL_LSE, (b, h, i, m, lse[b, h, i])


# ------------------------------------------------------------------ the five workloads

def test_cfg1_full(attn):
    q, k, v = make_workload_inputs(CFG1)
    check_full(attn, q, k, v, CFG1.causal, CFG1.softmax_scale, CFG1.name)


def test_cfg2_full(attn):
    q, k, v = make_workload_inputs(CFG2)
    check_full(attn, q, k, v, CFG2.causal, CFG2.softmax_scale, CFG2.name)


def test_cfg3_sampled(attn):
    q, k, v = make_workload_inputs(CFG3)
    check_sampled(attn, CFG3, q, k, v, full_heads=((0, 0), (15, 15)))


def test_cfg4_sampled(attn):
    q, k, v = make_workload_inputs(CFG4)
    check_sampled(attn, CFG4, q, k, v, full_heads=((7, 31),))


@pytest.mark.parametrize("w", sweep_points(), ids=lambda w: w.name)
def test_sweep_point(attn, w):
    q, k, v = make_workload_inputs(w)
    if w.N <= 2048:
        check_full(attn, q, k, v, w.causal, w.softmax_scale, w.name)
    else:
        check_sampled(attn, w, q, k, v, count=128, full_heads=())


@pytest.mark.parametrize("w", wide_points(), ids=lambda w: w.name)
def test_wide_point_sampled(attn, w):
    """Head dims 192 and 256 at every benchmark size (N = 2048 and 8192, causal and not):
    sampled rows (every tile edge of one head and seeded draws), each computed by the oracle on
    its own."""
    q, k, v = make_workload_inputs(w)
    check_sampled(attn, w, q, k, v, count=96, full_heads=())


# ------------------------------------------------------------------ edge shapes

EDGE = [
    # (B, Hq, Hkv, N, D, causal)
    (1, 1, 1, 1, 64, False), (1, 1, 1, 1, 128, True), (2, 2, 2, 7, 64, True), (1, 2, 1, 7, 128, False),
    (1, 2, 2, 127, 128, True), (1, 2, 2, 127, 64, False), (1, 2, 2, 128, 128, True),
    (1, 2, 2, 129, 128, True), (1, 2, 2, 129, 64, False), (1, 2, 2, 255, 64, True),
    (1, 2, 2, 256, 128, False), (1, 2, 2, 257, 128, True), (2, 4, 2, 383, 64, True),
    (1, 4, 1, 1000, 128, True), (1, 4, 1, 1000, 128, False), (1, 8, 1, 640, 64, True),
    (3, 8, 4, 300, 128, False), (1, 16, 2, 513, 128, True),
    # causal GQA past N = 2048 at D = 128 (two-tile kernel, units of two query heads of one KV head):
    # ragged tail, odd tile count (the middle step holds one unit), groups 2 and 4
    (1, 4, 2, 2100, 128, True), (2, 8, 2, 2304, 128, True),
    # non-causal GQA at D = 64 and 32 (the separate-P form): ragged tails, split last waves
    (2, 8, 2, 1000, 64, False), (2, 4, 1, 777, 32, False), (3, 6, 3, 2049, 64, False),
]


@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_edge_shapes(attn, shape):
    B, Hq, Hkv, N, D, causal = shape
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=3000 + N + D + Hq)
    check_full(attn, q, k, v, causal, 1.0 / math.sqrt(D), str(shape))


LONG = [
    # (B, Hq, Hkv, N, D, causal): sequences past the benchmark sizes, up to 128K keys per head
    (1, 2, 1, 131072, 128, True), (1, 2, 1, 131072, 128, False), (1, 2, 2, 65536, 64, True),
    (1, 3, 3, 100000, 128, False), (1, 4, 1, 131072, 64, False),
]


@pytest.mark.parametrize("shape", LONG, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_long_sequences_sampled(attn, shape):
    """Long sequences (1024 KV blocks per head at N = 128K): seeded rows against the oracle row
    by row, and the LSE bounds on those rows."""
    B, Hq, Hkv, N, D, causal = shape
    w = Workload(f"long_B{B}_Hq{Hq}_Hkv{Hkv}_N{N}_D{D}_{'c' if causal else 'nc'}", B, Hq, Hkv, N, D, causal,
                 4000 + N % 997 + D)
    q, k, v = make_workload_inputs(w)
    # rows on both sides of the edges of twelve query tiles (the first two, the last two and
    # eight seeded ones) of the last head, the first and last rows, and 48 seeded draws
    g = np.random.default_rng(w.seed)
    T = -(-N // 128)
    tiles = {0, 1, T - 2, T - 1} | set(int(x) for x in g.choice(T, 8, replace=False))
    rows = {(0, 0, 0), (B - 1, Hq - 1, N - 1)}
    for t in tiles:
        for i in (t * 128 - 1, t * 128, t * 128 + 127):
            if 0 <= i < N:
                rows.add((B - 1, Hq - 1, i))
    for x in g.integers(0, B * Hq * N, 48):
        b, rem = divmod(int(x), Hq * N)
        rows.add((b, rem // N, rem % N))
    check_sampled(attn, w, q, k, v, full_heads=(), rows=sorted(rows))


HEAD_DIMS = [
    # (B, Hq, Hkv, N, D, causal): head dims 32 and 96 (the last 64-column chunk partly used)
    (1, 2, 2, 1, 32, False), (1, 2, 1, 129, 32, True), (2, 4, 4, 700, 32, False), (1, 4, 2, 1025, 32, True),
    (1, 2, 2, 1, 96, True), (1, 2, 1, 255, 96, False), (2, 4, 4, 700, 96, True), (1, 4, 2, 1025, 96, False),
    (1, 8, 8, 2048, 96, False), (1, 8, 2, 2048, 96, True),
]


@pytest.mark.parametrize("shape", HEAD_DIMS, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_head_dims_32_and_96(attn, shape):
    B, Hq, Hkv, N, D, causal = shape
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=3500 + N + D + Hq)
    check_full(attn, q, k, v, causal, 1.0 / math.sqrt(D), str(shape))


WIDE_HEAD_DIMS = [
    # (B, Hq, Hkv, N, D, causal): head dims 192 and 256 (the one-tile, two-score-buffer kernel)
    (1, 2, 2, 1, 192, False), (1, 2, 1, 129, 192, True), (2, 4, 4, 700, 192, False), (1, 4, 2, 1025, 192, True),
    (1, 2, 2, 1, 256, True), (1, 2, 1, 255, 256, False), (2, 4, 4, 700, 256, True), (1, 4, 2, 1025, 256, False),
    (1, 4, 4, 2048, 256, False), (1, 8, 2, 2048, 256, True), (1, 2, 2, 384, 256, False),
]


@pytest.mark.parametrize("shape", WIDE_HEAD_DIMS,
                         ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_head_dims_192_and_256(attn, shape):
    B, Hq, Hkv, N, D, causal = shape
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=3600 + N + D + Hq)
    check_full(attn, q, k, v, causal, 1.0 / math.sqrt(D), str(shape))


WIDE_PERSISTENT = [
    # (B, Hq, Hkv, N, D, causal): the wide-head kernel's persistent CTAs walking many items
    (8, 16, 16, 2176, 192, True),    # causal tile pairs, 17 tiles per head: the middle tile is an item alone
    (4, 20, 4, 2048, 256, True),     # causal tile pairs, GQA group 5
    (10, 16, 16, 1920, 256, False),  # non-causal, 15 tiles per head, ~16 tiles per CTA
    (1, 6, 2, 1500, 192, True),      # causal, fewer pairs than SMs: single tiles, heaviest first
]


@pytest.mark.parametrize("shape", WIDE_PERSISTENT, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_wide_persistent_items_sampled(attn, shape):
    """Every item kind of the wide-head kernel's schedule, at sizes where CTAs take many items:
    rows on both sides of the first, middle and last tiles' edges of the first and last heads,
    plus seeded draws, each computed by the oracle on its own."""
    B, Hq, Hkv, N, D, causal = shape
    w = Workload(f"widep_B{B}_Hq{Hq}_N{N}_D{D}", B, Hq, Hkv, N, D, causal, 4200 + N + D)
    q, k, v = make_workload_inputs(w)
    T = -(-N // 128)
    rows = set()
    for b, h in ((0, 0), (B - 1, Hq - 1)):
        for t in (0, T // 2, T - 1):
            for i in (t * 128 - 1, t * 128, t * 128 + 127):
                if 0 <= i < N:
                    rows.add((b, h, i))
    g = np.random.default_rng(w.seed)
    for x in g.integers(0, B * Hq * N, 64):
        b, rem = divmod(int(x), Hq * N)
        rows.add((b, rem // N, rem % N))
    check_sampled(attn, w, q, k, v, full_heads=(), rows=sorted(rows))


@pytest.mark.parametrize("causal", [False, True])
def test_wide_head_dim_rescale_and_scales(attn, causal):
    """D = 256 with keys whose norm grows along the sequence (the lazy O rescale runs between
    the two score buffers) and with a negative and a zero scale."""
    B, Hq, Hkv, N, D = 1, 2, 1, 900, 256
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=3700 + causal)
    growth = torch.linspace(0.2, 3.0, N).reshape(1, 1, N, 1)
    k = (k.float() * growth).to(torch.bfloat16)
    check_full(attn, q, k, v, causal, 1.0 / math.sqrt(D), "wide growing keys")
    check_full(attn, q, k, v, causal, -0.05, "wide negative scale")
    check_full(attn, q, k, v, causal, 0.0, "wide zero scale")


@pytest.mark.parametrize("scale", [0.0, -0.0883883, 0.02, 0.5])
@pytest.mark.parametrize("causal", [False, True])
def test_scales(attn, scale, causal):
    q, k, v = make_qkv(1, 2, 2, 300, 128, seed=4001)
    check_full(attn, q, k, v, causal, scale, f"scale={scale}")


@pytest.mark.parametrize("causal", [False, True])
def test_growing_scores_exercise_rescale(attn, causal):
    """Keys whose norm grows along the sequence push each row's running max up by far
    more than the lazy-rescale threshold several times, so the O correction runs."""
    q, k, v = make_qkv(1, 2, 1, 1024, 128, seed=4002)
    grow = torch.linspace(0.2, 6.0, 1024).reshape(1, 1, 1024, 1)
    k = (k.float() * grow).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    check_full(attn, q, k, v, causal, 1.0 / math.sqrt(128), "growing scores")


def test_large_magnitude_inputs(attn):
    q, k, v = make_qkv(1, 2, 2, 512, 64, seed=4003)
    q = (q.float() * 8).to(torch.bfloat16)
    k = (k.float() * 8).to(torch.bfloat16)
    check_full(attn, q, k, v, True, 0.125, "large magnitude")


@pytest.mark.parametrize("D,N,causal", [(32, 300, False), (64, 300, False), (64, 300, True), (96, 300, False),
                                        (128, 300, True), (128, 300, False), (128, 2200, True), (192, 300, True),
                                        (256, 300, False)])
def test_one_dominant_key_per_row_at_every_column(attn, D, N, causal):
    """Row i's query is a * e_(i mod D) and key k's component k mod D is a, so row i's largest
    scores (all equal, ~300 above the others in log2 units) sit at the keys congruent to i modulo
    D.  Across a tile's rows every column of a key block then holds some row's maximum: a row
    maximum that skipped a column would leave 2^300 in that row's sum and a non-finite output.
    Covers the two-tile kernel (P over S and P beside O), the column-split and the wide kernels."""
    _, k, v = make_qkv(1, 2, 1, N, D, seed=4100 + N + D)
    scale = 1.0 / math.sqrt(D)
    a = float(torch.tensor(math.sqrt(300.0 / (scale * math.log2(math.e)))).to(torch.bfloat16))
    idx = torch.arange(N)
    qf = torch.zeros(1, 2, N, D)
    qf[:, :, idx, idx % D] = a
    kf = k.float().clone()
    kf[:, :, idx, idx % D] = a
    q, k = qf.to(torch.bfloat16), kf.to(torch.bfloat16)
    check_full(attn, q, k, v, causal, scale, f"dominant keys D{D} N{N} causal={causal}")


# ------------------------------------------------------------------ invariants on the GPU path

def test_identical_v_rows_give_that_row(attn):
    q, k, v = make_qkv(2, 4, 2, 700, 128, seed=4004)
    r = v[:, :, :1, :].expand(-1, -1, 700, -1).contiguous()
    for causal in (False, True):
        o, _ = gpu_forward(attn, q, k, r, causal, 1 / math.sqrt(128))
        ref = np.repeat(r.float().numpy()[:, :, :1, :].repeat(2, axis=1), 700, axis=2)
        assert np.max(np.abs(o - ref)) <= TOL_O_MAX


def test_causal_first_query_returns_v0(attn):
    q, k, v = make_qkv(2, 4, 1, 384, 64, seed=4005)
    o, lse = gpu_forward(attn, q, k, v, True, 0.125)
    v0 = v.float().numpy()[:, 0, 0, :]
    for h in range(4):
        assert np.max(np.abs(o[:, h, 0, :] - v0)) <= TOL_O_MAX
        lse0 = 0.125 * (q.double()[:, h, 0, :] * k.double()[:, 0, 0, :]).sum(-1).numpy()
        assert np.max(np.abs(lse[:, h, 0] - lse0)) <= TOL_LSE


def test_noncausal_kv_permutation_invariance(attn):
    q, k, v = make_qkv(1, 2, 2, 512, 128, seed=4006)
    perm = torch.randperm(512, generator=torch.Generator().manual_seed(1))
    o1, l1 = gpu_forward(attn, q, k, v, False, 0.09)
    o2, l2 = gpu_forward(attn, q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), False, 0.09)
    assert np.max(np.abs(o1 - o2)) <= TOL_O_MAX and np.max(np.abs(l1 - l2)) <= TOL_LSE


# ------------------------------------------------------------------ robustness

def test_every_output_written_and_guard_bands_untouched(attn):
    B, Hq, Hkv, N, D = 2, 4, 2, 333, 128
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hkv, N, D, seed=4007))
    guard = 4096
    o_buf = torch.full((B * Hq * N * D + guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * Hq * N + guard,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[: B * Hq * N * D].view(B, Hq, N, D)
    lse = l_buf[: B * Hq * N].view(B, Hq, N)
    attn.forward(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert torch.isnan(o_buf[B * Hq * N * D:]).all() and torch.isnan(l_buf[B * Hq * N:]).all()


def test_bitwise_deterministic(attn):
    q, k, v = (x.cuda() for x in make_qkv(2, 8, 2, 1536, 128, seed=4008))
    o1, l1 = attn.forward(q, k, v, causal=True)
    o2, l2 = attn.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_side_stream_and_host_path(attn):
    q, k, v = make_qkv(1, 4, 4, 640, 64, seed=4009)
    s = torch.cuda.Stream()
    o_h, l_h = attn.forward_from_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True, stream=s)
    o_ref, l_ref = attention_forward(q, k, v, True, 0.125)
    assert_close(o_h.float().numpy().astype(np.float64), l_h.numpy().astype(np.float64), o_ref, l_ref, "host path")


@pytest.mark.parametrize("B,Hq,Hkv,pieces", [(3, 4, 2, 4), (1, 8, 2, 4), (2, 2, 2, 1)])
def test_host_path_in_pieces_equals_device_call(attn, B, Hq, Hkv, pieces):
    """forward_from_host cuts the problem into batch rows (or KV-head groups when B == 1) and
    pipelines the copies; every piece is checked against the oracle.  (A small piece may take
    the split last wave, whose merge rounds differently from one whole call, so the pieces are
    not compared bit for bit with a single device call.)"""
    q, k, v = make_qkv(B, Hq, Hkv, 700, 128, seed=4011 + B)
    o_h, l_h = attn.forward_from_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=False, pieces=pieces)
    o_ref, l_ref = attention_forward(q, k, v, False, 128 ** -0.5)
    assert_close(o_h.float().numpy().astype(np.float64), l_h.numpy().astype(np.float64), o_ref, l_ref,
                 f"host path in {pieces} pieces")


def test_misaligned_device_pointer_rejected(attn):
    q, k, v = (x.cuda() for x in make_qkv(1, 1, 1, 128, 64, seed=4010))
    o = torch.empty(1 * 128 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(128, dtype=torch.float32, device="cuda")
    st = attn.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr() + 2, lse.data_ptr(),
                       1, 1, 1, 128, 64, 0, 0.125, torch.cuda.current_stream().cuda_stream)
    assert st == attn.ATTN_ERR_MISALIGNED


# ------------------------------------------------------------------ split last wave (workspace path)

SPLIT = [
    # (B, Hq, Hkv, N, D): non-causal shapes whose last wave is split into KV ranges
    (1, 1, 1, 2048, 128),   # 1 head x 8 pairs = 8 units, all in the split last wave
    (2, 3, 1, 1000, 128),   # ragged N, GQA 3:1
    (1, 4, 2, 1100, 64),    # tile 1 of the last pair empty, D=64
    (1, 2, 2, 1111, 128),   # ragged last block
    (4, 16, 16, 2048, 128), # the cfg2 shape: 3 whole waves + 68 units split in 2
    (1, 4, 4, 1500, 96),    # D=96
    (1, 3, 3, 2048, 32),    # D=32
]


@pytest.mark.parametrize("shape", SPLIT, ids=lambda s: "B{}_Hq{}_Hkv{}_N{}_D{}".format(*s))
def test_split_tail_matches_oracle_and_unsplit_path(attn, shape):
    B, Hq, Hkv, N, D = shape
    assert attn.attn_fwd_workspace_bytes(B, Hq, N, D, False) > 0, "shape does not exercise the split"
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=5000 + N + D)
    scale = 1 / math.sqrt(D)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o1, l1 = attn.forward(qd, kd, vd, causal=False, scale=scale, split=True)
    o2, l2 = attn.forward(qd, kd, vd, causal=False, scale=scale, split=False)
    torch.cuda.synchronize()
    assert attn.device_status() == (attn.ATTN_OK, 0)
    o_ref, l_ref = attention_forward(q, k, v, False, scale)
    for o, l in ((o1, l1), (o2, l2)):
        assert_close(o.float().cpu().numpy().astype(np.float64), l.cpu().numpy().astype(np.float64),
                     o_ref, l_ref, str(shape))
    # the two schedules differ only in fp32 summation order
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_split_tail_deterministic_across_calls_sharing_a_workspace(attn):
    q, k, v = (x.cuda() for x in make_qkv(1, 4, 4, 2048, 128, seed=5100))
    outs = [attn.forward(q, k, v, causal=False) for _ in range(3)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_split_workspace_too_small_is_rejected(attn):
    B, Hq, N, D = 1, 2, 2048, 128
    need = attn.attn_fwd_workspace_bytes(B, Hq, N, D, False)
    assert need > 0
    q, k, v = (x.cuda() for x in make_qkv(B, Hq, Hq, N, D, seed=5200))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hq, N, D, 0, 0.0883)
    assert attn.attn_fwd_ws(*args, ws.data_ptr(), need - 256, s) == attn.ATTN_ERR_INVALID_ARG
    assert attn.attn_fwd_ws(*args, ws.data_ptr(), need, s) == attn.ATTN_OK
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()


def test_default_calls_on_two_streams_at_once(attn):
    """forward() with its defaults (split last wave, cached workspace) on two streams whose
    kernels overlap: each stream gets its own workspace, so both results match the oracle.
    cfg2-sized non-causal problems (their last wave is split), different inputs per stream."""
    w = CFG2
    assert attn.attn_fwd_workspace_bytes(w.B, w.Hq, w.N, w.D, False) > 0
    inputs = [make_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed + 40 + i) for i in range(2)]
    dev_in = [tuple(x.cuda() for x in qkv) for qkv in inputs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    outs = []
    for _ in range(3):      # several rounds, so the two streams' launches interleave
        outs = []
        for (qd, kd, vd), s in zip(dev_in, streams):
            with torch.cuda.stream(s):
                outs.append(attn.forward(qd, kd, vd, causal=False, scale=w.softmax_scale, stream=s))
    torch.cuda.synchronize()
    assert attn.device_status() == (attn.ATTN_OK, 0)
    for (q, k, v), (o, lse) in zip(inputs, outs):
        o_ref, l_ref = attention_forward(q, k, v, False, w.softmax_scale)
        assert_close(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                     o_ref, l_ref, "two streams")


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal,pieces", [
    (3, 4, 2, 700, 128, False, 4), (1, 8, 2, 640, 64, True, 4), (2, 2, 2, 1, 128, False, 1),
    (1, 16, 4, 1100, 128, False, 3), (4, 16, 16, 2048, 128, False, 4), (2, 4, 1, 513, 96, True, 64),
])
def test_host_buffer_entry_point(attn, B, Hq, Hkv, N, D, causal, pieces):
    """attn_fwd_from_host through the C ABI: pinned host inputs, caller-owned device buffers,
    results in pinned host outputs; against the oracle, and the device buffers hold the same
    results."""
    q, k, v = make_qkv(B, Hq, Hkv, N, D, seed=4200 + N + pieces)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.full((B, Hq, N, D), float("nan"), dtype=torch.bfloat16).pin_memory()
    lh = torch.full((B, Hq, N), float("nan"), dtype=torch.float32).pin_memory()
    qd, kd, vd = (torch.empty(x.shape, dtype=x.dtype, device="cuda") for x in (q, k, v))
    od = torch.empty((B, Hq, N, D), dtype=torch.bfloat16, device="cuda")
    ld = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    need = attn.attn_fwd_from_host_workspace_bytes(B, Hq, Hkv, N, D, causal, pieces)
    assert need >= 0
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    scale = D ** -0.5
    s = torch.cuda.Stream()
    st = attn.attn_fwd_from_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(), lh.data_ptr(),
                                 qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), ld.data_ptr(),
                                 ws.data_ptr() if need > 0 else None, need, B, Hq, Hkv, N, D, causal, scale, pieces,
                                 s.cuda_stream)
    assert st == attn.ATTN_OK, attn.attn_status_string(st) + " " + attn.attn_last_cuda_error()
    # the call is synchronous: the host outputs are complete on return
    o_ref, l_ref = attention_forward(q, k, v, causal, scale)
    assert_close(oh.float().numpy().astype(np.float64), lh.numpy().astype(np.float64), o_ref, l_ref,
                 f"attn_fwd_from_host {pieces} pieces")
    torch.cuda.synchronize()
    assert torch.equal(od.cpu(), oh) and torch.equal(ld.cpu(), lh)
    assert attn.device_status() == (attn.ATTN_OK, 0)


def test_calls_from_several_host_threads(attn):
    """Four host threads, each on its own stream, call forward() (split last wave: a cached
    workspace per stream) and backward() on different inputs, several times and at once; every
    result equals the one computed beforehand on a single thread, bit for bit (the kernels are
    deterministic).  (attn_fwd_noalloc is left out: its one static array must not be used by
    kernels that overlap.)"""
    import threading

    B, Hq, Hkv, N, D = 2, 8, 4, 1100, 128        # non-causal: the last wave is split
    cases = [make_qkv(B, Hq, Hkv, N, D, seed=7000 + i) for i in range(4)]
    dev = [tuple(x.cuda() for x in c) for c in cases]
    dos = [torch.randn(B, Hq, N, D, generator=torch.Generator().manual_seed(7100 + i)).to(torch.bfloat16).cuda()
           for i in range(4)]
    expect = []
    for (q, k, v), do in zip(dev, dos):
        o, lse = attn.forward(q, k, v, causal=False)
        expect.append((o, lse, attn.backward(q, k, v, o, lse, do, causal=False)))
    torch.cuda.synchronize()
    errors = []

    def worker(i):
        try:
            q, k, v = dev[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(4):
                    o, lse = attn.forward(q, k, v, causal=False, stream=s)
                    grads = attn.backward(q, k, v, o, lse, dos[i], causal=False, stream=s)
                    s.synchronize()
                    eo, el, eg = expect[i]
                    assert torch.equal(o, eo) and torch.equal(lse, el), f"thread {i}: forward differs"
                    assert all(torch.equal(a, b) for a, b in zip(grads, eg)), f"thread {i}: backward differs"
        except Exception as exc:   # reported by the main thread
            errors.append(repr(exc))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    assert attn.device_status() == (attn.ATTN_OK, 0)
