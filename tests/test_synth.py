"""The seeded input recipe (CPU): workload shapes and seeds, counted FLOPs, and the generators'
determinism, dtype, layout and distribution.  Every parity case and every bench number rests on
these inputs, so the recipe is pinned here."""
import math

import pytest
import torch

import attn_inputs as synth


def test_the_four_configurations():
    want = {
        "cfg1": (1, 2, 2, 128, 64, False, 1001),
        "cfg2": (4, 16, 16, 2048, 128, False, 1002),
        "cfg3": (16, 16, 16, 4096, 128, True, 1003),
        "cfg4": (8, 32, 8, 8192, 128, True, 1004),
    }
    for name, (B, Hq, Hkv, N, D, causal, seed) in want.items():
        w = synth.get_workload(name)
        assert (w.B, w.Hq, w.Hkv, w.N, w.D, w.causal, w.seed) == (B, Hq, Hkv, N, D, causal, seed)
        assert w.softmax_scale == 1.0 / math.sqrt(D)


def test_counted_flops():
    """4 B Hq N^2 D, halved when causal: 137.4, 1099.5 and 4398.0 GFLOP for cfg2, 3, 4."""
    assert round(synth.get_workload("cfg2").flops / 1e9, 1) == 137.4
    assert round(synth.get_workload("cfg3").flops / 1e9, 1) == 1099.5
    assert round(synth.get_workload("cfg4").flops / 1e9, 1) == 4398.0
    assert synth.get_workload("cfg1").flops == 4.0 * 1 * 2 * 128 * 128 * 64


def test_sweep_points():
    pts = synth.sweep_points()
    assert len(pts) == 20
    assert [p.seed for p in pts] == list(range(2000, 2020))
    assert {(p.D, p.N, p.causal) for p in pts} == {(D, N, c) for D in (64, 128)
                                                    for N in (1024, 2048, 4096, 8192, 16384)
                                                    for c in (True, False)}
    for p in pts:
        assert p.B * p.N == 16384 and p.Hq == p.Hkv == 16


def test_wide_points():
    pts = synth.wide_points()
    assert {(p.D, p.N, p.causal) for p in pts} == {(D, N, c) for D in (192, 256) for N in (2048, 8192)
                                                    for c in (True, False)}
    assert [p.seed for p in pts] == list(range(3000, 3008))


def test_make_qkv_is_seeded_bf16_and_standard_normal():
    q, k, v = synth.make_qkv(2, 4, 2, 256, 64, seed=5)
    assert q.shape == (2, 4, 256, 64) and k.shape == v.shape == (2, 2, 256, 64)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    assert q.is_contiguous() and k.is_contiguous() and v.is_contiguous()
    q2, k2, v2 = synth.make_qkv(2, 4, 2, 256, 64, seed=5)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q3, _, _ = synth.make_qkv(2, 4, 2, 256, 64, seed=6)
    assert not torch.equal(q, q3)
    # q, k, v in that order from one generator: q of a bigger draw starts with the same values
    g = torch.Generator().manual_seed(5)
    ref = torch.randn((2, 4, 256, 64), generator=g, dtype=torch.float32)
    assert torch.equal(q, ref.to(torch.bfloat16))
    ref_k = torch.randn((2, 2, 256, 64), generator=g, dtype=torch.float32)
    assert torch.equal(k, ref_k.to(torch.bfloat16))
    x = torch.cat([t.float().flatten() for t in (q, k, v)])
    assert abs(x.mean().item()) < 0.02 and abs(x.std().item() - 1.0) < 0.02


def test_make_dout_and_e4m3_inputs():
    d = synth.make_dout(1, 2, 128, 64, seed=9)
    assert d.shape == (1, 2, 128, 64) and d.dtype == torch.bfloat16
    assert torch.equal(d, synth.make_dout(1, 2, 128, 64, seed=9))
    q8, k8, v8, descale = synth.make_qkv_e4m3(1, 2, 1, 128, 64, seed=9)
    assert q8.dtype == torch.float8_e4m3fn and q8.shape == (1, 2, 128, 64) and k8.shape == (1, 1, 128, 64)
    assert descale == 1.0 / synth.E4M3_AMPLITUDE
    # the E4M3 values are the same N(0,1) draws, times 16, rounded to E4M3
    g = torch.Generator().manual_seed(9)
    ref = torch.randn((1, 2, 128, 64), generator=g, dtype=torch.float32) * synth.E4M3_AMPLITUDE
    assert torch.equal(q8.float(), ref.to(torch.float8_e4m3fn).float())


@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (2, 3, 300), (4, 16, 2048)])
def test_sample_rows_cover_tile_edges(B, H, N):
    rows = synth.sample_rows(B, H, N, 50, seed=1)
    assert (0, 0, 0) in rows and (B - 1, H - 1, N - 1) in rows
    for t in range(0, N, 128):
        for i in (t - 1, t, t + 127):
            if 0 <= i < N:
                assert (B - 1, 0, i) in rows
    assert all(0 <= b < B and 0 <= h < H and 0 <= i < N for b, h, i in rows)
    assert rows == sorted(set(rows))
