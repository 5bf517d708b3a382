"""Where the E4M3-forward and backward tolerance bars come from (CPU only).

Neither path has a tolerance fixed by the method, so each bar is derived: the rounding the
kernel performs is emulated on the CPU, step by step, on seeded inputs; its error against
the fp64 oracle is the envelope; the bar the GPU parity tests use is then required to sit
between 2x and 4x that envelope (2x: room for the kernel's other rounding differences, such
as its summation order and its polynomial exponentials; at most 4x: the bar must not be
loose enough to hide a real mistake).

E4M3 forward (tests/test_parity_fp8.py): scores are exact fp32 sums of E4M3 products; the
running row maximum is replaced only when it grows by more than 8 (base 2); p = 2^(s*c - m)
in fp32; P is rounded to E4M3 (nearest even) as the A operand of P V; the row sums use the
fp32 p; O accumulates in fp32, is rescaled when the maximum moves, divided by l, scaled by
the V descale and rounded to bf16.

Backward (tests/test_parity_bwd.py): from the forward's bf16 O and fp32 LSE,
P = 2^(s * scale * log2 e - LSE * log2 e) in fp32 with s an fp32 sum of bf16 products;
delta = fp32 row sums of dO o O (bf16 values); dP = dO V^T in fp32; dS = P (dP - delta) in
fp32, rounded to bf16; P rounded to bf16; dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K
accumulated in fp32 and rounded to bf16 (scale applied before the rounding).
"""
import math

import numpy as np
import pytest
import torch

import test_parity_bwd as bwd_bars
import test_parity_fp8 as fp8_bars
from attn_inputs import make_dout, make_qkv, make_qkv_e4m3
from oracle import attention_backward, attention_forward

LOG2E = 1.4426950408889634
BLOCK = 128
RESCALE_LOG2 = 8.0


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def e4m3(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).float().numpy()


def emulate_fp8_head(q8, k8, v8, qd, kd, vd, causal, scale):
    """One head of the E4M3 forward, block by block as the kernel rounds it.
    q8, k8, v8: the stored E4M3 values (as fp64, exact); returns (O bf16 values, LSE fp32)."""
    N = q8.shape[0]
    c = np.float32(abs(scale * qd * kd) * LOG2E)
    sgn = 1.0 if scale * qd * kd >= 0 else -1.0
    s_all = (sgn * (q8 @ k8.T)).astype(np.float32)          # exact products; fp32 sums
    if causal:
        s_all = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, s_all).astype(np.float32)
    m = np.full(N, -np.inf, dtype=np.float32)
    l = np.zeros(N, dtype=np.float32)
    o = np.zeros((N, v8.shape[1]), dtype=np.float32)
    nblk = (N + BLOCK - 1) // BLOCK
    for j in range(nblk):
        rows = np.arange(N) if not causal else np.arange(N)[np.arange(N) // BLOCK >= j]
        if rows.size == 0:
            continue
        cols = slice(j * BLOCK, min(N, (j + 1) * BLOCK))
        s = s_all[rows, cols]
        m_new = np.maximum(m[rows], (s.max(axis=1) * c).astype(np.float32))
        first = np.isneginf(m[rows])
        upd = first | (m_new > m[rows] + np.float32(RESCALE_LOG2))
        alpha = np.where(first, np.float32(1.0), np.exp2(np.where(upd, m[rows] - m_new, 0.0)).astype(np.float32))
        m_use = np.where(upd, m_new, m[rows]).astype(np.float32)
        p = np.exp2((s * c - m_use[:, None]).astype(np.float32)).astype(np.float32)
        l[rows] = l[rows] * alpha + p.sum(axis=1, dtype=np.float32)
        o[rows] = o[rows] * alpha[:, None] + (e4m3(p).astype(np.float64) @ v8[cols]).astype(np.float32)
        m[rows] = m_use
    out = bf16(o * np.float32(vd) / l[:, None])
    lse = ((m + np.log2(l)) * np.float32(math.log(2.0))).astype(np.float32)
    return out, lse


FP8_SHAPES = [(512, 64, True), (1024, 128, True), (2048, 128, True), (2048, 128, False), (1024, 64, False),
              (512, 32, True), (1024, 32, False), (1024, 96, True), (2048, 96, False), (1024, 192, True),
              (1024, 256, False)]


@pytest.fixture(scope="module")
def fp8_envelope():
    """(max |dO|, the largest per-shape mean |dO|, max |dLSE|): the parity tests bound the
    mean per test case, so the envelope's mean is the worst shape's."""
    dmax, mean_worst, lmax = 0.0, 0.0, 0.0
    for n, d, causal in FP8_SHAPES:
        q8, k8, v8, ds = make_qkv_e4m3(1, 2, 2, n, d, 7000 + n + d)
        scale = d ** -0.5
        deq = [x.float().numpy().astype(np.float64) for x in (q8, k8, v8)]
        o_ref, l_ref = attention_forward(*(x * ds for x in deq), causal, scale)
        errs = []
        for h in range(2):
            o, l = emulate_fp8_head(deq[0][0, h], deq[1][0, h], deq[2][0, h], ds, ds, ds, causal, scale)
            errs.append(np.abs(o - o_ref[0, h]))
            lmax = max(lmax, np.abs(l - l_ref[0, h]).max())
        dmax = max(dmax, max(e.max() for e in errs))
        mean_worst = max(mean_worst, float(np.mean(errs)))
    return dmax, mean_worst, lmax


def test_fp8_bars_sit_two_to_four_times_above_the_emulated_envelope(fp8_envelope):
    emax, emean, elmax = fp8_envelope
    assert 2 * emax <= fp8_bars.TOL_O_MAX <= 4 * emax, (emax, fp8_bars.TOL_O_MAX)
    assert 2 * emean <= fp8_bars.TOL_O_MEAN <= 4 * emean, (emean, fp8_bars.TOL_O_MEAN)
    # the scores are exact, so LSE keeps the bf16 forward's bound with room to spare
    assert 2 * elmax <= fp8_bars.TOL_LSE


def test_fp8_emulation_is_sensitive_to_the_probability_rounding():
    """A check of the emulation itself: without the E4M3 rounding of P its error falls to the
    bf16 output rounding (at least 10x smaller), so the envelope above is the P rounding's."""
    q8, k8, v8, ds = make_qkv_e4m3(1, 1, 1, 512, 64, 7100)
    deq = [x.float().numpy().astype(np.float64)[0, 0] for x in (q8, k8, v8)]
    o_ref, _ = attention_forward(*(x[None, None] * ds for x in deq), True, 0.125)
    o, _ = emulate_fp8_head(*deq, ds, ds, ds, True, 0.125)
    global e4m3
    saved = e4m3
    try:
        e4m3 = lambda x: np.asarray(x, dtype=np.float32)  # noqa: E731
        o_exact, _ = emulate_fp8_head(*deq, ds, ds, ds, True, 0.125)
    finally:
        e4m3 = saved
    assert np.abs(o_exact - o_ref[0, 0]).mean() * 10 <= np.abs(o - o_ref[0, 0]).mean()


def emulate_bwd_head(q, k, v, o16, lse32, do, causal, scale):
    """One head's gradients as the backward kernels round them (inputs: bf16 values as fp64;
    o16 the forward's bf16 O, lse32 its fp32 LSE).  Returns (dq, dk, dv) as bf16 values."""
    N = q.shape[0]
    s = (q @ k.T).astype(np.float32)
    x = s * np.float32(scale * LOG2E) + (-lse32 * np.float32(LOG2E)).astype(np.float32)[:, None]
    p = np.exp2(x.astype(np.float32)).astype(np.float32)
    if causal:
        p = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], np.float32(0.0), p)
    delta = (do.astype(np.float32) * o16.astype(np.float32)).sum(axis=1, dtype=np.float32)
    dp = (do @ v.T).astype(np.float32)
    ds = bf16(p * (dp - delta[:, None]))
    pb = bf16(p)
    dv = bf16((pb.astype(np.float64).T @ do).astype(np.float32))
    dk = bf16(((ds.astype(np.float64).T @ q).astype(np.float32)) * np.float32(scale))
    dq = bf16(((ds.astype(np.float64) @ k).astype(np.float32)) * np.float32(scale))
    return dq, dk, dv


BWD_SHAPES = [(384, 64, True), (512, 128, False), (768, 128, True), (1024, 64, False), (1024, 128, True)]


@pytest.fixture(scope="module")
def bwd_envelope():
    worst_max, worst_mean = 0.0, 0.0
    for n, d, causal in BWD_SHAPES:
        q, k, v = make_qkv(1, 1, 1, n, d, 7200 + n + d)
        do = make_dout(1, 1, n, d, 7300 + n + d)
        scale = d ** -0.5
        o_ref, l_ref = attention_forward(q, k, v, causal, scale)
        refs = attention_backward(q, k, v, do, causal, scale)
        f = [x.float().numpy().astype(np.float64)[0, 0] for x in (q, k, v, do)]
        got = emulate_bwd_head(f[0], f[1], f[2], bf16(o_ref[0, 0]).astype(np.float64),
                               l_ref[0, 0].astype(np.float32), f[3], causal, scale)
        for g, r in zip(got, refs):
            e = np.abs(g - r[0, 0])
            worst_max = max(worst_max, e.max() / np.abs(r).max())
            worst_mean = max(worst_mean, e.mean() / np.abs(r).mean())
    return worst_max, worst_mean


def test_bwd_bars_sit_two_to_four_times_above_the_emulated_envelope(bwd_envelope):
    emax, emean = bwd_envelope
    assert 2 * emax <= bwd_bars.TOL_MAX <= 4 * emax, (emax, bwd_bars.TOL_MAX)
    assert 2 * emean <= bwd_bars.TOL_MEAN <= 4 * emean, (emean, bwd_bars.TOL_MEAN)
