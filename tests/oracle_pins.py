"""Pins for the fp64 oracle: facts fixed by the definition of attention, not by the oracle.

Each ``pin_*`` takes an implementation ``impl(q, k, v, causal, scale) -> (O, LSE)``
working on fp64 numpy arrays ``[B, H, N, D]`` and raises AssertionError when the
implementation disagrees with the fact.  tests/test_oracle.py runs every pin on
the oracle; tests/test_oracle_mutants.py plants mistakes in copies of the
oracle and checks that each planted mistake fails at least one pin.
"""
from __future__ import annotations

import functools
import json
import math
import os

import numpy as np
import torch
from threadpoolctl import threadpool_limits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_closed_form.json")
TIGHT = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


def _rand(shape, seed, scale=1.0):
    return _rng(seed).standard_normal(shape) * scale


# --- values worked out by hand ------------------------------------------------

def pin_golden(impl):
    """Hand-derived closed forms stored in tests/golden/tiny_closed_form.json."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v"))
        O, L = impl(q, k, v, c["causal"], c["scale"])
        _close(O, np.array(c["o"]), 1e-14, c["name"] + " O")
        _close(L, np.array(c["lse"]), 1e-14, c["name"] + " LSE")


# --- an independent scalar brute force on tiny inputs ---------------------------

def brute_force(q, k, v, causal, scale):
    """Triple loop in plain Python floats: math.exp and math.fsum, no numpy algebra."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    Dv = v.shape[3]
    group = Hq // Hkv
    O = np.zeros((B, Hq, N, Dv))
    L = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kh = h // group
            for i in range(N):
                allowed = [j for j in range(N) if (not causal) or j <= i]
                s = [scale * math.fsum(float(q[b, h, i, d]) * float(k[b, kh, j, d]) for d in range(D))
                     for j in allowed]
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                tot = math.fsum(w)
                for d in range(Dv):
                    O[b, h, i, d] = math.fsum(w[t] * float(v[b, kh, j, d]) for t, j in enumerate(allowed)) / tot
                L[b, h, i] = mx + math.log(tot)
    return O, L


def pin_brute_force(impl):
    """Agreement with the scalar brute force on tiny MHA and GQA problems."""
    for (B, Hq, Hkv, N, D, Dv, causal, scale, seed) in [
        (1, 1, 1, 5, 3, 3, False, 0.7, 1),
        (1, 1, 1, 6, 4, 2, True, 0.5, 2),
        (2, 2, 1, 7, 4, 4, False, 0.5, 3),
        (1, 4, 2, 8, 3, 5, True, 1.3, 4),
        (1, 2, 2, 1, 2, 2, True, 0.9, 5),
    ]:
        q = _rand((B, Hq, N, D), seed)
        k = _rand((B, Hkv, N, D), seed + 100)
        v = _rand((B, Hkv, N, Dv), seed + 200)
        O, L = impl(q, k, v, causal, scale)
        Ob, Lb = brute_force(q, k, v, causal, scale)
        _close(O, Ob, 1e-12, f"brute force O {B,Hq,Hkv,N,D,causal}")
        _close(L, Lb, 1e-12, f"brute force LSE {B,Hq,Hkv,N,D,causal}")


# --- a library special case ----------------------------------------------------

def pin_torch_sdpa(impl):
    """CPU fp64 torch SDPA (with GQA and causal flags) and torch.logsumexp agree."""
    for (B, Hq, Hkv, N, D, causal, seed) in [
        (2, 4, 4, 33, 16, False, 11), (1, 8, 2, 70, 32, True, 12), (1, 6, 3, 50, 8, False, 13),
    ]:
        scale = 1.0 / math.sqrt(D)
        q = _rand((B, Hq, N, D), seed)
        k = _rand((B, Hkv, N, D), seed + 1)
        v = _rand((B, Hkv, N, D), seed + 2)
        O, L = impl(q, k, v, causal, scale)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=(Hq != Hkv))
        kr = tk.repeat_interleave(Hq // Hkv, dim=1)
        s = scale * tq @ kr.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        _close(O, ref.numpy(), 1e-10, "torch sdpa O")
        _close(L, torch.logsumexp(s, dim=-1).numpy(), 1e-10, "torch logsumexp LSE")


# --- invariants and closed forms ----------------------------------------------

def pin_row_sums(impl):
    """With V = identity, O is the probability matrix: rows sum to 1, nonnegative, causal zeros."""
    for causal in (False, True):
        N, D = 9, 5
        q = _rand((1, 1, N, D), 21)
        k = _rand((1, 1, N, D), 22)
        v = np.eye(N)[None, None]
        P, _ = impl(q, k, v, causal, 0.8)
        _close(P.sum(axis=-1), np.ones((1, 1, N)), TIGHT, "row sums")
        assert np.all(P >= 0.0), "negative probability"
        if causal:
            _close(np.triu(P[0, 0], 1), np.zeros((N, N)), 0.0, "causal zeros above diagonal")
            assert np.all(np.diag(P[0, 0]) > 0.0), "diagonal key must carry weight"


def pin_identical_v_rows(impl):
    """Every V row equal to r gives O_i = r, causal or not."""
    for causal in (False, True):
        N, D = 11, 6
        r = _rand((D,), 31)
        v = np.broadcast_to(r, (1, 1, N, D)).copy()
        O, _ = impl(_rand((1, 2, N, D), 32), _rand((1, 1, N, D), 33), v, causal, 0.6)
        _close(O, np.broadcast_to(r, O.shape), TIGHT, "identical V rows")


def pin_causal_first_query(impl):
    """Causal row 0 sees key 0 only: O_0 = V_0 and LSE_0 = scale * q_0 . k_0 (per kv head)."""
    B, Hq, Hkv, N, D = 2, 4, 2, 7, 5
    q, k, v = _rand((B, Hq, N, D), 41), _rand((B, Hkv, N, D), 42), _rand((B, Hkv, N, D), 43)
    O, L = impl(q, k, v, True, 0.45)
    for b in range(B):
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            _close(O[b, h, 0], v[b, kh, 0], TIGHT, "causal O_0")
            _close(L[b, h, 0], 0.45 * float(q[b, h, 0] @ k[b, kh, 0]), TIGHT, "causal LSE_0")


def pin_permutation(impl):
    """Non-causal attention is unchanged by one permutation applied to K and V rows together."""
    N, D = 12, 4
    q, k, v = _rand((1, 2, N, D), 51), _rand((1, 2, N, D), 52), _rand((1, 2, N, D), 53)
    perm = _rng(54).permutation(N)
    O1, L1 = impl(q, k, v, False, 0.7)
    O2, L2 = impl(q, k[:, :, perm], v[:, :, perm], False, 0.7)
    _close(O1, O2, TIGHT, "permutation O")
    _close(L1, L2, TIGHT, "permutation LSE")


def pin_single_key(impl):
    """N = 1: O = V_0 and LSE = scale * q . k, causal or not."""
    for causal in (False, True):
        q, k, v = _rand((1, 1, 1, 3), 61), _rand((1, 1, 1, 3), 62), _rand((1, 1, 1, 3), 63)
        O, L = impl(q, k, v, causal, 1.7)
        _close(O, v, TIGHT, "N=1 O")
        _close(L, 1.7 * np.sum(q * k, axis=-1), TIGHT, "N=1 LSE")


def pin_uniform_scores(impl):
    """Q = 0 (or scale = 0): O_i is the mean of the allowed V rows and LSE_i = ln(#allowed)."""
    N, D = 10, 4
    k, v = _rand((1, 1, N, D), 71), _rand((1, 1, N, D), 72)
    for causal in (False, True):
        for q, scale in ((np.zeros((1, 1, N, D)), 0.9), (_rand((1, 1, N, D), 73), 0.0)):
            O, L = impl(q, k, v, causal, scale)
            counts = np.arange(1, N + 1) if causal else np.full(N, N)
            if causal:
                mean = np.cumsum(v[0, 0], axis=0) / counts[:, None]
            else:
                mean = np.broadcast_to(v[0, 0].mean(axis=0), (N, D))
            _close(O[0, 0], mean, TIGHT, "uniform O")
            _close(L[0, 0], np.log(counts), TIGHT, "uniform LSE")


def pin_causal_prefix(impl):
    """Causal row i equals non-causal attention over the prefix of length i + 1."""
    N, D = 9, 3
    q, k, v = _rand((1, 1, N, D), 81), _rand((1, 1, N, D), 82), _rand((1, 1, N, D), 83)
    Oc, Lc = impl(q, k, v, True, 0.8)
    for i in range(N):
        On, Ln = impl(q[:, :, : i + 1], k[:, :, : i + 1], v[:, :, : i + 1], False, 0.8)
        _close(Oc[0, 0, i], On[0, 0, i], TIGHT, f"prefix O row {i}")
        _close(Lc[0, 0, i], Ln[0, 0, i], TIGHT, f"prefix LSE row {i}")


def pin_gqa_is_repeated_mha(impl):
    """GQA equals MHA with each KV head repeated for its contiguous group of query heads."""
    for causal in (False, True):
        B, Hq, Hkv, N, D = 2, 8, 2, 6, 4
        q, k, v = _rand((B, Hq, N, D), 91), _rand((B, Hkv, N, D), 92), _rand((B, Hkv, N, D), 93)
        Og, Lg = impl(q, k, v, causal, 0.5)
        Om, Lm = impl(q, np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1), causal, 0.5)
        _close(Og, Om, TIGHT, "gqa O")
        _close(Lg, Lm, TIGHT, "gqa LSE")


def pin_key_shift(impl):
    """Adding u to every key shifts row i's scores by scale*q_i.u: O unchanged, LSE shifted."""
    N, D = 8, 4
    q, k, v = _rand((1, 1, N, D), 101), _rand((1, 1, N, D), 102), _rand((1, 1, N, D), 103)
    u = _rand((D,), 104) * 3.0
    for causal in (False, True):
        O1, L1 = impl(q, k, v, causal, 0.7)
        O2, L2 = impl(q, k + u, v, causal, 0.7)
        _close(O2, O1, 1e-11, "key shift O")
        _close(L2, L1 + 0.7 * (q @ u), 1e-11, "key shift LSE")


def pin_linear_in_v(impl):
    """O is linear in V: O(a V1 + V2) = a O(V1) + O(V2); LSE does not depend on V."""
    N, D = 7, 3
    q, k = _rand((1, 1, N, D), 111), _rand((1, 1, N, D), 112)
    v1, v2 = _rand((1, 1, N, 5), 113), _rand((1, 1, N, 5), 114)
    for causal in (False, True):
        Oa, La = impl(q, k, 2.5 * v1 + v2, causal, 1.1)
        O1, L1 = impl(q, k, v1, causal, 1.1)
        O2, _ = impl(q, k, v2, causal, 1.1)
        _close(Oa, 2.5 * O1 + O2, 1e-12, "linearity O")
        _close(La, L1, TIGHT, "LSE independent of V")


def pin_large_scores(impl):
    """Scores of magnitude ~1e3 stay finite: the max is subtracted before exponentiating."""
    q = np.array([[[[30.0, 0.0], [0.0, 0.0]]]])
    k = np.array([[[[30.0, 0.0], [29.0, 1.0]]]])
    v = np.array([[[[1.0], [2.0]]]])
    O, L = impl(q, k, v, False, 1.0)
    # row 0 scores (900, 870): weights (1, e^-30) / (1 + e^-30)
    w = math.exp(-30.0)
    _close(O[0, 0, 0], [(1.0 + 2.0 * w) / (1.0 + w)], 1e-15, "large-score O")
    _close(L[0, 0, 0], 900.0 + math.log1p(w), 1e-12, "large-score LSE")


def _single_threaded(pin):
    """Runs a pin with one BLAS thread and one torch thread.  The pins compare fp64 results at
    1e-10 and tighter; with several threads a library call was seen, rarely, to differ from its
    own single-threaded result by ~6e-10 (torch.logsumexp beside the oracle's LSE), which says
    nothing about the oracle."""
    @functools.wraps(pin)
    def run(impl):
        threads = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            with threadpool_limits(1):
                return pin(impl)
        finally:
            torch.set_num_threads(threads)
    return run


ALL_PINS = [_single_threaded(p) for p in (
    pin_golden, pin_brute_force, pin_torch_sdpa, pin_row_sums, pin_identical_v_rows,
    pin_causal_first_query, pin_permutation, pin_single_key, pin_uniform_scores,
    pin_causal_prefix, pin_gqa_is_repeated_mha, pin_key_shift, pin_linear_in_v,
    pin_large_scores,
)]
