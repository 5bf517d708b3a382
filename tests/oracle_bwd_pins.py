"""Pins for the fp64 backward oracle: facts fixed by the calculus of attention, not by the oracle.

Each ``pin_bwd_*`` takes an implementation
``impl(q, k, v, do, causal, scale) -> (dq, dk, dv)`` on fp64 numpy arrays
(q, do ``[B, Hq, N, D]``; k, v ``[B, Hkv, N, D]``) and raises AssertionError when
the implementation disagrees.  The gradients are those of the scalar
L = sum(O * do) with O the attention output.  tests/test_oracle_bwd.py runs the
pins on the oracle; the same file plants mistakes in copies of the oracle's
backward and checks that each fails at least one pin.

The finite-difference pin differentiates the oracle's forward, which is pinned on
its own (tests/oracle_pins.py); every other pin is independent of the oracle.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import attention_forward
from oracle_pins import _single_threaded


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


def _inputs(B, Hq, Hkv, N, D, seed):
    return (_rand((B, Hq, N, D), seed), _rand((B, Hkv, N, D), seed + 1), _rand((B, Hkv, N, D), seed + 2),
            _rand((B, Hq, N, D), seed + 3))


# --- derivatives by central differences of the (separately pinned) forward ----------

def pin_bwd_finite_differences(impl):
    """Every entry of dq, dk, dv against a central difference of L = sum(O * do)."""
    h = 1e-5
    for causal in (False, True):
        q, k, v, do = _inputs(1, 2, 1, 5, 3, 11 + causal)
        scale = 0.61
        dq, dk, dv = impl(q, k, v, do, causal, scale)

        def loss(qq, kk, vv):
            return float(np.sum(attention_forward(qq, kk, vv, causal, scale)[0] * do))

        for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy()
                xm = x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = [q, k, v]
                args_m = [q, k, v]
                pos = ("dq", "dk", "dv").index(name)
                args_p[pos] = xp
                args_m[pos] = xm
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            _close(g, num, 1e-7, f"finite differences {name} causal={causal}")


# --- a library routine: torch autograd through CPU fp64 SDPA ----------------------

def pin_bwd_torch_autograd(impl):
    """Agrees with autograd through torch's fp64 scaled_dot_product_attention (GQA enabled)."""
    for causal in (False, True):
        q, k, v, do = _inputs(2, 4, 2, 9, 4, 21 + causal)
        scale = 0.37
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale,
                                                               enable_gqa=True)
        out.backward(torch.tensor(do))
        dq, dk, dv = impl(q, k, v, do, causal, scale)
        _close(dq, tq.grad.numpy(), 1e-10, f"torch dq causal={causal}")
        _close(dk, tk.grad.numpy(), 1e-10, f"torch dk causal={causal}")
        _close(dv, tv.grad.numpy(), 1e-10, f"torch dv causal={causal}")


# --- an independent scalar brute force through the softmax Jacobian -----------------

def brute_force_bwd(q, k, v, do, causal, scale):
    """Plain Python loops: dS_ij = sum_l dP_il * dP_il/dS_ij with the softmax Jacobian
    P_il ([l == j] - P_ij), written out term by term with math.fsum."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            allowed = [[(j <= i) or not causal for j in range(N)] for i in range(N)]
            P = [[0.0] * N for _ in range(N)]
            for i in range(N):
                s = [scale * math.fsum(q[b, h, i, d] * k[b, kh, j, d] for d in range(D)) if allowed[i][j] else None
                     for j in range(N)]
                mx = max(x for x in s if x is not None)
                e = [math.exp(x - mx) if x is not None else 0.0 for x in s]
                tot = math.fsum(e)
                P[i] = [x / tot for x in e]
            dP = [[math.fsum(do[b, h, i, d] * v[b, kh, j, d] for d in range(D)) for j in range(N)]
                  for i in range(N)]
            dS = [[math.fsum(dP[i][l] * P[i][l] * ((1.0 if l == j else 0.0) - P[i][j]) for l in range(N))
                   for j in range(N)] for i in range(N)]
            for i in range(N):
                for d in range(D):
                    dq[b, h, i, d] = scale * math.fsum(dS[i][j] * k[b, kh, j, d] for j in range(N))
            for j in range(N):
                for d in range(D):
                    dk[b, kh, j, d] += scale * math.fsum(dS[i][j] * q[b, h, i, d] for i in range(N))
                    dv[b, kh, j, d] += math.fsum(P[i][j] * do[b, h, i, d] for i in range(N))
    return dq, dk, dv


def pin_bwd_brute_force(impl):
    for causal in (False, True):
        q, k, v, do = _inputs(1, 2, 1, 4, 3, 31 + causal)
        ref = brute_force_bwd(q, k, v, do, causal, 0.8)
        got = impl(q, k, v, do, causal, 0.8)
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            _close(a, b, 1e-12, f"brute force {name} causal={causal}")


# --- closed forms and invariants -------------------------------------------------------

def pin_bwd_dv_sums(impl):
    """Probability rows sum to 1, so the rows of dV of a KV head sum to the dO rows of its query heads."""
    for causal in (False, True):
        q, k, v, do = _inputs(2, 4, 2, 7, 3, 41 + causal)
        _, _, dv = impl(q, k, v, do, causal, 0.5)
        want = do.reshape(2, 2, 2, 7, 3).sum(axis=(2, 3))
        _close(dv.sum(axis=2), want, 1e-12, f"dV row sums causal={causal}")


def pin_bwd_dk_sums_zero(impl):
    """Each row of dS sums to 0 (softmax is shift-invariant), so the rows of dK sum to 0."""
    for causal in (False, True):
        q, k, v, do = _inputs(2, 4, 2, 7, 3, 51 + causal)
        _, dk, _ = impl(q, k, v, do, causal, 0.9)
        _close(dk.sum(axis=2), np.zeros((2, 2, 3)), 1e-12, f"dK row sums causal={causal}")


def pin_bwd_key_shift(impl):
    """Adding one vector to every key shifts each score row by a constant: no gradient changes."""
    for causal in (False, True):
        q, k, v, do = _inputs(1, 2, 2, 6, 3, 61 + causal)
        a = impl(q, k, v, do, causal, 0.7)
        b = impl(q, k + np.array([0.3, -1.1, 0.6]), v, do, causal, 0.7)
        for name, x, y in zip(("dq", "dk", "dv"), a, b):
            _close(x, y, 1e-12, f"key shift {name} causal={causal}")


def pin_bwd_uniform(impl):
    """scale = 0: uniform weights over the allowed keys; dq = dk = 0 and dV_j = sum_i dO_i / n_i."""
    for causal in (False, True):
        q, k, v, do = _inputs(1, 1, 1, 5, 2, 71 + causal)
        dq, dk, dv = impl(q, k, v, do, causal, 0.0)
        _close(dq, np.zeros_like(dq), 1e-15, "uniform dq")
        _close(dk, np.zeros_like(dk), 1e-15, "uniform dk")
        want = np.zeros((5, 2))
        for i in range(5):
            n_i = i + 1 if causal else 5
            for j in range(n_i):
                want[j] += do[0, 0, i] / n_i
        _close(dv[0, 0], want, 1e-14, f"uniform dv causal={causal}")


def pin_bwd_identical_v(impl):
    """All V rows equal: O does not depend on the weights, so dq = dk = 0."""
    for causal in (False, True):
        q, k, _, do = _inputs(1, 2, 1, 6, 3, 81 + causal)
        v = np.broadcast_to(np.array([0.4, -2.0, 1.5]), (1, 1, 6, 3)).copy()
        dq, dk, _ = impl(q, k, v, do, causal, 0.8)
        _close(dq, np.zeros_like(dq), 1e-12, "identical-V dq")
        _close(dk, np.zeros_like(dk), 1e-12, "identical-V dk")


def pin_bwd_single_key(impl):
    """N = 1: O = V, so dV = dO (summed over the group) and dq = dk = 0."""
    q, k, v, do = _inputs(1, 2, 1, 1, 4, 91)
    dq, dk, dv = impl(q, k, v, do, False, 1.3)
    _close(dv[0, 0, 0], do[0, 0, 0] + do[0, 1, 0], 1e-15, "single-key dv")
    _close(dq, np.zeros_like(dq), 1e-15, "single-key dq")
    _close(dk, np.zeros_like(dk), 1e-15, "single-key dk")


def pin_bwd_causal_first_query(impl):
    """Causal query 0 sees only key 0 with weight 1: dq_0 = 0, and key N-1 is seen only
    by query N-1, so dv_{N-1} = P_{N-1,N-1} do_{N-1} with P from the last query's scores."""
    q, k, v, do = _inputs(1, 1, 1, 5, 3, 101)
    scale = 0.9
    dq, _, dv = impl(q, k, v, do, True, scale)
    _close(dq[0, 0, 0], np.zeros(3), 1e-15, "causal dq_0")
    s = scale * k[0, 0] @ q[0, 0, 4]
    p_last = math.exp(s[4] - s.max()) / np.exp(s - s.max()).sum()
    _close(dv[0, 0, 4], p_last * do[0, 0, 4], 1e-14, "causal dv_last")


def pin_bwd_gqa_is_repeated_mha(impl):
    """GQA gradients: dq equals MHA's on repeated K/V; dk, dv are MHA's summed over each group."""
    for causal in (False, True):
        q, k, v, do = _inputs(1, 4, 2, 5, 3, 111 + causal)
        g = impl(q, k, v, do, causal, 0.6)
        kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
        m = impl(q, kr, vr, do, causal, 0.6)
        _close(g[0], m[0], 1e-12, "gqa dq")
        _close(g[1], m[1].reshape(1, 2, 2, 5, 3).sum(axis=2), 1e-12, "gqa dk")
        _close(g[2], m[2].reshape(1, 2, 2, 5, 3).sum(axis=2), 1e-12, "gqa dv")


def pin_bwd_linear_in_do(impl):
    """The gradients of sum(O * dO) are linear in dO."""
    q, k, v, d1 = _inputs(1, 2, 2, 6, 3, 121)
    d2 = _rand(d1.shape, 125)
    a = impl(q, k, v, d1, True, 0.5)
    b = impl(q, k, v, d2, True, 0.5)
    c = impl(q, k, v, 2.0 * d1 - 3.0 * d2, True, 0.5)
    for name, x, y, z in zip(("dq", "dk", "dv"), a, b, c):
        _close(z, 2.0 * x - 3.0 * y, 1e-12, f"linearity {name}")


GOLDEN_BWD = os.path.join(os.path.dirname(__file__), "golden", "tiny_backward_closed_form.json")


def pin_bwd_golden(impl):
    """Hand-derived closed forms stored in tests/golden/tiny_backward_closed_form.json (two keys,
    D = 1: non-causal at scale 1 and 2, causal, and two query heads sharing one KV head)."""
    with open(GOLDEN_BWD) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v, do = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v", "do"))
        dq, dk, dv = impl(q, k, v, do, c["causal"], c["scale"])
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            _close(got, np.array(c[name]), 1e-12, f"golden {c['name']} {name}")


# one BLAS thread and one torch thread, as for the forward pins (their tolerances are as tight)
ALL_BWD_PINS = [_single_threaded(p) for p in (
    pin_bwd_golden, pin_bwd_finite_differences, pin_bwd_torch_autograd, pin_bwd_brute_force, pin_bwd_dv_sums,
    pin_bwd_dk_sums_zero, pin_bwd_key_shift, pin_bwd_uniform, pin_bwd_identical_v, pin_bwd_single_key,
    pin_bwd_causal_first_query, pin_bwd_gqa_is_repeated_mha, pin_bwd_linear_in_do,
)]
