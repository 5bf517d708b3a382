"""Pins for the fp64 oracle of the RoPE backward, and planted mistakes that must fail them (CPU).

The backward of the rotary step is the rotation's transpose (each pair is turned by an
orthogonal 2x2 matrix), so the gradients with respect to q and k are R^T applied to the
attention backward's gradients at the rotated inputs.  The pins fix that transpose by facts
that do not depend on how it is computed -- it undoes the rotation, it is the rotation's adjoint
under the dot product, one pair worked by hand -- and fix the whole backward by central finite
differences of the (pinned) RoPE forward and by position 0, where the rotation is the identity.
"""
import math

import numpy as np
import pytest

from oracle import attention_backward, attention_backward_rope, attention_forward_rope, rope_rotate
from oracle import rope_rotate_transpose


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- the transpose alone

def pin_undoes_the_rotation(tr):
    x = np.random.default_rng(11).standard_normal((2, 3, 17, 16))
    _close(tr(rope_rotate(x, 500.0), 500.0), x, 1e-13, "R^T R x = x")
    _close(rope_rotate(tr(x, 500.0), 500.0), x, 1e-13, "R R^T x = x")


def pin_adjoint(tr):
    """<R x, y> = <x, R^T y> for random x, y (the defining property of the transpose)."""
    rng = np.random.default_rng(12)
    x, y = rng.standard_normal((9, 32)), rng.standard_normal((9, 32))
    _close(np.sum(rope_rotate(x, 10000.0) * y), np.sum(x * tr(y, 10000.0)), 1e-12, "adjoint")


def pin_hand_pair(tr):
    """D = 4, base = 100, position 2: pairs (0, 2) and (1, 3) turned back by 2 rad and 0.2 rad."""
    g = np.zeros((3, 4))
    g[2] = [1.0, 2.0, 3.0, 4.0]
    c2, s2, c02, s02 = math.cos(2.0), math.sin(2.0), math.cos(0.2), math.sin(0.2)
    want = [1 * c2 + 3 * s2, 2 * c02 + 4 * s02, 3 * c2 - 1 * s2, 4 * c02 - 2 * s02]
    _close(tr(g, 100.0)[2], want, 1e-14, "hand pair")


TRANSPOSE_PINS = [pin_undoes_the_rotation, pin_adjoint, pin_hand_pair]


@pytest.mark.parametrize("pin", TRANSPOSE_PINS, ids=lambda p: p.__name__)
def test_oracle_rope_transpose_pins(pin):
    pin(rope_rotate_transpose)


# ---------------------------------------------------------------- the whole backward

def _loss(q, k, v, do, causal, scale, base):
    O, _ = attention_forward_rope(q, k, v, causal, scale, base)
    return float(np.sum(O * do))


@pytest.mark.parametrize("causal", [False, True])
def test_oracle_rope_backward_matches_finite_differences(causal):
    rng = np.random.default_rng(13)
    B, Hq, Hkv, N, D, scale, base = 1, 2, 1, 5, 4, 0.6, 30.0
    q, k, v = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, Hkv, N, D))
    do = rng.standard_normal((B, Hq, N, D))
    grads = attention_backward_rope(q, k, v, do, causal, scale, base)
    h = 1e-6
    for name, x, g in zip(("dq", "dk", "dv"), (q, k, v), grads):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if t is x else t for t in (q, k, v)]
            args_m = [xm if t is x else t for t in (q, k, v)]
            num[idx] = (_loss(*args_p, do, causal, scale, base) - _loss(*args_m, do, causal, scale, base)) / (2 * h)
        _close(g, num, 1e-7, f"finite differences {name} causal={causal}")


def test_oracle_rope_backward_at_position_zero_is_the_plain_backward():
    rng = np.random.default_rng(14)
    q, k, v, do = (rng.standard_normal((2, 3, 1, 8)) for _ in range(4))
    for a, b in zip(attention_backward_rope(q, k, v, do, False, 0.5), attention_backward(q, k, v, do, False, 0.5)):
        _close(a, b, 1e-15, "N = 1")


# ---------------------------------------------------------------- planted mistakes

def _mutant(kind):
    def tr(g, base):
        g = np.asarray(g, dtype=np.float64)
        N, D = g.shape[-2], g.shape[-1]
        p = np.arange(N, dtype=np.float64)[:, None]
        d = np.arange(D // 2, dtype=np.float64)[None, :]
        th = p * base ** (-2.0 * d / D)
        c, s = np.cos(th), np.sin(th)
        a, b = g[..., : D // 2], g[..., D // 2:]
        if kind == "not_transposed":          # the forward rotation again
            u, w = a * c - b * s, b * c + a * s
        elif kind == "halves_swapped":
            u, w = b * c - a * s, a * c + b * s
        elif kind == "sin_dropped":
            u, w = a * c, b * c
        else:                                 # "angle_doubled"
            c2, s2 = np.cos(2 * th), np.sin(2 * th)
            u, w = a * c2 + b * s2, b * c2 - a * s2
        return np.concatenate([u, w], axis=-1)
    return tr


@pytest.mark.parametrize("kind", ["not_transposed", "halves_swapped", "sin_dropped", "angle_doubled"])
def test_planted_transpose_mistake_fails_a_pin(kind):
    caught = []
    for pin in TRANSPOSE_PINS:
        try:
            pin(_mutant(kind))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {kind} passed every pin"
