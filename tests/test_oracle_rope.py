"""Pins for the fp64 RoPE oracle, and planted mistakes that must fail them (CPU only).

Each pin takes ``rot(x, base) -> x'`` rotating x [..., N, D] by the angles of positions
0..N-1 ("rotate-half" pairing: element d with element d + D/2).  The values below are worked
out by hand from that definition with math.cos / math.sin on explicit numbers.
"""
import math

import numpy as np
import pytest

from oracle import attention_forward, attention_forward_rope, rope_angles, rope_rotate


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


def pin_hand_values(rot):
    """D = 4, base = 100: theta(p, 0) = p, theta(p, 1) = p * 100^(-1/2) = p / 10.
    Row p = 2 of x = [1, 2, 3, 4] pairs (1, 3) rotated by 2 rad and (2, 4) by 0.2 rad."""
    x = np.zeros((3, 4))
    x[2] = [1.0, 2.0, 3.0, 4.0]
    y = rot(x, 100.0)
    c2, s2, c02, s02 = math.cos(2.0), math.sin(2.0), math.cos(0.2), math.sin(0.2)
    want = [1 * c2 - 3 * s2, 2 * c02 - 4 * s02, 3 * c2 + 1 * s2, 4 * c02 + 2 * s02]
    _close(y[2], want, 1e-14, "hand values p=2")


def pin_last_frequency(rot):
    """D = 8, base = 10000, p = 5: the last pair (3, 7) turns by 5 * 10000^(-6/8) = 0.005 rad,
    the first pair (0, 4) by 5 rad."""
    x = np.zeros((6, 8))
    x[5] = [1.0, 0.0, 0.0, 2.0, 0.5, 0.0, 0.0, -1.0]
    y = rot(x, 10000.0)
    t = 0.005
    _close([y[5, 3], y[5, 7]], [2 * math.cos(t) + 1 * math.sin(t), -1 * math.cos(t) + 2 * math.sin(t)], 1e-14,
           "last pair")
    _close([y[5, 0], y[5, 4]], [1 * math.cos(5.0) - 0.5 * math.sin(5.0), 0.5 * math.cos(5.0) + 1 * math.sin(5.0)],
           1e-14, "first pair")


def pin_two_dims(rot):
    """D = 2: one pair turned by p radians (base^0 = 1) for every position p."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 7, 2))
    y = rot(x, 10000.0)
    p = np.arange(7)
    _close(y[..., 0], x[..., 0] * np.cos(p) - x[..., 1] * np.sin(p), 1e-14, "D=2 first")
    _close(y[..., 1], x[..., 1] * np.cos(p) + x[..., 0] * np.sin(p), 1e-14, "D=2 second")


def pin_position_zero(rot):
    x = np.random.default_rng(4).standard_normal((3, 5, 16))
    _close(rot(x, 10000.0)[:, 0], x[:, 0], 0.0, "position 0 unchanged")


def pin_norm_preserved(rot):
    x = np.random.default_rng(5).standard_normal((2, 9, 32))
    y = rot(x, 500.0)
    half = 16
    _close(y[..., :half] ** 2 + y[..., half:] ** 2, x[..., :half] ** 2 + x[..., half:] ** 2, 1e-12, "pair norms")


def pin_relative_position(rot):
    """rot(q at i) . rot(k at j) depends on i - j only."""
    rng = np.random.default_rng(6)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    N = 12
    Q = np.tile(q, (N, 1))
    K = np.tile(k, (N, 1))
    rq, rk = rot(Q, 10000.0), rot(K, 10000.0)
    for (i, j, t) in [(3, 1, 5), (7, 7, 2), (2, 6, 4)]:
        _close(rq[i] @ rk[j], rq[i + t] @ rk[j + t], 1e-12, f"relative position {(i, j, t)}")


ROPE_PINS = [pin_hand_values, pin_last_frequency, pin_two_dims, pin_position_zero, pin_norm_preserved,
             pin_relative_position]


@pytest.mark.parametrize("pin", ROPE_PINS, ids=lambda p: p.__name__)
def test_oracle_rope_pins(pin):
    pin(rope_rotate)


def test_rope_angles_table():
    th = rope_angles(4, 8, 10000.0)
    assert th.shape == (4, 4)
    _close(th[3], [3.0, 3.0 * 0.1, 3.0 * 0.01, 3.0 * 0.001], 1e-15, "angles")


def test_attention_forward_rope_is_attention_of_rotated_inputs():
    """A scalar rotation written out with math.cos/math.sin, then the (pinned) forward."""
    rng = np.random.default_rng(7)
    B, H, N, D = 1, 2, 5, 4
    q, k, v = (rng.standard_normal((B, H, N, D)) for _ in range(3))

    def scalar_rot(x, base):
        y = np.empty_like(x)
        for idx in np.ndindex(x.shape[:-2]):
            for p in range(N):
                for d in range(D // 2):
                    th = p * base ** (-2.0 * d / D)
                    a, b = x[idx + (p, d)], x[idx + (p, d + D // 2)]
                    y[idx + (p, d)] = a * math.cos(th) - b * math.sin(th)
                    y[idx + (p, d + D // 2)] = b * math.cos(th) + a * math.sin(th)
        return y

    for causal in (False, True):
        O, L = attention_forward_rope(q, k, v, causal, 0.7, base=50.0)
        O2, L2 = attention_forward(scalar_rot(q, 50.0), scalar_rot(k, 50.0), v, causal, 0.7)
        _close(O, O2, 1e-13, "rope attention O")
        _close(L, L2, 1e-13, "rope attention LSE")


# ---------------------------------------------------------------- planted mistakes

def _rot(pair="half", sign=1.0, expo=2.0, pos0=0, fixed_base=None, swap_out=False, swap_cs=False):
    def rot(x, base):
        x = np.asarray(x, dtype=np.float64)
        N, D = x.shape[-2], x.shape[-1]
        b = fixed_base if fixed_base is not None else base
        p = np.arange(pos0, pos0 + N, dtype=np.float64)[:, None]
        d = np.arange(D // 2, dtype=np.float64)[None, :]
        th = p * b ** (-expo * d / D)
        c, s = np.cos(th), sign * np.sin(th)
        if swap_cs:
            c, s = s, c
        if pair == "half":
            a, bb = x[..., : D // 2], x[..., D // 2:]
        else:
            a, bb = x[..., 0::2], x[..., 1::2]
        u, w = a * c - bb * s, bb * c + a * s
        if swap_out:
            u, w = w, u
        if pair == "half":
            return np.concatenate([u, w], axis=-1)
        y = np.empty_like(x)
        y[..., 0::2], y[..., 1::2] = u, w
        return y
    return rot


MUTANTS = {
    "interleaved_pairs": _rot(pair="interleaved"),
    "rotation_reversed": _rot(sign=-1.0),
    "frequency_exponent_d_over_D": _rot(expo=1.0),
    "positions_from_one": _rot(pos0=1),
    "base_ignored": _rot(fixed_base=10000.0),
    "halves_swapped": _rot(swap_out=True),
    "cos_sin_swapped": _rot(swap_cs=True),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_rope_mistake_fails_a_pin(name):
    caught = []
    for pin in ROPE_PINS:
        try:
            pin(MUTANTS[name])
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"


def test_unmutated_rope_copy_passes_every_pin():
    for pin in ROPE_PINS:
        pin(_rot())
