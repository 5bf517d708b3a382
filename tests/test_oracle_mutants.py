"""Planted mistakes in copies of the oracle must each fail at least one pin (CPU only).

Every mutant below is the oracle's definition with one plausible slip: a
dropped term, a wrong sign or index, a transposed operand.  If some mutant
passed every pin, the pins would not be pinning that part of the oracle.
"""
import numpy as np
import pytest

from oracle_pins import ALL_PINS


def _make(scores=None, probs=None, combine=None, lse=None, kvmap=None):
    def impl(q, k, v, causal, scale):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        B, Hq, N, _ = q.shape
        Hkv = k.shape[1]
        O = np.empty((B, Hq, N, v.shape[3]))
        L = np.empty((B, Hq, N))
        for b in range(B):
            for h in range(Hq):
                kh = kvmap(h, Hq, Hkv) if kvmap else h // (Hq // Hkv)
                qh, kk, vv = q[b, h], k[b, kh], v[b, kh]
                if scores:
                    S = scores(qh, kk, causal, scale)
                else:
                    S = scale * qh @ kk.T
                    if causal:
                        S = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, S)
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                l = E.sum(axis=1, keepdims=True)
                P = probs(E, l, S) if probs else E / l
                O[b, h] = combine(P, vv, E) if combine else P @ vv
                L[b, h] = lse(m[:, 0], l[:, 0]) if lse else m[:, 0] + np.log(l[:, 0])
        return O, L
    return impl


def _mask(S, keep):
    n = S.shape[0]
    i, j = np.arange(n)[:, None], np.arange(n)[None, :]
    return np.where(keep(i, j), S, -np.inf)


def _strict_causal(q, k, c, s):
    S = s * q @ k.T
    if not c:
        return S
    # keeps j < i, and row 0 keeps key 0 so that the row is not empty
    return _mask(S, lambda i, j: (j < i) | ((i == 0) & (j == 0)))


MUTANTS = {
    "causal_mask_upper": _make(scores=lambda q, k, c, s: _mask(s * q @ k.T, lambda i, j: (j >= i) | (not c))),
    "causal_excludes_diagonal": _make(scores=_strict_causal),
    "causal_ignored": _make(scores=lambda q, k, c, s: s * q @ k.T),
    "scale_dropped": _make(scores=lambda q, k, c, s: _mask(q @ k.T, lambda i, j: (j <= i) | (not c))),
    "scale_inverted": _make(scores=lambda q, k, c, s: _mask((1.0 / s if s else 0.0) * q @ k.T,
                                                           lambda i, j: (j <= i) | (not c))),
    "scores_transposed": _make(scores=lambda q, k, c, s: _mask(s * k @ q.T, lambda i, j: (j <= i) | (not c))),
    "gqa_heads_interleaved": _make(kvmap=lambda h, Hq, Hkv: h % Hkv),
    "unnormalised_output": _make(combine=lambda P, v, E: E @ v),
    "probs_transposed": _make(combine=lambda P, v, E: P.T @ v),
    "softmax_over_columns": _make(probs=lambda E, l, S: np.exp(S - S.max()) / np.exp(S - S.max()).sum(axis=0, keepdims=True)),
    "lse_without_max": _make(lse=lambda m, l: np.log(l)),
    "lse_base2": _make(lse=lambda m, l: (m + np.log(l)) / np.log(2.0)),
    "lse_max_only": _make(lse=lambda m, l: m),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    impl = MUTANTS[name]
    caught = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"


def test_unmutated_copy_passes_every_pin():
    impl = _make()
    for pin in ALL_PINS:
        pin(impl)
