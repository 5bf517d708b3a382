"""The fp64 backward oracle against its pins, and planted mistakes against the pins (CPU only)."""
import numpy as np
import pytest

from oracle import attention_backward
from oracle_bwd_pins import ALL_BWD_PINS


@pytest.mark.parametrize("pin", ALL_BWD_PINS, ids=lambda p: p.__name__)
def test_oracle_backward_pins(pin):
    pin(attention_backward)


def _make(ds=None, dq=None, dk=None, dv=None, scores=None, gqa_overwrite=False):
    """A copy of the backward definition with optional replaced steps."""
    def impl(q, k, v, do, causal, scale):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
        B, Hq, N, D = q.shape
        Hkv = k.shape[1]
        gq = np.empty_like(q)
        gk = np.zeros_like(k)
        gv = np.zeros_like(v)
        for b in range(B):
            for h in range(Hq):
                kh = h // (Hq // Hkv)
                qh, kk, vv, dd = q[b, h], k[b, kh], v[b, kh], do[b, h]
                S = scores(qh, kk, causal, scale) if scores else scale * qh @ kk.T
                if causal and not scores:
                    S = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, S)
                E = np.exp(S - S.max(axis=1, keepdims=True))
                P = E / E.sum(axis=1, keepdims=True)
                O = P @ vv
                dP = dd @ vv.T
                delta = np.sum(dd * O, axis=1, keepdims=True)
                dS = ds(P, dP, delta) if ds else P * (dP - delta)
                a = dq(dS, kk, scale) if dq else scale * dS @ kk
                c = dk(dS, qh, scale) if dk else scale * dS.T @ qh
                e = dv(P, dd) if dv else P.T @ dd
                gq[b, h] = a
                if gqa_overwrite:
                    gk[b, kh] = c
                    gv[b, kh] = e
                else:
                    gk[b, kh] += c
                    gv[b, kh] += e
        return gq, gk, gv
    return impl


MUTANTS = {
    "delta_dropped": _make(ds=lambda P, dP, d: P * dP),
    "ds_sign_flipped": _make(ds=lambda P, dP, d: P * (d - dP)),
    "delta_not_row_wise": _make(ds=lambda P, dP, d: P * (dP - d.T)),
    "dq_unscaled": _make(dq=lambda dS, k, s: dS @ k),
    "dq_transposed_ds": _make(dq=lambda dS, k, s: s * dS.T @ k),
    "dk_not_transposed": _make(dk=lambda dS, q, s: s * dS @ q),
    "dk_scaled_twice": _make(dk=lambda dS, q, s: s * s * dS.T @ q),
    "dv_not_transposed": _make(dv=lambda P, do: P @ do),
    "dv_from_unnormalised_p": _make(dv=lambda P, do: (P / P.max(axis=1, keepdims=True)).T @ do),
    "causal_ignored": _make(scores=lambda q, k, c, s: s * q @ k.T),
    "gqa_overwrites_group": _make(gqa_overwrite=True),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_backward_mistake_fails_a_pin(name):
    impl = MUTANTS[name]
    caught = []
    for pin in ALL_BWD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"


def test_unmutated_backward_copy_passes_every_pin():
    impl = _make()
    for pin in ALL_BWD_PINS:
        pin(impl)
