"""The fp64 oracle against facts the definition of attention fixes (CPU only)."""
import numpy as np
import pytest

from oracle import attention_forward, attention_rows
from oracle_pins import ALL_PINS


def rows_impl(q, k, v, causal, scale):
    """The oracle's row-at-a-time function, evaluated on every row."""
    B, Hq, N, _ = q.shape
    rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N)]
    O, L = attention_rows(q, k, v, rows, causal, scale)
    return O.reshape(B, Hq, N, -1), L.reshape(B, Hq, N)


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_forward_pins(pin):
    pin(attention_forward)


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_rows_pins(pin):
    pin(rows_impl)


def test_oracle_accepts_bf16_torch_tensors():
    """bf16 torch inputs are upcast exactly (bf16 -> fp32 -> fp64 loses nothing)."""
    import torch
    from attn_inputs import make_qkv

    q, k, v = make_qkv(1, 2, 1, 16, 8, seed=7)
    O1, L1 = attention_forward(q, k, v, True, 0.3)
    O2, L2 = attention_forward(q.to(torch.float64).numpy(), k.to(torch.float64).numpy(),
                               v.to(torch.float64).numpy(), True, 0.3)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)
