"""Plain fp64 CPU oracle for scaled-dot-product attention: forward pass and its gradients.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may call it.  It shares no code with the CUDA library.

What it computes
----------------
The pages ("Making AMD GPUs go brrr", section "Real kernel example"; and
"HipKittens: fast and furious AMD kernels", section "Performance results")
name a tiled attention forward kernel -- causal and non-causal, over several
head dims D and sequence lengths N -- whose hot loop is built from a score
matmul, ``exp2`` and row sums, but print no formula.  The definition used
here is the plain one that such a kernel reaches up to rounding order:

    S   = scale * Q_h K_{kv(h)}^T                     (N x N)
    S_ij = -inf        for j > i            (causal only, top-left aligned)
    P   = row-softmax(S)
    O_h = P V_{kv(h)}                                  (N x D)
    LSE_i = ln sum_j exp(S_ij)             (natural log of the scaled scores)

with kv(h) = h // (Hq / Hkv) (contiguous query-head groups share one KV head).
Everything is evaluated in float64 on the bf16 input values upcast exactly;
the full score matrix of one head is materialised, no blocking, no online
softmax.  The readings of what the pages leave open (formula, LSE base,
causal alignment, head mapping, layout) are listed in the design notes.

Parity status: every forward function below is pinned by tests/test_oracle.py
(closed forms, invariants, a scalar brute force and a library special case)
and by tests/test_oracle_mutants.py (planted mistakes must fail a pin).  The
backward functions are pinned by tests/test_oracle_bwd.py (central differences
of the forward, autograd through torch's fp64 SDPA, a scalar brute force through
the softmax Jacobian, closed forms and invariants, planted mistakes).  The RoPE
functions are pinned by tests/test_oracle_rope.py (hand-computed values, position 0,
norm preservation, relative-position property, planted mistakes).
"""
from __future__ import annotations

import numpy as np


def _as_f64(x) -> np.ndarray:
    """Upcast a numpy array or a CPU torch tensor (bf16/fp32/fp64) to fp64."""
    if hasattr(x, "detach"):  # torch tensor: go through float32, exact for bf16
        import torch

        x = x.detach().to("cpu")
        if x.dtype != torch.float64:
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """Query head h reads KV head h // (Hq/Hkv): contiguous groups of Hq/Hkv."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def head_scores(qh: np.ndarray, kh: np.ndarray, causal: bool, scale: float) -> np.ndarray:
    """Scaled, masked score matrix of one head: S = scale * q k^T, -inf above the diagonal if causal."""
    S = scale * (qh @ kh.T)
    if causal:
        n_q, n_k = S.shape
        i = np.arange(n_q)[:, None]
        j = np.arange(n_k)[None, :]
        S = np.where(j > i, -np.inf, S)
    return S


def head_forward(qh, kh, vh, causal: bool, scale: float):
    """One head: returns (O [N, D], LSE [N]) in fp64."""
    qh, kh, vh = _as_f64(qh), _as_f64(kh), _as_f64(vh)
    S = head_scores(qh, kh, causal, scale)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1, keepdims=True)
    O = (E / l) @ vh
    lse = m[:, 0] + np.log(l[:, 0])
    return O, lse


def attention_forward(q, k, v, causal: bool, scale: float):
    """Full forward: q [B,Hq,N,D], k/v [B,Hkv,N,D] -> (O [B,Hq,N,D], LSE [B,Hq,N]), fp64.

    Computed one (b, h) head at a time, each with its full N x N score matrix.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    O = np.empty((B, Hq, N, v.shape[3]), dtype=np.float64)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kh = kv_head(h, Hq, Hkv)
            O[b, h], lse[b, h] = head_forward(q[b, h], k[b, kh], v[b, kh], causal, scale)
    return O, lse


def attention_rows(q, k, v, rows, causal: bool, scale: float):
    """Selected output rows, each from its own score row (for full-size sampled checks).

    ``rows`` is a list of (b, h, i).  Row i of head (b, h) is the softmax of
    scale * q[b,h,i] . k[b,kv(h),j] over the allowed keys j (all j, or j <= i
    when causal), applied to V.  Returns (O [len(rows), D], LSE [len(rows)]).
    Accepts torch tensors without converting them whole.
    """
    Hq = q.shape[1]
    Hkv = k.shape[1]
    out_o = []
    out_l = []
    cache_key = None
    kh_arr = vh_arr = None
    for (b, h, i) in rows:
        kh = kv_head(h, Hq, Hkv)
        if cache_key != (b, kh):
            kh_arr = _as_f64(k[b, kh])
            vh_arr = _as_f64(v[b, kh])
            cache_key = (b, kh)
        qi = _as_f64(q[b, h, i])
        s = scale * (kh_arr @ qi)
        if causal:
            s = np.where(np.arange(s.shape[0]) > i, -np.inf, s)
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        out_o.append((e / l) @ vh_arr)
        out_l.append(m + np.log(l))
    return np.stack(out_o), np.asarray(out_l)


# ----------------------------------------------------------------------------------------
# Backward pass (gradients of the forward above), for the attention-backward extension.
#
# The pages name an attention backward kernel ("HipKittens: fast and furious AMD
# kernels", section "Performance results"; "State of the AMD ecosystem" for the SDPA
# backward baselines) without a formula.  The plain definition: with P the forward's
# probabilities and dO the gradient of a loss with respect to O,
#     dP = dO V^T,   delta_i = sum_d dO_id O_id  (= sum_j P_ij dP_ij),
#     dS = P o (dP - delta),   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO,
# and for grouped heads dK, dV of a KV head are summed over its query heads.

def head_backward(qh, kh, vh, doh, causal: bool, scale: float):
    """One head: returns (dQ [N, D], dK [N, D], dV [N, D]) in fp64."""
    qh, kh, vh, doh = _as_f64(qh), _as_f64(kh), _as_f64(vh), _as_f64(doh)
    S = head_scores(qh, kh, causal, scale)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    P = E / E.sum(axis=1, keepdims=True)
    O = P @ vh
    dP = doh @ vh.T
    delta = np.sum(doh * O, axis=1, keepdims=True)
    dS = P * (dP - delta)
    return scale * (dS @ kh), scale * (dS.T @ qh), P.T @ doh


def attention_backward(q, k, v, do, causal: bool, scale: float):
    """Gradients of sum(O * do) w.r.t. q [B,Hq,N,D], k and v [B,Hkv,N,D]; fp64.

    Each query head's contributions to its KV head's dK and dV are summed.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros((B, Hkv, N, v.shape[3]), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kh = kv_head(h, Hq, Hkv)
            gq, gk, gv = head_backward(q[b, h], k[b, kh], v[b, kh], do[b, h], causal, scale)
            dq[b, h] = gq
            dk[b, kh] += gk
            dv[b, kh] += gv
    return dq, dk, dv


# ----------------------------------------------------------------------------------------
# Rotary position embedding (RoPE) applied to Q and K before attention.
#
# The pages list a rotary kernel among the kernels built with the tile library ("HipKittens:
# fast and furious AMD kernels", section "Performance results") without its formula.  The
# definition used (the "rotate-half" pairing): for position p (the token index) and
# d < D/2, with theta = p * base^(-2d/D),
#     x'_d       = x_d cos(theta) - x_{d+D/2} sin(theta)
#     x'_{d+D/2} = x_{d+D/2} cos(theta) + x_d sin(theta)

def rope_angles(N: int, D: int, base: float = 10000.0) -> np.ndarray:
    """theta[p, d] = p * base^(-2d/D) for p < N, d < D/2, in fp64."""
    p = np.arange(N, dtype=np.float64)[:, None]
    d = np.arange(D // 2, dtype=np.float64)[None, :]
    return p * base ** (-2.0 * d / D)


def rope_rotate(x, base: float = 10000.0, angles=None):
    """Rotate the last dimension of x [..., N, D] by the RoPE angles of positions 0..N-1."""
    x = _as_f64(x)
    N, D = x.shape[-2], x.shape[-1]
    th = rope_angles(N, D, base) if angles is None else np.asarray(angles, dtype=np.float64)
    c, s = np.cos(th), np.sin(th)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def attention_forward_rope(q, k, v, causal: bool, scale: float, base: float = 10000.0):
    """Attention of RoPE(q), RoPE(k) and v (all fp64); returns (O, LSE) as attention_forward."""
    return attention_forward(rope_rotate(q, base), rope_rotate(k, base), v, causal, scale)


# The backward of the rotary step.  Each (x_d, x_{d+D/2}) pair is turned by the 2x2 rotation
# R(theta) = [[cos, -sin], [sin, cos]], so by the chain rule the gradient with respect to the
# unrotated pair is R(theta)^T times the gradient with respect to the rotated one:
#     g_d       =  g'_d cos(theta) + g'_{d+D/2} sin(theta)
#     g_{d+D/2} = -g'_d sin(theta) + g'_{d+D/2} cos(theta)

def rope_rotate_transpose(g, base: float = 10000.0, angles=None):
    """R(theta)^T applied to the last dimension of g [..., N, D] (the rotation by -theta)."""
    g = _as_f64(g)
    N, D = g.shape[-2], g.shape[-1]
    th = rope_angles(N, D, base) if angles is None else np.asarray(angles, dtype=np.float64)
    c, s = np.cos(th), np.sin(th)
    a, b = g[..., : D // 2], g[..., D // 2:]
    return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)


def attention_backward_rope(q, k, v, do, causal: bool, scale: float, base: float = 10000.0):
    """Gradients (dQ, dK, dV) of sum(O o dO) for O = attention(RoPE(q), RoPE(k), v): the
    attention backward at the rotated inputs, then the rotation's transpose on dQ and dK."""
    dqr, dkr, dv = attention_backward(rope_rotate(q, base), rope_rotate(k, base), v, do, causal, scale)
    return rope_rotate_transpose(dqr, base), rope_rotate_transpose(dkr, base), dv
