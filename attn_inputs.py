"""Seeded synthetic inputs for the attention forward pass.

This module only draws random numbers and names the workloads; it holds none
of the attention arithmetic.  Both the CUDA path's tests/bench and the CPU
oracle's tests take their inputs from here.

Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws Q, K and V, in
that order, as i.i.d. N(0, 1) float32 tensors of layout ``[B, H, N, D]``;
each is then rounded to bfloat16 (round-to-nearest-even).  ``scale`` defaults
to ``1/sqrt(D)``.  Workload ``cfg<k>`` uses seed ``1000 + k``; sweep point
number ``i`` (in the order of :func:`sweep_points`) uses seed ``2000 + i``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask mode and input seed."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    causal: bool
    seed: int
    scale: float = field(default=float("nan"))

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D) if math.isnan(self.scale) else self.scale

    @property
    def flops(self) -> float:
        """Counted FLOPs: 4*B*Hq*N^2*D, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.D
        return f / 2.0 if self.causal else f

    @property
    def algorithmic_bytes(self) -> int:
        """Q, K, V read once and O, LSE written once."""
        qo = 2 * self.B * self.Hq * self.N * self.D * 2
        kv = 2 * self.B * self.Hkv * self.N * self.D * 2
        lse = 4 * self.B * self.Hq * self.N
        return qo + kv + lse

    def describe(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv,
            "N": self.N, "D": self.D, "causal": self.causal,
            "scale": self.softmax_scale, "seed": self.seed,
        }


# The five workloads; the fifth is a sweep at a fixed B*N = 16384 tokens.
CFG1 = Workload("cfg1_B1_H2_N128_D64", 1, 2, 2, 128, 64, False, 1001)
CFG2 = Workload("cfg2_B4_H16_N2048_D128", 4, 16, 16, 2048, 128, False, 1002)
CFG3 = Workload("cfg3_B16_H16_N4096_D128_causal", 16, 16, 16, 4096, 128, True, 1003)
CFG4 = Workload("cfg4_gqa_B8_Hq32_Hkv8_N8192_D128_causal", 8, 32, 8, 8192, 128, True, 1004)

SWEEP_TOKENS = 16384


def sweep_points() -> list[Workload]:
    pts = []
    i = 0
    for D in (64, 128):
        for N in (1024, 2048, 4096, 8192, 16384):
            for causal in (True, False):
                B = SWEEP_TOKENS // N
                tag = "causal" if causal else "noncausal"
                pts.append(Workload(f"sweep_D{D}_N{N}_{tag}", B, 16, 16, N, D, causal, 2000 + i))
                i += 1
    return pts


def wide_points() -> list[Workload]:
    """Head dims 192 and 256 (beyond the sweep's 64 and 128), same token count per batch."""
    pts = []
    i = 0
    for D in (192, 256):
        for N in (2048, 8192):
            for causal in (True, False):
                tag = "causal" if causal else "noncausal"
                pts.append(Workload(f"wide_D{D}_N{N}_{tag}", SWEEP_TOKENS // N, 16, 16, N, D, causal, 3000 + i))
                i += 1
    return pts


WORKLOADS = {w.name: w for w in (CFG1, CFG2, CFG3, CFG4, *sweep_points(), *wide_points())}
ALIASES = {"cfg1": CFG1.name, "cfg2": CFG2.name, "cfg3": CFG3.name, "cfg4": CFG4.name}


def get_workload(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def make_qkv(B: int, Hq: int, Hkv: int, N: int, D: int, seed: int):
    """Draw (q, k, v) as contiguous CPU bfloat16 tensors [B, H, N, D]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, Hq, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


def make_dout(B: int, Hq: int, N: int, D: int, seed: int):
    """Draw the upstream gradient dL/dO as a contiguous CPU bfloat16 tensor [B, Hq, N, D]
    (i.i.d. N(0, 1) in fp32, rounded to bf16), from its own seed."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn((B, Hq, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)


E4M3_AMPLITUDE = 16.0  # inputs are drawn N(0,1), multiplied by this and rounded to E4M3


def make_qkv_e4m3(B: int, Hq: int, Hkv: int, N: int, D: int, seed: int):
    """Draw (q, k, v) as for make_qkv (same generator and order, fp32 N(0,1)), multiply by
    E4M3_AMPLITUDE and round to float8_e4m3fn (nearest even).  Returns the three CPU E4M3
    tensors and the descale factor 1 / E4M3_AMPLITUDE that maps them back to the inputs'
    scale (the values |x| * 16 >= 2^-6 are normal E4M3 numbers)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = []
    for shape in ((B, Hq, N, D), (B, Hkv, N, D), (B, Hkv, N, D)):
        x = torch.randn(shape, generator=g, dtype=torch.float32) * E4M3_AMPLITUDE
        out.append(x.to(torch.float8_e4m3fn))
    return out[0], out[1], out[2], 1.0 / E4M3_AMPLITUDE


def make_workload_inputs(w: Workload):
    return make_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, w.seed)


def sample_rows(B: int, H: int, N: int, count: int, seed: int) -> list[tuple[int, int, int]]:
    """Seeded (b, h, i) output rows for sampled checks at full size.

    Always includes the first and last rows and the rows on either side of
    every 128-row tile edge of one head, then ``count`` uniform draws.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rows = set()
    rows.add((0, 0, 0))
    rows.add((B - 1, H - 1, N - 1))
    for t in range(0, N, 128):
        for i in (t - 1, t, t + 127):
            if 0 <= i < N:
                rows.add((B - 1, 0, i))
    draws = torch.randint(0, B * H * N, (count,), generator=g).tolist()
    for x in draws:
        b, rem = divmod(x, H * N)
        h, i = divmod(rem, N)
        rows.add((b, h, i))
    return sorted(rows)
