#!/usr/bin/env python
"""Benchmark of the B200 bf16 attention forward (TFLOP/s, % of the dense BF16 peak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl ours|reference]
                    [--pass fwd|bwd|rope|fp8|bwd_rope]

One step = one attention forward pass over the workload's batch (one kernel
launch).  Default workload: the largest configuration, GQA B=8, Hq=32, Hkv=8,
N=8192, D=128, causal, bf16 inputs drawn i.i.d. N(0,1) from a seeded CPU
generator (768 MiB of inputs, 520 MiB of outputs).  A 512 MB buffer is written
between timed steps to flush the 126 MB L2 (smaller workloads' inputs would fit
in it); each step's kernel is timed with CUDA events on its launching stream.

FLOPs counted: 4*B*Hq*N^2*D, halved for causal.  `value` is the whole-job
throughput (all ranks' FLOPs / the slowest rank's time).  With N>1 GPUs
(torchrun), every rank runs its own batch of the workload (weak scaling): the
query heads are independent, so no collective touches the data path; NCCL only
carries the barrier and the max-over-ranks timing.

`--pass bwd` times the backward pass instead (one step = one attn_bwd call: the prep,
dK/dV and dQ launches), on the forward's o and lse computed once before timing; its
FLOP count is 2.5x the forward's (the five N x N x D matmuls of the gradient), the
usual convention.

`--pass rope` times attn_fwd_rope (the rotary kernel on Q and K, then the forward) with the
forward's FLOP count, and adds the rotary kernel alone against the HBM roofline.

`--pass fp8` times attn_fwd_fp8 on E4M3 inputs (N(0,1) x 16 rounded to E4M3, descale 1/16) with
the forward's FLOP count, against the measured bf16 peak x 2 (the nominal E4M3/bf16 ratio).

`--pass bwd_rope` times attn_bwd_rope (the rotary kernel on Q and K, the backward on the
rotated tensors, the inverse rotation of dQ and dK) on the outputs of attn_fwd_rope, with the
backward's FLOP count.

`--impl reference` times the fp64 CPU oracle instead (the only other
implementation of this path): each step is a bounded sample of the workload's
heads on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DATASHEET_BF16_TFLOPS = 2250.0   # B200 dense BF16 (no sparsity)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DEFAULT_WORKLOAD = "cfg4"
METRIC = "attention fwd TFLOP/s (bf16, 1 B200) and % of dense BF16 tensor peak"
METRIC_FP8 = "attention fwd E4M3 (FP8) TFLOP/s (1 B200) and % of dense FP8 tensor peak"
FP8_OVER_BF16 = 2.0  # nominal dense E4M3 / bf16 tensor rate (4.5 / 2.25 PFLOP/s)
METRIC_ROPE = "attention fwd with RoPE of Q and K TFLOP/s (bf16, 1 B200; forward FLOP count) and % of dense BF16 tensor peak"
METRIC_BWD = "attention bwd TFLOP/s (bf16, 1 B200; 2.5x the forward FLOP count) and % of dense BF16 tensor peak"
METRIC_BWD_ROPE = ("attention bwd through RoPE of Q and K TFLOP/s (bf16, 1 B200; 2.5x the forward FLOP count) "
                   "and % of dense BF16 tensor peak")
PASS_NAMES = {"fwd": "forward", "bwd": "backward", "rope": "forward with RoPE", "fp8": "forward, E4M3 inputs",
              "bwd_rope": "backward through RoPE"}
METRICS = {"fwd": METRIC, "bwd": METRIC_BWD, "rope": METRIC_ROPE, "fp8": METRIC_FP8, "bwd_rope": METRIC_BWD_ROPE}
BWD_FLOP_RATIO = 2.5      # counted backward FLOPs / forward FLOPs (five matmuls against two)
BWD_EXECUTED_RATIO = 7 / 5  # matmuls the kernels execute / matmuls counted (S and dP run twice)
L2_FLUSH_BYTES = 512 << 20
CPU_SAMPLE_SECONDS = 12.0


# ------------------------------------------------------------------ distributed helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (x itself on one rank)."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        import torch

        t = torch.zeros(1, device=device)
        dist.all_reduce(t)


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch of the workload."""
    return seed + 7919 * rank


# ------------------------------------------------------------------ peaks and clocks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 1400.0, FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples of one GPU while a region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w", prefix="clocks_", suffix=".csv", delete=False)
        self.path = self.f.name
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            self.f.close()
            os.unlink(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        busy = [r for r in rows if (num(r[4]) or 0) > 50] or rows
        sm = [num(r[1]) for r in busy if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(num(r[2]) or 0 for r in rows),
                "reasons": reasons, "samples": len(busy),
                "power_w_max": max(num(r[3]) or 0 for r in rows)}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


def profile_traffic(workload_name: str, which: str = "fwd"):
    """DRAM bytes per launch (per call for the backward) from the committed ncu summary, if
    it matches the current kernel sources."""
    path = os.path.join(ROOT, "profiles", f"attn_{which}_{workload_name}_dram.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    from tiled_attention_forward_03_b200.build import kernel_source_digest

    if d.get("kernel_source_sha256") != kernel_source_digest(which):
        return None
    return d.get("dram_bytes_per_launch")


def bench_config(w, pass_: str, world: int) -> dict:
    """The `config` object of the JSON line; both arms print the same one."""
    return {**w.describe(), "pass": PASS_NAMES[pass_],
            "l2": "flushed between timed steps (512 MB write)",
            "parallelism": f"replicas{world}: each rank its own batch, no collective on the data path"}


# ------------------------------------------------------------------ CPU oracle timing

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        import numpy  # noqa: F401

        info = threadpool_info()
        if info:
            return max(int(x.get("num_threads", 1)) for x in info)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def time_oracle(w, seconds: float, heads: int | None = None, backward: bool = False, rope: bool = False):
    """Run the fp64 oracle on whole heads of workload w for about `seconds` (or `heads` heads);
    the forward (of RoPE-rotated q and k with `rope`), or with `backward` the gradients of one
    query head.

    Returns (TFLOP/s, FLOPs done, seconds, heads done, sample description)."""
    from oracle import head_backward, head_forward, rope_rotate, rope_rotate_transpose
    from attn_inputs import make_dout, make_qkv, make_qkv_e4m3

    q, k, v = make_qkv(1, w.Hq, w.Hkv, w.N, w.D, w.seed)  # one batch row holds all heads
    do = make_dout(1, w.Hq, w.N, w.D, w.seed + 500) if backward else None
    g = w.Hq // w.Hkv
    per_head = w.flops / (w.B * w.Hq) * (BWD_FLOP_RATIO if backward else 1.0)
    done = 0
    t0 = time.perf_counter()
    while True:
        h = done % w.Hq
        if backward and rope:
            dq, dk, _ = head_backward(rope_rotate(q[0, h]), rope_rotate(k[0, h // g]), v[0, h // g], do[0, h],
                                      w.causal, w.softmax_scale)
            rope_rotate_transpose(dq), rope_rotate_transpose(dk)
        elif backward:
            head_backward(q[0, h], k[0, h // g], v[0, h // g], do[0, h], w.causal, w.softmax_scale)
        elif rope:
            head_forward(rope_rotate(q[0, h]), rope_rotate(k[0, h // g]), v[0, h // g], w.causal, w.softmax_scale)
        else:
            head_forward(q[0, h], k[0, h // g], v[0, h // g], w.causal, w.softmax_scale)
        done += 1
        el = time.perf_counter() - t0
        if heads is not None and done >= heads:
            break
        if heads is None and el >= seconds:
            break
    tflops = per_head * done / el / 1e12
    what = ("gradients through RoPE" if rope else "gradients") if backward else ("RoPE + forward" if rope else "forward")
    sample = (f"{what} of {done} heads, cycling over the {w.Hq} query heads of one batch row of {w.name} "
              f"(each head's full {w.N}x{w.N} fp64 score matrix), {el:.1f} s")
    return tflops, per_head * done, el, done, sample


# ------------------------------------------------------------------ our arm

def run_ours(args, w):
    import torch

    backward = args.pass_ in ("bwd", "bwd_rope")
    bwd_rope = args.pass_ == "bwd_rope"
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")

    import tiled_attention_forward_03_b200 as attn
    from attn_inputs import make_dout, make_qkv, make_qkv_e4m3

    fp8 = args.pass_ == "fp8"
    if fp8:
        q, k, v, ds = make_qkv_e4m3(w.B, w.Hq, w.Hkv, w.N, w.D, rank_seed(w.seed, rank))
    else:
        q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, rank_seed(w.seed, rank))
    qd, kd, vd = (x.to(device) for x in (q, k, v))
    o = torch.empty(qd.shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    scale = w.softmax_scale

    if backward:
        # the backward consumes the forward's saved o and lse: computed once, untimed
        do = make_dout(w.B, w.Hq, w.N, w.D, rank_seed(w.seed + 500, rank))
        dod = do.to(device)
        dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        if bwd_rope:
            cos_t, sin_t = attn.rope_tables(w.N, w.D, device=device)
            attn.forward_rope(qd, kd, vd, cos_t, sin_t, causal=w.causal, scale=scale, out=o, lse=lse, stream=stream)

            def step():
                attn.backward_rope(qd, kd, vd, cos_t, sin_t, o, lse, dod, causal=w.causal, scale=scale, dq=dq,
                                   dk=dk, dv=dv, stream=stream)
        else:
            attn.forward(qd, kd, vd, causal=w.causal, scale=scale, out=o, lse=lse, stream=stream)

            def step():
                attn.backward(qd, kd, vd, o, lse, dod, causal=w.causal, scale=scale, dq=dq, dk=dk, dv=dv,
                              stream=stream)
    elif fp8:
        def step():
            attn.forward_fp8(qd, kd, vd, ds, ds, ds, causal=w.causal, scale=scale, out=o, lse=lse, stream=stream)
    elif args.pass_ == "rope":
        cos_t, sin_t = attn.rope_tables(w.N, w.D, device=device)

        def step():
            attn.forward_rope(qd, kd, vd, cos_t, sin_t, causal=w.causal, scale=scale, out=o, lse=lse, stream=stream)
    else:
        def step():
            attn.forward(qd, kd, vd, causal=w.causal, scale=scale, out=o, lse=lse, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    st, site = attn.device_status()
    if st != attn.ATTN_OK:
        raise RuntimeError(f"kernel wait gave up during warm-up (site {site})")

    clocks = ClockSampler(physical_gpu_index(local)) if rank == 0 else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # keep the GPU busy long enough for the clock sampler to see the timed region
    barrier(dist, device)
    torch.cuda.synchronize(device)
    for i in range(args.steps):
        flush.zero_()                       # L2 flush between timed steps (not timed)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    clk = clocks.stop() if clocks else None
    kernel_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    local_ms = sum(kernel_ms)
    total_ms = max_over_ranks(local_ms, dist, device)
    st, site = attn.device_status()
    if st != attn.ATTN_OK:
        raise RuntimeError(f"kernel wait gave up during timing (site {site})")

    # ---- end to end through the public host-buffer call
    e2e_steps = max(3, min(args.steps, 20))
    if backward:
        host_in = tuple(x.pin_memory() for x in (q, k, v, o.cpu(), lse.cpu(), do))
        host_out = tuple(torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (dq, dk, dv))

        def e2e_call():
            attn.backward_from_host(*host_in, causal=w.causal, scale=scale, device=device, out_host=host_out,
                                    stream=stream, rope_tables=(cos_t, sin_t) if bwd_rope else None)
        h2d = sum(x.numel() * x.element_size() for x in host_in)
        d2h = sum(x.numel() * x.element_size() for x in host_out)
        e2e_path = ("backward_from_host: pinned host q,k,v,o,lse,dO -> device, "
                    + ("attn_bwd_rope (device-resident cos/sin tables)" if bwd_rope else "attn_bwd")
                    + ", dq,dk,dv -> pinned host; in 4 pieces (batch rows), copies overlapping the kernels")
    else:
        qh, kh, vh = (x.pin_memory() for x in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        tables = (cos_t, sin_t) if args.pass_ == "rope" else None
        descales = (ds, ds, ds) if fp8 else None

        def e2e_call():
            attn.forward_from_host(qh, kh, vh, causal=w.causal, scale=scale, device=device, out_host=oh,
                                   lse_host=lh, stream=stream, rope_tables=tables, fp8_descales=descales)
        h2d = sum(x.numel() * x.element_size() for x in (q, k, v))
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        if tables or fp8:
            e2e_path = ("forward_from_host: pinned host q,k,v -> device, "
                        + ("attn_fwd_rope (device-resident cos/sin tables)" if tables else "attn_fwd_fp8 (E4M3 inputs)")
                        + ", o,lse -> pinned host; in 8 pieces (batch rows), torch copies overlapping the kernels")
        else:
            e2e_path = ("attn_fwd_from_host (C ABI, called by forward_from_host): pinned host q,k,v -> device "
                        "buffers, attn_fwd_ws per piece, o,lse -> pinned host; 8 pieces (batch rows), the "
                        "library's copy streams overlapping the kernels; returns after the last download")
    for _ in range(2):
        e2e_call()
    barrier(dist, device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    barrier(dist, device)

    rope_ms = None
    if args.pass_ == "rope":
        # the rotary kernel alone (attn_rope_qk), L2 flushed between launches
        qo, ko = torch.empty_like(qd), torch.empty_like(kd)
        for _ in range(3):
            attn.rope(qd, kd, cos_t, sin_t, q_out=qo, k_out=ko, stream=stream)
        rs = [torch.cuda.Event(enable_timing=True) for _ in range(20)]
        re_ = [torch.cuda.Event(enable_timing=True) for _ in range(20)]
        for i in range(20):
            flush.zero_()
            rs[i].record(stream)
            attn.rope(qd, kd, cos_t, sin_t, q_out=qo, k_out=ko, stream=stream)
            re_[i].record(stream)
        torch.cuda.synchronize(device)
        rope_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(rs, re_))
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return None

    peak_burst, peak_sustained, hbm, peak_kind = measured_peaks()
    # The roofline denominator follows the regime the timed region ran in: the burst matmul
    # figure while the clock record shows no power capping (a short run of the kernel), the
    # sustained one once the power cap has brought the clocks down (a long run).
    capped = clk is not None and "sw_power_cap" in (clk.get("reasons") or [])
    peak = peak_sustained if capped else peak_burst
    peak_regime = ("sustained (the clock record shows sw_power_cap during the timed region)" if capped
                   else "burst (no power capping during the timed region)")
    flops_step = w.flops * (BWD_FLOP_RATIO if backward else 1.0)
    value = world * flops_step * args.steps / (total_ms * 1e-3) / 1e12
    achieved = flops_step / (statistics.mean(kernel_ms) * 1e-3) / 1e12
    e2e_value = world * flops_step * e2e_steps / (e2e_ms * 1e-3) / 1e12
    # DRAM traffic from a committed ncu record of this path and workload (bf16 forward and
    # backward only), if the record's kernel sources are the current ones
    traffic = profile_traffic(w.name, args.pass_) if args.pass_ in ("fwd", "bwd") else None
    if backward:
        kernel = (f"attn_bwd call: attn_bwd_prep + attn_bwd_sm100<{w.D}, dK/dV> + attn_bwd_sm100<{w.D}, dQ>, "
                  f"timed together")
        if bwd_rope:
            kernel = (f"attn_bwd_rope call: attn_rope_qk + attn_bwd_prep + attn_bwd_sm100<{w.D}, dK/dV> + "
                      f"attn_bwd_sm100<{w.D}, dQ> + attn_rope_qk_inverse, timed together")
        # read q, o, dO (query heads), k, v (KV heads), lse; write dq, dk, dv; all bf16 but lse
        q_side = w.B * w.Hq * w.N * w.D * 2
        kv_side = w.B * w.Hkv * w.N * w.D * 2
        algo_bytes = 4 * q_side + 4 * kv_side + 4 * w.B * w.Hq * w.N
    elif args.pass_ == "rope":
        kernel = f"attn_fwd_rope call: attn_rope_qk on Q and K + the forward kernel, timed together"
        algo_bytes = w.algorithmic_bytes
    elif fp8:
        kernel = f"attn_fwd_sm100<{w.D}, E4M3>" if w.D <= 128 else f"attn_fwd_wide_sm100<{w.D}, E4M3>"
        # q, k, v one byte per element; o bf16, lse fp32
        algo_bytes = (w.B * w.Hq + 2 * w.B * w.Hkv) * w.N * w.D + 2 * w.B * w.Hq * w.N * w.D + 4 * w.B * w.Hq * w.N
        peak_burst = peak_burst * FP8_OVER_BF16
        peak = peak * FP8_OVER_BF16
        peak_kind = f"{peak_kind} bf16 matmul x {FP8_OVER_BF16:g} (nominal E4M3/bf16 ratio)"
    else:
        # the kernel the library picks for this shape (bf16, no split last wave)
        colsplit = w.causal and w.D == 128 and w.N <= 2048
        sep_p = not w.causal and w.D <= 64          # P beside O, one MMA warp per tile
        kernel = f"attn_fwd_colsplit_sm100<{w.D}>" if colsplit else (
            f"attn_fwd_sm100<{w.D}, bf16, P beside O>" if sep_p else
            f"attn_fwd_sm100<{w.D}>" if w.D <= 128 else f"attn_fwd_wide_sm100<{w.D}>")
        algo_bytes = w.algorithmic_bytes

    line = {
        "metric": METRICS[args.pass_],
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16",
        "data": "synthetic",
        "config": bench_config(w, args.pass_, world),
        "pct_of_dense_bf16_peak" if not fp8 else "pct_of_dense_fp8_peak":
            round(100.0 * value / world / (DATASHEET_BF16_TFLOPS * (FP8_OVER_BF16 if fp8 else 1.0)), 2),
        "pct_of_measured_bf16_peak" if not fp8 else "pct_of_measured_fp8_peak": round(100.0 * value / world / peak_burst, 2),
        "hbm_gbs_algorithmic": round(algo_bytes / (statistics.mean(kernel_ms) * 1e-3) / 1e9, 1),
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "path": e2e_path},
        "gpu_launches": args.steps * {"fwd": 1, "bwd": 3, "rope": 2, "fp8": 1, "bwd_rope": 5}[args.pass_],
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": f"{peak_kind} bf16 matmul, {peak_regime}",
                     "kernel": kernel},
    }
    if backward:
        line["roofline"]["executed_tflops"] = round(achieved * BWD_EXECUTED_RATIO, 2)
        line["roofline"]["executed_note"] = ("the kernels run 7 N x N x D matmuls where 5 are counted "
                                             "(scores and dP are formed in both the dK/dV and dQ kernels)")
    if rope_ms is not None:
        # read q, k once, write their rotations once (the 2 x N x D/2 fp32 tables stay in L2)
        rope_bytes = 2 * 2 * (w.B * w.Hq + w.B * w.Hkv) * w.N * w.D
        gbs = rope_bytes / (rope_ms * 1e-3) / 1e9
        line["rope_kernel"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                               "frac": round(gbs / hbm, 4), "us_per_launch": round(rope_ms * 1e3, 2),
                               "algorithmic_bytes": rope_bytes, "kernel": "attn_rope_qk",
                               "peak_kind": "measured HBM copy bandwidth"}
    if world == 1 and not args.no_cpu_baseline:
        tf, _, el, done, sample = time_oracle(w, CPU_SAMPLE_SECONDS, backward=backward,
                                              rope=args.pass_ in ("rope", "bwd_rope"))
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": sample}
    if dist is not None:
        dist.destroy_process_group()
    return line


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    backward = args.pass_ in ("bwd", "bwd_rope")
    per_step = []
    for i in range(args.warmup + args.steps):
        tf, flops, el, done, sample = time_oracle(w, 0.0, heads=1, backward=backward,
                                                  rope=args.pass_ in ("rope", "bwd_rope"))
        if i >= args.warmup:
            per_step.append((flops, el))
    flops = sum(f for f, _ in per_step)
    secs = sum(e for _, e in per_step)
    value = flops / secs / 1e12
    cores = cpu_threads()
    what = "gradients of one head" if backward else "one head"
    sample = f"{what} of {w.name} per step (full {w.N}x{w.N} fp64 score matrix), {args.steps} steps"
    return {
        "impl": "reference",
        "metric": METRICS[args.pass_],
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(w, args.pass_, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)  # cfg4 forward: ~0.7 s of timed region (clock samples)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="cfg1..cfg4, a sweep point name (e.g. sweep_D128_N8192_causal), or 'all'")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd", "rope", "fp8", "bwd_rope"], default="fwd",
                    help="fwd: the attention forward (default); bwd: the backward pass (attn_bwd); "
                         "rope: RoPE of Q and K then the forward (attn_fwd_rope); fp8: the E4M3 forward "
                         "(attn_fwd_fp8)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from attn_inputs import WORKLOADS, get_workload

    names = list(WORKLOADS) if args.workload == "all" else [args.workload]
    for i, name in enumerate(names):
        w = get_workload(name)
        if args.impl == "reference":
            line = run_reference(args, w)
        else:
            if i > 0:
                args.no_cpu_baseline = True
            line = run_ours(args, w)
        if line is not None:
            print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
