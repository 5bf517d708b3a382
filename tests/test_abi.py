"""The C ABI on the host: the library loads, exports what include/attn.h declares,
and rejects bad arguments before any CUDA call (no GPU needed)."""
import ctypes
import math
import os
import re

import pytest

import tiled_attention_forward_03_b200 as attn

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")

OK, INVALID, UNSUPPORTED, MISALIGNED = (attn.ATTN_OK, attn.ATTN_ERR_INVALID_ARG,
                                        attn.ATTN_ERR_UNSUPPORTED, attn.ATTN_ERR_MISALIGNED)
P = 0x10000  # a 16-byte aligned fake device address; never dereferenced by a rejected call


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("attn_fwd", "attn_status_string", "attn_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(attn.lib_path)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_library_is_in_tree_and_built_for_sm100a():
    assert os.path.dirname(attn.lib_path) == os.path.dirname(os.path.abspath(attn.__file__))
    assert "sm_100a" in attn.attn_version()


def test_status_strings():
    assert attn.attn_status_string(OK) == "ATTN_OK"
    assert attn.attn_status_string(attn.ATTN_ERR_TIMEOUT) == "ATTN_ERR_TIMEOUT"
    assert attn.attn_status_string(12345) == "ATTN_ERR_UNKNOWN"


def call(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=1, N=128, D=128, causal=0, scale=0.125, stream=None)
    args.update(kw)
    return attn.attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"],
                         args["Hkv"], args["N"], args["D"], args["causal"], args["scale"], args["stream"])


@pytest.mark.parametrize("kw,expected", [
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(v=None), INVALID),
    (dict(o=None), INVALID), (dict(lse=None), INVALID),
    (dict(B=-1), INVALID), (dict(N=-5), INVALID), (dict(Hq=0), INVALID), (dict(Hkv=0), INVALID),
    (dict(Hq=3, Hkv=2), INVALID), (dict(scale=math.nan), INVALID), (dict(scale=math.inf), INVALID),
    (dict(D=80), UNSUPPORTED), (dict(D=384), UNSUPPORTED), (dict(D=0), UNSUPPORTED), (dict(D=48), UNSUPPORTED),
    (dict(D=160), UNSUPPORTED), (dict(q=P + 8), MISALIGNED), (dict(k=P + 2), MISALIGNED), (dict(v=P + 4), MISALIGNED),
    (dict(o=P + 1), MISALIGNED), (dict(lse=P + 2), MISALIGNED),
    # D = 192, 256: more than 2^30 query tiles (the wide-head kernel steps through them in 32 bits)
    (dict(B=1 << 10, Hq=1 << 10, Hkv=1 << 10, N=(1 << 17) + 1, D=256), UNSUPPORTED),
])
def test_rejected_before_any_cuda_call(kw, expected):
    assert call(**kw) == expected


@pytest.mark.parametrize("kw", [dict(B=0), dict(N=0), dict(B=0, q=None, k=None, v=None, o=None, lse=None)])
def test_empty_problem_is_ok_without_launch(kw):
    assert call(**kw) == OK


def test_lse_only_needs_4_byte_alignment():
    # Misalignment is checked after null/size checks; a 4-byte aligned lse passes it,
    # so the call only fails later, at the first CUDA call, when no GPU is present.
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a machine without a GPU")
    assert call(lse=P + 4) == attn.ATTN_ERR_CUDA


def test_num_units():
    assert attn.attn_num_units(4, 16, 2048) == 4 * 16 * 8
    assert attn.attn_num_units(1, 2, 129) == 2 * 1
    assert attn.attn_num_units(1, 1, 257) == 2
    assert attn.attn_num_units(0, 1, 100) == 0
    assert attn.attn_num_units(1, 0, 100) == -1


def call_ws(ws, nbytes, **kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=1, N=128, D=128, causal=0, scale=0.125, stream=None)
    args.update(kw)
    return attn.attn_fwd_ws(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"],
                            args["Hkv"], args["N"], args["D"], args["causal"], args["scale"], ws, nbytes, None)


def test_workspace_entry_point_host_checks():
    assert call_ws(P + 128, 1 << 20) == MISALIGNED          # workspace must be 256-byte aligned
    assert call_ws(None, 4096) == INVALID                  # size without a buffer
    assert call_ws(P, 1 << 20, D=80) == UNSUPPORTED        # the usual checks still apply first
    assert call_ws(P, 1 << 20, q=None) == INVALID
    assert call_ws(None, 0, B=0) == OK                     # empty problem


def test_wide_head_dims_need_no_workspace():
    # D = 192, 256 run on the one-tile kernel, which never splits its last wave
    assert attn.attn_fwd_workspace_bytes(4, 16, 2048, 256, 0) == 0
    assert attn.attn_fwd_workspace_bytes(4, 16, 2048, 192, 0) == 0


def test_workspace_bytes_host_cases():
    assert attn.attn_fwd_workspace_bytes(-1, 2, 128, 128, 0) == -1
    assert attn.attn_fwd_workspace_bytes(1, 2, 128, 80, 0) == -1
    assert attn.attn_fwd_workspace_bytes(4, 16, 2048, 128, 1) == 0   # causal never splits
    assert attn.attn_fwd_workspace_bytes(0, 16, 2048, 128, 0) == 0


# ---------------------------------------------------------------- backward entry point

def call_bwd(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, Hq=2, Hkv=1, N=128, D=128, causal=0,
                scale=0.125, ws=P, ws_bytes=1 << 20)
    args.update(kw)
    return attn.attn_bwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["dout"], args["dq"],
                         args["dk"], args["dv"], args["B"], args["Hq"], args["Hkv"], args["N"], args["D"],
                         args["causal"], args["scale"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=None), INVALID), (dict(dout=None), INVALID), (dict(dq=None), INVALID), (dict(dk=None), INVALID),
    (dict(dv=None), INVALID), (dict(o=None), INVALID), (dict(lse=None), INVALID), (dict(ws=None), INVALID),
    (dict(ws_bytes=1024), INVALID), (dict(B=-1), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(scale=math.nan), INVALID), (dict(D=80), UNSUPPORTED), (dict(D=256), UNSUPPORTED),
    (dict(dout=P + 8), MISALIGNED), (dict(dq=P + 2), MISALIGNED), (dict(dk=P + 4), MISALIGNED),
    (dict(dv=P + 1), MISALIGNED), (dict(lse=P + 2), MISALIGNED), (dict(ws=P + 128), MISALIGNED),
])
def test_backward_rejected_before_any_cuda_call(kw, expected):
    assert call_bwd(**kw) == expected


@pytest.mark.parametrize("kw", [dict(B=0), dict(N=0), dict(N=0, q=None, dout=None, ws=None, ws_bytes=0)])
def test_backward_empty_problem_is_ok_without_launch(kw):
    assert call_bwd(**kw) == OK


def test_backward_workspace_bytes():
    # two fp32 arrays [B*Hq][N rounded up to 128], each rounded up to 256 bytes
    assert attn.attn_bwd_workspace_bytes(4, 16, 2048) == 2 * 4 * 16 * 2048 * 4
    assert attn.attn_bwd_workspace_bytes(1, 1, 1) == 2 * 128 * 4
    assert attn.attn_bwd_workspace_bytes(1, 3, 129) == 2 * 3 * 256 * 4
    assert attn.attn_bwd_workspace_bytes(0, 4, 100) == 0
    assert attn.attn_bwd_workspace_bytes(2, 4, 0) == 0
    assert attn.attn_bwd_workspace_bytes(-1, 4, 100) == -1
    assert attn.attn_bwd_workspace_bytes(1, 0, 100) == -1


# ---------------------------------------------------------------- RoPE entry points

def call_rope(**kw):
    args = dict(q=P, k=P, c=P, s=P, qo=P, ko=P, B=1, Hq=2, Hkv=1, N=128, D=128)
    args.update(kw)
    return attn.attn_rope_qk(args["q"], args["k"], args["c"], args["s"], args["qo"], args["ko"], args["B"],
                             args["Hq"], args["Hkv"], args["N"], args["D"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(c=None), INVALID), (dict(s=None), INVALID),
    (dict(qo=None), INVALID), (dict(ko=None), INVALID), (dict(B=-1), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(D=80), UNSUPPORTED), (dict(D=384), UNSUPPORTED), (dict(q=P + 8), MISALIGNED),
    (dict(c=P + 4), MISALIGNED), (dict(ko=P + 2), MISALIGNED),
    (dict(B=1 << 20, Hq=1 << 10, Hkv=1 << 10, N=1 << 20), UNSUPPORTED),
    # rows of Q and K together at 2^32 (the kernel's 32-bit row index) and one below
    (dict(B=1, Hq=1 << 15, Hkv=1 << 15, N=1 << 16, D=32), UNSUPPORTED),
])
def test_rope_rejected_before_any_cuda_call(kw, expected):
    assert call_rope(**kw) == expected


def test_rope_empty_problem_is_ok():
    assert call_rope(B=0) == OK
    assert call_rope(N=0, q=None, k=None, c=None, s=None, qo=None, ko=None) == OK


def call_fwd_rope(**kw):
    args = dict(q=P, k=P, v=P, c=P, s=P, o=P, lse=P, B=1, Hq=2, Hkv=1, N=128, D=128, causal=0, scale=0.125,
                ws=P, nbytes=1 << 24)
    args.update(kw)
    return attn.attn_fwd_rope(args["q"], args["k"], args["v"], args["c"], args["s"], args["o"], args["lse"],
                              args["B"], args["Hq"], args["Hkv"], args["N"], args["D"], args["causal"],
                              args["scale"], args["ws"], args["nbytes"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(v=None), INVALID), (dict(ws=None), INVALID), (dict(nbytes=1024), INVALID), (dict(o=None), INVALID),
    (dict(scale=math.nan), INVALID), (dict(D=48), UNSUPPORTED), (dict(ws=P + 64), MISALIGNED),
    (dict(lse=P + 2), MISALIGNED), (dict(s=P + 8), MISALIGNED),
])
def test_fwd_rope_rejected_before_any_cuda_call(kw, expected):
    assert call_fwd_rope(**kw) == expected


def call_rope_inverse(**kw):
    args = dict(q=P, k=P, c=P, s=P, qo=P, ko=P, B=1, Hq=2, Hkv=1, N=128, D=128)
    args.update(kw)
    return attn.attn_rope_qk_inverse(args["q"], args["k"], args["c"], args["s"], args["qo"], args["ko"], args["B"],
                                     args["Hq"], args["Hkv"], args["N"], args["D"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=None), INVALID), (dict(ko=None), INVALID), (dict(c=None), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(D=80), UNSUPPORTED), (dict(k=P + 8), MISALIGNED), (dict(qo=P + 2), MISALIGNED),
])
def test_rope_inverse_rejected_before_any_cuda_call(kw, expected):
    assert call_rope_inverse(**kw) == expected
    assert call_rope_inverse(B=0) == OK


def call_bwd_rope(**kw):
    args = dict(q=P, k=P, v=P, c=P, s=P, o=P, lse=P, do=P, dq=P, dk=P, dv=P, B=1, Hq=2, Hkv=1, N=128, D=128,
                causal=0, scale=0.125, ws=P, nbytes=1 << 24)
    args.update(kw)
    return attn.attn_bwd_rope(args["q"], args["k"], args["v"], args["c"], args["s"], args["o"], args["lse"],
                              args["do"], args["dq"], args["dk"], args["dv"], args["B"], args["Hq"], args["Hkv"],
                              args["N"], args["D"], args["causal"], args["scale"], args["ws"], args["nbytes"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(v=None), INVALID), (dict(o=None), INVALID), (dict(lse=None), INVALID), (dict(do=None), INVALID),
    (dict(dq=None), INVALID), (dict(dk=None), INVALID), (dict(dv=None), INVALID), (dict(ws=None), INVALID),
    (dict(nbytes=1024), INVALID), (dict(scale=math.nan), INVALID), (dict(c=None), INVALID),
    (dict(D=192), UNSUPPORTED), (dict(D=48), UNSUPPORTED), (dict(ws=P + 64), MISALIGNED),
    (dict(dk=P + 8), MISALIGNED), (dict(lse=P + 2), MISALIGNED), (dict(do=P + 8), MISALIGNED),
])
def test_bwd_rope_rejected_before_any_cuda_call(kw, expected):
    assert call_bwd_rope(**kw) == expected


def test_bwd_rope_empty_problem_and_workspace_query():
    assert call_bwd_rope(B=0) == OK and call_bwd_rope(N=0) == OK
    need = attn.attn_bwd_rope_workspace_bytes(2, 4, 2, 300, 64)
    rot = -(-2 * 4 * 300 * 64 * 2 // 256) * 256 + -(-2 * 2 * 300 * 64 * 2 // 256) * 256
    assert need == rot + attn.attn_bwd_workspace_bytes(2, 4, 300)
    assert attn.attn_bwd_rope_workspace_bytes(1, 2, 1, 100, 256) == -1
    assert attn.attn_bwd_rope_workspace_bytes(0, 2, 1, 100, 64) == 0


# ---------------------------------------------------------------- E4M3 forward

def call_fp8(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=1, N=128, D=128, causal=0, scale=0.125, qd=0.1, kd=0.1,
                vd=0.1, ws=None, nbytes=0)
    args.update(kw)
    return attn.attn_fwd_fp8(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"],
                             args["Hkv"], args["N"], args["D"], args["causal"], args["scale"], args["qd"],
                             args["kd"], args["vd"], args["ws"], args["nbytes"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=None), INVALID), (dict(o=None), INVALID), (dict(qd=0.0), INVALID), (dict(kd=math.nan), INVALID),
    (dict(vd=math.inf), INVALID), (dict(scale=math.nan), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(D=160), UNSUPPORTED), (dict(D=80), UNSUPPORTED), (dict(D=512), UNSUPPORTED),
    (dict(v=P + 8), MISALIGNED), (dict(ws=P + 64, nbytes=4096), MISALIGNED), (dict(ws=None, nbytes=64), INVALID),
])
def test_fp8_rejected_before_any_cuda_call(kw, expected):
    assert call_fp8(**kw) == expected


def test_fp8_empty_problem_is_ok():
    assert call_fp8(B=0) == OK
    assert call_fp8(N=0, q=None, k=None, v=None, o=None, lse=None) == OK


def test_backward_grid_limit():
    # B * Hq * ceil(N/128) above 2^30 is refused on the host
    assert call_bwd(B=1 << 16, Hq=1 << 8, Hkv=1 << 8, N=128 * ((1 << 6) + 1)) == UNSUPPORTED


def test_fast_div_equals_floor_division():
    """The scheduler's division by launch-constant divisors (multiply-high by
    ceil(2^64 / d)) against exact integer division: every small divisor, powers of two and
    their neighbours, large divisors, and dividends at 0, around multiples of d and at the
    top of the 32-bit range (the kernel's counts stay below 2^31)."""
    import random

    rng = random.Random(11)
    divisors = list(range(1, 300))
    for e in range(1, 32):
        divisors += [(1 << e) - 1, 1 << e, (1 << e) + 1]
    divisors += [rng.randrange(2, 1 << 32) for _ in range(200)] + [(1 << 32) - 1, (1 << 31) - 1, 3 * 5 * 7 * 11 * 13]
    top = (1 << 32) - 1
    for d in divisors:
        if d > top:
            continue
        ns = {0, 1, d - 1, d, d + 1, 2 * d - 1, top, top - 1, (1 << 31) - 1, (top // d) * d, (top // d) * d - 1}
        ns |= {rng.randrange(0, 1 << 32) for _ in range(40)}
        ns |= {k * d + r for k in (rng.randrange(0, max(1, top // d)),) for r in (0, d - 1)}
        for n in ns:
            if 0 <= n <= top:
                assert attn.attn_selftest_fast_div(n, d) == n // d, (n, d)
    assert attn.attn_selftest_fast_div(5, 0) == 0


def test_work_unit_count_limit():
    """The scheduler indexes work units (256 query rows of one head) in 32 bits: a problem with
    2^31 or more of them is refused before any CUDA call, even when B*Hq itself fits."""
    B, Hq = 1 << 20, 1 << 10                      # B*Hq = 2^30
    assert call(B=B, Hq=Hq, Hkv=Hq, N=2048) == UNSUPPORTED   # 2^30 heads x 8 units
    assert call(B=B, Hq=Hq, Hkv=Hq, N=512) == UNSUPPORTED    # exactly 2^31 units


def call_host(**kw):
    a = dict(qh=P, kh=P, vh=P, oh=P, lh=P, qd=P, kd=P, vd=P, od=P, ld=P, ws=None, wsb=0, B=2, Hq=4, Hkv=2, N=128,
             D=128, causal=0, scale=0.125, pieces=4)
    a.update(kw)
    return attn.attn_fwd_from_host(a["qh"], a["kh"], a["vh"], a["oh"], a["lh"], a["qd"], a["kd"], a["vd"], a["od"],
                                   a["ld"], a["ws"], a["wsb"], a["B"], a["Hq"], a["Hkv"], a["N"], a["D"], a["causal"],
                                   a["scale"], a["pieces"], None)


@pytest.mark.parametrize("kw,expected", [
    (dict(qh=None), INVALID), (dict(oh=None), INVALID), (dict(lh=None), INVALID), (dict(qd=None), INVALID),
    (dict(ld=None), INVALID), (dict(pieces=0), INVALID), (dict(pieces=-3), INVALID), (dict(Hq=3), INVALID),
    (dict(scale=math.nan), INVALID), (dict(ws=None, wsb=256), INVALID), (dict(D=80), UNSUPPORTED),
    (dict(qd=P + 8), MISALIGNED), (dict(od=P + 2), MISALIGNED), (dict(ld=P + 2), MISALIGNED),
    (dict(ws=P + 128, wsb=4096), MISALIGNED), (dict(B=0), OK), (dict(N=0, qh=None, qd=None), OK),
])
def test_host_buffer_entry_point_rejects_before_any_cuda_call(kw, expected):
    assert call_host(**kw) == expected


def test_host_buffer_workspace_query_rejects_bad_sizes():
    assert attn.attn_fwd_from_host_workspace_bytes(1, 3, 2, 128, 128, 0, 4) == -1
    assert attn.attn_fwd_from_host_workspace_bytes(1, 2, 2, 128, 80, 0, 4) == -1
    assert attn.attn_fwd_from_host_workspace_bytes(1, 2, 2, 128, 128, 0, 0) == -1
    assert attn.attn_fwd_from_host_workspace_bytes(0, 2, 2, 128, 128, 0, 4) == 0


@pytest.mark.parametrize("args,expected", [
    ((P, P, -1, 64, 10000.0), INVALID), ((P, P, 16, 7, 10000.0), INVALID), ((P, P, 16, 0, 10000.0), INVALID),
    ((P, P, 16, 64, 0.0), INVALID), ((P, P, 16, 64, -2.0), INVALID), ((P, P, 16, 64, math.nan), INVALID),
    ((P, P, 16, 64, math.inf), INVALID), ((None, P, 16, 64, 10000.0), INVALID), ((P + 4, P, 16, 64, 10000.0), MISALIGNED),
    ((P, P + 8, 16, 64, 10000.0), MISALIGNED), ((None, None, 0, 64, 10000.0), OK),
])
def test_rope_tables_entry_point_rejects_before_any_cuda_call(args, expected):
    assert attn.attn_rope_tables(*args, None) == expected
