"""bf16 attention on B200 (sm_100a) -- forward, backward, RoPE: Python binding of the C ABI in include/attn.h.

The binding only marshals arguments: every step of the computation runs in the
CUDA kernel inside ``libattn_fwd.so``.  There is no CPU fallback; if the library
cannot be loaded, importing this package raises.

    import tiled_attention_forward_03_b200 as attn
    o, lse = attn.forward(q, k, v, causal=True)        # q,k,v: CUDA bf16 [B, H, N, D]
    dq, dk, dv = attn.backward(q, k, v, o, lse, do, causal=True)
    cos_t, sin_t = attn.rope_tables(N, D, device="cuda")
    o, lse = attn.forward_rope(q, k, v, cos_t, sin_t, causal=True)   # attention of RoPE(q), RoPE(k)
    dq, dk, dv = attn.backward_rope(q, k, v, cos_t, sin_t, o, lse, do, causal=True)
"""
from __future__ import annotations

import ctypes
import math
import os

from . import build as _build

__all__ = [
    "ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_MISALIGNED",
    "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT", "AttnError", "lib", "lib_path", "attn_fwd", "attn_fwd_ws",
    "attn_fwd_workspace_bytes", "attn_fwd_noalloc", "attn_fwd_noalloc_scratch_bytes", "attn_fwd_from_host",
    "attn_fwd_from_host_workspace_bytes", "attn_rope_tables",
    "attn_status_string", "attn_last_cuda_error", "attn_device_status", "attn_num_units",
    "attn_version", "attn_selftest_exp2_poly", "attn_selftest_wait_timeout", "forward",
    "forward_from_host", "device_status", "attn_bwd", "attn_bwd_workspace_bytes", "backward",
    "backward_from_host", "attn_rope_qk", "attn_fwd_rope", "attn_fwd_rope_workspace_bytes", "rope_tables",
    "rope", "forward_rope", "attn_fwd_fp8", "forward_fp8", "attn_rope_qk_inverse", "attn_bwd_rope",
    "attn_bwd_rope_workspace_bytes", "rope_inverse", "backward_rope",
]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_MISALIGNED = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str = "attn_fwd"):
        self.status = status
        detail = attn_last_cuda_error() if status in (ATTN_ERR_CUDA,) else ""
        super().__init__(f"{where} failed: {attn_status_string(status)}" + (f" ({detail})" if detail else ""))


def _load() -> ctypes.CDLL:
    path = _build.LIB_PATH
    if not _build.up_to_date():
        # Sources newer than the library (or no library): rebuild.  A failed build is an
        # error; only a machine without nvcc may use an existing library as shipped.
        if _build.have_nvcc():
            try:
                _build.build()
            except Exception as exc:
                raise ImportError(f"building the attention CUDA library failed: {exc}") from exc
        elif not os.path.exists(path):
            raise ImportError(f"attention CUDA library not found at {path} and nvcc is unavailable")
    if not os.path.exists(path):
        raise ImportError(f"attention CUDA library not found at {path}")
    L = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.attn_fwd.restype = i
    L.attn_fwd_ws.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    L.attn_bwd.restype = i
    L.attn_bwd_workspace_bytes.argtypes = [i, i, i]
    L.attn_bwd_workspace_bytes.restype = ctypes.c_longlong
    L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, f, vp, ctypes.c_size_t, vp]
    L.attn_fwd_fp8.restype = i
    L.attn_rope_qk.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    L.attn_rope_qk.restype = i
    L.attn_fwd_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    L.attn_fwd_rope.restype = i
    L.attn_fwd_rope_workspace_bytes.argtypes = [i, i, i, i, i]
    L.attn_fwd_rope_workspace_bytes.restype = ctypes.c_longlong
    L.attn_rope_qk_inverse.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    L.attn_rope_qk_inverse.restype = i
    L.attn_bwd_rope.argtypes = [vp] * 11 + [i, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    L.attn_bwd_rope.restype = i
    L.attn_bwd_rope_workspace_bytes.argtypes = [i, i, i, i, i]
    L.attn_bwd_rope_workspace_bytes.restype = ctypes.c_longlong
    L.attn_fwd_ws.restype = i
    L.attn_fwd_workspace_bytes.argtypes = [i, i, i, i, i]
    L.attn_fwd_workspace_bytes.restype = ctypes.c_longlong
    L.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.attn_fwd_noalloc.restype = i
    L.attn_fwd_from_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i, i, i, i, i, i,
                                     f, i, vp]
    L.attn_fwd_from_host.restype = i
    L.attn_fwd_from_host_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    L.attn_fwd_from_host_workspace_bytes.restype = ctypes.c_longlong
    L.attn_rope_tables.argtypes = [vp, vp, i, i, ctypes.c_double, vp]
    L.attn_rope_tables.restype = i
    L.attn_fwd_noalloc_scratch_bytes.argtypes = []
    L.attn_fwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
    L.attn_status_string.argtypes = [i]
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_last_cuda_error.argtypes = []
    L.attn_last_cuda_error.restype = ctypes.c_char_p
    L.attn_device_status.argtypes = [vp, ctypes.POINTER(i)]
    L.attn_device_status.restype = i
    L.attn_num_units.argtypes = [i, i, i]
    L.attn_num_units.restype = ctypes.c_longlong
    L.attn_version.argtypes = []
    L.attn_version.restype = ctypes.c_char_p
    L.attn_selftest_fast_div.argtypes = [ctypes.c_uint, ctypes.c_uint]
    L.attn_selftest_fast_div.restype = ctypes.c_uint
    L.attn_selftest_exp2_poly.argtypes = [vp, vp, i, vp]
    L.attn_selftest_exp2_poly.restype = i
    L.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    L.attn_selftest_wait_timeout.restype = i
    return L


lib = _load()
lib_path = _build.LIB_PATH


# ---------------------------------------------------------------- raw C calls

def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, stream) -> int:
    """Direct call of the C entry point; pointers and stream are integers (or None)."""
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, D, int(bool(causal)), float(scale), stream)


def attn_fwd_ws(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, workspace, workspace_bytes, stream) -> int:
    """Direct call of the workspace entry point (pointers, sizes and stream as integers)."""
    return lib.attn_fwd_ws(q, k, v, o, lse, B, Hq, Hkv, N, D, int(bool(causal)), float(scale),
                           workspace, workspace_bytes, stream)


def attn_fwd_noalloc(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, stream) -> int:
    """Direct call of the entry point that allocates nothing (its workspace is a static
    device array in the library); for callers that may not allocate device memory."""
    return lib.attn_fwd_noalloc(q, k, v, o, lse, B, Hq, Hkv, N, D, int(bool(causal)), float(scale), stream)


def attn_fwd_from_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev, workspace,
                       workspace_bytes, B, Hq, Hkv, N, D, causal, scale, pieces, stream) -> int:
    """Direct call of the host-buffer entry point (host and device pointers, sizes and stream as
    integers); returns once the host outputs hold the results."""
    return lib.attn_fwd_from_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev,
                                  workspace, workspace_bytes, B, Hq, Hkv, N, D, int(bool(causal)), float(scale),
                                  pieces, stream)


def attn_fwd_from_host_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int, causal: bool, pieces: int) -> int:
    return lib.attn_fwd_from_host_workspace_bytes(B, Hq, Hkv, N, D, int(bool(causal)), pieces)


def attn_rope_tables(cos_t, sin_t, N, D, base, stream) -> int:
    """Direct call of the RoPE table entry point (device pointers and stream as integers)."""
    return lib.attn_rope_tables(cos_t, sin_t, N, D, float(base), stream)


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, causal, scale, workspace, workspace_bytes,
             stream) -> int:
    """Direct call of the backward entry point (pointers, sizes and stream as integers)."""
    return lib.attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, int(bool(causal)), float(scale),
                        workspace, workspace_bytes, stream)


def attn_bwd_workspace_bytes(B: int, Hq: int, N: int) -> int:
    return lib.attn_bwd_workspace_bytes(B, Hq, N)


def attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, q_descale, k_descale, v_descale, workspace,
                 workspace_bytes, stream) -> int:
    """Direct call of the E4M3 forward entry point (pointers, sizes and stream as integers)."""
    return lib.attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, D, int(bool(causal)), float(scale), float(q_descale),
                            float(k_descale), float(v_descale), workspace, workspace_bytes, stream)


def attn_rope_qk(q, k, cos_t, sin_t, q_out, k_out, B, Hq, Hkv, N, D, stream) -> int:
    """Direct call of the RoPE entry point (pointers and stream as integers)."""
    return lib.attn_rope_qk(q, k, cos_t, sin_t, q_out, k_out, B, Hq, Hkv, N, D, stream)


def attn_fwd_rope(q, k, v, cos_t, sin_t, o, lse, B, Hq, Hkv, N, D, causal, scale, workspace, workspace_bytes,
                  stream) -> int:
    """Direct call of the RoPE + forward entry point."""
    return lib.attn_fwd_rope(q, k, v, cos_t, sin_t, o, lse, B, Hq, Hkv, N, D, int(bool(causal)), float(scale),
                             workspace, workspace_bytes, stream)


def attn_fwd_rope_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int) -> int:
    return lib.attn_fwd_rope_workspace_bytes(B, Hq, Hkv, N, D)


def attn_rope_qk_inverse(dq_rot, dk_rot, cos_t, sin_t, dq, dk, B, Hq, Hkv, N, D, stream) -> int:
    """Direct call of the inverse RoPE entry point (pointers and stream as integers)."""
    return lib.attn_rope_qk_inverse(dq_rot, dk_rot, cos_t, sin_t, dq, dk, B, Hq, Hkv, N, D, stream)


def attn_bwd_rope(q, k, v, cos_t, sin_t, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, causal, scale, workspace,
                  workspace_bytes, stream) -> int:
    """Direct call of the RoPE backward entry point."""
    return lib.attn_bwd_rope(q, k, v, cos_t, sin_t, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D,
                             int(bool(causal)), float(scale), workspace, workspace_bytes, stream)


def attn_bwd_rope_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int) -> int:
    return lib.attn_bwd_rope_workspace_bytes(B, Hq, Hkv, N, D)


def attn_fwd_noalloc_scratch_bytes() -> int:
    return lib.attn_fwd_noalloc_scratch_bytes()


def attn_fwd_workspace_bytes(B: int, Hq: int, N: int, D: int, causal: bool) -> int:
    return lib.attn_fwd_workspace_bytes(B, Hq, N, D, int(bool(causal)))


def attn_status_string(status: int) -> str:
    return lib.attn_status_string(status).decode()


def attn_last_cuda_error() -> str:
    return lib.attn_last_cuda_error().decode()


def attn_device_status(stream=None):
    site = ctypes.c_int(0)
    st = lib.attn_device_status(stream, ctypes.byref(site))
    return st, site.value


def attn_num_units(B: int, Hq: int, N: int) -> int:
    return lib.attn_num_units(B, Hq, N)


def attn_version() -> str:
    return lib.attn_version().decode()


def attn_selftest_fast_div(n: int, d: int) -> int:
    return lib.attn_selftest_fast_div(n, d)


def attn_selftest_exp2_poly(x_ptr, y_ptr, n: int, stream) -> int:
    return lib.attn_selftest_exp2_poly(x_ptr, y_ptr, n, stream)


def attn_selftest_wait_timeout(timeout_us: int, stream) -> int:
    return lib.attn_selftest_wait_timeout(timeout_us, stream)


# ---------------------------------------------------------------- torch conveniences

def _check(t, name, dtype, shape):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_workspaces: dict = {}


def _workspace(device, nbytes: int, purpose: str, stream):
    """A cached device buffer of at least nbytes, per device, purpose ("fwd": the split-tail
    schedule, "bwd": the backward pass's per-row delta and LSE, "rope": the rotated q and k,
    "bwd_rope": the rotated q and k and the backward's per-row data)
    and stream.  Calls on one stream run in order, so they may share a buffer; calls on
    different streams get different buffers and may overlap on the GPU.  The buffer is marked
    as used on ``stream``, so that when a larger one replaces it, torch's allocator does not
    hand its memory to another stream's allocation before the kernels enqueued on ``stream``
    have finished with it."""
    import torch

    key = (device.type, device.index, purpose, stream.cuda_stream)
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    buf.record_stream(stream)
    return buf


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None, stream=None,
            split: bool = True):
    """Attention forward on CUDA bf16 tensors [B, H, N, D]; returns (o bf16, lse fp32 [B, Hq, N]).

    Runs on ``stream`` (a torch.cuda.Stream) or torch's current stream.  With ``split``
    (default) a non-causal problem whose last wave would leave the GPU half idle splits
    that wave's KV ranges across SMs (attn_fwd_ws, with a workspace cached per device and
    stream, so calls on different streams may run at once); ``split=False`` calls attn_fwd.
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, N, D]")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    _check(q, "q", torch.bfloat16, (B, Hq, N, D))
    _check(k, "k", torch.bfloat16, (B, Hkv, N, D))
    _check(v, "v", torch.bfloat16, (B, Hkv, N, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, (B, Hq, N, D))
    _check(lse, "lse", torch.float32, (B, Hq, N))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        ws_bytes = attn_fwd_workspace_bytes(B, Hq, N, D, causal) if split else 0
        if ws_bytes < 0:
            raise AttnError(ATTN_ERR_CUDA, "attn_fwd_workspace_bytes")
        if ws_bytes > 0:
            ws = _workspace(q.device, ws_bytes, "fwd", s)
            st = attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, Hq, Hkv, N, D, causal, scale, ws.data_ptr(), ws.numel(), s.cuda_stream)
        else:
            st = attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, Hq, Hkv, N, D, causal, scale, s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st)
    return out, lse


def _pieces(B: int, Hq: int, Hkv: int, n: int):
    """Up to n independent pieces of a [B, H, ...] attention problem, as (batch slice, query-head
    slice, KV-head slice): ranges of batch rows, or for B == 1 ranges of whole KV-head groups.
    Each piece is a contiguous block of every tensor."""
    if B >= 2 or Hkv == 1:
        n = max(1, min(n, B))
        e = [B * i // n for i in range(n + 1)]
        return [(slice(e[i], e[i + 1]), slice(None), slice(None)) for i in range(n) if e[i] < e[i + 1]]
    g = Hq // Hkv
    n = max(1, min(n, Hkv))
    e = [Hkv * i // n for i in range(n + 1)]
    return [(slice(0, 1), slice(e[i] * g, e[i + 1] * g), slice(e[i], e[i + 1])) for i in range(n) if e[i] < e[i + 1]]


_streams: dict = {}


def _side_streams(dev):
    """The two copy streams of the host-buffer calls, created once per device."""
    import torch

    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    pair = _streams.get(key)
    if pair is None:
        pair = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        _streams[key] = pair
    return pair


def _pipelined(dev, stream, pieces, inputs, outputs, compute):
    """Run `compute(piece)` for each piece with its inputs copied in and its outputs copied out,
    the copies on two side streams so that piece i+1's upload and piece i-1's download overlap
    piece i's kernels.  inputs / outputs: lists of (host tensor, device tensor, piece -> index).
    Returns after every copy has completed.  The side streams are shared by all calls on a
    device: calls from several host threads at once must not overlap."""
    import torch

    s_in, s_out = _side_streams(dev)
    s_in.wait_stream(stream)
    for pc in pieces:
        with torch.cuda.stream(s_in):
            for host, devt, idx in inputs:
                devt[idx(pc)].copy_(host[idx(pc)], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
        stream.wait_event(ev_in)
        with torch.cuda.stream(stream):
            compute(pc)
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
        s_out.wait_event(ev_c)
        with torch.cuda.stream(s_out):
            for host, devt, idx in outputs:
                host[idx(pc)].copy_(devt[idx(pc)], non_blocking=True)
    s_out.synchronize()
    stream.synchronize()
    s_in.synchronize()


def forward_from_host(q, k, v, causal: bool = False, scale: float | None = None, device=None,
                      out_host=None, lse_host=None, stream=None, rope_tables=None, fp8_descales=None,
                      pieces: int = 8):
    """End-to-end call on host (ideally pinned) tensors: copy in, attention, copy out.

    Returns host tensors (o, lse).  The problem is cut into up to ``pieces`` independent parts
    (batch rows, or KV-head groups when B == 1); each part's upload, kernel and download are
    enqueued so that the copies of neighbouring parts overlap the kernels.  The bf16 forward
    is the library's own host-buffer call, attn_fwd_from_host (device buffers and the split
    workspace come from torch, on ``stream``).  With ``rope_tables`` = (cos_t, sin_t) (device
    tables from rope_tables()), the attention is that of RoPE(q), RoPE(k) and v (forward_rope),
    and with ``fp8_descales`` = (q_descale, k_descale, v_descale), q, k, v are float8_e4m3fn and
    the call is forward_fp8: those two are pipelined here, with torch copies on two side streams.
    """
    import torch

    dev = torch.device(device if device is not None else "cuda")
    if dev.index is None:
        dev = torch.device(dev.type, torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    with torch.cuda.stream(s):
        qd, kd, vd = (torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (q, k, v))
        od = torch.empty((B, Hq, N, D), dtype=torch.bfloat16, device=dev)
        ld = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    if out_host is None:
        out_host = torch.empty(od.shape, dtype=od.dtype, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty(ld.shape, dtype=ld.dtype, pin_memory=True)
    if rope_tables is None and fp8_descales is None:
        for name, t, shape in (("q", q, (B, Hq, N, D)), ("k", k, (B, Hkv, N, D)), ("v", v, (B, Hkv, N, D)),
                               ("out_host", out_host, (B, Hq, N, D))):
            if t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 host tensor of shape {shape}")
        if lse_host.is_cuda or lse_host.dtype != torch.float32 or tuple(lse_host.shape) != (B, Hq, N) \
                or not lse_host.is_contiguous():
            raise ValueError(f"lse_host must be a contiguous fp32 host tensor of shape {(B, Hq, N)}")
        with torch.cuda.device(dev):
            ws_bytes = attn_fwd_from_host_workspace_bytes(B, Hq, Hkv, N, D, causal, pieces)
            if ws_bytes < 0:
                raise AttnError(ATTN_ERR_INVALID_ARG, "attn_fwd_from_host_workspace_bytes")
            ws = _workspace(dev, ws_bytes, "fwd", s) if ws_bytes > 0 else None
            st = attn_fwd_from_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out_host.data_ptr(),
                                    lse_host.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                                    ld.data_ptr(), ws.data_ptr() if ws is not None else None,
                                    ws.numel() if ws is not None else 0, B, Hq, Hkv, N, D, causal, scale, pieces,
                                    s.cuda_stream)
        if st != ATTN_OK:
            raise AttnError(st, "attn_fwd_from_host")
        return out_host, lse_host
    qi = lambda pc: (pc[0], pc[1])
    ki = lambda pc: (pc[0], pc[2])

    def compute(pc):
        a, b, c, o, lse = qd[qi(pc)], kd[ki(pc)], vd[ki(pc)], od[qi(pc)], ld[qi(pc)]
        if rope_tables is not None:
            forward_rope(a, b, c, rope_tables[0], rope_tables[1], causal=causal, scale=scale, out=o, lse=lse, stream=s)
        else:
            forward_fp8(a, b, c, *fp8_descales, causal=causal, scale=scale, out=o, lse=lse, stream=s)

    _pipelined(dev, s, _pieces(B, Hq, Hkv, pieces), [(q, qd, qi), (k, kd, ki), (v, vd, ki)],
               [(out_host, od, qi), (lse_host, ld, qi)], compute)
    return out_host, lse_host


def backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None, dq=None, dk=None,
             dv=None, stream=None):
    """Attention backward on CUDA tensors: returns (dq, dk, dv), bf16, shaped like q, k, v.

    ``o`` and ``lse`` are the forward's outputs for the same q, k, v, causal and scale;
    ``dout`` is the bf16 gradient of the loss with respect to o.  The workspace (per-row
    delta and LSE) is cached per device and stream.
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, N, D]")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    _check(q, "q", torch.bfloat16, (B, Hq, N, D))
    _check(k, "k", torch.bfloat16, (B, Hkv, N, D))
    _check(v, "v", torch.bfloat16, (B, Hkv, N, D))
    _check(o, "o", torch.bfloat16, (B, Hq, N, D))
    _check(lse, "lse", torch.float32, (B, Hq, N))
    _check(dout, "dout", torch.bfloat16, (B, Hq, N, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", torch.bfloat16, (B, Hq, N, D))
    _check(dk, "dk", torch.bfloat16, (B, Hkv, N, D))
    _check(dv, "dv", torch.bfloat16, (B, Hkv, N, D))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        ws_bytes = attn_bwd_workspace_bytes(B, Hq, N)
        if ws_bytes < 0:
            raise AttnError(ATTN_ERR_INVALID_ARG, "attn_bwd_workspace_bytes")
        ws = _workspace(q.device, max(ws_bytes, 256), "bwd", s)
        st = attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, N, D, causal, scale,
                      ws.data_ptr(), ws.numel(), s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def backward_from_host(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None, device=None,
                       out_host=None, stream=None, pieces: int = 4, rope_tables=None):
    """End-to-end backward on host (ideally pinned) tensors: copy q, k, v, o, lse and dout in,
    run attn_bwd, copy dq, dk, dv out.  Returns host tensors (dq, dk, dv); ``out_host`` may
    hold three preallocated host tensors for them.  Pipelined in up to ``pieces`` independent
    parts as forward_from_host (batch rows, or whole KV-head groups when B == 1, so that each
    KV head's gradient is complete within one part).  With ``rope_tables`` = (cos_t, sin_t)
    (device tables from rope_tables()) the gradients are those through RoPE (backward_rope;
    o and lse from forward_rope).  Returns after the last download."""
    import torch

    dev = torch.device(device if device is not None else "cuda")
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    host_in = (q, k, v, o, lse, dout)
    with torch.cuda.stream(s):
        dev_in = tuple(torch.empty(x.shape, dtype=x.dtype, device=dev) for x in host_in)
        grads = tuple(torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (q, k, v))
    if out_host is None:
        out_host = tuple(torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in grads)
    qi = lambda pc: (pc[0], pc[1])
    ki = lambda pc: (pc[0], pc[2])
    in_idx = (qi, ki, ki, qi, qi, qi)

    def compute(pc):
        qd, kd, vd, od, ld, dd = (x[f(pc)] for x, f in zip(dev_in, in_idx))
        if rope_tables is not None:
            backward_rope(qd, kd, vd, rope_tables[0], rope_tables[1], od, ld, dd, causal=causal, scale=scale,
                          dq=grads[0][qi(pc)], dk=grads[1][ki(pc)], dv=grads[2][ki(pc)], stream=s)
        else:
            backward(qd, kd, vd, od, ld, dd, causal=causal, scale=scale, dq=grads[0][qi(pc)], dk=grads[1][ki(pc)],
                     dv=grads[2][ki(pc)], stream=s)

    _pipelined(dev, s, _pieces(B, Hq, Hkv, pieces), list(zip(host_in, dev_in, in_idx)),
               list(zip(out_host, grads, (qi, ki, ki))), compute)
    return tuple(out_host)


def forward_fp8(q, k, v, q_descale: float, k_descale: float, v_descale: float, causal: bool = False,
                scale: float | None = None, out=None, lse=None, stream=None, split: bool = True):
    """Attention forward on CUDA float8_e4m3fn q, k, v [B, H, N, D] with per-tensor descales
    (the inputs' values are descale * stored value); returns (o bf16, lse fp32 [B, Hq, N]).
    Workspace handling as forward()."""
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, N, D]")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    f8 = torch.float8_e4m3fn
    _check(q, "q", f8, (B, Hq, N, D))
    _check(k, "k", f8, (B, Hkv, N, D))
    _check(v, "v", f8, (B, Hkv, N, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.empty((B, Hq, N, D), dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", torch.bfloat16, (B, Hq, N, D))
    _check(lse, "lse", torch.float32, (B, Hq, N))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        ws_bytes = attn_fwd_workspace_bytes(B, Hq, N, D, causal) if split else 0
        if ws_bytes < 0:
            raise AttnError(ATTN_ERR_CUDA, "attn_fwd_workspace_bytes")
        ws = _workspace(q.device, ws_bytes, "fwd", s) if ws_bytes > 0 else None
        st = attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N,
                          D, causal, scale, q_descale, k_descale, v_descale, ws.data_ptr() if ws is not None else None,
                          ws.numel() if ws is not None else 0, s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return out, lse


def rope_tables(N: int, D: int, base: float = 10000.0, device=None, stream=None):
    """cos and sin tables [N, D/2] (fp32) of the angles p * base^(-2d/D), filled on the device by
    attn_rope_tables (fp64 arithmetic rounded to fp32).  ``device`` defaults to the current CUDA
    device; the tables are written on ``stream`` (or torch's current stream)."""
    import torch

    dev = torch.device(device if device is not None else "cuda")
    with torch.cuda.device(dev):
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        cos_t = torch.empty((N, D // 2), dtype=torch.float32, device=dev)
        sin_t = torch.empty((N, D // 2), dtype=torch.float32, device=dev)
        st = attn_rope_tables(cos_t.data_ptr(), sin_t.data_ptr(), N, D, base, s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_rope_tables")
    return cos_t, sin_t


def rope(q, k, cos_t, sin_t, q_out=None, k_out=None, stream=None):
    """RoPE of CUDA bf16 q [B, Hq, N, D] and k [B, Hkv, N, D] with tables [N, D/2] (fp32, on the
    device); returns (q_out, k_out).  Pass q_out=q, k_out=k to rotate in place."""
    import torch

    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    _check(q, "q", torch.bfloat16, (B, Hq, N, D))
    _check(k, "k", torch.bfloat16, (B, Hkv, N, D))
    _check(cos_t, "cos_t", torch.float32, (N, D // 2))
    _check(sin_t, "sin_t", torch.float32, (N, D // 2))
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    _check(q_out, "q_out", torch.bfloat16, (B, Hq, N, D))
    _check(k_out, "k_out", torch.bfloat16, (B, Hkv, N, D))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = attn_rope_qk(q.data_ptr(), k.data_ptr(), cos_t.data_ptr(), sin_t.data_ptr(), q_out.data_ptr(),
                          k_out.data_ptr(), B, Hq, Hkv, N, D, s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_rope_qk")
    return q_out, k_out


def rope_inverse(dq_rot, dk_rot, cos_t, sin_t, dq=None, dk=None, stream=None):
    """The inverse (= transpose) of rope(): rotates by -theta.  Maps gradients with respect to
    RoPE(q), RoPE(k) to gradients with respect to q, k; returns (dq, dk).  Pass dq=dq_rot,
    dk=dk_rot to work in place."""
    import torch

    B, Hq, N, D = dq_rot.shape
    Hkv = dk_rot.shape[1]
    _check(dq_rot, "dq_rot", torch.bfloat16, (B, Hq, N, D))
    _check(dk_rot, "dk_rot", torch.bfloat16, (B, Hkv, N, D))
    _check(cos_t, "cos_t", torch.float32, (N, D // 2))
    _check(sin_t, "sin_t", torch.float32, (N, D // 2))
    dq = torch.empty_like(dq_rot) if dq is None else dq
    dk = torch.empty_like(dk_rot) if dk is None else dk
    _check(dq, "dq", torch.bfloat16, (B, Hq, N, D))
    _check(dk, "dk", torch.bfloat16, (B, Hkv, N, D))
    s = stream if stream is not None else torch.cuda.current_stream(dq_rot.device)
    with torch.cuda.device(dq_rot.device):
        st = attn_rope_qk_inverse(dq_rot.data_ptr(), dk_rot.data_ptr(), cos_t.data_ptr(), sin_t.data_ptr(),
                                  dq.data_ptr(), dk.data_ptr(), B, Hq, Hkv, N, D, s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_rope_qk_inverse")
    return dq, dk


def backward_rope(q, k, v, cos_t, sin_t, o, lse, dout, causal: bool = False, scale: float | None = None,
                  dq=None, dk=None, dv=None, stream=None):
    """Backward of forward_rope (attn_bwd_rope): gradients (dq, dk, dv) with respect to the
    unrotated q, k and v, given the forward's o and lse and dout.  The workspace (rotated q and k,
    the backward's per-row data) is cached per device and stream."""
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, N, D]")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    _check(q, "q", torch.bfloat16, (B, Hq, N, D))
    _check(k, "k", torch.bfloat16, (B, Hkv, N, D))
    _check(v, "v", torch.bfloat16, (B, Hkv, N, D))
    _check(cos_t, "cos_t", torch.float32, (N, D // 2))
    _check(sin_t, "sin_t", torch.float32, (N, D // 2))
    _check(o, "o", torch.bfloat16, (B, Hq, N, D))
    _check(lse, "lse", torch.float32, (B, Hq, N))
    _check(dout, "dout", torch.bfloat16, (B, Hq, N, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", torch.bfloat16, (B, Hq, N, D))
    _check(dk, "dk", torch.bfloat16, (B, Hkv, N, D))
    _check(dv, "dv", torch.bfloat16, (B, Hkv, N, D))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        ws_bytes = attn_bwd_rope_workspace_bytes(B, Hq, Hkv, N, D)
        if ws_bytes < 0:
            raise AttnError(ATTN_ERR_UNSUPPORTED, "attn_bwd_rope_workspace_bytes")
        ws = _workspace(q.device, max(ws_bytes, 256), "bwd_rope", s)
        st = attn_bwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), cos_t.data_ptr(), sin_t.data_ptr(),
                           o.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                           dv.data_ptr(), B, Hq, Hkv, N, D, causal, scale, ws.data_ptr(), ws.numel(), s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_rope")
    return dq, dk, dv


def forward_rope(q, k, v, cos_t, sin_t, causal: bool = False, scale: float | None = None, out=None, lse=None,
                 stream=None):
    """Attention forward of RoPE(q), RoPE(k), v in one call (attn_fwd_rope); returns (o, lse).
    The workspace (rotated q and k, split tail) is cached per device and stream."""
    import torch

    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    _check(q, "q", torch.bfloat16, (B, Hq, N, D))
    _check(k, "k", torch.bfloat16, (B, Hkv, N, D))
    _check(v, "v", torch.bfloat16, (B, Hkv, N, D))
    _check(cos_t, "cos_t", torch.float32, (N, D // 2))
    _check(sin_t, "sin_t", torch.float32, (N, D // 2))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", torch.bfloat16, (B, Hq, N, D))
    _check(lse, "lse", torch.float32, (B, Hq, N))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        nbytes = attn_fwd_rope_workspace_bytes(B, Hq, Hkv, N, D)
        if nbytes < 0:
            raise AttnError(ATTN_ERR_CUDA, "attn_fwd_rope_workspace_bytes")
        ws = _workspace(q.device, max(nbytes, 256), "rope", s)
        st = attn_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), cos_t.data_ptr(), sin_t.data_ptr(),
                           out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, D, causal, scale, ws.data_ptr(),
                           ws.numel(), s.cuda_stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_rope")
    return out, lse


def device_status(stream=None):
    """Synchronise and report whether a kernel wait gave up: (status, site)."""
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return attn_device_status(s.cuda_stream)
