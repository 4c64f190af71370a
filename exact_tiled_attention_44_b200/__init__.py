"""Exact tiled attention for B200 (sm_100a): Python binding of libattn.so.

Argument marshalling only.  Every arithmetic step of the forward, the backward
and the decoding step runs in the CUDA kernels behind the C ABI declared in
``include/attn.h``; PyTorch supplies device memory and streams.  There is no
CPU fallback: if the library is not built, or the device is not an sm_100 GPU,
the calls raise.

    import exact_tiled_attention_44_b200 as A
    o, lse = A.attention(q, k, v, causal=True)        # q,k,v: CUDA bf16/fp16 [B,H,N,d]
    dq, dk, dv = A.attention_backward(q, k, v, o, do, lse, causal=True)
    o_new, lse_new = A.decode(q_new, k_cache, v_cache)
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "AttnError", "attention", "attention_from_host", "attn_fwd_raw", "attn_fwd_alibi_raw",
    "alibi_slopes", "decode", "decode_workspace_bytes", "attn_decode_raw",
    "attn_decode_noalloc_raw", "attention_backward", "attn_bwd_raw", "bwd_workspace_bytes",
    "unmasked_pairs",
    "visited_blocks", "fwd_unit_kind", "get_status", "set_watchdog_ns", "launch_count", "test_withhold_loads",
    "test_count_blocks", "test_force_units", "error_string",
    "library_path", "load_library", "EXPORTED_SYMBOLS", "ATTN_OK", "ATTN_ERR_INVALID_ARG",
    "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_MISALIGNED", "ATTN_ERR_CUDA", "ATTN_ERR_DEVICE_TIMEOUT",
    "ATTN_BF16", "ATTN_FP16", "ATTN_OUT_F32",
]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_MISALIGNED = -3
ATTN_ERR_CUDA = -4
ATTN_ERR_DEVICE_TIMEOUT = -5
ATTN_BF16 = 0
ATTN_FP16 = 1
ATTN_OUT_F32 = 0x10

EXPORTED_SYMBOLS = ("attn_fwd", "attn_fwd_host", "attn_fwd_alibi", "attn_alibi_slopes",
                    "attn_decode", "attn_decode_workspace_bytes", "attn_decode_noalloc",
                    "attn_error_string", "attn_unmasked_pairs", "attn_visited_blocks",
                    "attn_fwd_unit_kind",
                    "attn_get_status", "attn_set_watchdog_ns", "attn_launch_count",
                    "attn_test_withhold_loads", "attn_test_count_blocks", "attn_test_force_units",
                    "attn_bwd", "attn_bwd_workspace_bytes")

_LIB = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str = "attn_fwd"):
        self.status = status
        super().__init__(f"{what} failed: {error_string(status)} ({status})")


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")


def load_library():
    """Loads libattn.so (built in-tree); raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built: run `python -m exact_tiled_attention_44_b200._build`")
    lib = ctypes.CDLL(path)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp]
    lib.attn_fwd.restype = ci
    lib.attn_fwd_host.argtypes = [vp] * 10 + [ci] * 8 + [cf, ci, vp]
    lib.attn_fwd_host.restype = ci
    lib.attn_fwd_alibi.argtypes = [vp] * 6 + [ci] * 8 + [cf, ci, vp]
    lib.attn_fwd_alibi.restype = ci
    lib.attn_alibi_slopes.argtypes = [ci, ctypes.POINTER(ctypes.c_float)]
    lib.attn_alibi_slopes.restype = ci
    lib.attn_decode.argtypes = [vp] * 6 + [ctypes.c_longlong] + [ci] * 9 + [cf, ci, vp]
    lib.attn_decode.restype = ci
    lib.attn_decode_workspace_bytes.argtypes = [ci] * 6
    lib.attn_decode_workspace_bytes.restype = ctypes.c_longlong
    lib.attn_decode_noalloc.argtypes = [vp] * 5 + [ci] * 9 + [cf, ci, vp]
    lib.attn_decode_noalloc.restype = ci
    lib.attn_error_string.argtypes = [ci]
    lib.attn_error_string.restype = ctypes.c_char_p
    lib.attn_unmasked_pairs.argtypes = [ci, ci, ci, ci]
    lib.attn_unmasked_pairs.restype = ctypes.c_longlong
    lib.attn_visited_blocks.argtypes = [ci, ci, ci, ci]
    lib.attn_visited_blocks.restype = ctypes.c_longlong
    lib.attn_get_status.argtypes = []
    lib.attn_get_status.restype = ci
    lib.attn_set_watchdog_ns.argtypes = [ctypes.c_ulonglong]
    lib.attn_set_watchdog_ns.restype = ctypes.c_ulonglong
    lib.attn_launch_count.argtypes = []
    lib.attn_launch_count.restype = ctypes.c_ulonglong
    lib.attn_test_withhold_loads.argtypes = [ci]
    lib.attn_test_withhold_loads.restype = ci
    lib.attn_test_count_blocks.argtypes = [vp]
    lib.attn_test_count_blocks.restype = ci
    lib.attn_fwd_unit_kind.argtypes = [ci] * 7
    lib.attn_fwd_unit_kind.restype = ci
    lib.attn_test_force_units.argtypes = [ci]
    lib.attn_test_force_units.restype = ci
    lib.attn_bwd.argtypes = [vp] * 11 + [ctypes.c_longlong] + [ci] * 8 + [cf, ci, vp]
    lib.attn_bwd.restype = ci
    lib.attn_bwd_workspace_bytes.argtypes = [ci] * 5
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_longlong
    _LIB = lib
    return lib


def error_string(status: int) -> str:
    return load_library().attn_error_string(int(status)).decode()


def unmasked_pairs(N: int, causal: bool, window: int = 0, n_sink: int = 0) -> int:
    """Kept (query, key) pairs of one head (host-only helper of the library)."""
    return int(load_library().attn_unmasked_pairs(N, int(causal), window, n_sink))


def visited_blocks(N: int, causal: bool, window: int = 0, n_sink: int = 0) -> int:
    """128x128 block pairs the kernel's schedule computes for one head."""
    return int(load_library().attn_visited_blocks(N, int(causal), window, n_sink))


def fwd_unit_kind(B: int, H: int, H_kv: int, N: int, window: int = 0, alibi: bool = False,
                  sm_count: int = 0) -> int:
    """Work-unit shape attn_fwd runs for these sizes (0 tile pairs, 1 split
    tiles, 2 head pairs; host only, see include/attn.h); sm_count 0 asks the
    current device."""
    return int(load_library().attn_fwd_unit_kind(B, H, H_kv, N, window, int(alibi), sm_count))


def get_status() -> int:
    """Reads and clears the device watchdog status (synchronises the device)."""
    return int(load_library().attn_get_status())


def set_watchdog_ns(ns: int) -> int:
    return int(load_library().attn_set_watchdog_ns(int(ns)))


def launch_count() -> int:
    return int(load_library().attn_launch_count())


def test_withhold_loads(n_launches: int) -> int:
    """Failure-detection hook: the next n launches issue no copies, so their
    waits run into the watchdog (see include/attn.h)."""
    return int(load_library().attn_test_withhold_loads(int(n_launches)))


def test_force_units(mode: int) -> int:
    """Work-unit shape hook for tests: 0 forces pairs of Q tiles, 1 single
    tiles shared by both softmax warpgroups, 2 pairs of query heads sharing a
    K/V head, -1 the automatic choice (see include/attn.h)."""
    return int(load_library().attn_test_force_units(int(mode)))


def test_count_blocks(counter: torch.Tensor | None) -> int:
    """Schedule test hook: while set, forward and backward launches add the
    score tiles (forward) or steps (backward) they compute to ``counter``, a
    one-element int64 CUDA tensor the caller zeroes; None turns it off (see
    include/attn.h)."""
    if counter is None:
        return int(load_library().attn_test_count_blocks(None))
    if (not counter.is_cuda or counter.dtype != torch.int64 or counter.numel() != 1
            or not counter.is_contiguous()):
        raise ValueError("counter must be a one-element contiguous int64 CUDA tensor")
    return int(load_library().attn_test_count_blocks(counter.data_ptr()))


def alibi_slopes(H: int, device=None) -> torch.Tensor:
    """The library's ALiBi slopes for H heads (attn_alibi_slopes: 2^(-8 h / H),
    h = 1..H) as a float32 tensor, moved to ``device`` when given."""
    buf = (ctypes.c_float * max(H, 1))()
    rc = int(load_library().attn_alibi_slopes(int(H), buf))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_alibi_slopes")
    t = torch.tensor(list(buf)[:H], dtype=torch.float32)
    return t if device is None else t.to(device)


def default_scale(d: int) -> float:
    """1/sqrt(d) rounded once to float32 (the "HEAD_DIM ** -0.5" of the Hands-On guide)."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float16:
        return ATTN_FP16
    raise TypeError(f"q/k/v must be bfloat16 or float16, got {t.dtype}")


def attn_fwd_raw(q, k, v, o, lse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                 stream) -> int:
    """Direct C-ABI call with integer pointers; returns the status code."""
    return int(load_library().attn_fwd(q, k, v, o, lse, B, H, H_kv, N, d, int(causal), window,
                                       n_sink, ctypes.c_float(scale), dtype, stream))


def attn_fwd_alibi_raw(q, k, v, o, lse, slopes, B, H, H_kv, N, d, causal, window, n_sink, scale,
                       dtype, stream) -> int:
    """Direct C-ABI call of attn_fwd_alibi with integer pointers; returns the status code."""
    return int(load_library().attn_fwd_alibi(q, k, v, o, lse, slopes, B, H, H_kv, N, d,
                                             int(causal), window, n_sink, ctypes.c_float(scale),
                                             dtype, stream))


def decode_workspace_bytes(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int) -> int:
    """Scratch bytes attn_decode needs for these sizes (0: the cache is not split)."""
    return int(load_library().attn_decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d))


def attn_decode_raw(q, k, v, o, lse, ws, ws_bytes, B, H, H_kv, N_q, N_kv, d, causal, window,
                    n_sink, scale, dtype, stream) -> int:
    """Direct C-ABI call of attn_decode with integer pointers; returns the status code."""
    return int(load_library().attn_decode(q, k, v, o, lse, ws, ctypes.c_longlong(ws_bytes), B, H,
                                          H_kv, N_q, N_kv, d, int(causal), window, n_sink,
                                          ctypes.c_float(scale), dtype, stream))


def attn_decode_noalloc_raw(q, k, v, o, lse, B, H, H_kv, N_q, N_kv, d, causal, window, n_sink,
                            scale, dtype, stream) -> int:
    """Direct C-ABI call of attn_decode_noalloc (static scratch); returns the status code."""
    return int(load_library().attn_decode_noalloc(q, k, v, o, lse, B, H, H_kv, N_q, N_kv, d,
                                                  int(causal), window, n_sink,
                                                  ctypes.c_float(scale), dtype, stream))


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = True,
           window: int = 0, n_sink: int = 0, scale: float | None = None, out_f32: bool = False,
           out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
           return_lse: bool = True, workspace: torch.Tensor | None = None):
    """Attention of the new query rows q [B, H, N_q, d] against the cache k, v
    [B, H_kv, N_kv, d] (attn_decode).  Query row i sits at cache position
    N_kv - N_q + i.  ``workspace``: a CUDA uint8 tensor of at least
    decode_workspace_bytes(...) bytes; allocated here (torch) when omitted.
    Returns (o [B, H, N_q, d], lse [B, H, N_q] or None)."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4 or k.shape != v.shape:
        raise ValueError("q [B, H, N_q, d] and k, v [B, H_kv, N_kv, d] expected")
    if q.shape[0] != k.shape[0] or q.shape[3] != k.shape[3]:
        raise ValueError(f"shape mismatch q={tuple(q.shape)} k={tuple(k.shape)}")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    B, H, N_q, d = q.shape
    H_kv, N_kv = k.shape[1], k.shape[2]
    if out is not None:
        _expect(out, "out", (B, H, N_q, d), torch.float32 if out_f32 else q.dtype, q.device)
    if lse is not None:
        _expect(lse, "lse", (B, H, N_q), torch.float32, q.device)
    if workspace is not None:
        _expect_workspace(workspace, q.device)
    if not q.is_cuda:
        raise ValueError("decode() takes CUDA tensors")
    if scale is None:
        scale = default_scale(d)
    code = _dtype_code(q) | (ATTN_OUT_F32 if out_f32 else 0)
    if out is None:
        out = torch.empty((B, H, N_q, d), dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = decode_workspace_bytes(B, H, H_kv, N_q, N_kv, d)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    stream = torch.cuda.current_stream(q.device).cuda_stream
    with _Device(q.device):
        rc = attn_decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr() if lse is not None else None, ws_ptr, ws_bytes, B, H,
                             H_kv, N_q, N_kv, d, causal, window, n_sink, scale, code, stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_decode")
    return out, lse


def bwd_workspace_bytes(B: int, H: int, N: int, d: int, dtype: int) -> int:
    """Scratch bytes attn_bwd needs (dtype: the status-style code incl. ATTN_OUT_F32)."""
    return int(load_library().attn_bwd_workspace_bytes(B, H, N, d, dtype))


def attn_bwd_raw(q, k, v, o, dout, lse, slopes, dq, dk, dv, ws, ws_bytes, B, H, H_kv, N, d,
                 causal, window, n_sink, scale, dtype, stream) -> int:
    """Direct C-ABI call of attn_bwd with integer pointers; returns the status code."""
    return int(load_library().attn_bwd(q, k, v, o, dout, lse, slopes, dq, dk, dv, ws,
                                       ctypes.c_longlong(ws_bytes), B, H, H_kv, N, d, int(causal),
                                       window, n_sink, ctypes.c_float(scale), dtype, stream))


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                       dout: torch.Tensor, lse: torch.Tensor, *, causal: bool = False,
                       window: int = 0, n_sink: int = 0, scale: float | None = None,
                       alibi_slopes: torch.Tensor | None = None, out_f32: bool = False,
                       workspace: torch.Tensor | None = None, grads=None):
    """dQ, dK, dV of attention()'s output for the upstream gradient ``dout``
    (attn_bwd).  ``o`` and ``dout`` are [B, H, N, d] in q's 16-bit dtype and
    ``lse`` the forward's float32 [B, H, N]; mask, scale and slopes must be
    those of the forward.  ``workspace``: CUDA uint8 tensor of at least
    bwd_workspace_bytes(...) bytes (allocated here with torch when omitted);
    ``grads``: optional preallocated (dq, dk, dv).  Returns (dq, dk, dv),
    float32 when ``out_f32``."""
    _check(q, k, v)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    for name, t in (("o", o), ("dout", dout)):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous [B, H, N, d] tensor like q")
    if (lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous()
            or lse.device != q.device):
        raise ValueError("lse must be a contiguous float32 [B, H, N] tensor on q's device")
    if alibi_slopes is not None:
        if (alibi_slopes.dtype != torch.float32 or alibi_slopes.device != q.device
                or tuple(alibi_slopes.shape) != (H,) or not alibi_slopes.is_contiguous()):
            raise ValueError("alibi_slopes must be a contiguous float32 [H] tensor on q's device")
    odt = torch.float32 if out_f32 else q.dtype
    if grads is not None:
        if len(grads) != 3:
            raise ValueError("grads must be (dq, dk, dv)")
        _expect(grads[0], "dq", (B, H, N, d), odt, q.device)
        _expect(grads[1], "dk", (B, H_kv, N, d), odt, q.device)
        _expect(grads[2], "dv", (B, H_kv, N, d), odt, q.device)
    if workspace is not None:
        _expect_workspace(workspace, q.device)
    if not q.is_cuda:
        raise ValueError("attention_backward() takes CUDA tensors")
    if scale is None:
        scale = default_scale(d)
    code = _dtype_code(q) | (ATTN_OUT_F32 if out_f32 else 0)
    if grads is None:
        dq = torch.empty((B, H, N, d), dtype=odt, device=q.device)
        dk = torch.empty((B, H_kv, N, d), dtype=odt, device=q.device)
        dv = torch.empty((B, H_kv, N, d), dtype=odt, device=q.device)
    else:
        dq, dk, dv = grads
    need = bwd_workspace_bytes(B, H, N, d, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    stream = torch.cuda.current_stream(q.device).cuda_stream
    with _Device(q.device):
        rc = attn_bwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                          lse.data_ptr(), alibi_slopes.data_ptr() if alibi_slopes is not None else None,
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws_ptr, ws_bytes, B, H,
                          H_kv, N, d, causal, window, n_sink, scale, code, stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return dq, dk, dv


class _Device:
    """Makes `dev` the current CUDA device for a library call; a no-op (no
    device switch) when it already is, the common case."""
    __slots__ = ("dev", "ctx")

    def __init__(self, dev):
        self.dev = dev
        self.ctx = None

    def __enter__(self):
        if self.dev.index is not None and self.dev.index != torch.cuda.current_device():
            self.ctx = torch.cuda.device(self.dev)
            self.ctx.__enter__()
        return self

    def __exit__(self, *exc):
        if self.ctx is not None:
            self.ctx.__exit__(*exc)
        return False


def _check(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, N, d] / [B, H_kv, N, d]")
    if k.shape != v.shape or q.shape[0] != k.shape[0] or q.shape[2:] != k.shape[2:]:
        raise ValueError(f"shape mismatch q={tuple(q.shape)} k={tuple(k.shape)} v={tuple(v.shape)}")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    _dtype_code(q)
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")


def _expect(t: torch.Tensor, name: str, shape, dtype, device=None):
    """Caller-provided buffers must match what the C ABI will write: it sizes
    every tensor from B, H, H_kv, N and d alone."""
    if (tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous()
            or (device is not None and t.device != device)):
        where = f" on {device}" if device is not None else ""
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}{where}, "
                         f"got {tuple(t.shape)} {t.dtype} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _expect_workspace(ws: torch.Tensor, device):
    if ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous() or ws.device != device:
        raise ValueError(f"workspace must be a contiguous 1-D uint8 tensor on {device}")


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
              window: int = 0, n_sink: int = 0, scale: float | None = None,
              out_f32: bool = False, out: torch.Tensor | None = None,
              lse: torch.Tensor | None = None, return_lse: bool = True,
              alibi_slopes: torch.Tensor | None = None):
    """O = softmax(scale * q k^T + mask) v and the per-row natural-log LSE.

    q: [B, H, N, d] CUDA bf16/fp16; k, v: [B, H_kv, N, d] (H % H_kv == 0).
    ``alibi_slopes``: optional float32 CUDA tensor [H]; the logits then get
    -slopes[h] * |i - j| added (attn_fwd_alibi).
    Returns (o, lse) with o [B, H, N, d] (float32 when ``out_f32``) and lse
    [B, H, N] float32 (None when ``return_lse`` is False).
    """
    _check(q, k, v)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if out is not None:
        _expect(out, "out", (B, H, N, d), torch.float32 if out_f32 else q.dtype, q.device)
    if lse is not None:
        _expect(lse, "lse", (B, H, N), torch.float32, q.device)
    if not q.is_cuda:
        raise ValueError("attention() takes CUDA tensors; use attention_from_host() for host tensors")
    if scale is None:
        scale = default_scale(d)
    code = _dtype_code(q) | (ATTN_OUT_F32 if out_f32 else 0)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    if alibi_slopes is not None:
        if (alibi_slopes.dtype != torch.float32 or alibi_slopes.device != q.device
                or tuple(alibi_slopes.shape) != (H,) or not alibi_slopes.is_contiguous()):
            raise ValueError("alibi_slopes must be a contiguous float32 [H] tensor on q's device")
    with _Device(q.device):
        if alibi_slopes is None:
            rc = attn_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              lse.data_ptr() if lse is not None else None, B, H, H_kv, N, d,
                              causal, window, n_sink, scale, code, stream)
        else:
            rc = attn_fwd_alibi_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr() if lse is not None else None,
                                    alibi_slopes.data_ptr(), B, H, H_kv, N, d, causal, window,
                                    n_sink, scale, code, stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd" if alibi_slopes is None else "attn_fwd_alibi")
    return out, lse


def attention_from_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, staging: dict,
                        out: torch.Tensor, lse: torch.Tensor | None = None, causal: bool = False,
                        window: int = 0, n_sink: int = 0, scale: float | None = None,
                        out_f32: bool = False, stream: torch.cuda.Stream | None = None):
    """Host-resident forward through ``attn_fwd_host``: copies in, computes, copies out.

    q, k, v, out, lse are CPU tensors (page-locked for asynchronous copies);
    ``staging`` holds device tensors "q", "k", "v", "o" and optionally "lse"
    of the matching shapes.  Enqueues on ``stream`` (default: current) and
    returns without synchronising.
    """
    _check(q, k, v)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    odt = torch.float32 if out_f32 else q.dtype
    cpu = torch.device("cpu")
    _expect(out, "out", (B, H, N, d), odt, cpu)
    if lse is not None:
        _expect(lse, "lse", (B, H, N), torch.float32, cpu)
        if staging.get("lse") is None:
            raise ValueError("staging needs an 'lse' tensor when lse is requested")
    dev = staging["q"].device
    _expect(staging["q"], "staging['q']", q.shape, q.dtype, dev)
    _expect(staging["k"], "staging['k']", k.shape, k.dtype, dev)
    _expect(staging["v"], "staging['v']", v.shape, v.dtype, dev)
    _expect(staging["o"], "staging['o']", (B, H, N, d), odt, dev)
    if staging.get("lse") is not None:
        _expect(staging["lse"], "staging['lse']", (B, H, N), torch.float32, dev)
    if dev.type != "cuda":
        raise ValueError("staging tensors must be CUDA tensors")
    if scale is None:
        scale = default_scale(d)
    code = _dtype_code(q) | (ATTN_OUT_F32 if out_f32 else 0)
    s = (stream or torch.cuda.current_stream(dev)).cuda_stream
    dl = staging.get("lse")
    with _Device(dev):
        rc = int(load_library().attn_fwd_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
            lse.data_ptr() if lse is not None else None,
            staging["q"].data_ptr(), staging["k"].data_ptr(), staging["v"].data_ptr(),
            staging["o"].data_ptr(), dl.data_ptr() if dl is not None else None,
            B, H, H_kv, N, d, int(causal), window, n_sink, ctypes.c_float(scale), code, s))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_host")
    return out, lse
