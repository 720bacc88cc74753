"""B200 (sm_100a) gated delta rule decode library: thin Python binding.

Every step of the computation runs in the CUDA kernels of ``libgdn.so``
(see ``include/gdn.h``); this module only marshals torch tensors (device
memory and the current stream) into the C ABI through ctypes.  There is no
CPU fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB_PATH, build_library

__all__ = [
    "GdnError", "load_library", "decode_step", "decode_step_ex", "fused_decode_step",
    "get_error", "last_error_string", "version", "F32", "BF16", "F16", "STATUS_SLOT_RANGE",
    "STATUS_ACCEPT_RANGE", "STATUS_SEQ_RANGE", "EXPORTED_SYMBOLS", "chunk_prefill",
    "chunk_prefill_noalloc", "prefill_workspace_size", "lowrank_decode_step", "lowrank_prefill",
]

F32, BF16, F16 = 0, 1, 2
OK, ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_SLOT_RANGE, ERR_SLOT_DUP = 0, -1, -2, -3, -4, -5
ERR_ACCEPT_RANGE, ERR_SEQ_RANGE, ERR_TIMEOUT = -6, -7, -8
STATUS_SLOT_RANGE = 0x1
STATUS_ACCEPT_RANGE = 0x2
STATUS_SEQ_RANGE = 0x4
STATUS_TIMEOUT = 0x8

EXPORTED_SYMBOLS = (
    "gdn_decode_step", "gdn_decode_step_ex", "gdn_fused_decode_step", "gdn_chunk_prefill",
    "gdn_chunk_prefill_noalloc", "gdn_prefill_workspace_size", "gdn_prefill_workspace_size_ex",
    "gdn_lowrank_decode_step", "gdn_lowrank_prefill",
    "gdn_get_error", "gdn_last_error_string", "gdn_version",
)


class GdnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"gdn error {code}: {message}")
        self.code = code


class StepArgs(ctypes.Structure):
    """Mirror of ``gdn_step_args`` in include/gdn.h (field order matters)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("state", ctypes.c_void_p),
        ("slot_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hk", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int),
        ("dv", ctypes.c_int), ("T", ctypes.c_int), ("n_slots", ctypes.c_int),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("state_dtype", ctypes.c_int),
        ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int), ("l2_eps", ctypes.c_float),
        ("dev_status", ctypes.c_void_p), ("check_slots", ctypes.c_int),
        ("n_accept", ctypes.c_void_p), ("token_slots", ctypes.c_void_p),
        ("stream", ctypes.c_void_p),
    ]


class PrefillArgs(ctypes.Structure):
    """Mirror of ``gdn_prefill_args`` in include/gdn.h (field order matters)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("state", ctypes.c_void_p),
        ("slot_idx", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("N", ctypes.c_int), ("total_tokens", ctypes.c_int), ("Hk", ctypes.c_int),
        ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("n_slots", ctypes.c_int),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int), ("l2_eps", ctypes.c_float),
        ("initial_state", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("dev_status", ctypes.c_void_p), ("stream", ctypes.c_void_p),
    ]


class LowrankArgs(ctypes.Structure):
    """Mirror of ``gdn_lowrank_args`` in include/gdn.h (field order matters)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("win_k", ctypes.c_void_p),
        ("win_u", ctypes.c_void_p), ("win_c", ctypes.c_void_p), ("win_count", ctypes.c_void_p),
        ("slot_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hk", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int),
        ("dv", ctypes.c_int), ("T", ctypes.c_int), ("R", ctypes.c_int), ("n_slots", ctypes.c_int),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int), ("l2_eps", ctypes.c_float),
        ("dev_status", ctypes.c_void_p), ("stream", ctypes.c_void_p),
    ]


class LowrankPrefillArgs(ctypes.Structure):
    """Mirror of ``gdn_lowrank_prefill_args`` in include/gdn.h (field order matters)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("win_k", ctypes.c_void_p),
        ("win_u", ctypes.c_void_p), ("win_c", ctypes.c_void_p), ("win_count", ctypes.c_void_p),
        ("slot_idx", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("N", ctypes.c_int), ("total_tokens", ctypes.c_int), ("Hk", ctypes.c_int),
        ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("R", ctypes.c_int),
        ("n_slots", ctypes.c_int), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int), ("l2_eps", ctypes.c_float),
        ("initial_window", ctypes.c_int), ("dev_status", ctypes.c_void_p),
        ("stream", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load ``libgdn.so`` (building the in-tree one first if it is missing and
    nvcc is available).  The environment variable ``GDN_LIBRARY`` names
    another build of the library to load instead.  Raises if it cannot be
    loaded."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or os.environ.get("GDN_LIBRARY") or LIB_PATH
    if p == LIB_PATH and not os.path.exists(p):
        build_library()
    lib = ctypes.CDLL(p)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.gdn_decode_step.restype = i
    lib.gdn_decode_step.argtypes = [vp] * 8 + [i] * 5 + [vp]
    lib.gdn_decode_step_ex.restype = i
    lib.gdn_decode_step_ex.argtypes = [ctypes.POINTER(StepArgs)]
    lib.gdn_fused_decode_step.restype = i
    lib.gdn_fused_decode_step.argtypes = ([vp, vp, vp, i, vp, vp, vp, vp, vp, vp, f, vp, vp, vp]
                                          + [i] * 6 + [i, vp, vp])
    lib.gdn_chunk_prefill.restype = i
    lib.gdn_chunk_prefill.argtypes = [ctypes.POINTER(PrefillArgs)]
    lib.gdn_chunk_prefill_noalloc.restype = i
    lib.gdn_chunk_prefill_noalloc.argtypes = [ctypes.POINTER(PrefillArgs)]
    lib.gdn_prefill_workspace_size.restype = ctypes.c_size_t
    lib.gdn_prefill_workspace_size.argtypes = [i] * 5
    lib.gdn_prefill_workspace_size_ex.restype = ctypes.c_size_t
    lib.gdn_prefill_workspace_size_ex.argtypes = [i] * 6
    lib.gdn_lowrank_decode_step.restype = i
    lib.gdn_lowrank_decode_step.argtypes = [ctypes.POINTER(LowrankArgs)]
    lib.gdn_lowrank_prefill.restype = i
    lib.gdn_lowrank_prefill.argtypes = [ctypes.POINTER(LowrankPrefillArgs)]
    lib.gdn_get_error.restype = i
    lib.gdn_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.gdn_last_error_string.restype = ctypes.c_char_p
    lib.gdn_last_error_string.argtypes = []
    lib.gdn_version.restype = i
    lib.gdn_version.argtypes = []
    if path is None:
        _lib = lib
    return lib


def _check(rc: int) -> None:
    if rc != OK:
        msg = load_library().gdn_last_error_string()
        raise GdnError(rc, msg.decode() if msg else "")


def last_error_string() -> str:
    msg = load_library().gdn_last_error_string()
    return msg.decode() if msg else ""


def version() -> int:
    return load_library().gdn_version()


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def decode_step(q, k, v, g, beta, state, slot_idx, out=None, *, stream=None):
    """``gdn_decode_step``: bf16 q/k/v [B,T,H,dk|dv], fp32 g/beta [B,T,H],
    fp32 state pool [n_slots,H,dv,dk] (in place), int32 slot_idx [B].
    Returns out fp32 [B,T,H,dv]."""
    torch = _torch()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if state.dtype != torch.float32:
        raise TypeError("gdn_decode_step takes an fp32 state pool; use decode_step_ex")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    rc = load_library().gdn_decode_step(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(state, "state"), _dev(slot_idx, "slot_idx"), _dev(out, "out"),
        B, H, dk, dv, T, _stream(stream))
    _check(rc)
    return out


def decode_step_ex(q, k, v, g, beta, state, slot_idx, out=None, *, scale: float = 0.0,
                   qk_l2norm: bool = True, l2_eps: float = 1e-6, out_dtype=None,
                   dev_status=None, check_slots: bool = False, n_slots: int | None = None,
                   n_accept=None, token_slots=None, stream=None):
    """``gdn_decode_step_ex``: q, k [B,T,Hk,dk]; v [B,T,H,dv] (both fp32 or
    both bf16); g, beta fp32 [B,T,H]; state [n_slots,H,dv,dk] of fp32, bf16
    or fp16 (in place; its dtype selects the state storage type); slot_idx
    int32 [B]; out [B,T,H,dv] of ``out_dtype`` (default fp32).
    ``n_slots`` defaults to ``state.shape[0]``; pass 0 for "unknown".
    Speculative decoding: ``n_accept`` int32 [B] commits the state after the
    first n_accept[b] tokens (0: nothing written); ``token_slots`` int32
    [B,T] stores the state after every token in those pool slots instead."""
    torch = _torch()
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    a = StepArgs()
    a.q, a.k, a.v = _dev(q, "q"), _dev(k, "k"), _dev(v, "v")
    a.g, a.beta = _dev(g, "g"), _dev(beta, "beta")
    a.state, a.slot_idx, a.out = _dev(state, "state"), _dev(slot_idx, "slot_idx"), _dev(out, "out")
    a.B, a.Hk, a.H, a.dk, a.dv, a.T = B, Hk, H, dk, dv, T
    a.n_slots = state.shape[0] if n_slots is None else int(n_slots)
    a.in_dtype = _dtype_code(q)
    if _dtype_code(k) != a.in_dtype or _dtype_code(v) != a.in_dtype:
        raise TypeError("q, k and v must share one dtype")
    a.out_dtype = _dtype_code(out)
    a.state_dtype = _dtype_code(state)
    a.scale = float(scale)
    a.qk_l2norm = 1 if qk_l2norm else 0
    a.l2_eps = float(l2_eps)
    a.dev_status = _dev(dev_status, "dev_status") if dev_status is not None else None
    a.check_slots = 1 if check_slots else 0
    a.n_accept = _dev(n_accept, "n_accept") if n_accept is not None else None
    a.token_slots = _dev(token_slots, "token_slots") if token_slots is not None else None
    a.stream = _stream(stream)
    _check(load_library().gdn_decode_step_ex(ctypes.byref(a)))
    return out


def fused_decode_step(mixed_x, conv_state, conv_w, a, b, A_log, dt_bias, z, norm_w, state,
                      slot_idx, out=None, *, Hk: int, H: int, dk: int, dv: int,
                      norm_eps: float = 1e-6, out_dtype=None, dev_status=None, stream=None):
    """``gdn_fused_decode_step`` (T = 1): mixed_x bf16 [B,C]; conv_state bf16
    [n_slots,C,3] (in place); conv_w [C,4] fp32 or bf16; a, b bf16 [B,H];
    A_log, dt_bias fp32 [H]; z bf16 [B,H*dv]; norm_w fp32 [dv]; state fp32
    [n_slots,H,dv,dk] (in place); slot_idx int32 [B].  Returns out [B,H,dv]."""
    torch = _torch()
    B = mixed_x.shape[0]
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype or torch.float32, device=mixed_x.device)
    rc = load_library().gdn_fused_decode_step(
        _dev(mixed_x, "mixed_x"), _dev(conv_state, "conv_state"), _dev(conv_w, "conv_w"),
        _dtype_code(conv_w), _dev(a, "a"), _dev(b, "b"), _dev(A_log, "A_log"),
        _dev(dt_bias, "dt_bias"), _dev(z, "z"), _dev(norm_w, "norm_w"), float(norm_eps),
        _dev(state, "state"), _dev(slot_idx, "slot_idx"), _dev(out, "out"),
        B, Hk, H, dk, dv, state.shape[0], _dtype_code(out),
        _dev(dev_status, "dev_status") if dev_status is not None else None, _stream(stream))
    _check(rc)
    return out


def prefill_workspace_size(N: int, total_tokens: int, H: int, dk: int, dv: int,
                           in_dtype=None) -> int:
    """Bytes of scratch a prefill call needs: ``gdn_prefill_workspace_size_ex``
    for inputs of ``in_dtype`` (a torch dtype), or, without it,
    ``gdn_prefill_workspace_size`` (enough for either input dtype)."""
    lib = load_library()
    if in_dtype is None:
        return int(lib.gdn_prefill_workspace_size(N, total_tokens, H, dk, dv))
    torch = _torch()
    code = {torch.float32: F32, torch.bfloat16: BF16}[in_dtype]
    return int(lib.gdn_prefill_workspace_size_ex(N, total_tokens, H, dk, dv, code))


def chunk_prefill(q, k, v, g, beta, state, slot_idx, cu_seqlens, out=None, *, workspace=None,
                  initial_state: bool = True, scale: float = 0.0, qk_l2norm: bool = True,
                  l2_eps: float = 1e-6, out_dtype=None, dev_status=None, stream=None,
                  _noalloc: bool = False):
    """``gdn_chunk_prefill``: q, k [total,Hk,dk]; v [total,H,dv] (fp32 or
    bf16); g, beta fp32 [total,H]; state fp32 [n_slots,H,dv,dk] (final states
    stored in place); slot_idx int32 [N]; cu_seqlens int32 [N+1] on the
    device.  ``workspace`` is a device byte buffer of at least
    prefill_workspace_size(...) bytes (allocated here when not given).
    Returns out [total,H,dv]."""
    torch = _torch()
    total, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    N = slot_idx.shape[0]
    if out is None:
        out = torch.zeros((total, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    if not _noalloc and workspace is None:
        need = prefill_workspace_size(N, total, H, dk, dv, q.dtype)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    a = PrefillArgs()
    a.q, a.k, a.v = _dev(q, "q"), _dev(k, "k"), _dev(v, "v")
    a.g, a.beta = _dev(g, "g"), _dev(beta, "beta")
    a.state, a.slot_idx = _dev(state, "state"), _dev(slot_idx, "slot_idx")
    a.cu_seqlens, a.out = _dev(cu_seqlens, "cu_seqlens"), _dev(out, "out")
    a.N, a.total_tokens, a.Hk, a.H, a.dk, a.dv = N, total, Hk, H, dk, dv
    a.n_slots = state.shape[0]
    a.in_dtype = _dtype_code(q)
    if _dtype_code(k) != a.in_dtype or _dtype_code(v) != a.in_dtype:
        raise TypeError("q, k and v must share one dtype")
    a.out_dtype = _dtype_code(out)
    a.scale, a.qk_l2norm, a.l2_eps = float(scale), 1 if qk_l2norm else 0, float(l2_eps)
    a.initial_state = 1 if initial_state else 0
    if _noalloc:
        a.workspace, a.workspace_bytes = None, 0
    else:
        a.workspace = _dev(workspace, "workspace")
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.dev_status = _dev(dev_status, "dev_status") if dev_status is not None else None
    a.stream = _stream(stream)
    lib = load_library()
    _check(lib.gdn_chunk_prefill_noalloc(ctypes.byref(a)) if _noalloc
           else lib.gdn_chunk_prefill(ctypes.byref(a)))
    return out


def chunk_prefill_noalloc(q, k, v, g, beta, state, slot_idx, cu_seqlens, out=None, **kw):
    """``gdn_chunk_prefill_noalloc``: chunk_prefill without a workspace; the
    library's built-in 64 MiB device scratch is used instead (see
    include/gdn.h for the limit and for calls that overlap on the GPU).
    ``out`` must be given by callers that cannot allocate."""
    kw.pop("workspace", None)
    return chunk_prefill(q, k, v, g, beta, state, slot_idx, cu_seqlens, out, _noalloc=True, **kw)


def lowrank_decode_step(q, k, v, g, beta, win_k, win_u, win_c, win_count, slot_idx, out=None, *,
                        scale: float = 0.0, qk_l2norm: bool = True, l2_eps: float = 1e-6,
                        out_dtype=None, dev_status=None, stream=None):
    """``gdn_lowrank_decode_step``: q, k [B,T,Hk,dk]; v [B,T,H,dv]; g, beta
    fp32 [B,T,H]; window win_k fp32 [n_slots,H,R,dk], win_u [n_slots,H,R,dv],
    win_c [n_slots,H,R], win_count int32 [n_slots,H] (all in place);
    slot_idx int32 [B].  Returns out [B,T,H,dv]."""
    torch = _torch()
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    n_slots, _, R, _ = win_k.shape
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    a = LowrankArgs()
    a.q, a.k, a.v = _dev(q, "q"), _dev(k, "k"), _dev(v, "v")
    a.g, a.beta = _dev(g, "g"), _dev(beta, "beta")
    a.win_k, a.win_u = _dev(win_k, "win_k"), _dev(win_u, "win_u")
    a.win_c, a.win_count = _dev(win_c, "win_c"), _dev(win_count, "win_count")
    a.slot_idx, a.out = _dev(slot_idx, "slot_idx"), _dev(out, "out")
    a.B, a.Hk, a.H, a.dk, a.dv, a.T, a.R, a.n_slots = B, Hk, H, dk, dv, T, R, n_slots
    a.in_dtype = _dtype_code(q)
    if _dtype_code(k) != a.in_dtype or _dtype_code(v) != a.in_dtype:
        raise TypeError("q, k and v must share one dtype")
    a.out_dtype = _dtype_code(out)
    a.scale, a.qk_l2norm, a.l2_eps = float(scale), 1 if qk_l2norm else 0, float(l2_eps)
    a.dev_status = _dev(dev_status, "dev_status") if dev_status is not None else None
    a.stream = _stream(stream)
    _check(load_library().gdn_lowrank_decode_step(ctypes.byref(a)))
    return out


def lowrank_prefill(q, k, v, g, beta, win_k, win_u, win_c, win_count, slot_idx, cu_seqlens,
                    out=None, *, initial_window: bool = True, scale: float = 0.0,
                    qk_l2norm: bool = True, l2_eps: float = 1e-6, out_dtype=None,
                    dev_status=None, stream=None):
    """``gdn_lowrank_prefill``: q, k [total,Hk,dk]; v [total,H,dv] (fp32 or
    bf16); g, beta fp32 [total,H]; the window as in lowrank_decode_step (in
    place); slot_idx int32 [N]; cu_seqlens int32 [N+1] on the device.
    Returns out [total,H,dv]."""
    torch = _torch()
    total, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    n_slots, _, R, _ = win_k.shape
    if out is None:
        out = torch.zeros((total, H, dv), dtype=out_dtype or torch.float32, device=q.device)
    a = LowrankPrefillArgs()
    a.q, a.k, a.v = _dev(q, "q"), _dev(k, "k"), _dev(v, "v")
    a.g, a.beta = _dev(g, "g"), _dev(beta, "beta")
    a.win_k, a.win_u = _dev(win_k, "win_k"), _dev(win_u, "win_u")
    a.win_c, a.win_count = _dev(win_c, "win_c"), _dev(win_count, "win_count")
    a.slot_idx, a.cu_seqlens = _dev(slot_idx, "slot_idx"), _dev(cu_seqlens, "cu_seqlens")
    a.out = _dev(out, "out")
    a.N, a.total_tokens, a.Hk, a.H, a.dk, a.dv = slot_idx.shape[0], total, Hk, H, dk, dv
    a.R, a.n_slots = R, n_slots
    a.in_dtype = _dtype_code(q)
    if _dtype_code(k) != a.in_dtype or _dtype_code(v) != a.in_dtype:
        raise TypeError("q, k and v must share one dtype")
    a.out_dtype = _dtype_code(out)
    a.scale, a.qk_l2norm, a.l2_eps = float(scale), 1 if qk_l2norm else 0, float(l2_eps)
    a.initial_window = 1 if initial_window else 0
    a.dev_status = _dev(dev_status, "dev_status") if dev_status is not None else None
    a.stream = _stream(stream)
    _check(load_library().gdn_lowrank_prefill(ctypes.byref(a)))
    return out


def get_error(dev_status) -> tuple[int, int]:
    """``gdn_get_error``: returns (status code, raw bits) of a device status word."""
    bits = ctypes.c_int(0)
    rc = load_library().gdn_get_error(_dev(dev_status, "dev_status"), ctypes.byref(bits))
    return rc, bits.value
