"""Plain fp64 CPU oracle for the gated delta rule decode step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never imports, links or calls it, and the two share no code.

The arithmetic lives in ``gdn_oracle.c`` (double precision, sequential, the
definition written out; see its header for the definition and its sources).
This module only compiles it with gcc and marshals numpy float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

SLOT_RANGE = 2  # return code for a slot outside [-1, n_slots)

_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle.so`` (strict IEEE fp64)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        d, i, p = ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        for name in ("oracle_sigmoid", "oracle_softplus", "oracle_silu"):
            getattr(lib, name).restype = d
            getattr(lib, name).argtypes = [d]
        lib.oracle_gate_g.restype = d
        lib.oracle_gate_g.argtypes = [d, d, d]
        lib.oracle_conv4.restype = d
        lib.oracle_conv4.argtypes = [p, d, p]
        lib.oracle_l2norm.restype = None
        lib.oracle_l2norm.argtypes = [p, i, d, p]
        lib.oracle_gated_rmsnorm.restype = None
        lib.oracle_gated_rmsnorm.argtypes = [p, p, p, i, d, p]
        lib.oracle_gdn_token.restype = None
        lib.oracle_gdn_token.argtypes = [p, i, i, p, p, p, d, d, d, p]
        lib.oracle_decode_step.restype = i
        lib.oracle_decode_step.argtypes = [p] * 8 + [i] * 7 + [d, i, d, i]
        lib.oracle_decode_step_spec.restype = i
        lib.oracle_decode_step_spec.argtypes = [p] * 10 + [i] * 7 + [d, i, d, i]
        lib.oracle_prefill.restype = i
        lib.oracle_prefill.argtypes = [p] * 9 + [i] * 6 + [d, i, d, i, i]
        lib.oracle_lowrank_decode_step.restype = i
        lib.oracle_lowrank_decode_step.argtypes = [p] * 11 + [i] * 8 + [d, i, d]
        lib.oracle_lowrank_prefill.restype = i
        lib.oracle_lowrank_prefill.argtypes = [p] * 12 + [i] * 7 + [d, i, d, i]
        lib.oracle_round_to.restype = d
        lib.oracle_round_to.argtypes = [d, i, i, d]
        lib.oracle_round_storage.restype = d
        lib.oracle_round_storage.argtypes = [d, i]
        lib.oracle_fused_step.restype = i
        lib.oracle_fused_step.argtypes = [p] * 9 + [d, p, p, p] + [i] * 6 + [d, d]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---- scalar and vector pieces (exported so the tests can pin each) --------

def sigmoid(x: float) -> float:
    return _load().oracle_sigmoid(float(x))


def softplus(x: float) -> float:
    return _load().oracle_softplus(float(x))


def silu(x: float) -> float:
    return _load().oracle_silu(float(x))


def gate_g(a: float, A_log: float, dt_bias: float) -> float:
    return _load().oracle_gate_g(float(a), float(A_log), float(dt_bias))


def conv4(cs, x: float, w) -> float:
    cs, w = _f64(cs), _f64(w)
    assert cs.size == 3 and w.size == 4
    return _load().oracle_conv4(_ptr(cs), float(x), _ptr(w))


def l2norm(x, eps: float = 0.0) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _load().oracle_l2norm(_ptr(x), x.size, float(eps), _ptr(y))
    return y


def gated_rmsnorm(o, z, w, eps: float = 0.0) -> np.ndarray:
    o, z, w = _f64(o), _f64(z), _f64(w)
    y = np.empty_like(o)
    _load().oracle_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(w), o.size, float(eps), _ptr(y))
    return y


def gdn_token(S, q, k, v, alpha: float, beta: float, scale: float):
    """One token on one head.  ``S`` is the storage layout [dv][dk] and is
    updated in place; returns o [dv]."""
    assert S.dtype == np.float64 and S.flags.c_contiguous
    dv, dk = S.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.empty(dv, dtype=np.float64)
    _load().oracle_gdn_token(_ptr(S), dk, dv, _ptr(q), _ptr(k), _ptr(v),
                             float(alpha), float(beta), float(scale), _ptr(o))
    return o


STORAGE = {None: 0, "fp64": 0, "fp32": 1, "bf16": 2, "fp16": 3}


def round_storage(x: float, kind: str) -> float:
    """Round to the nearest value of a storage format ("fp32", "bf16",
    "fp16"), ties to even."""
    return _load().oracle_round_storage(float(x), STORAGE[kind])


def round_to(x: float, p: int, emin: int, maxv: float) -> float:
    return _load().oracle_round_to(float(x), int(p), int(emin), float(maxv))


# ---- the batched steps ------------------------------------------------------

def decode_step(q, k, v, g, beta, state: np.ndarray, slot_idx, *, scale=None,
                qk_l2norm: bool = True, eps: float = 1e-6, state_round=None):
    """Batched decode step.  Shapes: q, k [B,T,Hk,dk]; v [B,T,H,dv];
    g, beta [B,T,H]; state [n_slots,H,dv,dk] float64, updated in place and,
    if ``state_round`` names a storage format ("fp32", "bf16", "fp16"),
    rounded to it once at the end of the call; slot_idx [B] int.
    Returns (out [B,T,H,dv] float64, return code)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    assert state.dtype == np.float64 and state.flags.c_contiguous
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    n_slots = state.shape[0]
    assert state.shape == (n_slots, H, dv, dk)
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().oracle_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(slots),
        _ptr(out), B, T, Hk, H, dk, dv, n_slots, float(scale), int(bool(qk_l2norm)),
        float(eps), STORAGE[state_round])
    return out, rc


ACCEPT_RANGE = 4  # return bit for an n_accept entry outside [0, T]


def decode_step_spec(q, k, v, g, beta, state: np.ndarray, slot_idx, *, n_accept=None,
                     token_slots=None, scale=None, qk_l2norm: bool = True, eps: float = 1e-6,
                     state_round=None):
    """Decode step with accept-length commit (``n_accept`` [B]) or per-token
    snapshots into pool slots (``token_slots`` [B,T]); see gdn_oracle.c.
    Returns (out [B,T,H,dv] float64, return code bits)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    assert state.dtype == np.float64 and state.flags.c_contiguous
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    n_slots = state.shape[0]
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    na = None if n_accept is None else np.ascontiguousarray(np.asarray(n_accept, dtype=np.int32))
    tsl = (None if token_slots is None
           else np.ascontiguousarray(np.asarray(token_slots, dtype=np.int32)))
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().oracle_decode_step_spec(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(slots),
        None if na is None else _ptr(na), None if tsl is None else _ptr(tsl), _ptr(out),
        B, T, Hk, H, dk, dv, n_slots, float(scale), int(bool(qk_l2norm)), float(eps),
        STORAGE[state_round])
    return out, rc


def prefill(q, k, v, g, beta, state: np.ndarray, slot_idx, cu_seqlens, *, scale=None,
            qk_l2norm: bool = True, eps: float = 1e-6, initial_state: bool = True,
            state_round=None):
    """Prefill over packed variable-length sequences (see gdn_oracle.c).
    q, k [total,Hk,dk]; v [total,H,dv]; g, beta [total,H]; state
    [n_slots,H,dv,dk] float64 (final states stored in place); slot_idx [N];
    cu_seqlens [N+1].  Returns (out [total,H,dv] float64, return code)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    assert state.dtype == np.float64 and state.flags.c_contiguous
    total, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    N = slots.size
    assert cu.size == N + 1 and cu[-1] <= total
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((total, H, dv), dtype=np.float64)
    rc = _load().oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(slots), _ptr(cu),
        _ptr(out), N, Hk, H, dk, dv, state.shape[0], float(scale), int(bool(qk_l2norm)),
        float(eps), int(bool(initial_state)), STORAGE[state_round])
    return out, rc


def lowrank_decode_step(q, k, v, g, beta, win_k: np.ndarray, win_u: np.ndarray,
                        win_c: np.ndarray, win_count: np.ndarray, slot_idx, *, scale=None,
                        qk_l2norm: bool = True, eps: float = 1e-6):
    """Low-rank sliding-window decode step (see gdn_oracle.c).  win_k
    [n_slots,H,R,dk], win_u [n_slots,H,R,dv], win_c [n_slots,H,R] float64 and
    win_count [n_slots,H] int32 are updated in place.
    Returns (out [B,T,H,dv] float64, return code)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    for a in (win_k, win_u, win_c):
        assert a.dtype == np.float64 and a.flags.c_contiguous
    assert win_count.dtype == np.int32 and win_count.flags.c_contiguous
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    n_slots, _, R, _ = win_k.shape
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().oracle_lowrank_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(win_k), _ptr(win_u), _ptr(win_c),
        _ptr(win_count), _ptr(slots), _ptr(out), B, T, Hk, H, dk, dv, R, n_slots, float(scale),
        int(bool(qk_l2norm)), float(eps))
    return out, rc


def lowrank_prefill(q, k, v, g, beta, win_k: np.ndarray, win_u: np.ndarray, win_c: np.ndarray,
                    win_count: np.ndarray, slot_idx, cu_seqlens, *, scale=None,
                    qk_l2norm: bool = True, eps: float = 1e-6, initial_window: bool = True):
    """Low-rank window over packed prompts (see gdn_oracle.c): q, k
    [total,Hk,dk]; v [total,H,dv]; g, beta [total,H]; the window arrays as in
    lowrank_decode_step (updated in place); slot_idx [N]; cu_seqlens [N+1].
    Returns (out [total,H,dv] float64, return code)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    for a in (win_k, win_u, win_c):
        assert a.dtype == np.float64 and a.flags.c_contiguous
    assert win_count.dtype == np.int32 and win_count.flags.c_contiguous
    total, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    n_slots, _, R, _ = win_k.shape
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    N = slots.size
    assert cu.size == N + 1 and cu[-1] <= total
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((total, H, dv), dtype=np.float64)
    rc = _load().oracle_lowrank_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(win_k), _ptr(win_u), _ptr(win_c),
        _ptr(win_count), _ptr(slots), _ptr(cu), _ptr(out), N, Hk, H, dk, dv, R, n_slots,
        float(scale), int(bool(qk_l2norm)), float(eps), int(bool(initial_window)))
    return out, rc


def fused_step(mixed_x, conv_state: np.ndarray, conv_w, a, b, A_log, dt_bias, z,
               norm_w, state: np.ndarray, slot_idx, *, Hk: int, H: int, dk: int,
               dv: int, norm_eps: float = 1e-6, scale=None, l2_eps: float = 1e-6):
    """Fused conv + gates + recurrence + gated RMSNorm, T = 1.
    mixed_x [B,C]; conv_state [n_slots,C,3] float64 (updated in place);
    conv_w [C,4]; a, b [B,H]; A_log, dt_bias [H]; z [B,H*dv]; norm_w [dv];
    state [n_slots,H,dv,dk] float64 (updated in place).
    Returns (out [B,H,dv] float64, return code)."""
    mixed_x, conv_w, a, b, A_log, dt_bias, z, norm_w = (
        _f64(x) for x in (mixed_x, conv_w, a, b, A_log, dt_bias, z, norm_w))
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert state.dtype == np.float64 and state.flags.c_contiguous
    B = mixed_x.shape[0]
    n_slots = state.shape[0]
    assert mixed_x.shape[1] == 2 * Hk * dk + H * dv
    slots = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().oracle_fused_step(
        _ptr(mixed_x), _ptr(conv_state), _ptr(conv_w), _ptr(a), _ptr(b), _ptr(A_log),
        _ptr(dt_bias), _ptr(z), _ptr(norm_w), float(norm_eps), _ptr(state), _ptr(slots),
        _ptr(out), B, Hk, H, dk, dv, n_slots, float(scale), float(l2_eps))
    return out, rc
