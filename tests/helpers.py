"""Shared helpers of the GPU parity tests: running the oracle on the same
seeded inputs and the tolerances of the comparison.

Tolerances (from the acceptance bar of the decode step):
  * outputs: max |o_gpu - o_ref| <= 2e-3 * rms(o_ref) over each call's
    output tensor, for bf16 (and fp32) inputs with fp32 outputs;
  * state: per (slot, head) ||S_gpu - S_ref||_F / ||S_ref||_F <= 1e-4,
    including after 64 consecutive steps;
  * bf16 outputs add the storage rounding of the output itself,
    2^-8 * |o_ref| (half an ulp of an 8-bit significand).
"""
import numpy as np
import torch

import oracle

O_TOL = 2e-3
STATE_TOL = 1e-4


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).contiguous().numpy()


def oracle_decode(inp: dict, *, scale=None, qk_l2norm=True, eps=1e-6, state=None):
    """Run the oracle on the (host copies of the) exact inputs the GPU gets.
    Returns (out, state_after) as float64 arrays."""
    st = f64(inp["state"] if state is None else state).copy()
    out, rc = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                 f64(inp["beta"]), st, inp["slot_idx"].cpu().numpy(),
                                 scale=scale, qk_l2norm=qk_l2norm, eps=eps)
    return out, st, rc


def assert_out_close(o_gpu: torch.Tensor, o_ref: np.ndarray, bf16_out: bool = False):
    og = f64(o_gpu)
    rms = float(np.sqrt(np.mean(o_ref * o_ref)))
    err = np.abs(og - o_ref)
    bound = O_TOL * rms + (2.0 ** -8) * np.abs(o_ref) if bf16_out else O_TOL * rms
    worst = float((err - bound).max()) if err.size else 0.0
    assert worst <= 0.0, f"max |do| = {err.max():.3e} vs bound {O_TOL}*rms = {O_TOL * rms:.3e}"
    return float(err.max() / rms) if rms > 0 else 0.0


def state_rel_err(s_gpu: np.ndarray, s_ref: np.ndarray) -> float:
    """max over (slot, head) of ||dS||_F / ||S_ref||_F; arrays [..., dv, dk]."""
    d = (s_gpu - s_ref).reshape(-1, s_ref.shape[-2] * s_ref.shape[-1])
    r = s_ref.reshape(-1, s_ref.shape[-2] * s_ref.shape[-1])
    num = np.sqrt((d * d).sum(axis=1))
    den = np.sqrt((r * r).sum(axis=1))
    return float((num / np.maximum(den, 1e-300)).max()) if num.size else 0.0


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: v.to(device).contiguous() for k, v in inp.items()}


# significand bits and smallest normal exponent of the 16-bit state formats
STORAGE_FORMAT = {"bf16": (8, -126), "fp16": (11, -14)}
# one unit in the last place, relative: 2^(1-p)
STORAGE_U = {"bf16": 2.0 ** -7, "fp16": 2.0 ** -10}


def storage_ulp(x: np.ndarray, kind: str) -> np.ndarray:
    """Spacing of the storage format at |x| (subnormal spacing below the
    smallest normal)."""
    p, emin = STORAGE_FORMAT[kind]
    _, e = np.frexp(np.abs(x))
    E = np.maximum(e - 1, emin)
    return np.ldexp(1.0, E - p + 1)


GUARD_BYTES = 4096
GUARD_FILL = 0xA7  # an arbitrary byte value; as fp32/bf16 it is a large negative number


class Guarded:
    """A device tensor with GUARD_BYTES of sentinel bytes on each side.

    Stands in for a memory checker: a kernel that writes past either end of
    the tensor changes a sentinel, and check() says which side and where.
    The tensor itself starts at a 256-byte boundary (the allocator's
    alignment plus the guard size), as any caller's allocation would."""

    def __init__(self, like: torch.Tensor):
        nbytes = like.numel() * like.element_size()
        self.nbytes = nbytes
        self.buf = torch.full((GUARD_BYTES + nbytes + GUARD_BYTES,), GUARD_FILL,
                              dtype=torch.uint8, device="cuda")
        body = self.buf[GUARD_BYTES:GUARD_BYTES + nbytes]
        self.t = body.view(like.dtype).view(like.shape)
        self.t.copy_(like.to("cuda"))

    def check(self, name: str = "tensor"):
        torch.cuda.synchronize()
        lo = self.buf[:GUARD_BYTES].cpu()
        hi = self.buf[GUARD_BYTES + self.nbytes:].cpu()
        for side, g in (("before", lo), ("after", hi)):
            bad = (g != GUARD_FILL).nonzero()
            assert bad.numel() == 0, (
                f"{name}: {bad.numel()} guard bytes {side} the buffer changed "
                f"(first at offset {int(bad[0])} of the {side} guard)")
