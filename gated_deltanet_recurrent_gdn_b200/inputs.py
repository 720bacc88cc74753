"""Seeded synthetic inputs for the decode-step workloads.

This module draws random tensors and nothing else: it holds none of the
decode step's arithmetic and serves both the CUDA path and the CPU checker.
Every workload is drawn from one ``torch.Generator`` seeded per call, in a
fixed order, on the requested device; bf16 inputs are drawn in fp32 and
rounded once, so every consumer reads the identical rounded values.

Workloads (sizes from the target configurations; distributions as stated):
  tiny      B=1,   H=4,  dk=dv=128, T=8, fp32 q/k/v, identity slots
  layer     B=64,  H=48, dk=dv=128, T=1, bf16 q/k/v, identity slots
  serving   B=256, H=48, dk=dv=128, T=1, bf16, 48 layers, each with its own
            512-slot pool; slot_idx = a random permutation of 512, first 256
  mtp       B=128, H=48, dk=dv=128, T=4, bf16, identity slots
  fused     B=256, Hk=16, H=48, dk=dv=128, C = 2*16*128 + 48*128 = 10240,
            26 (10%) padding rows at random positions, identity slots
  prefill   8 prompts of 777..4096 tokens (19,101 in all), H=48, dk=dv=128,
            bf16 q/k/v, packed with cu_seqlens
Distributions: q, k, v ~ N(0,1); g ~ U(-0.5, 0); beta = sigmoid(N(0,1));
state ~ N(0, 0.02^2) (std 0.02); fused extras: conv state ~ N(0,1) bf16,
conv weights ~ N(0, 0.5^2) fp32, a, b, z ~ N(0,1) bf16,
A_log = log(U(1,16)), dt_bias ~ N(0, 0.5^2), norm_w = 1 + N(0, 0.1^2).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    T: int
    Hk: int | None = None        # None: Hk = H
    n_slots: int | None = None   # None: n_slots = B
    in_dtype: torch.dtype = torch.bfloat16
    state_dtype: torch.dtype = torch.float32
    slots: str = "identity"      # identity | perm | padded
    layers: int = 1
    pad_frac: float = 0.0

    @property
    def hk(self) -> int:
        return self.H if self.Hk is None else self.Hk

    @property
    def pool(self) -> int:
        return self.B if self.n_slots is None else self.n_slots


@dataclass(frozen=True)
class FusedWorkload:
    name: str
    B: int
    Hk: int
    H: int
    dk: int
    dv: int
    n_slots: int | None = None
    pad_frac: float = 0.0
    conv_w_dtype: torch.dtype = torch.float32

    @property
    def C(self) -> int:
        return 2 * self.Hk * self.dk + self.H * self.dv

    @property
    def pool(self) -> int:
        return self.B if self.n_slots is None else self.n_slots


TINY = DecodeWorkload("tiny", B=1, H=4, dk=128, dv=128, T=8, in_dtype=torch.float32)
LAYER = DecodeWorkload("layer", B=64, H=48, dk=128, dv=128, T=1)
SERVING = DecodeWorkload("serving", B=256, H=48, dk=128, dv=128, T=1, n_slots=512,
                         slots="perm", layers=48)
MTP = DecodeWorkload("mtp", B=128, H=48, dk=128, dv=128, T=4)
FUSED = FusedWorkload("fused", B=256, Hk=16, H=48, dk=128, dv=128, pad_frac=0.1)

WORKLOADS = {w.name: w for w in (TINY, LAYER, SERVING, MTP)}


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, gen, device, std=1.0, dtype=torch.float32):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def slot_map(kind: str, B: int, n_slots: int, gen, device, pad_frac: float = 0.0) -> torch.Tensor:
    """int32 [B] slot map: identity, a random permutation of the pool
    (first B entries), or identity with round(pad_frac*B) rows set to -1."""
    if kind == "identity":
        s = torch.arange(B, dtype=torch.int32)
    elif kind == "perm":
        s = torch.randperm(n_slots, generator=gen, device=device)[:B].to(torch.int32).cpu()
    elif kind == "padded":
        s = torch.arange(B, dtype=torch.int32)
        n_pad = int(round(pad_frac * B))
        pad = torch.randperm(B, generator=gen, device=device)[:n_pad].cpu()
        s[pad] = -1
    else:
        raise ValueError(kind)
    return s.to(device)


def decode_inputs(w: DecodeWorkload, seed: int = 0, device="cpu", layer: int = 0,
                  with_state: bool = True) -> dict:
    """One layer's inputs, drawn in the order q, k, v, g, b_logit, state, slot."""
    gen = generator(seed * 1000 + layer, device)
    B, T, H, Hk, dk, dv = w.B, w.T, w.H, w.hk, w.dk, w.dv
    d = {}
    d["q"] = _normal((B, T, Hk, dk), gen, device, dtype=w.in_dtype)
    d["k"] = _normal((B, T, Hk, dk), gen, device, dtype=w.in_dtype)
    d["v"] = _normal((B, T, H, dv), gen, device, dtype=w.in_dtype)
    d["g"] = torch.rand((B, T, H), generator=gen, device=device, dtype=torch.float32) * -0.5
    d["beta"] = torch.sigmoid(_normal((B, T, H), gen, device))
    if with_state:
        d["state"] = _normal((w.pool, H, dv, dk), gen, device, std=0.02, dtype=w.state_dtype)
    d["slot_idx"] = slot_map(w.slots, B, w.pool, gen, device, w.pad_frac)
    return d


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    lens: tuple            # tokens per sequence
    H: int
    dk: int
    dv: int
    Hk: int | None = None
    n_slots: int | None = None
    in_dtype: torch.dtype = torch.bfloat16

    @property
    def hk(self) -> int:
        return self.H if self.Hk is None else self.Hk

    @property
    def N(self) -> int:
        return len(self.lens)

    @property
    def total(self) -> int:
        return int(sum(self.lens))

    @property
    def pool(self) -> int:
        return self.N if self.n_slots is None else self.n_slots


# prompts of a serving prefill: 8 prompts of 1024..4096 tokens, 48 heads
PREFILL = PrefillWorkload("prefill", lens=(4096, 1024, 3000, 2048, 1500, 4096, 777, 2560),
                          H=48, dk=128, dv=128)


def prefill_inputs(w: PrefillWorkload, seed: int = 0, device="cpu") -> dict:
    """Packed prompts, drawn in the order q, k, v, g, b_logit, state; identity
    slots; cu_seqlens from the lengths."""
    gen = generator(seed, device)
    T, H, Hk, dk, dv = w.total, w.H, w.hk, w.dk, w.dv
    d = {}
    d["q"] = _normal((T, Hk, dk), gen, device, dtype=w.in_dtype)
    d["k"] = _normal((T, Hk, dk), gen, device, dtype=w.in_dtype)
    d["v"] = _normal((T, H, dv), gen, device, dtype=w.in_dtype)
    d["g"] = torch.rand((T, H), generator=gen, device=device, dtype=torch.float32) * -0.5
    d["beta"] = torch.sigmoid(_normal((T, H), gen, device))
    d["state"] = _normal((w.pool, H, dv, dk), gen, device, std=0.02)
    d["slot_idx"] = torch.arange(w.N, dtype=torch.int32, device=device)
    cu = [0]
    for L in w.lens:
        cu.append(cu[-1] + int(L))
    d["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    return d


def lowrank_window(w: DecodeWorkload, R: int, seed: int = 0, device="cpu") -> dict:
    """A full low-rank window per (slot, head): cached k ~ unit vectors of
    N(0,1) draws, cached u ~ N(0, 0.1^2), decay weights ~ U(0.05, 1) and a
    count past R (every ring position holds an update)."""
    gen = generator(seed, device)
    k = _normal((w.pool, w.H, R, w.dk), gen, device)
    d = {"win_k": k / k.norm(dim=-1, keepdim=True)}
    d["win_u"] = _normal((w.pool, w.H, R, w.dv), gen, device, std=0.1)
    d["win_c"] = 0.05 + 0.95 * torch.rand((w.pool, w.H, R), generator=gen, device=device)
    d["win_count"] = torch.full((w.pool, w.H), 4 * R + 3, dtype=torch.int32, device=device)
    return d


def fused_inputs(w: FusedWorkload, seed: int = 0, device="cpu") -> dict:
    gen = generator(seed, device)
    B, Hk, H, dk, dv, C = w.B, w.Hk, w.H, w.dk, w.dv, w.C
    bf = torch.bfloat16
    d = {}
    d["mixed_x"] = _normal((B, C), gen, device, dtype=bf)
    d["conv_state"] = _normal((w.pool, C, 3), gen, device, dtype=bf)
    d["conv_w"] = _normal((C, 4), gen, device, std=0.5, dtype=w.conv_w_dtype)
    d["a"] = _normal((B, H), gen, device, dtype=bf)
    d["b"] = _normal((B, H), gen, device, dtype=bf)
    d["A_log"] = torch.log(1.0 + 15.0 * torch.rand((H,), generator=gen, device=device))
    d["dt_bias"] = _normal((H,), gen, device, std=0.5)
    d["z"] = _normal((B, H * dv), gen, device, dtype=bf)
    d["norm_w"] = 1.0 + _normal((dv,), gen, device, std=0.1)
    d["state"] = _normal((w.pool, H, dv, dk), gen, device, std=0.02)
    d["slot_idx"] = slot_map("padded" if w.pad_frac > 0 else "identity", B, w.pool, gen,
                             device, w.pad_frac)
    return d


def shrink(w, **kw):
    """A copy of a workload with some sizes changed (for small test cases)."""
    return replace(w, **kw)
