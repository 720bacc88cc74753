"""The invariants the definition of the step fixes, checked on the GPU
(through the C ABI), and the edge cases of its gates and inputs.

* decay only (beta = 0): after T tokens the state is S0 * prod(alpha), to
  fp32 rounding (a few ulps per element);
* projection (beta = 1, unit k): after the update S'^T k = v, so with q = k
  the read-out is scale * v, to fp32 rounding;
* extreme gates (g down to -200, where alpha underflows to 0 in fp32;
  beta exactly 0 or 1) and all-zero q or k rows (the epsilon inside the
  L2 norm decides them) against the fp64 oracle at the usual tolerances;
* a chain of 64 four-token calls (the block form of the recurrence) against
  the oracle carried in fp64: state within 1e-4.
Each runs both the token-by-token kernel and the block form (calls of 2..4
tokens on an fp32 pool)."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STATE_TOL, assert_out_close, f64, oracle_decode, state_rel_err, to_dev

import oracle

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24  # unit roundoff of fp32


def run_gpu(inp, **kw):
    d = to_dev(inp)
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                             d["slot_idx"], **kw)
    torch.cuda.synchronize()
    return out, d["state"]


@pytest.mark.parametrize("T", [1, 3, 4, 6])
def test_decay_only_scales_the_state_by_the_product_of_the_alphas(T):
    w = inputs.DecodeWorkload("decay", B=3, H=4, dk=128, dv=128, T=T, n_slots=5, slots="perm")
    inp = inputs.decode_inputs(w, seed=T)
    inp["beta"].zero_()
    s0 = f64(inp["state"])
    out, st = run_gpu(inp)
    prod = np.exp(f64(inp["g"]).sum(axis=1))  # [B, H]
    slots = inp["slot_idx"].numpy()
    got = f64(st)
    for b in range(w.B):
        want = s0[slots[b]] * prod[b][:, None, None]
        # exp and each of the T products or the unrolled product round once
        tol = (4 * T + 4) * U32 * np.abs(want) + 1e-30
        assert np.all(np.abs(got[slots[b]] - want) <= tol)
    untouched = sorted(set(range(w.pool)) - set(slots.tolist()))
    assert torch.equal(st[untouched].cpu(), inp["state"][untouched])
    o_ref, _, _ = oracle_decode(inp)
    assert_out_close(out, o_ref)


def _unit_k(n_rows, dk, gen):
    """Rows of dk values with four entries of +-1/2 at random places: exactly
    unit length in every floating-point format."""
    k = torch.zeros((n_rows, dk))
    for r in range(n_rows):
        idx = torch.randperm(dk, generator=gen)[:4]
        k[r, idx] = torch.where(torch.rand(4, generator=gen) < 0.5, -0.5, 0.5)
    return k


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
def test_projection_with_beta_one_and_unit_k_reads_back_v(T, in_dtype):
    """With beta = 1 and |k| = 1 every token makes S^T k = v; with q = k and
    no in-kernel normalisation the read-out is scale * v."""
    w = inputs.DecodeWorkload("proj", B=2, H=3, dk=128, dv=128, T=T, in_dtype=in_dtype)
    inp = inputs.decode_inputs(w, seed=40 + T)
    gen = torch.Generator().manual_seed(T)
    k = _unit_k(w.B * T * w.H, w.dk, gen).reshape(w.B, T, w.H, w.dk).to(in_dtype)
    inp["k"], inp["q"] = k, k.clone()
    inp["beta"].fill_(1.0)
    scale = 0.25
    out, st = run_gpu(inp, scale=scale, qk_l2norm=False)
    v = f64(inp["v"])
    o = f64(out)
    s = f64(st)
    # |o - scale v| at fp32 rounding of sums of terms of size |v| and |S|
    mag = np.abs(v).max() + np.abs(s).max() * 4
    assert np.abs(o - scale * v).max() <= 64 * U32 * scale * mag
    # and the stored state projects the last token's k onto its v
    slots = inp["slot_idx"].numpy()
    kl = f64(k)[:, T - 1]  # [B, H, dk]
    for b in range(w.B):
        proj = np.einsum("hji,hi->hj", s[slots[b]], kl[b])
        assert np.abs(proj - v[b, T - 1]).max() <= 64 * U32 * mag


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_extreme_gates_and_zero_rows(T):
    """g in {0, -30, -100, -200} (alpha from 1 down to an fp32 underflow),
    beta exactly 0 or 1 on some tokens, and all-zero q or k rows, against the
    fp64 oracle (whose alpha does not underflow at g = -200: the difference
    is far below the tolerance)."""
    w = inputs.DecodeWorkload("edge", B=6, H=4, dk=128, dv=128, T=T, n_slots=9, slots="perm")
    inp = inputs.decode_inputs(w, seed=70 + T)
    gen = torch.Generator().manual_seed(T)
    choice = torch.randint(0, 5, inp["g"].shape, generator=gen)
    g = inp["g"]
    g[choice == 1] = -30.0
    g[choice == 2] = -100.0
    g[choice == 3] = -200.0
    g[choice == 4] = 0.0
    bsel = torch.randint(0, 3, inp["beta"].shape, generator=gen)
    inp["beta"][bsel == 1] = 0.0
    inp["beta"][bsel == 2] = 1.0
    inp["k"][0, 0, 1].zero_()          # a zero k row
    inp["q"][1, T - 1, 2].zero_()      # a zero q row
    inp["k"][2, :, 3].zero_()          # zero k on every token of one head
    inp["q"][2, :, 3].zero_()
    o_ref, s_ref, _ = oracle_decode(inp)
    out, st = run_gpu(inp)
    assert torch.isfinite(out).all() and torch.isfinite(st).all()
    assert_out_close(out, o_ref)
    # a head decayed by exp(-100) or exp(-200) and not updated since (beta = 0
    # or k = 0) holds about 1e-45 or 1e-89 times S0 in the fp64 oracle: in
    # fp32 that is a few subnormal units or exactly 0, with no relative
    # precision left.  The relative bound therefore applies with a floor of
    # 1e-30 on the reference norm (far below any state the step leaves
    # otherwise, far above fp32's subnormal spacing).
    d = (f64(st) - s_ref).reshape(-1, w.dv * w.dk)
    r = s_ref.reshape(-1, w.dv * w.dk)
    num, den = np.sqrt((d * d).sum(1)), np.sqrt((r * r).sum(1))
    assert np.all(num <= STATE_TOL * np.maximum(den, 1e-30)), float((num / np.maximum(den, 1e-30)).max())


def test_state_error_after_64_four_token_calls():
    """64 calls of T = 4 (the block form) chained on one pool against the
    oracle carried in fp64 over the same 256 tokens."""
    w = inputs.DecodeWorkload("chain4", B=4, H=8, dk=128, dv=128, T=4, n_slots=6, slots="perm")
    inp0 = inputs.decode_inputs(w, seed=3)
    s_ref = f64(inp0["state"]).copy()
    st = inp0["state"].cuda().contiguous()
    slots = inp0["slot_idx"]
    for step in range(64):
        inp = inputs.decode_inputs(w, seed=500 + step, with_state=False)
        o_ref, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                      f64(inp["beta"]), s_ref, slots.numpy())
        d = to_dev(inp)
        out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, slots.cuda())
        assert_out_close(out, o_ref)
    torch.cuda.synchronize()
    err = state_rel_err(f64(st)[slots.long().numpy()], s_ref[slots.long().numpy()])
    assert err <= STATE_TOL, err
