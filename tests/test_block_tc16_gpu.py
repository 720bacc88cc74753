"""GPU parity of calls of 2..4 tokens on a 16-bit state pool (bf16 and fp16)
with dk = dv = 128: the block form of the recurrence with both contractions
on the tensor cores (decode_block_tc16_kernel).  The same criteria as the other 16-bit pool
tests, from the storage format's arithmetic:

  * outputs within 2e-3 * rms(o) of the fp64 oracle run from the same stored
    state (fp32 arithmetic);
  * every stored element within one storage ulp of the exact (fp64) state
    after the call, plus 1e-5 of the head's largest magnitude;
  * padded (-1) rows: zero outputs, their slots untouched; an out-of-range
    slot sets GDN_STATUS_SLOT_RANGE;
  * n_accept = n stores the state after the first n tokens (n = 0 keeps the
    slot), with the outputs of a call without commit, bit for bit;
  * 64 chained four-token calls, GPU and oracle each carrying its own
    rounded state: per-head relative Frobenius difference at most one ulp.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STORAGE_U, assert_out_close, f64, storage_ulp, to_dev

import oracle

pytestmark = pytest.mark.gpu

KINDS = {"bf16": torch.bfloat16, "fp16": torch.float16}


def within_ulp(s_gpu, s_ref, kind):
    g = f64(s_gpu)
    slack = 1e-5 * np.abs(s_ref).reshape(-1, s_ref.shape[-1] * s_ref.shape[-2]).max()
    err = np.abs(g - s_ref)
    bound = storage_ulp(s_ref, kind) + slack
    assert (err <= bound).all(), f"max err/ulp {(err / storage_ulp(s_ref, kind)).max():.3f}"


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
@pytest.mark.parametrize("T", [2, 3, 4])
@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
def test_one_call_against_the_oracle(T, in_dtype, kind):
    w = inputs.DecodeWorkload("tc16", B=10, H=6, Hk=2, dk=128, dv=128, T=T, n_slots=16,
                              slots="perm", in_dtype=in_dtype, state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=10 + T)
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                  f64(inp["beta"]), st_ref, inp["slot_idx"].numpy())
    d = to_dev(inp)
    pre = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"])
    torch.cuda.synchronize()
    assert_out_close(out, o_ref)
    used = inp["slot_idx"].long()
    within_ulp(d["state"][used.cuda()], st_ref[used.numpy()], kind)
    unused = sorted(set(range(w.pool)) - set(used.tolist()))
    ui = torch.tensor(unused, device="cuda")
    assert torch.equal(d["state"][ui], pre[ui])


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_padded_and_out_of_range_slots(kind):
    w = inputs.DecodeWorkload("tc16p", B=6, H=4, dk=128, dv=128, T=4, n_slots=8,
                              state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=5)
    inp["slot_idx"] = torch.tensor([3, -1, 0, 9, 5, 1], dtype=torch.int32)
    d = to_dev(inp)
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                             dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & gdn.STATUS_SLOT_RANGE
    for b in (1, 3):  # padding and out of range: zero outputs
        assert torch.count_nonzero(out[b]) == 0
    for s in (2, 4, 6, 7):  # slots nobody names
        assert torch.equal(d["state"][s], pre[s])
    ok = [0, 2, 4, 5]
    sub = {k: (v[ok] if k != "state" else v) for k, v in inp.items()}
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.decode_step(f64(sub["q"]), f64(sub["k"]), f64(sub["v"]), f64(sub["g"]),
                                  f64(sub["beta"]), st_ref, sub["slot_idx"].numpy())
    assert_out_close(out[ok], o_ref)
    sl = sub["slot_idx"].long()
    within_ulp(d["state"][sl.cuda()], st_ref[sl.numpy()], kind)


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_accept_lengths(kind):
    w = inputs.DecodeWorkload("tc16a", B=10, H=4, dk=128, dv=128, T=4, n_slots=12, slots="perm",
                              state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=9)
    n_acc = torch.tensor([0, 1, 2, 3, 4, 4, 2, 0, 1, 3], dtype=torch.int32)
    d = to_dev(inp)
    st = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                             n_accept=n_acc.cuda())
    plain = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"].clone(),
                               d["slot_idx"])
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
    slots = inp["slot_idx"].long()
    for b in range(w.B):
        n = int(n_acc[b])
        s = int(slots[b])
        if n == 0:
            assert torch.equal(st[s], d["state"][s])
            continue
        ref = f64(inp["state"][s:s + 1]).copy()
        oracle.decode_step(*(f64(inp[x][b:b + 1, :n]) for x in ("q", "k", "v", "g", "beta")),
                           ref, np.array([0], dtype=np.int32))
        within_ulp(st[s], ref[0], kind)


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_64_chained_four_token_calls(kind):
    w = inputs.DecodeWorkload("tc16c", B=4, H=6, dk=128, dv=128, T=4, state_dtype=KINDS[kind])
    inp0 = inputs.decode_inputs(w, seed=0)
    st = inp0["state"].cuda()
    s_round = f64(inp0["state"]).copy()
    for step in range(64):
        inp = inputs.decode_inputs(w, seed=900 + step, with_state=False)
        s_sync = f64(st).copy()
        o_sync, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                       f64(inp["g"]), f64(inp["beta"]), s_sync,
                                       inp["slot_idx"].numpy())
        args = [f64(inp[x]) for x in ("q", "k", "v", "g", "beta")]
        oracle.decode_step(*args, s_round, inp["slot_idx"].numpy(), state_round=kind)
        d = to_dev(inp)
        out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"])
        torch.cuda.synchronize()
        assert_out_close(out, o_sync)
        within_ulp(st, s_sync, kind)
    g = f64(st).reshape(w.B * w.H, -1)
    r = s_round.reshape(w.B * w.H, -1)
    rel = np.linalg.norm(g - r, axis=1) / np.linalg.norm(r, axis=1)
    assert rel.max() <= STORAGE_U[kind], rel.max()


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_unknown_pool_size_takes_the_token_loop(kind):
    """n_slots = 0 ("unknown"): the tensor map cannot be made, so the call
    runs the token loop; same criteria against the oracle, and the outputs
    agree with the tensor-core path's to the output tolerance."""
    w = inputs.DecodeWorkload("tc16u", B=6, H=4, dk=128, dv=128, T=3, n_slots=8, slots="perm",
                              state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=21)
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                  f64(inp["beta"]), st_ref, inp["slot_idx"].numpy())
    d = to_dev(inp)
    st0 = d["state"].clone()
    out_loop = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st0, d["slot_idx"],
                                  n_slots=0)
    out_tc = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                d["slot_idx"])
    torch.cuda.synchronize()
    assert_out_close(out_loop, o_ref)
    assert_out_close(out_tc, f64(out_loop))
    used = inp["slot_idx"].long()
    within_ulp(st0[used.cuda()], st_ref[used.numpy()], kind)


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_many_units_per_cta_with_padding_and_commits(kind):
    """More (sequence, head) units than resident CTAs (64 x 48 = 3072 against
    4 per SM), so every CTA walks several units in turn; 10% padding rows and
    accept lengths 0..4 interleave units that skip the update (or all the
    work) with units that store, which is what the CTA's count of barrier
    phases has to follow.  Outputs against the oracle; every committed slot
    within one storage ulp of the exact state after its accepted prefix;
    padding rows zero; uncommitted and unnamed slots untouched."""
    w = inputs.DecodeWorkload("tc16m", B=64, H=48, dk=128, dv=128, T=4, n_slots=64,
                              slots="padded", pad_frac=0.1, state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=31)
    rng = np.random.default_rng(31)
    n_acc = torch.tensor(rng.integers(0, 5, size=w.B), dtype=torch.int32)
    st_ref = f64(inp["state"]).copy()
    o_ref, rc = oracle.decode_step_spec(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                        f64(inp["g"]), f64(inp["beta"]), st_ref,
                                        inp["slot_idx"].numpy(), n_accept=n_acc.numpy())
    assert rc == 0
    d = to_dev(inp)
    pre = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                             n_accept=n_acc.cuda())
    torch.cuda.synchronize()
    assert_out_close(out, o_ref)
    slots = inp["slot_idx"].long()
    pad = slots < 0
    assert int(pad.sum()) > 0 and torch.count_nonzero(out[pad.cuda()]) == 0
    stored = [int(s) for s, n in zip(slots.tolist(), n_acc.tolist()) if s >= 0 and n > 0]
    kept = sorted(set(range(w.pool)) - set(stored))
    assert len(stored) > 0 and len(kept) > 0
    si = torch.tensor(stored)
    within_ulp(d["state"][si.cuda()], st_ref[si.numpy()], kind)
    ki = torch.tensor(kept, device="cuda")
    assert torch.equal(d["state"][ki], pre[ki])
