"""GPU parity of the speculative-decoding state handling of
gdn_decode_step_ex (through the C ABI) against the fp64 oracle:

  * accept-length commit (n_accept): outputs of all T tokens, the state of
    the accepted prefix; bit-identical to a plain call on that prefix;
  * per-token snapshots (token_slots): every snapshot bit-identical to the
    state after a plain call on the corresponding prefix;
  * the two-pass verify/commit flow, bad values, 16-bit pools.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STATE_TOL, assert_out_close, f64, state_rel_err, storage_ulp, to_dev

import oracle

pytestmark = pytest.mark.gpu


def prefix(d, n):
    return {k: (v[:, :n].contiguous() if k in ("q", "k", "v", "g", "beta") else v)
            for k, v in d.items()}


def plain(d, state):
    return gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], state, d["slot_idx"])


def same_state(a, b):
    """fp32 pools: bit-identical.  16-bit pools: single-token calls run a
    different lane partition (packed rows), so the stored values may differ
    by the rounding of the fp32 arithmetic, at most one storage ulp."""
    if a.dtype == torch.float32:
        return torch.equal(a, b)
    kind = "bf16" if a.dtype == torch.bfloat16 else "fp16"
    ref = f64(b)
    return bool((np.abs(f64(a) - ref) <= storage_ulp(ref, kind) + 1e-6 * np.abs(ref).max()).all())


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.bfloat16])
def test_accept_length_commit(state_dtype):
    w = inputs.DecodeWorkload("acc", B=12, H=6, dk=128, dv=128, T=4, n_slots=16, slots="perm",
                              state_dtype=state_dtype)
    inp = inputs.decode_inputs(w, seed=7)
    n_acc = torch.tensor([0, 1, 2, 3, 4, 4, 2, 0, 1, 3, 4, 2], dtype=torch.int32)
    d = to_dev(inp)
    st = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                             n_accept=n_acc.cuda())
    torch.cuda.synchronize()
    # outputs: the same bits as a call without commit
    ref_out = plain(d, d["state"].clone())
    assert torch.equal(out, ref_out)
    # state of each row: the same bits as a plain call on its accepted prefix
    slots = inp["slot_idx"].long()
    for b in range(w.B):
        n = int(n_acc[b])
        want = d["state"].clone()
        if n > 0:
            pre = prefix({k: v[b:b + 1] for k, v in d.items()}, n)
            plain(pre, want)
        assert same_state(st[slots[b]], want[slots[b]]), (b, n)
    # and against the oracle
    o_ref = f64(inp["state"]).copy()
    out_ref, rc = oracle.decode_step_spec(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                          f64(inp["g"]), f64(inp["beta"]), o_ref,
                                          inp["slot_idx"].numpy(), n_accept=n_acc.numpy())
    assert rc == 0
    assert_out_close(out, out_ref)
    if state_dtype == torch.float32:
        assert state_rel_err(f64(st[slots.cuda()]), o_ref[slots.numpy()]) <= STATE_TOL


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.float16])
def test_token_snapshots(state_dtype):
    B, T = 5, 3
    w = inputs.DecodeWorkload("snap", B=B, H=4, dk=128, dv=128, T=T, n_slots=B + B * T,
                              state_dtype=state_dtype)
    inp = inputs.decode_inputs(w, seed=8)
    tsl = (B + torch.arange(B * T, dtype=torch.int32)).reshape(B, T)
    tsl[2, 1] = -1
    d = to_dev(inp)
    st = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                             token_slots=tsl.cuda(), check_slots=True)
    torch.cuda.synchronize()
    if state_dtype == torch.float32:
        assert torch.equal(out, plain(d, d["state"].clone()))
    else:
        # a 16-bit pool at dk = dv = 128: snapshots take the token loop, a plain
        # call of 3 tokens the tensor-core block form; outputs agree to fp32
        # rounding (within the output tolerance of the oracle's)
        assert_out_close(out, f64(plain(d, d["state"].clone())))
    assert torch.equal(st[:B], d["state"][:B])  # source slots untouched
    for t in range(T):
        want = d["state"].clone()
        plain(prefix(d, t + 1), want)
        for b in range(B):
            ts = int(tsl[b, t])
            if ts >= 0:
                assert same_state(st[ts], want[b]), (b, t)
            else:
                assert torch.equal(st[B + b * T + t], d["state"][B + b * T + t])


def test_verify_then_commit_two_passes():
    """Pass 1 with n_accept = 0 reads the state and writes none; pass 2
    commits the accepted prefix.  Together: outputs of pass 1 and the state
    of a single committing call."""
    w = inputs.DecodeWorkload("vc", B=8, H=4, dk=128, dv=128, T=4)
    inp = inputs.decode_inputs(w, seed=9)
    d = to_dev(inp)
    st = d["state"].clone()
    zeros = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    out1 = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                              n_accept=zeros)
    torch.cuda.synchronize()
    assert torch.equal(st, d["state"])
    n_acc = torch.tensor([1, 4, 2, 3, 0, 4, 1, 2], dtype=torch.int32, device="cuda")
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                       n_accept=n_acc)
    st1 = d["state"].clone()
    out_once = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st1, d["slot_idx"],
                                  n_accept=n_acc)
    torch.cuda.synchronize()
    assert torch.equal(out1, out_once)
    assert torch.equal(st, st1)


def test_bad_accept_and_token_slot_values():
    w = inputs.DecodeWorkload("bad", B=3, H=2, dk=128, dv=128, T=2, n_slots=8)
    inp = inputs.decode_inputs(w)
    d = to_dev(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = d["state"].clone()
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                       n_accept=torch.tensor([3, -1, 1], dtype=torch.int32, device="cuda"),
                       dev_status=status)
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_ACCEPT_RANGE and bits == gdn.STATUS_ACCEPT_RANGE
    assert torch.equal(st[:2], d["state"][:2]) and not torch.equal(st[2], d["state"][2])
    status.zero_()
    tsl = torch.tensor([[3, 4], [9, -1], [6, 7]], dtype=torch.int32, device="cuda")
    st = d["state"].clone()
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                       token_slots=tsl, dev_status=status)
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_SLOT_RANGE and bits == gdn.STATUS_SLOT_RANGE
    with pytest.raises(gdn.GdnError) as e:   # host check: a token slot that is a source slot
        gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                           token_slots=torch.tensor([[0, 4], [5, 6], [3, 7]], dtype=torch.int32,
                                                    device="cuda"), check_slots=True)
    assert e.value.code == gdn.ERR_SLOT_DUP


@pytest.mark.parametrize("state_dtype", [torch.bfloat16, torch.float16])
def test_single_token_commit_and_snapshot_on_16bit_pools(state_dtype):
    """One token on a 16-bit pool (the kernel that stages its tile in shared
    memory): n_accept = 1 stores what a plain call stores, n_accept = 0 stores
    nothing, a snapshot slot receives the state instead of the source slot,
    and the outputs are those of the plain call in every mode."""
    B = 6
    w = inputs.DecodeWorkload("st1", B=B, H=4, dk=128, dv=128, T=1, n_slots=2 * B,
                              state_dtype=state_dtype)
    inp = inputs.decode_inputs(w, seed=12)
    d = to_dev(inp)
    plain_st = d["state"].clone()
    ref_out = plain(d, plain_st)
    st = d["state"].clone()
    n_acc = torch.tensor([1, 0, 1, 1, 0, 1], dtype=torch.int32, device="cuda")
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"],
                             n_accept=n_acc)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    for b in range(B):
        s = int(inp["slot_idx"][b])
        want = plain_st[s] if int(n_acc[b]) == 1 else d["state"][s]
        assert torch.equal(st[s], want), b
    st2 = d["state"].clone()
    tsl = torch.tensor([[B + b] if b != 3 else [-1] for b in range(B)], dtype=torch.int32,
                       device="cuda")
    out2 = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st2, d["slot_idx"],
                              token_slots=tsl)
    torch.cuda.synchronize()
    assert torch.equal(out2, ref_out)
    assert torch.equal(st2[:B], d["state"][:B])  # the source slots are not written
    for b in range(B):
        if b == 3:
            assert torch.equal(st2[B + b], d["state"][B + b])
        else:
            assert torch.equal(st2[B + b], plain_st[int(inp["slot_idx"][b])]), b
