"""GPU parity of the fused step (conv k=4 + SiLU, gates, GQA, recurrence,
gated RMSNorm) through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STATE_TOL, assert_out_close, f64, state_rel_err, to_dev

import oracle

pytestmark = pytest.mark.gpu


def run_fused_gpu(d, w, **kw):
    out = gdn.fused_decode_step(d["mixed_x"], d["conv_state"], d["conv_w"], d["a"], d["b"],
                                d["A_log"], d["dt_bias"], d["z"], d["norm_w"], d["state"],
                                d["slot_idx"], Hk=w.Hk, H=w.H, dk=w.dk, dv=w.dv, **kw)
    torch.cuda.synchronize()
    return out


def oracle_fused(inp, w, rows=None):
    """Oracle on the sequences ``rows`` (all by default), each on its own
    one-slot pool so that only the touched slots are converted."""
    rows = range(w.B) if rows is None else rows
    res = {}
    for b in rows:
        s = int(inp["slot_idx"][b])
        if s < 0:
            res[b] = (np.zeros((w.H, w.dv)), None, None)
            continue
        st = f64(inp["state"][s:s + 1]).copy()
        cs = f64(inp["conv_state"][s:s + 1]).copy()
        out, rc = oracle.fused_step(f64(inp["mixed_x"][b:b + 1]), cs, f64(inp["conv_w"]),
                                    f64(inp["a"][b:b + 1]), f64(inp["b"][b:b + 1]),
                                    f64(inp["A_log"]), f64(inp["dt_bias"]),
                                    f64(inp["z"][b:b + 1]), f64(inp["norm_w"]), st, [0],
                                    Hk=w.Hk, H=w.H, dk=w.dk, dv=w.dv)
        assert rc == 0
        res[b] = (out[0], st[0], cs[0])
    return res


def check(w, seed=0, rows=None, out_dtype=None):
    inp = inputs.fused_inputs(w, seed=seed)
    d = to_dev(inp)
    out = run_fused_gpu(d, w, out_dtype=out_dtype)
    ref = oracle_fused(inp, w, rows)
    bf16 = out.dtype == torch.bfloat16
    o_ref = np.stack([ref[b][0] for b in ref])
    assert_out_close(out[list(ref)], o_ref, bf16_out=bf16)
    for b, (_, st, cs) in ref.items():
        s = int(inp["slot_idx"][b])
        if s < 0:
            assert torch.all(out[b] == 0)
            continue
        assert state_rel_err(f64(d["state"][s]), st) <= STATE_TOL
        # the conv state holds bf16 copies of inputs: bit-exact
        assert np.array_equal(f64(d["conv_state"][s]), cs)
    # padding rows: their slots (identity map) are untouched
    pad = (inp["slot_idx"] < 0).nonzero().flatten().tolist()
    for b in pad:
        assert torch.all(out[b] == 0)
        if b < w.pool and b not in inp["slot_idx"].tolist():
            assert torch.equal(d["state"][b].cpu(), inp["state"][b])
            assert torch.equal(d["conv_state"][b].cpu(), inp["conv_state"][b])
    return inp, d, out


def test_fused_small_full_compare():
    w = inputs.shrink(inputs.FUSED, B=20)
    check(w)


def test_fused_full_size_sampled():
    w = inputs.FUSED
    inp = inputs.fused_inputs(w)
    pads = (inp["slot_idx"] < 0).nonzero().flatten().tolist()
    rng = np.random.default_rng(2)
    rows = sorted(set(rng.integers(0, w.B, 10).tolist()) | set(pads[:2]) | {0, w.B - 1})
    check(w, rows=rows)


@pytest.mark.parametrize("Hk,H", [(4, 4), (4, 8), (2, 16), (1, 3)])
def test_fused_group_sizes(Hk, H):
    """cluster sizes 1, 2, 8 and 3"""
    w = inputs.FusedWorkload("g", B=9, Hk=Hk, H=H, dk=128, dv=128, pad_frac=0.2)
    check(w, seed=Hk * 10 + H)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_fused_head_sizes(dk, dv):
    w = inputs.FusedWorkload("hs", B=6, Hk=2, H=6, dk=dk, dv=dv, pad_frac=0.2)
    check(w, seed=dk + dv)


def test_fused_bf16_weights_and_bf16_out():
    w = inputs.FusedWorkload("bf", B=8, Hk=2, H=6, dk=128, dv=128, conv_w_dtype=torch.bfloat16)
    check(w, out_dtype=torch.bfloat16)


def test_fused_two_steps_carry_conv_and_state():
    w = inputs.FusedWorkload("two", B=5, Hk=2, H=6, dk=128, dv=128)
    inp = inputs.fused_inputs(w, seed=4)
    d = to_dev(inp)
    st = f64(inp["state"]).copy()
    cs = f64(inp["conv_state"]).copy()
    for step in range(3):
        x = inputs.fused_inputs(w, seed=50 + step)["mixed_x"]
        d["mixed_x"] = x.cuda()
        out = run_fused_gpu(d, w)
        o_ref, rc = oracle.fused_step(f64(x), cs, f64(inp["conv_w"]), f64(inp["a"]), f64(inp["b"]),
                                      f64(inp["A_log"]), f64(inp["dt_bias"]), f64(inp["z"]),
                                      f64(inp["norm_w"]), st, inp["slot_idx"].numpy(),
                                      Hk=w.Hk, H=w.H, dk=w.dk, dv=w.dv)
        assert_out_close(out, o_ref)
    assert np.array_equal(f64(d["conv_state"]), cs)
    assert state_rel_err(f64(d["state"]), st) <= STATE_TOL


def test_fused_bad_slot_sets_status():
    w = inputs.FusedWorkload("bad", B=3, Hk=1, H=3, dk=64, dv=64)
    inp = inputs.fused_inputs(w)
    inp["slot_idx"] = torch.tensor([0, 7, 2], dtype=torch.int32)
    d = to_dev(inp)
    pre = d["state"].clone()
    pre_cs = d["conv_state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_fused_gpu(d, w, dev_status=status)
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_SLOT_RANGE and bits == gdn.STATUS_SLOT_RANGE
    assert torch.all(out[1] == 0)
    assert torch.equal(d["state"][1], pre[1]) and torch.equal(d["conv_state"][1], pre_cs[1])
