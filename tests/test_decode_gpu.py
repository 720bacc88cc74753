"""GPU parity of the batched decode step (through the C ABI) against the fp64
oracle on the same seeded inputs, plus its bit-exact and edge-case behaviour.

Calls of 2..4 tokens on an fp32 pool run the block form of the recurrence
(all tokens' dot products against the starting state, then a scalar
recurrence and one rank-n update); other calls run token by token."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import (STATE_TOL, assert_out_close, f64, oracle_decode, state_rel_err, to_dev)

import oracle

pytestmark = pytest.mark.gpu


def run_gpu(inp, **kw):
    d = to_dev(inp)
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                             d["slot_idx"], **kw)
    torch.cuda.synchronize()
    return out, d["state"]


def check_against_oracle(w, seed=0, **kw):
    inp = inputs.decode_inputs(w, seed=seed)
    o_ref, s_ref, rc = oracle_decode(inp, **{k: v for k, v in kw.items()
                                            if k in ("scale", "qk_l2norm")})
    out, st = run_gpu(inp, **kw)
    ratio = assert_out_close(out, o_ref, bf16_out=(out.dtype == torch.bfloat16))
    err = state_rel_err(f64(st), s_ref)
    assert err <= STATE_TOL, err
    return ratio, err


def test_library_loads_on_gpu():
    lib = gdn.load_library()
    assert lib.gdn_version() == 10000


def test_tiny_T8_single_call():
    check_against_oracle(inputs.TINY)


def test_tiny_T8_as_eight_calls_bit_exact_with_one_call():
    inp = inputs.decode_inputs(inputs.TINY)
    out8, st8 = run_gpu(inp)
    d = to_dev(inp)
    outs = []
    for t in range(8):
        sl = slice(t, t + 1)
        outs.append(gdn.decode_step_ex(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                                       d["v"][:, sl].contiguous(), d["g"][:, sl].contiguous(),
                                       d["beta"][:, sl].contiguous(), d["state"], d["slot_idx"]))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, dim=1), out8)
    assert torch.equal(d["state"], st8)


def test_layer_full_size():
    check_against_oracle(inputs.LAYER)


def test_mtp_T4_full_size():
    check_against_oracle(inputs.MTP)


def _single_token_calls(d, T):
    outs = []
    for t in range(T):
        sl = slice(t, t + 1)
        outs.append(gdn.decode_step(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                                    d["v"][:, sl].contiguous(), d["g"][:, sl].contiguous(),
                                    d["beta"][:, sl].contiguous(), d["state"], d["slot_idx"]))
    torch.cuda.synchronize()
    return torch.cat(outs, dim=1)


def test_mtp_T4_first_token_bit_exact_with_a_T1_call():
    """Calls of 2..4 tokens run the block form of the recurrence; for the
    first token it performs the single-token operations, so that token's
    output has the bits of a one-token call (fp32 pool)."""
    w = inputs.shrink(inputs.MTP, B=16)
    inp = inputs.decode_inputs(w)
    out4, _ = run_gpu(inp)
    d = to_dev(inp)
    out1 = _single_token_calls(d, 1)
    assert torch.equal(out1[:, 0], out4[:, 0])


def test_mtp_T4_agrees_with_four_T1_calls():
    """The block form and four sequential single-token calls differ only by
    fp32 rounding: a few ulps of the state and of the outputs."""
    w = inputs.shrink(inputs.MTP, B=16)
    inp = inputs.decode_inputs(w)
    out4, st4 = run_gpu(inp)
    d = to_dev(inp)
    outs = _single_token_calls(d, 4)
    rms = float(f64(outs).std())
    assert float(np.abs(f64(outs) - f64(out4)).max()) <= 1e-5 * rms
    assert state_rel_err(f64(st4), f64(d["state"])) <= 1e-6


@pytest.mark.parametrize("T", [2, 3, 4])
@pytest.mark.parametrize("dk,dv,Hk,H", [(128, 128, 6, 6), (64, 128, 2, 6), (128, 64, 3, 6),
                                        (64, 64, 1, 4)])
def test_block_tokens_against_oracle(T, dk, dv, Hk, H):
    w = inputs.DecodeWorkload("blk", B=7, H=H, Hk=Hk, dk=dk, dv=dv, T=T, n_slots=11,
                              slots="perm")
    check_against_oracle(w, seed=T)


@pytest.mark.parametrize("w", [inputs.TINY, inputs.shrink(inputs.LAYER, B=8)],
                         ids=["tiny", "layer_slice"])
def test_state_error_after_64_steps(w):
    w = inputs.shrink(w, T=1)
    inp0 = inputs.decode_inputs(w, seed=0)
    s_ref = f64(inp0["state"]).copy()
    st = inp0["state"].cuda().contiguous()
    for step in range(64):
        inp = inputs.decode_inputs(w, seed=100 + step, with_state=False)
        inp["slot_idx"] = inp0["slot_idx"]
        o_ref, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                      f64(inp["beta"]), s_ref, inp["slot_idx"].numpy())
        d = to_dev(inp)
        out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"])
        assert_out_close(out, o_ref)
    torch.cuda.synchronize()
    err = state_rel_err(f64(st), s_ref)
    assert err <= STATE_TOL, err


def test_serving_layer_full_size_sampled():
    """The benchmarked launch (B=256, H=48, 512-slot pool, permuted slots) at
    full size: 40 whole sequences (1,920 of the 12,288 (sequence, head)
    units, the first and the last among them) against the oracle in one
    batched call, every unused slot bit-identical, and every used slot
    changed."""
    w = inputs.SERVING
    dev_inp = inputs.decode_inputs(w, seed=0, device="cuda")
    pre = dev_inp["state"].clone()
    out = gdn.decode_step_ex(dev_inp["q"], dev_inp["k"], dev_inp["v"], dev_inp["g"],
                             dev_inp["beta"], dev_inp["state"], dev_inp["slot_idx"])
    torch.cuda.synchronize()
    slots = dev_inp["slot_idx"].cpu().numpy()
    unused = np.setdiff1d(np.arange(w.pool), slots)
    ui = torch.as_tensor(unused, device="cuda")
    assert torch.equal(dev_inp["state"][ui], pre[ui])
    used = torch.as_tensor(slots.astype(np.int64), device="cuda")
    changed = (dev_inp["state"][used] != pre[used]).flatten(1).any(dim=1)
    assert bool(changed.all())
    rng = np.random.default_rng(1)
    bs = np.sort(np.concatenate([[0, w.B - 1], 1 + rng.choice(w.B - 2, 38, replace=False)]))
    bt = torch.as_tensor(bs, device="cuda")
    st = f64(pre[used[bt]]).copy()  # a compact pool: sequence i uses slot i
    o_ref, _ = oracle.decode_step(f64(dev_inp["q"][bt]), f64(dev_inp["k"][bt]),
                                  f64(dev_inp["v"][bt]), f64(dev_inp["g"][bt]),
                                  f64(dev_inp["beta"][bt]), st, np.arange(len(bs)))
    assert_out_close(out[bt], o_ref)
    assert state_rel_err(f64(dev_inp["state"][used[bt]]), st) <= STATE_TOL


def test_ragged_gqa_fp32_small_heads():
    """Odd batch, GQA (H = 3 Hk), T = 3, dk = dv = 64, fp32 inputs, padding
    and permuted slots in one call."""
    w = inputs.DecodeWorkload("ragged", B=7, H=6, Hk=2, dk=64, dv=64, T=3, n_slots=11,
                              in_dtype=torch.float32, slots="perm")
    inp = inputs.decode_inputs(w, seed=3)
    inp["slot_idx"][2] = -1
    check = oracle_decode(inp)
    out, st = run_gpu(inp)
    assert_out_close(out, check[0])
    assert state_rel_err(f64(st), check[1]) <= STATE_TOL
    assert torch.all(out[2] == 0)


@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128), (64, 64)])
def test_other_head_sizes(dk, dv):
    w = inputs.DecodeWorkload("hs", B=5, H=3, dk=dk, dv=dv, T=2)
    check_against_oracle(w, seed=dk + dv)


def test_bf16_output():
    w = inputs.shrink(inputs.LAYER, B=4)
    check_against_oracle(w, out_dtype=torch.bfloat16)


def test_no_in_kernel_l2norm_and_custom_scale():
    w = inputs.shrink(inputs.TINY, T=2, in_dtype=torch.float32)
    inp = inputs.decode_inputs(w)
    for key in ("q", "k"):
        inp[key] = inp[key] / inp[key].norm(dim=-1, keepdim=True)
    o_ref, s_ref, _ = oracle_decode(inp, scale=0.3, qk_l2norm=False)
    out, st = run_gpu(inp, scale=0.3, qk_l2norm=False)
    assert_out_close(out, o_ref)
    assert state_rel_err(f64(st), s_ref) <= STATE_TOL


def test_alpha1_beta0_leaves_state_bit_exact():
    w = inputs.shrink(inputs.LAYER, B=4, H=8)
    inp = inputs.decode_inputs(w)
    inp["g"].zero_()
    inp["beta"].zero_()
    o_ref, _, _ = oracle_decode(inp)
    out, st = run_gpu(inp)
    assert torch.equal(st.cpu(), inp["state"])
    assert_out_close(out, o_ref)


def test_permuted_slots_bit_exact_with_identity_on_prepermuted_pool():
    w = inputs.DecodeWorkload("perm", B=12, H=4, dk=128, dv=128, T=2, n_slots=20, slots="perm")
    inp = inputs.decode_inputs(w, seed=5)
    perm = inp["slot_idx"].long()
    out_p, st_p = run_gpu(inp)
    inp2 = dict(inp)
    inp2["state"] = inp["state"][perm].clone()
    inp2["slot_idx"] = torch.arange(w.B, dtype=torch.int32)
    out_i, st_i = run_gpu(inp2)
    assert torch.equal(out_p, out_i)
    assert torch.equal(st_p[perm.cuda()], st_i)


def test_out_of_range_slots_set_status_and_skip():
    w = inputs.DecodeWorkload("bad", B=4, H=2, dk=128, dv=128, T=1, n_slots=4)
    inp = inputs.decode_inputs(w)
    inp["slot_idx"] = torch.tensor([0, 4, -3, 2], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = to_dev(inp)
    pre = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                             dev_status=status)
    torch.cuda.synchronize()
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_SLOT_RANGE and bits & gdn.STATUS_SLOT_RANGE
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)
    assert torch.equal(d["state"][1], pre[1]) and torch.equal(d["state"][3], pre[3])
    o_ref, s_ref, rc_ref = oracle_decode(inp)
    assert rc_ref == oracle.SLOT_RANGE
    assert_out_close(out, o_ref)


def test_clean_status_stays_zero():
    w = inputs.shrink(inputs.LAYER, B=3, H=2)
    inp = inputs.decode_inputs(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run_gpu(inp, dev_status=status)
    assert gdn.get_error(status) == (gdn.OK, 0)


def test_check_slots_rejects_duplicates_before_launch():
    w = inputs.DecodeWorkload("dup", B=3, H=2, dk=64, dv=64, T=1, n_slots=5)
    inp = inputs.decode_inputs(w)
    inp["slot_idx"] = torch.tensor([1, 3, 1], dtype=torch.int32)
    d = to_dev(inp)
    pre = d["state"].clone()
    with pytest.raises(gdn.GdnError) as e:
        gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                           check_slots=True)
    assert e.value.code == gdn.ERR_SLOT_DUP
    inp["slot_idx"] = torch.tensor([1, 5, 0], dtype=torch.int32)
    d = to_dev(inp)
    with pytest.raises(gdn.GdnError) as e:
        gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                           check_slots=True)
    assert e.value.code == gdn.ERR_SLOT_RANGE
    torch.cuda.synchronize()
    assert torch.equal(d["state"], pre)


def test_empty_batch_and_max_T():
    w = inputs.DecodeWorkload("e", B=0, H=2, dk=128, dv=128, T=1)
    inp = inputs.decode_inputs(w)
    out, _ = run_gpu(inp)
    assert out.shape == (0, 1, 2, 128)
    check_against_oracle(inputs.DecodeWorkload("t8", B=3, H=2, dk=128, dv=128, T=8), seed=9)
    w9 = inputs.DecodeWorkload("t9", B=1, H=1, dk=128, dv=128, T=9)
    with pytest.raises(gdn.GdnError) as e:
        run_gpu(inputs.decode_inputs(w9))
    assert e.value.code == gdn.ERR_UNSUPPORTED


def test_simple_entry_matches_ex_on_nondefault_stream():
    w = inputs.shrink(inputs.LAYER, B=6, H=4)
    inp = inputs.decode_inputs(w)
    d1, d2 = to_dev(inp), to_dev(inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1 = gdn.decode_step(d1["q"], d1["k"], d1["v"], d1["g"], d1["beta"], d1["state"],
                             d1["slot_idx"])
    o2 = gdn.decode_step_ex(d2["q"], d2["k"], d2["v"], d2["g"], d2["beta"], d2["state"],
                            d2["slot_idx"], n_slots=0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(d1["state"], d2["state"])
