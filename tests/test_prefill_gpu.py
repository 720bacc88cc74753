"""GPU parity of the chunked prefill (through the C ABI) against the fp64
oracle's token-by-token recurrence on the same packed prompts: outputs
within 2e-3 * rms(o) and final states within 1e-4 relative (Frobenius, per
sequence and head), across ragged chunk boundaries, GQA, head sizes,
initial-state modes, padding sequences and bad ranges."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STATE_TOL, assert_out_close, f64, state_rel_err, to_dev

import oracle

pytestmark = pytest.mark.gpu


def run(w, seed=0, initial_state=True, slots=None, out_dtype=None, **kw):
    inp = inputs.prefill_inputs(w, seed=seed)
    if slots is not None:
        inp["slot_idx"] = torch.tensor(slots, dtype=torch.int32)
    st_ref = f64(inp["state"]).copy()
    o_ref, rc = oracle.prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                               f64(inp["beta"]), st_ref, inp["slot_idx"].numpy(),
                               inp["cu_seqlens"].numpy(), initial_state=initial_state)
    d = to_dev(inp)
    out = gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                            d["cu_seqlens"], initial_state=initial_state, out_dtype=out_dtype, **kw)
    torch.cuda.synchronize()
    return inp, d, out, o_ref, st_ref


@pytest.mark.parametrize("lens", [(1, 63, 64, 65, 130, 7), (200,), (64, 64)])
def test_ragged_chunk_boundaries(lens):
    w = inputs.PrefillWorkload("p", lens=lens, H=4, Hk=2, dk=128, dv=128)
    inp, d, out, o_ref, st_ref = run(w, seed=len(lens))
    assert_out_close(out, o_ref)
    assert state_rel_err(f64(d["state"]), st_ref) <= STATE_TOL


@pytest.mark.parametrize("n_prompts", [9, 300])
def test_many_prompts_in_any_length_order(n_prompts):
    """Phase B hands out its CTAs longest prompt first (up to 256 prompts;
    beyond that, in prompt order): both orders, with lengths shuffled and
    repeated, give the oracle's outputs and states."""
    rng = np.random.default_rng(n_prompts)
    lens = tuple(int(x) for x in rng.integers(1, 150 if n_prompts < 100 else 12, n_prompts))
    w = inputs.PrefillWorkload("many", lens=lens, H=2, dk=64, dv=64)
    inp, d, out, o_ref, st_ref = run(w, seed=n_prompts)
    assert_out_close(out, o_ref)
    assert state_rel_err(f64(d["state"]), st_ref) <= STATE_TOL


def test_long_prompt():
    w = inputs.PrefillWorkload("long", lens=(2048, 333), H=2, dk=128, dv=128)
    inp, d, out, o_ref, st_ref = run(w, seed=5)
    assert_out_close(out, o_ref)
    assert state_rel_err(f64(d["state"]), st_ref) <= STATE_TOL


@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (128, 128)])
def test_head_sizes(dk, dv, in_dtype):
    """Every product path of phase A: fp32 inputs (warp-level 3xTF32), bf16
    inputs with the Gram products on tcgen05, and bf16 with dk = dv = 128,
    where W and U run on tcgen05 as well."""
    w = inputs.PrefillWorkload("hs", lens=(70, 5, 129), H=3, dk=dk, dv=dv, in_dtype=in_dtype)
    inp, d, out, o_ref, st_ref = run(w, seed=dk + dv)
    assert_out_close(out, o_ref)
    assert state_rel_err(f64(d["state"]), st_ref) <= STATE_TOL


def test_zero_initial_state_padding_and_bf16_out():
    w = inputs.PrefillWorkload("z", lens=(100, 40, 66), H=2, dk=128, dv=128, n_slots=5)
    inp, d, out, o_ref, st_ref = run(w, seed=7, initial_state=False, slots=[4, -1, 0],
                                     out_dtype=torch.bfloat16)
    assert_out_close(out, o_ref, bf16_out=True)
    assert torch.all(out[100:140] == 0)
    used = [4, 0]
    assert state_rel_err(f64(d["state"][used]), st_ref[used]) <= STATE_TOL
    for s in (1, 2, 3):
        assert torch.equal(d["state"][s].cpu(), inp["state"][s])


def test_prefill_then_decode_continues_the_recurrence():
    """Prefill of the first L tokens followed by a decode step on token L+1
    equals the oracle over L+1 tokens."""
    w = inputs.PrefillWorkload("pd", lens=(97,), H=4, dk=128, dv=128)
    inp = inputs.prefill_inputs(w, seed=9)
    d = to_dev(inp)
    cu = torch.tensor([0, 96], dtype=torch.int32, device="cuda")
    gdn.chunk_prefill(d["q"][:96].contiguous(), d["k"][:96].contiguous(), d["v"][:96].contiguous(),
                      d["g"][:96].contiguous(), d["beta"][:96].contiguous(), d["state"],
                      d["slot_idx"], cu)
    o_last = gdn.decode_step(d["q"][96:97, None].contiguous(), d["k"][96:97, None].contiguous(),
                             d["v"][96:97, None].contiguous(), d["g"][96:97, None].contiguous(),
                             d["beta"][96:97, None].contiguous(), d["state"], d["slot_idx"])
    torch.cuda.synchronize()
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                              f64(inp["beta"]), st_ref, [0], [0, 97])
    assert_out_close(o_last[0, 0], o_ref[96])
    assert state_rel_err(f64(d["state"]), st_ref) <= STATE_TOL


def test_serving_prefill_shape_sampled():
    """The benchmarked prefill (8 prompts, 19,101 tokens, 48 heads): sampled
    (sequence, head) pairs against the oracle one by one."""
    w = inputs.PREFILL
    d = inputs.prefill_inputs(w, seed=0, device="cuda")
    pre = d["state"].clone()
    out = gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                            d["cu_seqlens"])
    torch.cuda.synchronize()
    cu = d["cu_seqlens"].cpu().numpy()
    rng = np.random.default_rng(4)
    for n, h in [(0, 0), (7, 47)] + list(zip(rng.integers(0, w.N, 4), rng.integers(0, w.H, 4))):
        n, h = int(n), int(h)
        t0, t1 = int(cu[n]), int(cu[n + 1])
        st = f64(pre[n, h])[None, None].copy()
        o_ref, _ = oracle.prefill(f64(d["q"][t0:t1, h:h + 1]), f64(d["k"][t0:t1, h:h + 1]),
                                  f64(d["v"][t0:t1, h:h + 1]), f64(d["g"][t0:t1, h:h + 1]),
                                  f64(d["beta"][t0:t1, h:h + 1]), st, [0], [0, t1 - t0])
        assert_out_close(out[t0:t1, h:h + 1], o_ref)
        assert state_rel_err(f64(d["state"][n, h])[None], st[0]) <= STATE_TOL


def test_bad_sequence_range_is_skipped_and_reported():
    w = inputs.PrefillWorkload("bad", lens=(10, 20), H=2, dk=64, dv=64)
    inp = inputs.prefill_inputs(w)
    inp["cu_seqlens"] = torch.tensor([0, 10, 99], dtype=torch.int32)  # past total_tokens
    d = to_dev(inp)
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                      d["cu_seqlens"], dev_status=status)
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_SEQ_RANGE and bits == gdn.STATUS_SEQ_RANGE
    assert torch.equal(d["state"][1], pre[1]) and not torch.equal(d["state"][0], pre[0])
