"""GPU parity of the decode step with a 16-bit state pool (bf16 or fp16
storage, fp32 arithmetic; the state is rounded to nearest-even once per call).

Criteria, from the storage format's arithmetic:
  * one call from the same stored state: outputs within 2e-3 * rms(o) (the
    in-call arithmetic is the fp32 path's), and every stored element within
    one ulp of the storage format of the exact (fp64) result, plus 1e-5 of
    the head's largest magnitude for the fp32 arithmetic;
  * 64 chained calls, GPU and oracle each carrying its own rounded state:
    per-head relative Frobenius difference at most u = 2^(1-p) (one ulp
    everywhere);
  * drift against the exact fp64 recurrence (no rounding): the update map
    S -> alpha (I - beta k k^T) S is non-expansive for alpha <= 1,
    0 <= beta |k|^2 <= 1, so errors add at most linearly:
    ||E_T|| <= sum_t (u/2 + 1e-6) ||S_t||.
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


def check_state_within_ulp(s_gpu, s_ref, kind):
    g = f64(s_gpu)
    slack = 1e-5 * np.abs(s_ref).reshape(-1, s_ref.shape[-1] * s_ref.shape[-2]).max()
    bound = storage_ulp(s_ref, kind) + slack
    err = np.abs(g - s_ref)
    assert (err <= bound).all(), f"max err/ulp {(err / storage_ulp(s_ref, kind)).max():.3f}"


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
@pytest.mark.parametrize("T", [1, 4])
def test_one_call_from_the_same_stored_state(kind, T):
    w = inputs.DecodeWorkload("s16", B=16, H=8, dk=128, dv=128, T=T, n_slots=24, slots="perm",
                              state_dtype=KINDS[kind])
    inp = inputs.decode_inputs(w, seed=T)
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                  f64(inp["beta"]), st_ref, inp["slot_idx"].numpy())
    d = to_dev(inp)
    pre = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"])
    torch.cuda.synchronize()
    assert d["state"].dtype == KINDS[kind]
    assert_out_close(out, o_ref)
    used = inp["slot_idx"].long()
    check_state_within_ulp(d["state"][used.cuda()], st_ref[used.numpy()], kind)
    unused = sorted(set(range(w.pool)) - set(used.tolist()))
    ui = torch.tensor(unused, device="cuda")
    assert torch.equal(d["state"][ui], pre[ui])


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_64_chained_calls(kind):
    w = inputs.DecodeWorkload("c16", B=4, H=6, dk=128, dv=128, T=1, state_dtype=KINDS[kind])
    inp0 = inputs.decode_inputs(w, seed=0)
    st = inp0["state"].cuda()
    s_round = f64(inp0["state"]).copy()    # oracle carrying a rounded state
    s_exact = s_round.copy()               # oracle carrying the exact state
    norms = [np.linalg.norm(s_exact.reshape(w.B * w.H, -1), axis=1)]
    for step in range(64):
        inp = inputs.decode_inputs(w, seed=500 + step, with_state=False)
        # per-step parity from the GPU's own stored state
        s_sync = f64(st).copy()
        o_sync, _ = oracle.decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                       f64(inp["g"]), f64(inp["beta"]), s_sync,
                                       inp["slot_idx"].numpy())
        args = [f64(inp[x]) for x in ("q", "k", "v", "g", "beta")]
        oracle.decode_step(*args, s_round, inp["slot_idx"].numpy(), state_round=kind)
        oracle.decode_step(*args, s_exact, inp["slot_idx"].numpy())
        norms.append(np.linalg.norm(s_exact.reshape(w.B * w.H, -1), axis=1))
        d = to_dev(inp)
        out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st, d["slot_idx"])
        torch.cuda.synchronize()
        assert_out_close(out, o_sync)
        check_state_within_ulp(st, s_sync, kind)
    u = STORAGE_U[kind]
    g = f64(st).reshape(w.B * w.H, -1)
    r = s_round.reshape(w.B * w.H, -1)
    rel = np.linalg.norm(g - r, axis=1) / np.linalg.norm(r, axis=1)
    assert rel.max() <= u, rel.max()
    e = s_exact.reshape(w.B * w.H, -1)
    drift = np.linalg.norm(g - e, axis=1)
    bound = (u / 2 + 1e-6) * np.sum(norms[1:], axis=0)
    assert (drift <= bound).all(), (drift / bound).max()


@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_serving_shape_sampled(kind):
    w = inputs.shrink(inputs.SERVING, state_dtype=KINDS[kind])
    d = inputs.decode_inputs(w, seed=1, device="cuda")
    pre = d["state"].clone()
    out = gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"])
    torch.cuda.synchronize()
    slots = d["slot_idx"].cpu().numpy()
    rng = np.random.default_rng(3)
    for b, h in zip(rng.integers(0, w.B, 12), rng.integers(0, w.H, 12)):
        s = int(slots[b])
        st = f64(pre[s, h])[None, None].copy()
        o_ref, _ = oracle.decode_step(f64(d["q"][b:b + 1, :, h:h + 1]),
                                      f64(d["k"][b:b + 1, :, h:h + 1]),
                                      f64(d["v"][b:b + 1, :, h:h + 1]),
                                      f64(d["g"][b:b + 1, :, h:h + 1]),
                                      f64(d["beta"][b:b + 1, :, h:h + 1]), st, [0])
        assert_out_close(out[b:b + 1, :, h:h + 1], o_ref)
        check_state_within_ulp(d["state"][s, h], st[0, 0], kind)


def test_simple_entry_refuses_16bit_state():
    w = inputs.DecodeWorkload("r", B=1, H=1, dk=128, dv=128, T=1, state_dtype=torch.bfloat16)
    d = to_dev(inputs.decode_inputs(w))
    with pytest.raises(TypeError):
        gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"])
