"""GPU parity of the low-rank sliding-window decode (through the C ABI)
against the fp64 oracle: outputs of every step within 2e-3 * rms(o), and
the window (cached k, u, decay weights; counts exactly) within 1e-4 relative
after the window has wrapped several times."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import assert_out_close, f64, to_dev

import oracle

pytestmark = pytest.mark.gpu


def fresh_window(n_slots, H, R, dk, dv):
    return [torch.zeros((n_slots, H, R, dk)), torch.zeros((n_slots, H, R, dv)),
            torch.zeros((n_slots, H, R)), torch.zeros((n_slots, H), dtype=torch.int32)]


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def chain(w, R, steps, T=1, seed=0, slots=None):
    win_ref = [f64(x).copy() for x in fresh_window(w.pool, w.H, R, w.dk, w.dv)]
    win_ref[3] = win_ref[3].astype(np.int32)
    win_gpu = [x.cuda() for x in fresh_window(w.pool, w.H, R, w.dk, w.dv)]
    ww = inputs.shrink(w, T=T)
    for step in range(steps):
        inp = inputs.decode_inputs(ww, seed=seed + step, with_state=False)
        if slots is not None:
            inp["slot_idx"] = torch.tensor(slots, dtype=torch.int32)
        o_ref, rc = oracle.lowrank_decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                               f64(inp["g"]), f64(inp["beta"]), *win_ref,
                                               inp["slot_idx"].numpy())
        d = to_dev(inp)
        out = gdn.lowrank_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], *win_gpu,
                                      d["slot_idx"])
        torch.cuda.synchronize()
        assert_out_close(out, o_ref)
    assert np.array_equal(win_gpu[3].cpu().numpy(), win_ref[3])
    for x, y in zip(win_gpu[:3], win_ref[:3]):
        assert rel(f64(x), y) <= 1e-4
    return win_gpu, win_ref


@pytest.mark.parametrize("R", [8, 16, 32, 64])
def test_window_wraps_several_times(R):
    w = inputs.DecodeWorkload("lr", B=6, H=4, dk=128, dv=128, T=1)
    chain(w, R, steps=2 * R + 3, seed=R)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_head_sizes_and_gqa(dk, dv):
    w = inputs.DecodeWorkload("lr", B=3, H=6, Hk=2, dk=dk, dv=dv, T=1, in_dtype=torch.float32)
    chain(w, 8, steps=19, seed=dk + dv)


def test_multi_token_calls_with_padding_and_permuted_slots():
    w = inputs.DecodeWorkload("lr", B=4, H=3, dk=128, dv=128, T=1, n_slots=7)
    win_gpu, win_ref = chain(w, 16, steps=9, T=4, seed=3, slots=[5, -1, 0, 3])
    # slots never used keep an empty window
    for s in (1, 2, 4, 6):
        assert int(win_gpu[3][s].sum()) == 0


def test_equals_full_rank_step_before_the_window_is_full():
    """From an empty window, the first R updates reproduce the full-rank
    decode from a zero state (GPU against GPU)."""
    R = 16
    w = inputs.DecodeWorkload("lr", B=8, H=4, dk=128, dv=128, T=1)
    win = [x.cuda() for x in fresh_window(w.B, w.H, R, w.dk, w.dv)]
    full = torch.zeros((w.B, w.H, w.dv, w.dk), device="cuda")
    for step in range(R):
        d = to_dev(inputs.decode_inputs(w, seed=100 + step, with_state=False))
        o_lr = gdn.lowrank_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], *win,
                                       d["slot_idx"])
        o_full = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], full, d["slot_idx"])
        torch.cuda.synchronize()
        rms = float(o_full.pow(2).mean().sqrt())
        assert float((o_lr - o_full).abs().max()) <= 2e-3 * rms
