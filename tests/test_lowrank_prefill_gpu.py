"""GPU parity of the low-rank window over whole prompts (gdn_lowrank_prefill,
through the C ABI) against the fp64 oracle's token-by-token window: outputs
within 2e-3 * rms(o), the window left behind (cached k, u, decay weights)
within 1e-4 relative, counts exactly; across every window length, partial
and full chunks, prompts shorter than the window, continuing a stored
window, padding, head sizes and input types; and 256 prompts in one call
(the load at which the page's chunked low-rank kernel crashed)."""
import numpy as np
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import assert_out_close, f64, to_dev

import oracle

pytestmark = pytest.mark.gpu


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run(w, R, seed, slots=None, count=None, initial_window=True, out_dtype=None):
    inp = inputs.prefill_inputs(w, seed=seed)
    if slots is not None:
        inp["slot_idx"] = torch.tensor(slots, dtype=torch.int32)
    dw = inputs.DecodeWorkload("lw", B=w.N, H=w.H, dk=w.dk, dv=w.dv, T=1, n_slots=w.pool)
    win = inputs.lowrank_window(dw, R, seed=seed + 1)
    if count is not None:
        win["win_count"] = torch.as_tensor(count, dtype=torch.int32).expand(w.pool, w.H).contiguous()
    ref = [f64(win[x]).copy() for x in ("win_k", "win_u", "win_c")]
    ref.append(win["win_count"].numpy().astype(np.int32).copy())
    o_ref, rc = oracle.lowrank_prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                       f64(inp["beta"]), *ref, inp["slot_idx"].numpy(),
                                       inp["cu_seqlens"].numpy(), initial_window=initial_window)
    d = to_dev(inp)
    gw = [win[x].cuda().contiguous() for x in ("win_k", "win_u", "win_c", "win_count")]
    out = gdn.lowrank_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], *gw, d["slot_idx"],
                              d["cu_seqlens"], initial_window=initial_window, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out, o_ref, gw, ref


def check_window(gw, ref):
    assert np.array_equal(gw[3].cpu().numpy(), ref[3])
    for x, y in zip(gw[:3], ref[:3]):
        assert rel(f64(x), y) <= 1e-4


@pytest.mark.parametrize("R", [8, 16, 32, 64])
def test_every_window_length_over_full_and_partial_chunks(R):
    w = inputs.PrefillWorkload("lp", lens=(200, 5, 64, 129), H=3, dk=128, dv=128)
    out, o_ref, gw, ref = run(w, R, seed=R, count=3 * R + 1)
    assert_out_close(out, o_ref)
    check_window(gw, ref)


@pytest.mark.parametrize("count", [0, 3, 70])
def test_windows_not_full_and_fresh_starts(count):
    """Entering windows of 0 and 3 updates (not full) and a long-running one;
    prompts shorter than the window."""
    w = inputs.PrefillWorkload("lp", lens=(2, 40, 9), H=2, dk=128, dv=128)
    out, o_ref, gw, ref = run(w, 32, seed=count, count=count)
    assert_out_close(out, o_ref)
    check_window(gw, ref)


def test_empty_start_padding_and_bf16_out():
    w = inputs.PrefillWorkload("lp", lens=(90, 17, 66), H=2, dk=128, dv=128, n_slots=5)
    out, o_ref, gw, ref = run(w, 16, seed=7, slots=[4, -1, 0], initial_window=False,
                              out_dtype=torch.bfloat16)
    assert_out_close(out, o_ref, bf16_out=True)
    assert torch.all(out[90:107] == 0)
    check_window(gw, ref)


@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_head_sizes_gqa_and_input_types(dk, dv, in_dtype):
    w = inputs.PrefillWorkload("lp", lens=(70, 130), H=4, Hk=2, dk=dk, dv=dv, in_dtype=in_dtype)
    out, o_ref, gw, ref = run(w, 16, seed=dk + dv, count=50)
    assert_out_close(out, o_ref)
    check_window(gw, ref)


def test_prefill_then_decode_continues_the_window():
    """The window a prompt leaves is the one the decode step continues."""
    w = inputs.PrefillWorkload("lp", lens=(150,), H=2, dk=128, dv=128)
    R = 16
    inp = inputs.prefill_inputs(w, seed=3)
    d = to_dev(inp)
    z = [torch.zeros((1, 2, R, 128), device="cuda"), torch.zeros((1, 2, R, 128), device="cuda"),
         torch.zeros((1, 2, R), device="cuda"), torch.zeros((1, 2), dtype=torch.int32, device="cuda")]
    cu = torch.tensor([0, 149], dtype=torch.int32, device="cuda")
    sl = lambda x: x[:149].contiguous()
    gdn.lowrank_prefill(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]), *z,
                        d["slot_idx"], cu, initial_window=False)
    tok = lambda x: x[149:150, None].contiguous()
    o_last = gdn.lowrank_decode_step(tok(d["q"]), tok(d["k"]), tok(d["v"]), tok(d["g"]),
                                     tok(d["beta"]), *z, d["slot_idx"])
    torch.cuda.synchronize()
    ref = [np.zeros((1, 2, R, 128)), np.zeros((1, 2, R, 128)), np.zeros((1, 2, R)),
           np.zeros((1, 2), dtype=np.int32)]
    o_ref, _ = oracle.lowrank_prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                      f64(inp["beta"]), *ref, [0], [0, 150], initial_window=False)
    assert_out_close(o_last[0, 0], o_ref[149])
    check_window(z, ref)


def test_256_prompts_in_one_call():
    """256 concurrent prompts of mixed lengths (the concurrency at which the
    page's chunked low-rank prefill crashed): every output and window
    against the oracle."""
    rng = np.random.default_rng(256)
    lens = tuple(int(x) for x in rng.integers(1, 200, 256))
    w = inputs.PrefillWorkload("lp256", lens=lens, H=2, dk=128, dv=128)
    out, o_ref, gw, ref = run(w, 32, seed=11, count=40)
    assert_out_close(out, o_ref)
    check_window(gw, ref)
