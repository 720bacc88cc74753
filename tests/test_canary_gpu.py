"""Guard bytes around every buffer a kernel writes (the stand-in for a
device memory checker, which this pool does not offer).

Each output, state pool, conv-state pool and low-rank window is allocated
with 4 KB of sentinel bytes on either side (helpers.Guarded); after the call
every sentinel must be unchanged, and the call's results must still match
the fp64 oracle.  The cases are the ones whose indexing reaches the ends of
the buffers: the last slot of a pool, padding rows, out-of-range slots,
ragged prompt ends, every kernel variant (token loop, block form, 16-bit
pools, speculative commit and snapshots, fused, prefill, low-rank)."""
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import Guarded, STATE_TOL, assert_out_close, f64, oracle_decode, state_rel_err, to_dev

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,state_dtype", [(1, torch.float32), (3, torch.float32),
                                           (6, torch.float32), (1, torch.bfloat16),
                                           (2, torch.float16), (2, torch.bfloat16),
                                           (4, torch.bfloat16)])
def test_decode_writes_stay_inside_out_and_state(T, state_dtype):
    w = inputs.DecodeWorkload("g", B=5, H=3, dk=128, dv=128, T=T, n_slots=7, slots="perm",
                              state_dtype=state_dtype)
    inp = inputs.decode_inputs(w, seed=T)
    # the pool's last slot first (the top end of the pool) and a padding row
    inp["slot_idx"] = torch.tensor([6, 2, 0, 4, -1], dtype=torch.int32)
    d = to_dev(inp)
    out = Guarded(torch.empty((w.B, T, w.H, w.dv)))
    st = Guarded(inp["state"])
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st.t, d["slot_idx"], out.t)
    out.check("out")
    st.check("state")
    if state_dtype == torch.float32:
        o_ref, s_ref, _ = oracle_decode(inp)
        assert_out_close(out.t, o_ref)
        assert state_rel_err(f64(st.t), s_ref) <= STATE_TOL


@pytest.mark.parametrize("dim,state_dtype", [(64, torch.float32), (128, torch.bfloat16)])
def test_decode_bad_slots_and_speculative_paths_stay_inside(dim, state_dtype):
    """dk = dv = 64 on an fp32 pool (the token loop and the block form), and
    128 on a bf16 pool (the tensor-core block form, whose tile goes back by
    TMA; the snapshots take the token loop)."""
    w = inputs.DecodeWorkload("g", B=6, H=2, dk=dim, dv=dim, T=4, n_slots=16,
                              state_dtype=state_dtype)
    inp = inputs.decode_inputs(w, seed=9)
    inp["slot_idx"] = torch.tensor([0, 15, -1, 99, -7, 3], dtype=torch.int32)
    d = to_dev(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = Guarded(torch.empty((w.B, w.T, w.H, w.dv)))
    st = Guarded(inp["state"])
    n_acc = torch.tensor([4, 2, 1, 0, 3, 4], dtype=torch.int32, device="cuda")
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st.t, d["slot_idx"], out.t,
                       n_accept=n_acc, dev_status=status)
    out.check("out")
    st.check("state")
    tok = torch.tensor([[4, 5, 6, 15], [7, -1, 8, 9], [-1, -1, -1, -1], [10, 11, 12, 13],
                        [-1, 14, -1, -1], [1, 2, -1, -1]], dtype=torch.int32, device="cuda")
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], st.t,
                       torch.tensor([0, -1, -1, -1, -1, 3], dtype=torch.int32, device="cuda"),
                       out.t, token_slots=tok)
    out.check("out")
    st.check("state")
    assert gdn.get_error(status)[0] == gdn.ERR_SLOT_RANGE


def test_fused_writes_stay_inside_out_state_and_conv_state():
    fw = inputs.FusedWorkload("g", B=6, Hk=2, H=6, dk=128, dv=128, pad_frac=0.2)
    fi = inputs.fused_inputs(fw, seed=2)
    s = fi["slot_idx"].clone()
    s[s >= 0] = torch.flip(s[s >= 0], dims=[0])  # the last slot in the first active row
    fi["slot_idx"] = s
    st_ref, cs_ref = f64(fi["state"]).copy(), f64(fi["conv_state"]).copy()
    o_ref, _ = oracle.fused_step(f64(fi["mixed_x"]), cs_ref, f64(fi["conv_w"]), f64(fi["a"]),
                                 f64(fi["b"]), f64(fi["A_log"]), f64(fi["dt_bias"]),
                                 f64(fi["z"]), f64(fi["norm_w"]), st_ref,
                                 fi["slot_idx"].numpy(), Hk=fw.Hk, H=fw.H, dk=fw.dk, dv=fw.dv)
    d = to_dev(fi)
    out = Guarded(torch.empty((fw.B, fw.H, fw.dv)))
    st = Guarded(fi["state"])
    cs = Guarded(fi["conv_state"])
    gdn.fused_decode_step(d["mixed_x"], cs.t, d["conv_w"], d["a"], d["b"], d["A_log"],
                          d["dt_bias"], d["z"], d["norm_w"], st.t, d["slot_idx"], out.t,
                          Hk=fw.Hk, H=fw.H, dk=fw.dk, dv=fw.dv)
    for g, name in ((out, "out"), (st, "state"), (cs, "conv_state")):
        g.check(name)
    assert_out_close(out.t, o_ref)
    assert state_rel_err(f64(st.t), st_ref) <= STATE_TOL


@pytest.mark.parametrize("dk,dv,in_dtype", [(128, 128, torch.bfloat16), (64, 128, torch.float32),
                                            (128, 64, torch.bfloat16)])
def test_prefill_writes_stay_inside_out_and_state(dk, dv, in_dtype):
    w = inputs.PrefillWorkload("g", lens=(65, 1, 130, 63), H=3, Hk=1, dk=dk, dv=dv,
                               in_dtype=in_dtype, n_slots=6)
    inp = inputs.prefill_inputs(w, seed=dk + dv)
    inp["slot_idx"] = torch.tensor([5, 0, -1, 2], dtype=torch.int32)
    st_ref = f64(inp["state"]).copy()
    o_ref, _ = oracle.prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                              f64(inp["beta"]), st_ref, inp["slot_idx"].numpy(),
                              inp["cu_seqlens"].numpy())
    d = to_dev(inp)
    out = Guarded(torch.zeros((w.total, w.H, w.dv)))
    st = Guarded(inp["state"])
    # exactly the size the call needs for its input dtype, so that a write past
    # the part the kernels use shows in the guard
    ws_bytes = gdn.prefill_workspace_size(w.N, w.total, w.H, w.dk, w.dv, in_dtype)
    ws = Guarded(torch.zeros(ws_bytes, dtype=torch.uint8))
    gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], st.t, d["slot_idx"],
                      d["cu_seqlens"], out.t, workspace=ws.t)
    for g, name in ((out, "out"), (st, "state"), (ws, "workspace")):
        g.check(name)
    assert_out_close(out.t, o_ref)
    assert state_rel_err(f64(st.t), st_ref) <= STATE_TOL


@pytest.mark.parametrize("R", [8, 64])
def test_lowrank_writes_stay_inside_the_window_pools(R):
    w = inputs.DecodeWorkload("g", B=4, H=2, dk=128, dv=128, T=2, n_slots=5)
    inp = inputs.decode_inputs(w, seed=R, with_state=False)
    inp["slot_idx"] = torch.tensor([4, -1, 0, 2], dtype=torch.int32)
    win = inputs.lowrank_window(w, R, seed=R)
    win["win_count"][0, 0] = 1  # one head of a window that is not full yet
    ref = [f64(win[x]).copy() for x in ("win_k", "win_u", "win_c")]
    ref.append(win["win_count"].numpy().copy())
    o_ref, _ = oracle.lowrank_decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                          f64(inp["g"]), f64(inp["beta"]), *ref,
                                          inp["slot_idx"].numpy())
    d = to_dev(inp)
    g = [Guarded(win[x]) for x in ("win_k", "win_u", "win_c", "win_count")]
    out = Guarded(torch.empty((w.B, w.T, w.H, w.dv)))
    gdn.lowrank_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], *[x.t for x in g],
                            d["slot_idx"], out.t)
    for x, name in zip(g + [out], ("win_k", "win_u", "win_c", "win_count", "out")):
        x.check(name)
    assert_out_close(out.t, o_ref)
    assert torch.equal(g[3].t.cpu(), torch.from_numpy(ref[3]))
