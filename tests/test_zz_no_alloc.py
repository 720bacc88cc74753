"""The allocation-free prefill entry point, gdn_chunk_prefill_noalloc.

Some callers cannot hand the library a workspace (their device memory is
planned and owned elsewhere, or the call sits on a path that must not
allocate); this entry point gives them the chunked prefill with a scratch
array built into the library instead.  Called through the C ABI, it must
give the results of gdn_chunk_prefill with a workspace, within the parity
tolerances of the other tests, on two calls in a row (the second call
reuses the scratch the first one left behind), and it must refuse a
request larger than its scratch with a clear error.
"""
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import inputs
from helpers import STATE_TOL, assert_out_close, f64, state_rel_err, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20


def test_noalloc_prefill_matches_workspace_prefill_on_two_calls():
    w = inputs.PrefillWorkload("na", lens=(100, 37, 64, 129), H=6, Hk=3, dk=128, dv=128)
    assert gdn.prefill_workspace_size(w.N, w.total, w.H, w.dk, w.dv) <= SCRATCH_BYTES
    first = to_dev(inputs.prefill_inputs(w, seed=11))
    st_ref = first["state"].clone()
    st_na = first["state"].clone()
    for call, seed in enumerate((11, 12)):
        d = first if call == 0 else to_dev(inputs.prefill_inputs(w, seed=seed))
        out_ref = torch.empty((w.total, w.H, w.dv), device="cuda")
        out_na = torch.empty((w.total, w.H, w.dv), device="cuda")
        gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], st_ref, d["slot_idx"],
                          d["cu_seqlens"], out_ref)
        gdn.chunk_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], st_na,
                                  d["slot_idx"], d["cu_seqlens"], out_na)
        torch.cuda.synchronize()
        assert_out_close(out_na, f64(out_ref))
        assert state_rel_err(f64(st_na), f64(st_ref)) <= STATE_TOL


def test_noalloc_prefill_refuses_requests_beyond_its_scratch():
    w = inputs.PrefillWorkload("big", lens=(64 * 200,), H=4, dk=128, dv=128)
    assert gdn.prefill_workspace_size(w.N, w.total, w.H, w.dk, w.dv) > SCRATCH_BYTES
    d = to_dev(inputs.prefill_inputs(w))
    out = torch.empty((w.total, w.H, w.dv), device="cuda")
    with pytest.raises(gdn.GdnError) as e:
        gdn.chunk_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                  d["slot_idx"], d["cu_seqlens"], out)
    assert e.value.code == gdn.ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
