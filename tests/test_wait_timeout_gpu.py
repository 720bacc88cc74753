"""The timeout branches of the library's bounded waits, driven on the GPU
without a fault.

The multi-token block forms (calls of 2..4 tokens on an fp32 pool, and on a
bf16 pool the tensor-core form, whose tile comes by TMA), the single-token
kernel on 16-bit pools and the low-rank kernel wait for their own copy into
shared memory, for at most a set time, and on running out set
GDN_STATUS_TIMEOUT, leave the state as it was and return.  A test build of the library (see
_build.WAIT_TEST_DEFINES) shortens the limit to 200 us and makes those waits
expect 16 bytes more than their copy delivers: every byte lands, in bounds,
but the wait's mbarrier phase never completes, so the wait runs out.  The
tests check the status word, that the pools are untouched and that the
context stays usable afterwards (the shipped library then runs normally)."""
import pytest
import torch

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import _build, inputs
from helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wait_test_lib():
    return gdn.load_library(_build.build_wait_test_library())


def test_block_form_wait_runs_out_and_leaves_the_state(wait_test_lib, monkeypatch):
    w = inputs.DecodeWorkload("to", B=2, H=2, dk=128, dv=128, T=4, n_slots=3)
    d = to_dev(inputs.decode_inputs(w, seed=1))
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setattr(gdn, "_lib", wait_test_lib)
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                       dev_status=status)
    torch.cuda.synchronize()
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_TIMEOUT and bits == gdn.STATUS_TIMEOUT
    assert torch.equal(d["state"], pre)
    # single-token calls take no bulk copy: the test build runs them normally
    status.zero_()
    d1 = to_dev(inputs.decode_inputs(inputs.shrink(w, T=1), seed=2))
    gdn.decode_step_ex(d1["q"], d1["k"], d1["v"], d1["g"], d1["beta"], d["state"],
                       d1["slot_idx"], dev_status=status)
    torch.cuda.synchronize()
    assert gdn.get_error(status) == (gdn.OK, 0)
    assert not torch.equal(d["state"], pre)


def test_tensor_core_block_form_wait_runs_out_and_leaves_the_state(wait_test_lib, monkeypatch):
    """bf16 pool, four tokens, dk = dv = 128: the tile's TMA wait runs out
    (the tensor memory is released, no product was issued)."""
    w = inputs.DecodeWorkload("to", B=3, H=2, dk=128, dv=128, T=4, n_slots=4,
                              state_dtype=torch.bfloat16)
    d = to_dev(inputs.decode_inputs(w, seed=6))
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setattr(gdn, "_lib", wait_test_lib)
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                       dev_status=status)
    torch.cuda.synchronize()
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_TIMEOUT and bits == gdn.STATUS_TIMEOUT
    assert torch.equal(d["state"], pre)


@pytest.mark.parametrize("state_dtype", [torch.bfloat16, torch.float16])
def test_staged_16bit_wait_runs_out_and_leaves_the_state(wait_test_lib, monkeypatch, state_dtype):
    w = inputs.DecodeWorkload("to", B=2, H=2, dk=128, dv=128, T=1, n_slots=3,
                              state_dtype=state_dtype)
    d = to_dev(inputs.decode_inputs(w, seed=4))
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setattr(gdn, "_lib", wait_test_lib)
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                       dev_status=status)
    torch.cuda.synchronize()
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_TIMEOUT and bits == gdn.STATUS_TIMEOUT
    assert torch.equal(d["state"], pre)


@pytest.mark.parametrize("R", [16, 64])
def test_lowrank_wait_runs_out_and_leaves_the_window(wait_test_lib, monkeypatch, R):
    w = inputs.DecodeWorkload("to", B=3, H=2, dk=128, dv=128, T=1, n_slots=3)
    inp = inputs.decode_inputs(w, seed=R, with_state=False)
    win = to_dev(inputs.lowrank_window(w, R, seed=R))
    pre = {k: v.clone() for k, v in win.items()}
    d = to_dev(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setattr(gdn, "_lib", wait_test_lib)
    gdn.lowrank_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], win["win_k"],
                            win["win_u"], win["win_c"], win["win_count"], d["slot_idx"],
                            dev_status=status)
    torch.cuda.synchronize()
    rc, bits = gdn.get_error(status)
    assert rc == gdn.ERR_TIMEOUT and bits == gdn.STATUS_TIMEOUT
    for k in win:
        assert torch.equal(win[k], pre[k]), k


def test_shipped_library_runs_normally_after_the_timeouts(wait_test_lib):
    """The context survives: the shipped library's block form completes."""
    w = inputs.DecodeWorkload("to", B=2, H=2, dk=128, dv=128, T=4, n_slots=3)
    d = to_dev(inputs.decode_inputs(w, seed=1))
    pre = d["state"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["slot_idx"],
                       dev_status=status)
    torch.cuda.synchronize()
    assert gdn.get_error(status) == (gdn.OK, 0)
    assert not torch.equal(d["state"], pre)
