"""The C-ABI library loads, exports every symbol include/gdn.h declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import gated_deltanet_recurrent_gdn_b200 as gdn
from gated_deltanet_recurrent_gdn_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    _build.build_library()
    return gdn.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_rebuild_check_watches_every_kernel_source():
    """A change to any source or header the library is compiled from makes
    the in-tree library stale, so the next load rebuilds it."""
    sources = [os.path.join(_build.CSRC, f) for f in os.listdir(_build.CSRC)
               if f.endswith((".cu", ".cuh", ".h"))]
    assert sources
    for f in sources + [HEADER]:
        assert f in _build.DEPS, f


def test_header_declares_the_abi():
    syms = declared_symbols()
    assert syms == sorted(gdn.EXPORTED_SYMBOLS), syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for s in declared_symbols():
        assert s in exported, s
        assert hasattr(lib, s)
    # nothing else with C linkage leaks out under the gdn_ prefix
    assert {s for s in exported if s.startswith("gdn_")} == set(declared_symbols())


def test_library_is_built_for_sm100a_only(lib):
    # the build line pins the architecture; the ELF carries no host fallback
    assert "arch=compute_100a,code=sm_100a" in " ".join(_build.NVCC_FLAGS)


def test_version(lib):
    assert lib.gdn_version() == 10000


def _args(**kw):
    a = gdn.StepArgs()
    fake = 0x10000  # 16-byte aligned, never dereferenced by host validation
    a.q = a.k = a.v = a.g = a.beta = a.state = a.slot_idx = a.out = fake
    a.B, a.Hk, a.H, a.dk, a.dv, a.T, a.n_slots = 2, 4, 4, 128, 128, 1, 2
    a.in_dtype, a.out_dtype, a.state_dtype = gdn.BF16, gdn.F32, gdn.F32
    a.scale, a.qk_l2norm, a.l2_eps = 0.0, 1, 1e-6
    a.dev_status, a.check_slots, a.stream = None, 0, None
    a.n_accept, a.token_slots = None, None
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=96), gdn.ERR_UNSUPPORTED),
    (dict(dv=32), gdn.ERR_UNSUPPORTED),
    (dict(T=0), gdn.ERR_UNSUPPORTED),
    (dict(T=9), gdn.ERR_UNSUPPORTED),
    (dict(H=6, Hk=4), gdn.ERR_ARG),
    (dict(Hk=0), gdn.ERR_ARG),
    (dict(B=-1), gdn.ERR_ARG),
    (dict(in_dtype=7), gdn.ERR_ARG),
    (dict(in_dtype=gdn.F16), gdn.ERR_ARG),
    (dict(state_dtype=3), gdn.ERR_ARG),
    (dict(q=None), gdn.ERR_ARG),
    (dict(state=None), gdn.ERR_ARG),
    (dict(out=0x10004), gdn.ERR_ARG),
    (dict(v=0x10008), gdn.ERR_ARG),
    (dict(g=0x10002), gdn.ERR_ARG),
    (dict(n_accept=0x10000, token_slots=0x10010, T=2), gdn.ERR_ARG),
    (dict(n_accept=0x10002), gdn.ERR_ARG),
])
def test_host_validation_rejects(lib, kw, code):
    a = _args(**kw)
    rc = lib.gdn_decode_step_ex(ctypes.byref(a))
    assert rc == code
    assert lib.gdn_last_error_string()


def test_empty_batch_is_a_noop(lib):
    a = _args(B=0, q=None, k=None, v=None, state=None)
    assert lib.gdn_decode_step_ex(ctypes.byref(a)) == gdn.OK


def test_null_args_struct(lib):
    assert lib.gdn_decode_step_ex(None) == gdn.ERR_ARG


def test_simple_entry_validates_too(lib):
    f = 0x10000
    assert lib.gdn_decode_step(f, f, f, f, f, f, f, f, 1, 4, 100, 128, 1, None) == gdn.ERR_UNSUPPORTED
    assert lib.gdn_decode_step(None, f, f, f, f, f, f, f, 1, 4, 128, 128, 1, None) == gdn.ERR_ARG
    assert lib.gdn_decode_step(None, None, None, None, None, None, None, None, 0, 4, 128, 128, 1,
                               None) == gdn.OK


def _fused(lib, **kw):
    f = 0x10000
    args = dict(mixed_x=f, conv_state=f, conv_w=f, w_dtype=gdn.F32, a=f, b=f, A_log=f,
                dt_bias=f, z=f, norm_w=f, norm_eps=1e-6, state=f, slot_idx=f, out=f, B=2,
                Hk=16, H=48, dk=128, dv=128, n_slots=4, out_dtype=gdn.F32, status=None,
                stream=None)
    args.update(kw)
    return lib.gdn_fused_decode_step(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(H=40), gdn.ERR_ARG),
    (dict(Hk=1, H=16), gdn.ERR_UNSUPPORTED),   # group 16 > 8
    (dict(dk=32), gdn.ERR_UNSUPPORTED),
    (dict(n_slots=0), gdn.ERR_ARG),
    (dict(mixed_x=None), gdn.ERR_ARG),
    (dict(conv_w=0x10008), gdn.ERR_ARG),
    (dict(out_dtype=5), gdn.ERR_ARG),
    (dict(norm_eps=-1.0), gdn.ERR_ARG),
])
def test_fused_host_validation_rejects(lib, kw, code):
    assert _fused(lib, **kw) == code


def test_fused_empty_batch_is_a_noop(lib):
    assert _fused(lib, B=0, mixed_x=None) == gdn.OK


def test_get_error_null(lib):
    assert lib.gdn_get_error(None, None) == gdn.ERR_ARG


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.decode_step(q, q, q, torch.zeros(1, 1, 4), torch.zeros(1, 1, 4),
                        torch.zeros(1, 4, 128, 128), torch.zeros(1, dtype=torch.int32))


def test_prefill_workspace_size(lib):
    one = lib.gdn_prefill_workspace_size(1, 64, 1, 128, 128)
    assert one > 0 and one % 16 == 0
    # an upper bound over any split of the tokens: grows with N and tokens
    assert lib.gdn_prefill_workspace_size(4, 64, 1, 128, 128) > one
    assert lib.gdn_prefill_workspace_size(1, 640, 1, 128, 128) > one
    assert lib.gdn_prefill_workspace_size(1, 64, 48, 128, 128) == 48 * one
    assert lib.gdn_prefill_workspace_size(1, 64, 1, 96, 128) == 0


def test_prefill_workspace_size_by_input_dtype(lib):
    """bf16 inputs at dk = dv = 128 keep only the chunk's (I + A)^-1 (64 x 64
    fp32) per chunk slot and head; fp32 inputs keep the general path's chunk
    matrices; the dtype-free size covers both."""
    ex = lib.gdn_prefill_workspace_size_ex
    slots = 64 // 64 + 1 + 1
    assert ex(1, 64, 1, 128, 128, gdn.BF16) == slots * 64 * 64 * 4
    assert ex(1, 64, 1, 128, 128, gdn.F32) > ex(1, 64, 1, 128, 128, gdn.BF16)
    assert lib.gdn_prefill_workspace_size(1, 64, 1, 128, 128) == ex(1, 64, 1, 128, 128, gdn.F32)
    for dk, dv in ((64, 64), (128, 64), (64, 128)):
        assert ex(2, 300, 3, dk, dv, gdn.BF16) == ex(2, 300, 3, dk, dv, gdn.F32)
    assert ex(1, 64, 1, 128, 128, 7) == 0


def _prefill_args(**kw):
    a = gdn.PrefillArgs()
    f = 0x10000
    a.q = a.k = a.v = a.g = a.beta = a.state = a.slot_idx = a.cu_seqlens = a.out = f
    a.N, a.total_tokens, a.Hk, a.H, a.dk, a.dv, a.n_slots = 2, 100, 4, 4, 128, 128, 2
    a.in_dtype, a.out_dtype = gdn.BF16, gdn.F32
    a.scale, a.qk_l2norm, a.l2_eps, a.initial_state = 0.0, 1, 1e-6, 1
    a.workspace = f
    a.workspace_bytes = 1 << 40
    a.dev_status, a.stream = None, None
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=32), gdn.ERR_UNSUPPORTED),
    (dict(H=6), gdn.ERR_ARG),
    (dict(N=-1), gdn.ERR_ARG),
    (dict(n_slots=0), gdn.ERR_ARG),
    (dict(workspace=None), gdn.ERR_ARG),
    (dict(workspace_bytes=1024), gdn.ERR_ARG),
    (dict(cu_seqlens=0x10002), gdn.ERR_ARG),
    (dict(out_dtype=9), gdn.ERR_ARG),
])
def test_prefill_host_validation_rejects(lib, kw, code):
    a = _prefill_args(**kw)
    assert lib.gdn_chunk_prefill(ctypes.byref(a)) == code
    assert lib.gdn_last_error_string()


def test_prefill_no_sequences_is_a_noop(lib):
    a = _prefill_args(N=0, q=None, workspace=None)
    assert lib.gdn_chunk_prefill(ctypes.byref(a)) == gdn.OK


@pytest.mark.parametrize("kw,code", [
    (dict(dk=32), gdn.ERR_UNSUPPORTED),
    (dict(H=6), gdn.ERR_ARG),
    (dict(N=-1), gdn.ERR_ARG),
    (dict(n_slots=0), gdn.ERR_ARG),
    (dict(cu_seqlens=0x10002), gdn.ERR_ARG),
    (dict(out_dtype=9), gdn.ERR_ARG),
    (dict(q=None), gdn.ERR_ARG),
    # argument errors come first even when the request is also too large for
    # the built-in scratch, and even when there is nothing to do (N = 0)
    (dict(H=6, total_tokens=1 << 20), gdn.ERR_ARG),
    (dict(N=0, H=6), gdn.ERR_ARG),
    (dict(N=0, dk=96), gdn.ERR_UNSUPPORTED),
    # a well-formed request beyond the scratch
    (dict(total_tokens=1 << 20), gdn.ERR_UNSUPPORTED),
])
def test_noalloc_prefill_host_validation_matches_the_workspace_entry(lib, kw, code):
    """gdn_chunk_prefill_noalloc checks its arguments exactly as
    gdn_chunk_prefill does (the workspace fields aside), before it looks at
    the size of its built-in scratch."""
    a = _prefill_args(workspace=None, workspace_bytes=0, **kw)
    assert lib.gdn_chunk_prefill_noalloc(ctypes.byref(a)) == code
    assert lib.gdn_last_error_string()
    if "total_tokens" not in kw:
        # the workspace entry point gives the same answer for the same error
        b = _prefill_args(**kw)
        assert lib.gdn_chunk_prefill(ctypes.byref(b)) == code


def test_noalloc_prefill_no_sequences_is_a_noop(lib):
    a = _prefill_args(N=0, q=None, workspace=None, workspace_bytes=0)
    assert lib.gdn_chunk_prefill_noalloc(ctypes.byref(a)) == gdn.OK
