"""The seeded input generators: deterministic, correctly shaped, valid slot maps."""
import torch

from gated_deltanet_recurrent_gdn_b200 import inputs


def test_decode_inputs_deterministic_and_shaped():
    w = inputs.shrink(inputs.LAYER, B=3, H=5)
    a = inputs.decode_inputs(w, seed=0)
    b = inputs.decode_inputs(w, seed=0)
    c = inputs.decode_inputs(w, seed=1)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert not torch.equal(a["q"], c["q"])
    assert a["q"].shape == (3, 1, 5, 128) and a["q"].dtype == torch.bfloat16
    assert a["v"].shape == (3, 1, 5, 128)
    assert a["g"].shape == (3, 1, 5) and a["g"].dtype == torch.float32
    assert float(a["g"].max()) <= 0.0 and float(a["g"].min()) >= -0.5
    assert 0.0 < float(a["beta"].min()) and float(a["beta"].max()) < 1.0
    assert a["state"].shape == (3, 5, 128, 128)
    assert torch.equal(a["slot_idx"], torch.arange(3, dtype=torch.int32))


def test_tiny_is_fp32():
    a = inputs.decode_inputs(inputs.TINY)
    assert a["q"].dtype == torch.float32 and a["q"].shape == (1, 8, 4, 128)


def test_serving_slot_map_is_a_partial_permutation():
    w = inputs.shrink(inputs.SERVING, H=1, dk=64, dv=64)
    a = inputs.decode_inputs(w, with_state=False)
    s = a["slot_idx"]
    assert s.shape == (256,) and s.dtype == torch.int32
    assert len(set(s.tolist())) == 256
    assert int(s.min()) >= 0 and int(s.max()) < 512
    assert not torch.equal(s, torch.arange(256, dtype=torch.int32))


def test_fused_inputs_padding_rows():
    w = inputs.shrink(inputs.FUSED, H=3, Hk=1, dk=64, dv=64)
    a = inputs.fused_inputs(w)
    s = a["slot_idx"]
    assert int((s == -1).sum()) == 26
    keep = s[s >= 0]
    assert len(set(keep.tolist())) == keep.numel()
    assert a["mixed_x"].shape == (256, w.C) and w.C == 2 * 64 + 3 * 64
    assert a["conv_state"].shape == (256, w.C, 3)
    assert a["conv_w"].shape == (w.C, 4) and a["conv_w"].dtype == torch.float32
    assert float(a["A_log"].min()) >= 0.0 and float(a["A_log"].max()) <= torch.log(torch.tensor(16.0))
    assert inputs.FUSED.C == 10240


def test_prefill_inputs_packed_and_seeded():
    w = inputs.PrefillWorkload("t", lens=(70, 5, 129), H=3, Hk=1, dk=64, dv=128)
    a = inputs.prefill_inputs(w, seed=2)
    b = inputs.prefill_inputs(w, seed=2)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert a["q"].shape == (204, 1, 64) and a["q"].dtype == torch.bfloat16
    assert a["v"].shape == (204, 3, 128)
    assert a["cu_seqlens"].tolist() == [0, 70, 75, 204]
    assert a["cu_seqlens"].dtype == torch.int32 and a["slot_idx"].tolist() == [0, 1, 2]
    assert a["state"].shape == (3, 3, 128, 64)
    assert float(a["g"].max()) <= 0.0 and float(a["g"].min()) >= -0.5
    assert 0.0 < float(a["beta"].min()) and float(a["beta"].max()) < 1.0


def test_benchmark_prefill_mix():
    w = inputs.PREFILL
    assert w.N == 8 and w.total == 19_101
    assert min(w.lens) == 777 and max(w.lens) == 4096
    # 64-token chunks: 300 of them; the workspace (and phase A's grid) reserves
    # the bound total // 64 + N + 1 = 307 chunk slots per head
    assert sum((L + 63) // 64 for L in w.lens) == 300
    assert w.total // 64 + w.N + 1 == 307


def test_lowrank_window_is_full_and_unit_norm():
    w = inputs.shrink(inputs.LAYER, B=2, H=3, n_slots=2)
    d = inputs.lowrank_window(w, R=16, seed=0)
    assert d["win_k"].shape == (2, 3, 16, 128) and d["win_u"].shape == (2, 3, 16, 128)
    assert torch.allclose(d["win_k"].norm(dim=-1), torch.ones(2, 3, 16), atol=1e-5)
    assert float(d["win_c"].min()) >= 0.05 and float(d["win_c"].max()) <= 1.0
    assert bool((d["win_count"] > 16).all())
