"""Host-side arithmetic of bench.py, no GPU: the algorithmic byte counts the
roofline divides by (checked against the figures written out from the
workloads' shapes), the kernel each workload's launch runs, the whole-job
throughput and the config block of the JSON line."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_serving_step_bytes():
    # 256 sequences x 48 heads of 128 x 128 fp32 state read and written, bf16
    # q, k, v, fp32 g and beta, the int32 slot map and fp32 out
    state = 2 * 256 * 48 * 128 * 128 * 4
    assert state == 805_306_368 * 2
    qkv = 256 * (2 * 48 * 128 + 48 * 128) * 2
    gb = 256 * 48 * 8
    total = state + qkv + gb + 256 * 4 + 256 * 48 * 128 * 4
    assert total == 1_626_440_704
    assert bench.algorithmic_bytes_per_launch(256, 48, 48, 128, 128, 1, 256) == total


def test_layer_and_mtp_bytes():
    assert bench.algorithmic_bytes_per_launch(64, 48, 48, 128, 128, 1, 64) == 406_610_176
    # T = 4: the state moves once, the per-token inputs and outputs four times
    assert bench.algorithmic_bytes_per_launch(128, 48, 48, 128, 128, 4, 128) == 836_960_768


def test_padding_rows_move_no_state():
    full = bench.algorithmic_bytes_per_launch(8, 4, 4, 128, 128, 1, 8)
    padded = bench.algorithmic_bytes_per_launch(8, 4, 4, 128, 128, 1, 6)
    assert full - padded == 2 * 2 * 4 * 128 * 128 * 4


def test_sixteen_bit_pools_halve_the_state_bytes():
    f32 = bench.algorithmic_bytes_per_launch(256, 48, 48, 128, 128, 1, 256)
    b16 = bench.algorithmic_bytes_per_launch(256, 48, 48, 128, 128, 1, 256, state_bytes=2)
    assert f32 - b16 == 256 * 48 * 128 * 128 * 4


@pytest.mark.parametrize("name,state,label", [
    ("serving", "f32", "gdn::decode_kernel"),
    ("mtp", "f32", "gdn::decode_block_smem_kernel"),
    ("mtp", "bf16", "gdn::decode_block_tc16_kernel"),
    ("mtp", "f16", "gdn::decode_block_tc16_kernel"),
    ("serving", "bf16", "gdn::decode_staged16_kernel"),
    ("serving", "f16", "gdn::decode_staged16_kernel"),
    ("tiny", "f32", "gdn::decode_kernel"),
    ("fused", "f32", "gdn::fused_kernel"),
    ("lowrank", "f32", "gdn::lowrank_kernel"),
])
def test_kernel_label_follows_the_call_shape(name, state, label):
    wl = bench.workloads(state)[name] if state != "f32" else bench.workloads()[name]
    assert bench.decode_kernel_label(wl, state) == label


def test_weak_scaling_value_counts_every_rank():
    # 2 ranks x 12,288 units x 10 steps in 100 ms (the slowest rank)
    assert bench.weak_scaling_value(12_288, 10, 2, 100.0) == pytest.approx(2_457_600.0)


def test_config_names_the_workload_and_its_shape():
    wl = bench.workloads()["serving"]
    c = bench.workload_config(wl, 48, 1, "graph")
    assert "B=256" in c["workload"] and "48 layers" in c["workload"]
    assert (c["B"], c["H"], c["dk"], c["dv"], c["T"], c["layers"]) == (256, 48, 128, 128, 1, 48)
    assert c["n_slots"] == 512 and c["state_dtype"] == "float32"
    assert "model" not in c


def test_measured_peaks_are_read_from_the_file(tmp_path):
    f = tmp_path / "peaks.json"
    f.write_text('{"hbm_gbs": 6540.2, "bf16_tflops": 1632.8, "bf16_tflops_sustained": 1373.9}')
    peaks, source = bench.measured_peaks(str(f))
    assert source == "measured"
    assert peaks == {"hbm_gbs": 6540.2, "bf16_tflops": 1632.8, "bf16_tflops_sustained": 1373.9}
    assert bench.measured_peak(str(f)) == (6540.2, "measured")


def test_measured_peaks_fall_back_when_the_file_is_absent(tmp_path):
    peaks, source = bench.measured_peaks(str(tmp_path / "absent.json"))
    assert source == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_groups_split_the_timed_steps():
    assert bench.group_bounds(100, 7) == [0, 14, 28, 42, 57, 71, 85, 100]
    assert bench.group_bounds(3, 7) == [0, 1, 2, 3]
    s = bench.spread([2.0, 1.0, 3.0, 2.5, 1.5])
    assert s == {"groups": 5, "median_ms_per_step": 2.0, "min_ms_per_step": 1.0,
                 "max_ms_per_step": 3.0}


def test_recorded_traffic_needs_the_current_sources(tmp_path):
    import json
    wl = bench.workloads()["serving"]
    rec = {"entries": {"serving/f32": {"kernel": "gdn::decode_kernel", "units_per_launch": 100,
                                        "dram_bytes_per_launch": 5000,
                                        "source_hash": bench.kernel_source_hash("decode")}}}
    f = tmp_path / "t.json"
    f.write_text(json.dumps(rec))
    b, src = bench.recorded_traffic(wl, "f32", 200, path=str(f))
    assert b == 10000 and "ncu" in src
    rec["entries"]["serving/f32"]["source_hash"] = "stale"
    f.write_text(json.dumps(rec))
    assert bench.recorded_traffic(wl, "f32", 200, path=str(f))[0] is None
    assert bench.recorded_traffic(wl, "bf16", 200, path=str(f))[0] is None


def test_threaded_oracle_sample_counts_every_thread():
    wl = bench.workloads()["tiny"]
    v1, s1, _ = bench.cpu_oracle_sample(0.0, wl, max_calls=2, threads=1)
    v2, s2, _ = bench.cpu_oracle_sample(0.0, wl, max_calls=2, threads=2)
    assert v1 > 0 and v2 > 0
    assert "1 thread" in s1 and "2 threads" in s2 and "4 oracle calls" in s2


def test_host_cpu_names_the_model_and_cores():
    model, cores = bench.host_cpu()
    assert isinstance(model, str) and cores >= 1


def test_prefill_roofline_counts_the_split_operand_products():
    """Per chunk of 64 tokens and head (dk = dv = 128): 10,573,141 algorithmic
    flops (Gram products 2 x 2,097,152 / 2, solve 87,381, K S and Q S
    4,194,304, T R and P Delta 2,097,152, K^T Delta 2,097,152) and 32,505,856
    bf16 MMA flops executed (the two M = 128 Gram passes, S in 3 parts, T R
    in 6 part pairs, P Delta in 3, K^T Delta' in 3).  frac is the executed
    rate over the measured bf16 peak."""
    wl = bench.workloads()["prefill"]
    chunks = sum((L + 63) // 64 for L in wl.spec.lens)
    assert chunks == 300
    assert wl.flops_per_launch() == pytest.approx(chunks * 48 * (10_485_760 + 64 ** 3 / 3))
    assert wl.tensor_flops_per_launch() == chunks * 48 * 32_505_856
    peaks = ({"hbm_gbs": 6540.2, "bf16_tflops": 1632.8, "bf16_tflops_sustained": 1373.9},
             "measured")
    r = bench.prefill_roofline(wl, 2e-3, 1.0e9, peaks=peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(wl.tensor_flops_per_launch() / 2e-3 / 1e12 / 1632.8,
                                      rel=1e-3)
    assert r["achieved"] == pytest.approx(wl.flops_per_launch() / 2e-3 / 1e12, rel=1e-3)


def test_lowrank_prefill_counts():
    """Per chunk of 64 tokens and head at R = 16, dk = dv = 128: 5,330,261
    flops (q k^T and k k^T 2 x 2,097,152 / 2 ... as the chunk form computes
    them) and the bytes of the inputs, the outputs and each head's window
    read and written once."""
    wl = bench.workloads()["lowrank_prefill"]
    wl.rank = 16
    C, dk, R = 64, 128, 16
    per = 4 * C * C * dk + 4 * C * R * dk + C ** 3 / 3 + 4 * C * R * dk + 4 * C * C * dk
    assert wl.lowrank_prefill_flops_per_launch() == pytest.approx(300 * 48 * per)
    w = wl.spec
    window = R * (dk + dk + 1) * 4 + 4
    want = (w.total * 3 * 48 * 128 * 2 + w.total * 48 * 8 + 2 * 8 * 48 * window
            + w.total * 48 * 128 * 4 + 9 * 4 + 8 * 4)
    assert wl.bytes_per_launch(8) == want
    assert bench.decode_kernel_label(wl, "f32") == "gdn::lowrank_prefill_kernel"
    assert bench.traffic_key(wl, "f32", 16) == "lowrank_prefill/f32/R16"
