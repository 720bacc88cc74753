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
    ("mtp", "bf16", "gdn::decode_kernel"),
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


def test_measured_peak_is_read_from_the_file():
    peak, source = bench.measured_peak()
    assert source == "measured" and peak > 1000.0
