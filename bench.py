#!/usr/bin/env python
"""Benchmark of the batched gated delta rule decode step on B200.

Workload (one "step"): the serving decode step B=256 sequences, H=48 heads,
dk=dv=128, T=1, fp32 state, bf16 q/k/v, called back to back over 48 layers;
each layer has its own 512-slot state pool and slot_idx is a random
permutation of the pool (first 256 entries).  One step moves 48 x 1.61 GB of
state, far more than the 126 MB L2, so no L2 flush is needed between steps.

Printed JSON line (rank 0):
  value      token-heads/s = (layers * B * H * T per step) / device time,
             inputs resident in HBM, the step replayed as a CUDA graph
  e2e        the same metric through the same C-ABI call with host buffers:
             each step copies every layer's inputs from pinned host memory
             and reads every layer's output back, pipelined on 3 streams
  roofline   HBM roofline of the decode kernel (the only kernel in the step)
  cpu_baseline  the fp64 CPU oracle timed on a bounded sample (rank 0, N=1)

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (independent sequences, no data-path collective) and the time
is the max over ranks: weak scaling.

``--impl reference`` times the CPU oracle instead (the only reference
implementation of this path) on the same workload, in bounded samples.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN decode token-heads/s and achieved HBM GB/s (% of 8 TB/s) at B=256,H=48"
UNIT = "token-heads/s"
NOMINAL_HBM_GBS = 8000.0
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
# an earlier measurement on this machine, used only when the file is absent
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA peak of a B200: 148 SMs x 128 fp32 lanes x 2 flop per cycle at the 1965 MHz maximum
# SM clock (the recipe's unit counts and clocks)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
_CSRC = os.path.join(ROOT, "gated_deltanet_recurrent_gdn_b200", "csrc")
# the sources each kernel family is built from (a change to any of them
# makes its recorded DRAM counters stale)
KERNEL_SOURCES = {
    "decode": [os.path.join(_CSRC, f) for f in ("gdn_kernels.cuh", "gdn_prefill.cuh",
                                                 "gdn_prefill_tc.cuh", "gdn_decode_tc.cuh",
                                                 "gdn_api.cu")],
    "fused": [os.path.join(_CSRC, f) for f in ("gdn_kernels.cuh", "gdn_api.cu")],
    "lowrank": [os.path.join(_CSRC, f) for f in ("gdn_kernels.cuh", "gdn_lowrank.cuh",
                                                  "gdn_api.cu")],
    "prefill": [os.path.join(_CSRC, f) for f in ("gdn_kernels.cuh", "gdn_prefill.cuh",
                                                  "gdn_prefill_tc.cuh", "gdn_api.cu")],
    "lowrank_prefill": [os.path.join(_CSRC, f) for f in ("gdn_kernels.cuh", "gdn_prefill.cuh",
                                                          "gdn_lowrank.cuh",
                                                          "gdn_lowrank_prefill.cuh", "gdn_api.cu")],
}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="serving",
                   choices=["serving", "layer", "mtp", "tiny", "fused", "prefill", "lowrank",
                            "lowrank_prefill"],
                   help="serving (the default and the headline) or another workload")
    p.add_argument("--state-dtype", default="f32", choices=["f32", "bf16", "f16"],
                   help="storage type of the state pool (decode workloads; f32 is the headline)")
    p.add_argument("--rank", type=int, default=16, choices=[8, 16, 32, 64],
                   help="window length of the low-rank workload")
    p.add_argument("--layers", type=int, default=0,
                   help="layers per step (0 = the workload's default; fewer only for profiling)")
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=20.0,
                   help="target wall time of all oracle baseline samples together")
    p.add_argument("--groups", type=int, default=7,
                   help="the timed steps are split into this many groups for the spread")
    return p.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def group_bounds(steps: int, groups: int):
    """Step indices at which the timed steps are split into (at most)
    ``groups`` groups of near-equal size: [0, ..., steps]."""
    g = max(1, min(groups, steps))
    return [steps * i // g for i in range(g + 1)]


def spread(per_step_ms):
    """Median, min and max of the per-step time of each group."""
    return {"groups": len(per_step_ms),
            "median_ms_per_step": round(statistics.median(per_step_ms), 4),
            "min_ms_per_step": round(min(per_step_ms), 4),
            "max_ms_per_step": round(max(per_step_ms), 4)}


def weak_scaling_value(units_per_rank_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed its own units; the job took
    as long as its slowest rank."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# bytes and peaks


def algorithmic_bytes_per_launch(B, H, Hk, dk, dv, T, n_active, in_bytes=2, out_bytes=4,
                                 state_bytes=4):
    """State read + write of the active slots, q/k/v, g/beta, slot map, out."""
    state = 2 * n_active * H * dk * dv * state_bytes
    qkv = B * T * (2 * Hk * dk + H * dv) * in_bytes
    gb = B * T * H * 8
    slots = B * 4
    out = B * T * H * dv * out_bytes
    return state + qkv + gb + slots + out


def measured_peaks(path=PEAKS_FILE):
    """(peaks, source): the machine's measured peaks (HBM copy GB/s, bf16 dense
    TFLOP/s as a burst and sustained), or the earlier measurement on this
    pool when the file is absent or unreadable."""
    try:
        with open(path) as f:
            d = json.load(f)
        peaks = {"hbm_gbs": float(d["hbm_gbs"])}
        for key in ("bf16_tflops", "bf16_tflops_sustained"):
            peaks[key] = float(d.get(key, FALLBACK_PEAKS[key]))
        return peaks, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def measured_peak(path=PEAKS_FILE):
    peaks, source = measured_peaks(path)
    return peaks["hbm_gbs"], source


def kernel_source_hash(kind: str = "decode"):
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kind]:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_kernel_label(wl, state_dtype):
    """The kernel one launch of the workload runs (the library picks it by
    the call's shape: calls of 2..4 tokens take the block form, on the CUDA
    cores for an fp32 pool and on the tensor cores for a 16-bit pool with
    dk = dv = 128; single tokens on a 16-bit pool with dk = 128 take the
    staged kernel)."""
    if wl.kind == "fused":
        return "gdn::fused_kernel"
    if wl.kind == "lowrank":
        return "gdn::lowrank_kernel"
    if wl.kind == "prefill":
        return "gdn::prefill_chunk_kernel + gdn::prefill_state_tc_kernel"
    if wl.kind == "lowrank_prefill":
        return "gdn::lowrank_prefill_kernel"
    if 2 <= wl.spec.T <= 4 and state_dtype == "f32":
        return "gdn::decode_block_smem_kernel"
    if 2 <= wl.spec.T <= 4 and state_dtype in ("bf16", "f16") and wl.spec.dk == wl.spec.dv == 128:
        return "gdn::decode_block_tc16_kernel"
    if wl.spec.T == 1 and state_dtype in ("bf16", "f16") and wl.spec.dk == 128:
        return "gdn::decode_staged16_kernel"
    return "gdn::decode_kernel"


def traffic_key(wl, state_dtype, rank=None):
    key = f"{wl.name}/{state_dtype}"
    return key + f"/R{rank}" if wl.kind in ("lowrank", "lowrank_prefill") else key


def recorded_traffic(wl, state_dtype, units_per_launch, path=None):
    """(DRAM bytes per launch, source text) from the committed summary of ncu
    counters for this workload, scaled to this launch's units; (None, why)
    when there is no record or the kernel's sources changed since the
    counters were taken."""
    try:
        with open(path or TRAFFIC_FILE) as f:
            d = json.load(f)
    except Exception:
        return None, "no recorded ncu counters"
    e = d.get("entries", {}).get(traffic_key(wl, state_dtype, getattr(wl, "rank", None)))
    if e is None:
        return None, "no recorded ncu counters for this workload"
    if e.get("source_hash") != kernel_source_hash(wl.kind):
        return None, "kernel sources changed since the ncu counters were taken"
    per_unit = e["dram_bytes_per_launch"] / e["units_per_launch"]
    return (int(round(per_unit * units_per_launch)),
            f"ncu dram__bytes_read.sum + dram__bytes_write.sum recorded in "
            f"profiles/dram_traffic.json ({e.get('capture', 'small-case capture')})")


# ---------------------------------------------------------------------------
# clocks


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs without CUDA_VISIBLE_DEVICES remapping
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [x.strip() for x in vis.split(",") if x.strip()]
            if gpu_index < len(ids):
                gpu_index = ids[gpu_index]
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in load),
                "samples": len(load), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# workloads


class Workload:
    """One benchmarked workload: how to build a layer's device tensors, how to
    launch one layer, and its units (token-heads) and algorithmic bytes per
    launch."""

    def __init__(self, name, spec, layers, kind, description):
        self.name, self.spec, self.default_layers = name, spec, layers
        self.kind, self.description = kind, description

    # --- sizes
    rank = 16  # window length of the low-rank workload

    def units_per_launch(self):
        w = self.spec
        if self.kind in ("prefill", "lowrank_prefill"):
            return w.total * w.H
        if self.kind == "lowrank":
            return w.B * w.H * w.T
        return w.B * w.H * (w.T if self.kind == "decode" else 1)

    def flops_per_launch(self):
        """Algorithmic arithmetic of the chunked prefill per call (a
        multiply-add counts 2), per chunk of C = 64 tokens and head: the Gram
        products k k^T and q k^T (2 x 2 C^2 dk), the triangular solve for
        (I + A)^-1 (C^3 / 3), K S and Q S (2 x 2 C dk dv), Delta = T R and
        P Delta (2 x 2 C^2 dv) and the state update K^T Delta (2 C dk dv)."""
        w = self.spec
        C = 64
        per = (2 * 2 * C * C * w.dk + C ** 3 / 3 + 2 * 2 * C * w.dk * w.dv
               + 2 * 2 * C * C * w.dv + 2 * C * w.dk * w.dv)
        chunks = sum((L + C - 1) // C for L in w.lens)
        return chunks * w.H * per

    def lowrank_prefill_flops_per_launch(self):
        """Arithmetic of the chunked low-rank window over the prompts, as the
        chunk form computes it on the CUDA cores (a multiply-add counts 2), per
        chunk of C = 64 tokens and head: q k^T and k k^T (2 x 2 C^2 dk), q and
        k against the entering window's k (2 x 2 C R dk), the triangular solve
        (C^3 / 3), the window's u against both (2 x 2 C R dv), Delta = T rhs
        and PQ Delta (2 x 2 C^2 dv)."""
        w = self.spec
        C, R = 64, self.rank
        per = (2 * 2 * C * C * w.dk + 2 * 2 * C * R * w.dk + C ** 3 / 3 + 2 * 2 * C * R * w.dv
               + 2 * 2 * C * C * w.dv)
        chunks = sum((L + C - 1) // C for L in w.lens)
        return chunks * w.H * per

    def tensor_flops_per_launch(self):
        """bf16 tensor-core arithmetic one call executes (bf16 inputs, dk = dv
        = 128): fp32 operands run as sums of bf16 parts, so a product costs
        one pass per part pair kept.  Per chunk and head: phase A's Gram
        [k; q] k^T (1 pass, M = 2C); phase B's Y, Z (S in 3 parts: 3 passes of
        2 x 2 C dk dv), q k^T (1 pass, M = 2C), T R (6 passes), P Delta (3
        passes) and K^T Delta' (3 passes)."""
        w = self.spec
        C = 64
        per = (2 * 2 * C * C * w.dk + 3 * 2 * 2 * C * w.dk * w.dv + 2 * 2 * C * C * w.dk
               + 6 * 2 * C * C * w.dv + 3 * 2 * C * C * w.dv + 3 * 2 * C * w.dk * w.dv)
        chunks = sum((L + C - 1) // C for L in w.lens)
        return chunks * w.H * per

    def n_active(self, d):
        return int((d["slot_idx"] >= 0).sum().item())

    def bytes_per_launch(self, n_active):
        w = self.spec
        if self.kind == "lowrank":
            R = self.rank
            per_head = R * (w.dk + w.dv) * 4 + R * 4 + 4 + (w.dk + w.dv + R) * 4 + 4
            return (n_active * w.H * per_head + w.B * w.T * (2 * w.hk * w.dk + w.H * w.dv) * 2
                    + w.B * w.T * w.H * 8 + w.B * 4 + w.B * w.T * w.H * w.dv * 4)
        if self.kind == "prefill":
            in_b = 2 if str(w.in_dtype) == "torch.bfloat16" else 4
            return (w.total * (2 * w.hk * w.dk + w.H * w.dv) * in_b + w.total * w.H * 8
                    + 2 * n_active * w.H * w.dk * w.dv * 4 + w.total * w.H * w.dv * 4
                    + (w.N + 1) * 4 + w.N * 4)
        if self.kind == "lowrank_prefill":
            in_b = 2 if str(w.in_dtype) == "torch.bfloat16" else 4
            R = self.rank
            window = R * (w.dk + w.dv + 1) * 4 + 4  # k, u, c and the count of a head
            return (w.total * (2 * w.hk * w.dk + w.H * w.dv) * in_b + w.total * w.H * 8
                    + 2 * n_active * w.H * window + w.total * w.H * w.dv * 4
                    + (w.N + 1) * 4 + w.N * 4)
        if self.kind == "decode":
            in_b = 2 if str(w.in_dtype) == "torch.bfloat16" else 4
            st_b = 4 if str(w.state_dtype) == "torch.float32" else 2
            return algorithmic_bytes_per_launch(w.B, w.H, w.hk, w.dk, w.dv, w.T, n_active,
                                                in_bytes=in_b, out_bytes=4, state_bytes=st_b)
        C = w.C
        w_b = 4 if str(w.conv_w_dtype) == "torch.float32" else 2
        return (2 * n_active * w.H * w.dk * w.dv * 4      # state read + write
                + n_active * C * 2                         # mixed projection row
                + n_active * C * 3 * 2 * 2                 # conv state read + write
                + C * 4 * w_b                              # conv weights
                + n_active * w.H * 2 * 2                   # a, b
                + n_active * w.H * w.dv * 2                # z
                + w.H * 8 + w.dv * 4 + w.B * 4             # A_log, dt_bias, norm_w, slots
                + w.B * w.H * w.dv * 4)                    # out (padding rows are zeroed)

    # --- tensors and launches
    def build(self, layer, device, seed):
        import torch

        from gated_deltanet_recurrent_gdn_b200 import inputs
        w = self.spec
        if self.kind == "decode":
            d = inputs.decode_inputs(w, seed=seed, layer=layer, device=device)
            d["out"] = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
        elif self.kind == "lowrank":
            d = inputs.decode_inputs(w, seed=seed, layer=layer, device=device, with_state=False)
            d.update(inputs.lowrank_window(w, self.rank, seed=seed * 1000 + layer, device=device))
            d["out"] = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
        elif self.kind == "lowrank_prefill":
            d = inputs.prefill_inputs(w, seed=seed * 1000 + layer, device=device)
            dw = inputs.DecodeWorkload("lw", B=w.N, H=w.H, dk=w.dk, dv=w.dv, T=1, n_slots=w.pool)
            d.update(inputs.lowrank_window(dw, self.rank, seed=seed * 1000 + layer, device=device))
            d["out"] = torch.empty((w.total, w.H, w.dv), dtype=torch.float32, device=device)
        elif self.kind == "prefill":
            import gated_deltanet_recurrent_gdn_b200 as gdn
            d = inputs.prefill_inputs(w, seed=seed * 1000 + layer, device=device)
            d["out"] = torch.empty((w.total, w.H, w.dv), dtype=torch.float32, device=device)
            need = gdn.prefill_workspace_size(w.N, w.total, w.H, w.dk, w.dv, w.in_dtype)
            d["workspace"] = torch.empty(need, dtype=torch.uint8, device=device)
        else:
            d = inputs.fused_inputs(w, seed=seed * 1000 + layer, device=device)
            d["out"] = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device=device)
        return d

    def host_keys(self):
        if self.kind in ("decode", "lowrank"):
            return ("q", "k", "v", "g", "beta", "slot_idx")
        if self.kind in ("prefill", "lowrank_prefill"):
            return ("q", "k", "v", "g", "beta", "slot_idx", "cu_seqlens")
        return ("mixed_x", "a", "b", "z", "slot_idx")

    def launch(self, d, stream):
        import gated_deltanet_recurrent_gdn_b200 as gdn
        w = self.spec
        if self.kind == "lowrank":
            gdn.lowrank_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["win_k"],
                                    d["win_u"], d["win_c"], d["win_count"], d["slot_idx"],
                                    d["out"], stream=stream)
        elif self.kind == "lowrank_prefill":
            gdn.lowrank_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["win_k"], d["win_u"],
                                d["win_c"], d["win_count"], d["slot_idx"], d["cu_seqlens"],
                                d["out"], stream=stream)
        elif self.kind == "prefill":
            gdn.chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                              d["slot_idx"], d["cu_seqlens"], d["out"], workspace=d["workspace"],
                              stream=stream)
        elif self.kind == "fused":
            gdn.fused_decode_step(d["mixed_x"], d["conv_state"], d["conv_w"], d["a"], d["b"],
                                  d["A_log"], d["dt_bias"], d["z"], d["norm_w"], d["state"],
                                  d["slot_idx"], d["out"], Hk=w.Hk, H=w.H, dk=w.dk, dv=w.dv,
                                  stream=stream)
        elif (str(w.in_dtype) == "torch.bfloat16" and w.hk == w.H
              and str(w.state_dtype) == "torch.float32"):
            # the plain entry point: bf16 q/k/v, fp32 out
            gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                            d["slot_idx"], d["out"], stream=stream)
        else:
            gdn.decode_step_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                               d["slot_idx"], d["out"], stream=stream)


def workloads(state_dtype: str = "f32"):
    import torch

    from gated_deltanet_recurrent_gdn_b200 import inputs
    st = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[state_dtype]
    if state_dtype != "f32":
        ws = {name: w for name, w in _workloads(inputs).items() if w.kind == "decode"}
        for w in ws.values():
            w.spec = inputs.shrink(w.spec, state_dtype=st)
            w.description = w.description.replace("fp32 state", f"{state_dtype} state")
        return ws
    return _workloads(inputs)


def _workloads(inputs):
    return {
        "serving": Workload("serving", inputs.SERVING, 48, "decode",
                            "serving decode step: B=256 H=48 dk=dv=128 T=1 fp32 state, bf16 q/k/v, "
                            "{L} layers back to back, 512-slot pool per layer, slot_idx = random "
                            "permutation"),
        "layer": Workload("layer", inputs.LAYER, 16, "decode",
                          "single-layer decode step: B=64 H=48 dk=dv=128 T=1 fp32 state, bf16 "
                          "q/k/v, identity slots, {L} layers back to back"),
        "mtp": Workload("mtp", inputs.MTP, 8, "decode",
                        "MTP verify step: B=128 H=48 dk=dv=128 T=4, fp32 state, bf16 q/k/v, "
                        "identity slots, {L} layers back to back"),
        "tiny": Workload("tiny", inputs.TINY, 16, "decode",
                         "tiny decode: B=1 H=4 dk=dv=128 T=8 fp32 state, fp32 inputs, {L} layers back "
                         "to back (launch-bound)"),
        "lowrank": Workload("lowrank", inputs.shrink(inputs.SERVING, n_slots=256,
                                                     slots="identity"), 16, "lowrank",
                            "low-rank sliding-window decode: B=256 H=48 dk=dv=128 T=1, full "
                            "windows of r updates, {L} layers back to back"),
        "lowrank_prefill": Workload("lowrank_prefill", inputs.PREFILL, 1, "lowrank_prefill",
                                    "low-rank window over whole prompts in chunks: 8 prompts of "
                                    "777..4096 tokens (19,101 tokens) H=48 dk=dv=128, bf16 q/k/v, "
                                    "windows of r updates continued from full ones, {L} layer(s)"),
        "prefill": Workload("prefill", inputs.PREFILL, 1, "prefill",
                            "chunked prefill: 8 prompts of 777..4096 tokens (19,101 tokens) "
                            "H=48 dk=dv=128, bf16 q/k/v, fp32 state, {L} layer(s)"),
        "fused": Workload("fused", inputs.FUSED, 8, "fused",
                          "fused conv+gates+recurrence+gated RMSNorm: B=256 (26 padding rows) "
                          "Hk=16 H=48 dk=dv=128 T=1, C=10240, {L} layers back to back"),
    }


def prefill_roofline(wl, launch_s, bpl, state_dtype="f32", peaks=None):
    """Roofline of one prefill call: the products run on the tensor cores in
    bf16 with fp32 operands split into bf16 parts, so the peak for its
    fp32-accurate arithmetic is the measured dense bf16 peak (burst: the call
    is timed on its own) divided by the bf16 flops executed per algorithmic
    flop; frac is then the tensor pipe's share of that peak."""
    peaks, source = peaks or measured_peaks()
    flops = wl.flops_per_launch()
    executed = wl.tensor_flops_per_launch()
    ratio = executed / flops
    peak = peaks["bf16_tflops"] / ratio
    tflops = flops / launch_s / 1e12
    traffic, traffic_src = recorded_traffic(wl, state_dtype, wl.units_per_launch())
    return {"bound": "tensor", "achieved": round(tflops, 2), "peak": round(peak, 1),
            "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
            "traffic": traffic, "traffic_source": traffic_src,
            "peak_source": (f"{source} bf16 dense peak {peaks['bf16_tflops']} TFLOP/s / "
                            f"{ratio:.3f} bf16 MMA flops executed per algorithmic flop"),
            "kernel": decode_kernel_label(wl, state_dtype),
            "algorithmic_flops_per_launch": flops,
            "bf16_mma_flops_per_launch": executed,
            "algorithmic_bytes_per_launch": bpl,
            "achieved_GBs": round(bpl / launch_s / 1e9, 1),
            "bytes_frac_of_peak_hbm": round(bpl / launch_s / 1e9 / peaks["hbm_gbs"], 4),
            "us_per_layer": round(launch_s * 1e6, 2)}


def workload_config(wl, L, world, timing):
    w = wl.spec
    if wl.kind == "lowrank_prefill":
        return {"workload": wl.description.format(L=L), "N": w.N, "tokens": w.total, "H": w.H,
                "dk": w.dk, "dv": w.dv, "R": wl.rank, "layers": L,
                "parallelism": f"replicas x{world}",
                "l2": "inputs (0.7 GB) and outputs (0.47 GB) larger than L2", "timing": timing}
    if wl.kind == "prefill":
        return {"workload": wl.description.format(L=L), "N": w.N, "tokens": w.total, "H": w.H,
                "dk": w.dk, "dv": w.dv, "layers": L, "parallelism": f"replicas x{world}",
                "l2": "inputs (0.7 GB) and outputs (0.47 GB) larger than L2", "timing": timing}
    config = {"workload": wl.description.format(L=L), "B": w.B, "H": w.H, "dk": w.dk,
              "dv": w.dv, "T": getattr(w, "T", 1), "layers": L, "n_slots": w.pool,
              "parallelism": f"replicas x{world}",
              "l2": "inputs larger than L2 (state moved per step >> 126 MB)",
              "timing": timing}
    if wl.kind == "fused":
        config["Hk"] = w.Hk
    else:
        config["state_dtype"] = str(w.state_dtype).replace("torch.", "")
    return config


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same workload


def _oracle_call_factory(wl):
    """(factory, token-heads per call, description of one call) for the
    oracle on a slice of the workload: its first sequences, all heads, a
    compact pool.  ``factory()`` builds fresh host copies of the inputs and
    state and returns a zero-argument call, so that threads never share a
    mutable array."""
    import numpy as np
    import torch

    import oracle
    from gated_deltanet_recurrent_gdn_b200 import inputs

    f64 = lambda t: t.to(torch.float64).numpy()
    if wl.kind == "prefill":
        w = inputs.PrefillWorkload("sample", lens=(256,), H=wl.spec.H, dk=wl.spec.dk,
                                   dv=wl.spec.dv)
        inp = inputs.prefill_inputs(w, seed=0)
        args = [f64(inp[x]) for x in ("q", "k", "v", "g", "beta")]
        slots, cu = inp["slot_idx"].numpy(), inp["cu_seqlens"].numpy()
        st0 = f64(inp["state"])

        def factory():
            st = st0.copy()
            return lambda: oracle.prefill(*args, st, slots, cu)
        desc = f"prefill of one 256-token prompt x {w.H} heads (dk={w.dk}, dv={w.dv})"
        return factory, w.total * w.H, desc
    if wl.kind == "lowrank_prefill":
        w = inputs.PrefillWorkload("sample", lens=(256,), H=wl.spec.H, dk=wl.spec.dk,
                                   dv=wl.spec.dv)
        inp = inputs.prefill_inputs(w, seed=0)
        dw = inputs.DecodeWorkload("lw", B=1, H=w.H, dk=w.dk, dv=w.dv, T=1)
        win = inputs.lowrank_window(dw, wl.rank, seed=0)
        args = [f64(inp[x]) for x in ("q", "k", "v", "g", "beta")]
        slots, cu = inp["slot_idx"].numpy(), inp["cu_seqlens"].numpy()

        def factory():
            wk, wu, wc = (f64(win[x]).copy() for x in ("win_k", "win_u", "win_c"))
            wn = win["win_count"].numpy().astype(np.int32).copy()
            return lambda: oracle.lowrank_prefill(*args, wk, wu, wc, wn, slots, cu)
        desc = (f"low-rank prefill (R={wl.rank}) of one 256-token prompt x {w.H} heads "
                f"(dk={w.dk}, dv={w.dv})")
        return factory, w.total * w.H, desc
    if wl.kind == "lowrank":
        Bs = 64
        w = inputs.shrink(wl.spec, B=Bs, n_slots=Bs)
        inp = inputs.decode_inputs(w, seed=0, with_state=False)
        win = inputs.lowrank_window(w, wl.rank, seed=0)
        args = [f64(inp[x]) for x in ("q", "k", "v", "g", "beta")]
        slots = inp["slot_idx"].numpy()

        def factory():
            wk, wu, wc = (f64(win[x]).copy() for x in ("win_k", "win_u", "win_c"))
            wn = win["win_count"].numpy().astype(np.int32).copy()
            return lambda: oracle.lowrank_decode_step(*args, wk, wu, wc, wn, slots)
        desc = f"{wl.name} (R={wl.rank}) step on {Bs} sequences x {w.H} heads"
        return factory, w.B * w.H * w.T, desc
    if wl.kind == "decode":
        Bs = min(wl.spec.B, 64 if wl.spec.T == 1 else 16)
        w = inputs.shrink(wl.spec, B=Bs, n_slots=Bs, slots="identity")
        inp = inputs.decode_inputs(w, seed=0)
        q, k, v, g, beta = (f64(inp[x]) for x in ("q", "k", "v", "g", "beta"))
        slots = inp["slot_idx"].numpy()
        st0 = f64(inp["state"])

        def factory():
            st = st0.copy()
            return lambda: oracle.decode_step(q, k, v, g, beta, st, slots)
        desc = (f"{wl.name} step on {Bs} sequences x {w.H} heads (dk={w.dk}, dv={w.dv}, "
                f"T={w.T})")
        return factory, w.B * w.H * w.T, desc
    Bs = 32
    w = inputs.shrink(wl.spec, B=Bs, n_slots=Bs, pad_frac=0.0)
    inp = inputs.fused_inputs(w, seed=0)
    x = f64(inp["mixed_x"])
    rest = {n: f64(inp[n]) for n in ("conv_w", "a", "b", "A_log", "dt_bias", "z", "norm_w")}
    slots = inp["slot_idx"].numpy()
    cs0, st0 = f64(inp["conv_state"]), f64(inp["state"])

    def factory():
        cs, st = cs0.copy(), st0.copy()
        return lambda: oracle.fused_step(x, cs, rest["conv_w"], rest["a"], rest["b"],
                                         rest["A_log"], rest["dt_bias"], rest["z"],
                                         rest["norm_w"], st, slots, Hk=w.Hk, H=w.H, dk=w.dk,
                                         dv=w.dv)
    desc = f"fused step on {Bs} sequences x {w.H} v-heads ({w.Hk} k-heads, C={w.C})"
    return factory, w.B * w.H, desc


def host_cpu():
    """(CPU model, cores this process may run on) of the host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        cores = os.cpu_count() or 1
    return model, cores


def cpu_oracle_sample(target_seconds: float, wl=None, max_calls: int = 10_000, threads: int = 1):
    """Time the fp64 oracle on a slice of the workload, repeated until about
    ``target_seconds`` of wall time; with ``threads`` > 1 every thread runs
    its own copy of the slice (the (b, h) units of the oracle are
    independent; the oracle's C calls release the interpreter lock).
    Returns (token-heads/s, sample text, seconds)."""
    import threading

    wl = wl or workloads()["serving"]
    factory, units_per_call, desc = _oracle_call_factory(wl)
    calls_fn = [factory() for _ in range(threads)]
    counts = [0] * threads
    start = threading.Barrier(threads + 1)
    stop = [False]

    def worker(i):
        start.wait()
        while not stop[0] and counts[i] < max_calls:
            calls_fn[i]()
            counts[i] += 1

    pool = [threading.Thread(target=worker, args=(i,)) for i in range(threads)]
    for t in pool:
        t.start()
    start.wait()
    t0 = time.perf_counter()
    while True:
        time.sleep(0.005)
        el = time.perf_counter() - t0
        if min(counts) >= max_calls or (el >= target_seconds and min(counts) >= 1):
            break
    stop[0] = True
    for t in pool:
        t.join()
    el = time.perf_counter() - t0
    units = sum(counts) * units_per_call
    sample = (f"{sum(counts)} oracle calls ({desc}), {units} token-heads in {el:.1f} s, "
              f"{threads} thread{'s' if threads > 1 else ''}")
    return units / el, sample, el


def cpu_baseline_line(wl, seconds: float):
    """The cpu_baseline object of the JSON line: the oracle as it stands on
    the host's cores, single-threaded (the headline value) and on every core,
    plus single-threaded samples of the other decode configurations."""
    model, cores = host_cpu()
    v1, sample1, _ = cpu_oracle_sample(seconds * 0.5, wl)
    vn, samplen, _ = cpu_oracle_sample(seconds * 0.25, wl, threads=cores) if cores > 1 else (
        v1, sample1, 0.0)
    others = {}
    if wl.kind == "decode" and wl.name == "serving":
        for name in ("layer", "mtp", "fused"):
            v, smp, _ = cpu_oracle_sample(seconds * 0.25 / 3, workloads()[name])
            others[name] = {"value": round(v, 1), "sample": smp, "cores": 1}
    return {"value": round(v1, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": sample1, "host_cpu": model, "host_cores": cores,
            "all_cores": {"value": round(vn, 1), "cores": cores, "sample": samplen},
            "other_configs": others or None}


# ---------------------------------------------------------------------------
# the GPU arm


def run_ours(args, rank, world, local):
    import torch

    import gated_deltanet_recurrent_gdn_b200 as gdn

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    gdn.load_library()

    wl = workloads(args.state_dtype)[args.workload]
    wl.rank = args.rank
    if wl.kind in ("lowrank", "lowrank_prefill"):
        wl.description = wl.description.replace("r updates", f"{args.rank} updates")
    L = args.layers or wl.default_layers
    layers = [wl.build(l, device, seed=rank) for l in range(L)]
    torch.cuda.synchronize()
    n_active = wl.n_active(layers[0])

    stream = torch.cuda.Stream(device=device)

    def step():
        for d in layers:
            wl.launch(d, stream)

    with torch.cuda.stream(stream):
        step()  # first launch outside any capture
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        torch.cuda.synchronize()
    run = (lambda: graph.replay()) if graph is not None else step

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run()
    torch.cuda.synchronize()

    # events at the group boundaries: recorded on the launching stream
    # between replays, they add no synchronisation inside the timed region
    bounds = group_bounds(args.steps, args.groups)
    evs = [torch.cuda.Event(enable_timing=True) for _ in bounds]
    barrier(dist, device)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        with torch.cuda.stream(stream):
            evs[0].record(stream)
            for i in range(1, len(bounds)):
                for _ in range(bounds[i] - bounds[i - 1]):
                    run()
                evs[i].record(stream)
        torch.cuda.synchronize()
    barrier(dist, device)
    ms_total = max_over_ranks(evs[0].elapsed_time(evs[-1]), dist, device)
    group_ms = [evs[i - 1].elapsed_time(evs[i]) / (bounds[i] - bounds[i - 1])
                for i in range(1, len(bounds))]
    clocks = clk.summary()

    launches = L * args.steps
    ms_per_step = ms_total / args.steps
    units_per_step = L * wl.units_per_launch()
    value = weak_scaling_value(units_per_step, args.steps, world, ms_total)

    bpl = wl.bytes_per_launch(n_active)
    launch_s = ms_total / 1e3 / launches
    achieved = bpl / launch_s / 1e9
    if wl.kind == "prefill":
        roofline = prefill_roofline(wl, launch_s, bpl, args.state_dtype)
    elif wl.kind == "lowrank_prefill":
        flops = wl.lowrank_prefill_flops_per_launch()
        tflops = flops / launch_s / 1e12
        traffic, traffic_src = recorded_traffic(wl, args.state_dtype, wl.units_per_launch())
        roofline = {"bound": "alu", "achieved": round(tflops, 2),
                    "peak": round(FP32_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
                    "frac": round(tflops / FP32_PEAK_TFLOPS, 4), "traffic": traffic,
                    "traffic_source": traffic_src,
                    "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz",
                    "kernel": decode_kernel_label(wl, args.state_dtype),
                    "algorithmic_flops_per_launch": flops,
                    "algorithmic_bytes_per_launch": bpl,
                    "achieved_GBs": round(achieved, 1),
                    "us_per_layer": round(launch_s * 1e6, 2)}
    else:
        peak, peak_kind = measured_peak()
        traffic, traffic_src = recorded_traffic(wl, args.state_dtype, wl.units_per_launch())
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4), "traffic": traffic,
                    "traffic_source": traffic_src,
                    "peak_source": f"{peak_kind} HBM copy bandwidth",
                    "kernel": decode_kernel_label(wl, args.state_dtype),
                    "algorithmic_bytes_per_launch": bpl,
                    "us_per_layer": round(launch_s * 1e6, 2),
                    "frac_of_8TBs": round(achieved / NOMINAL_HBM_GBS, 4)}
        if achieved > peak:
            roofline["note"] = (
                "above 1.0: the measured peak is a plain copy kernel's rate, a floor on what "
                "HBM sustains rather than its ceiling (this kernel's read-modify-write stream "
                "overlaps reads and writes better); frac_of_8TBs is the fraction of nominal")

    # ---- end to end: host buffers, copies inside the timed region ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, layers, device, dist, stream, world)

    timing = "CUDA graph of the step, replayed" if graph is not None else "eager launches"
    # release the graph before tearing anything down
    graph = None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_line(wl, args.cpu_seconds)

    config = workload_config(wl, L, world, timing)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clocks,
        "spread": spread(group_ms),
    }
    if dist is not None:
        barrier(dist, device)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, wl, layers, device, dist, compute, world):
    """Same step through the public call with host buffers: per layer, H2D of
    the per-token inputs from pinned memory, the kernel, D2H of out."""
    import torch

    keys = wl.host_keys()
    host = []
    for d in layers:
        h = {k: d[k].to("cpu").pin_memory() for k in keys}
        h["out"] = torch.empty(d["out"].shape, dtype=d["out"].dtype).pin_memory()
        host.append(h)
    h2d = sum(h[k].numel() * h[k].element_size() for h in host for k in keys)
    d2h = sum(h["out"].numel() * h["out"].element_size() for h in host)
    up = torch.cuda.Stream(device=device)
    down = torch.cuda.Stream(device=device)
    L = len(layers)
    ev_in = [torch.cuda.Event() for _ in range(L)]
    ev_k = [torch.cuda.Event() for _ in range(L)]
    ev_out = [torch.cuda.Event() for _ in range(L)]
    first = [True]

    def step():
        for l, (d, h) in enumerate(zip(layers, host)):
            with torch.cuda.stream(up):
                if not first[0]:
                    up.wait_event(ev_k[l])       # previous step's kernel has read the inputs
                for k in keys:
                    d[k].copy_(h[k], non_blocking=True)
                ev_in[l].record(up)
            compute.wait_event(ev_in[l])
            if not first[0]:
                compute.wait_event(ev_out[l])    # previous step's out has been read back
            wl.launch(d, compute)
            ev_k[l].record(compute)
            with torch.cuda.stream(down):
                down.wait_event(ev_k[l])
                h["out"].copy_(d["out"], non_blocking=True)
                ev_out[l].record(down)
        first[0] = False

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize()
    e0.record(compute)
    up.wait_event(e0)
    for _ in range(args.steps):
        step()
    compute.wait_event(ev_out[-1])
    e1.record(compute)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    units = world * L * wl.units_per_launch() * args.steps
    return {"value": round(units / (ms / 1e3), 1), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.steps, 4),
            "how": "pinned host -> device copies, kernel, device -> pinned host, per layer, "
                   "pipelined on 3 streams"}


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle


def run_reference(args, rank, world):
    if rank != 0:
        return
    per_step = max(1.0, args.cpu_seconds / max(args.steps, 1))
    wl = workloads(args.state_dtype)[args.workload]
    for _ in range(args.warmup):
        cpu_oracle_sample(0.0, wl, max_calls=1)
    total_units_s = []
    t_all = 0.0
    samples = []
    for _ in range(args.steps):
        v, sample, el = cpu_oracle_sample(per_step, wl)
        total_units_s.append(v)
        t_all += el
        samples.append(sample)
    value = statistics.median(total_units_s)
    ms_per_step = t_all / args.steps * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.layers or wl.default_layers, world,
                                  "CPU oracle, one bounded sample of the workload per step"),
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": samples[-1]},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.warmup < 3 and args.impl == "ours" and args.layers == 0:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
