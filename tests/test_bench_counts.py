"""Host logic of bench.py's roofline (CPU): the algorithmic counts per kernel and
per layer, and the source-hash guard on the committed ncu traffic.

The whole-layer FLOP counts are the ones the measurement plan fixes for each
configuration (169.1 GFLOP for the 340M-shaped layer, 244.9 for the
single-scale GLA layer of the same width, 338.2 at L = 32768, 1224.2 and 342.5
for the d = 2048 layer and its {2,4} ablation); the per-kernel split must add
up to them.
"""
import math

import pytest

import bench
from scale_gated_linear_b200 import workloads as wl

PLAN_GFLOP = {
    "msgla_340m": 169.1,
    "gla_340m": 244.9,
    "long_32k": 338.2,
    "wide_8k": 1224.2,
    "wide_8k_no_fine": 342.5,
}


@pytest.mark.parametrize("name", sorted(PLAN_GFLOP))
def test_total_flops_match_the_measurement_plan(name):
    w = wl.WORKLOADS[name]
    c = bench.algorithmic_counts(w, w.B, w.L)
    assert c["total_flops"] / 1e9 == pytest.approx(PLAN_GFLOP[name], abs=0.06)
    # the per-kernel FLOPs plus the 6 d elementwise operations per token are the total
    kernel_flops = sum(k.get("flops", 0) for k in c["kernels"].values())
    assert kernel_flops + w.B * w.L * 6 * w.d == pytest.approx(c["total_flops"])


def test_gla_term_uses_the_configured_chunk():
    w = wl.WORKLOADS["msgla_340m"]
    base = bench.algorithmic_counts(w, w.B, w.L)["kernels"]["gla"]["flops"]
    wide = bench.algorithmic_counts(w.replace(chunk=128), w.B, w.L)["kernels"]["gla"]["flops"]
    pooled_steps = sum(w.B * math.ceil(w.L / s) * h for s, h in zip(w.scales, w.heads))
    # the intra-chunk term C (d_k + d_v) per head and pooled step grows with C
    assert wide - base == pytest.approx(pooled_steps * (128 - w.chunk) * (w.d_k + w.d_v))


def test_layer_without_a_fine_branch_counts_the_hold_and_fusion_pass():
    w = wl.WORKLOADS["wide_8k_no_fine"]
    k = bench.algorithmic_counts(w, w.B, w.L)["kernels"]
    assert "out_gemm_fused" not in k
    held = sum(w.B * math.ceil(w.L / s) * w.d * 2 for s in w.scales)
    assert k["hold_fuse"]["bytes"] == held + w.B * w.L * len(w.scales) * 4 + w.B * w.L * w.d * 2
    # every kernel the plan can pick as the dominant one has a count
    for name in ("pool_u", "gate", "proj_gemm", "gla", "out_gemm_coarse", "hold_fuse"):
        assert name in k


def test_traffic_needs_matching_sources():
    # a kernel or workload without a committed capture reports no traffic
    assert bench.traffic_for("gla", "no_such_workload/B1/L1") is None
    assert bench.traffic_for("no_such_kernel", "msgla_340m/B8/L2048") is None
