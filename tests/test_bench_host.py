"""Host logic of bench.py (CPU): the algorithmic work behind the roofline
fractions, the L2 policy, the fused-combine rule and the lookup of committed
ncu traffic. The expected values are the per-workload totals (active-expert
FLOPs, expert weight bytes) recomputed here from the shapes."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_mixture_experts_renorm_b200 import build as build_mod  # noqa: E402
from sparse_mixture_experts_renorm_b200 import _binding as B  # noqa: E402
from sparse_mixture_experts_renorm_b200.workloads import WORKLOADS  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def library():
    """The launch plan comes from the library (a host-side query)."""
    build_mod.build()


def balanced(wl):
    c = np.full(wl.E, wl.T * wl.k // wl.E)
    c[: wl.T * wl.k - c.sum()] += 1
    return c


def test_prefill_gemm_work():
    wl = WORKLOADS["mixtral_prefill"]
    w = bench.algorithmic(wl, balanced(wl))
    gu, dn = w["grouped_gemm_gateup_swiglu"], w["grouped_gemm_down"]
    # 4 d I T k and 2 d I T k (+ the folded combine's 2 T k d)
    assert gu["flops"] == pytest.approx(1.924e12, rel=1e-3)
    assert dn["flops"] == pytest.approx(0.962e12, rel=1e-3)
    # weights once (W_gate + W_up = 1.879 GB), Xp read, H written
    assert gu["bytes"] == pytest.approx(2 * 8 * 14336 * 4096 * 2 + 8192 * 4096 * 2 + 8192 * 14336 * 2)
    assert w["combine"]["bytes"] == 0  # k = 2: inside the down GEMM


def test_decode_streams_all_weights_once():
    """At 32 tokens both projections run in one kernel: its slot streams the
    three weight matrices of every used expert once, reads the dispatched x,
    and accumulates the fp32 output in place; H stays between the two steps
    and is not counted."""
    wl = WORKLOADS["mixtral_decode"]
    w = bench.algorithmic(wl, balanced(wl))
    weights = 3 * 8 * 4096 * 14336 * 2
    assert weights == pytest.approx(2.819e9, rel=1e-3)
    assert w["grouped_gemm_down"]["bytes"] == 0 and w["grouped_gemm_down"]["flops"] == 0
    streamed = w["grouped_gemm_gateup_swiglu"]["bytes"] - 64 * 4096 * 2 - 2 * 32 * 4096 * 4 - 64 * 8
    assert streamed == weights
    assert w["grouped_gemm_gateup_swiglu"]["flops"] == pytest.approx(6.0 * 64 * 4096 * 14336 + 2.0 * 64 * 4096)


def test_unused_experts_are_not_streamed():
    wl = WORKLOADS["mixtral_decode"]
    c = balanced(wl)
    c[3] += c[5]
    c[5] = 0
    full = bench.algorithmic(wl, balanced(wl))["grouped_gemm_gateup_swiglu"]["bytes"]
    part = bench.algorithmic(wl, c)["grouped_gemm_gateup_swiglu"]["bytes"]
    assert full - part == 3 * 4096 * 14336 * 2


def test_capacity_counts_only_kept_rows():
    wl = WORKLOADS["fine_grained"]
    c = np.zeros(wl.E, dtype=np.int64)
    c[0], c[1], c[2] = wl.T * wl.k - 200, 150, 50
    w = bench.algorithmic(wl, c, {"cap": 100})
    assert w["grouped_gemm_down"]["flops"] == 2.0 * (100 + 100 + 50) * wl.d * wl.I


def test_fused_combine_rule():
    assert bench.fused_combine(WORKLOADS["mixtral_prefill"])
    assert not bench.fused_combine(WORKLOADS["mixtral_prefill"], n_shared=1)
    assert not bench.fused_combine(WORKLOADS["fine_grained"])  # k = 6
    assert not bench.fused_combine(WORKLOADS["tiny_f32"])  # fp32 path
    # the fold_combine option: every k, the down GEMM's slot carrying the combine
    fine, fold = WORKLOADS["fine_grained"], {"fold_combine": True}
    assert bench.plan_of(fine, fold) & B.MOE_PLAN_FUSED_COMBINE
    assert bench.launches_per_step(fine, fold) == 5
    assert bench.slot_names(fine, fold)[5] == "combine (in grouped_gemm_down)"
    w = bench.algorithmic(fine, balanced(fine), fold)
    R = fine.T * fine.k
    assert w["combine"]["bytes"] == 0
    assert w["grouped_gemm_down"]["bytes"] == (64 * 2048 * 1408 * 2 + R * 1408 * 2 + 2 * fine.T * 2048 * 4 + R * 8)


def test_fused_gemms_rule():
    """Both projections share one kernel for bf16 batches of at most 32 tokens."""
    assert bench.fused_gemms(WORKLOADS["mixtral_decode"])
    assert not bench.fused_gemms(WORKLOADS["mixtral_prefill"])
    assert not bench.fused_gemms(WORKLOADS["tiny_f32"])  # fp32 path
    assert bench.launches_per_step(WORKLOADS["mixtral_decode"]) == 3  # router (with the scan), permute, GEMMs
    assert bench.launches_per_step(WORKLOADS["mixtral_prefill"]) == 4  # the permute does the scan
    assert bench.launches_per_step(WORKLOADS["fine_grained"]) == 6  # 128 router blocks x 64 experts: scan kernel
    assert bench.launches_per_step(WORKLOADS["mixtral_prefill"], {"norm": 1}) == 5  # + the router weight split


@pytest.mark.parametrize("name,flush", [("tiny_f32", True), ("small_bf16", True), ("mixtral_prefill", False),
                                        ("fine_grained", False), ("mixtral_decode", False)])
def test_l2_policy(name, flush):
    wl = WORKLOADS[name]
    assert bench.needs_flush(wl) == flush
    text = bench.config_of(wl, 1)["l2"]
    assert ("flushed" in text) == flush and ("larger than L2" in text) == (not flush)


def test_traffic_lookup():
    """A committed capture of the current gemm_tc2.cu gives the per-launch
    DRAM bytes; a capture of an older source gives none (the bench then
    reports null)."""
    assert bench.load_traffic("no_such_workload", "grouped_gemm_down") is None
    v = bench.load_traffic("mixtral_prefill", "grouped_gemm_gateup_swiglu")
    if v is None:
        pytest.skip("gemm_tc2.cu changed since the committed capture: traffic is reported as null")
    assert 2.0e9 < v < 3.0e9  # about the 2.18 GB of algorithmic bytes
