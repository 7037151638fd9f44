"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, at every workload size and on the edge cases."""
import numpy as np
import pytest
import torch

import parity
from sparse_mixture_experts_renorm_b200 import _binding as B
from sparse_mixture_experts_renorm_b200 import get_permutation, moe_forward
from sparse_mixture_experts_renorm_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def run(wl, inp=None, seed=0):
    if inp is None:
        inp = make_inputs(wl, "cuda", seed)
    res = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    torch.cuda.synchronize()
    perm = get_permutation(res, wl.T, wl.d, wl.E, wl.k, wl.I, inp.x.dtype)
    torch.cuda.synchronize()
    return inp, res, perm


def check(wl, inp, res, perm, tokens=None):
    rep = parity.check(inp, res, perm, wl.k, wl.renorm, wl.dtype, tokens=tokens)
    print(f"\n[{wl.name}] {rep}")
    return rep


# --------------------------------------------------------------- edge cases --

EDGE = [
    Workload("f32_ragged", T=300, d=64, E=6, k=3, I=96, renorm=True, dtype="f32", router_std=0.5),
    Workload("f32_norenorm", T=77, d=36, E=5, k=2, I=20, renorm=False, dtype="f32", router_std=0.5),
    Workload("f32_dense_E1", T=33, d=32, E=1, k=1, I=48, renorm=True, dtype="f32"),
    Workload("f32_T1", T=1, d=128, E=4, k=2, I=256, renorm=True, dtype="f32", router_std=0.5),
    Workload("bf16_T1", T=1, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16", router_std=0.3),
    Workload("bf16_T7", T=7, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16", router_std=0.3),
    Workload("bf16_ragged_tails", T=129, d=192, E=5, k=3, I=320, renorm=True, dtype="bf16", router_std=0.3),
    Workload("bf16_norenorm_bias", T=300, d=256, E=8, k=2, I=512, renorm=False, dtype="bf16", zipf_bias=True),
    Workload("bf16_dense_E1", T=200, d=128, E=1, k=1, I=256, renorm=True, dtype="bf16"),
    Workload("bf16_k_eq_E", T=150, d=128, E=4, k=4, I=192, renorm=True, dtype="bf16"),
    Workload("bf16_max_E256_k8", T=96, d=64, E=256, k=8, I=64, renorm=True, dtype="bf16", router_std=0.5),
    Workload("bf16_many_tiles", T=1000, d=256, E=3, k=2, I=384, renorm=True, dtype="bf16", router_std=0.1),
    # the GEMMs' configurations: at most 32 tokens (every tile in the 16-row
    # token box), one more token, and an expert that receives all 32 tokens
    Workload("bf16_T32_all_experts_full", T=32, d=256, E=8, k=8, I=256, renorm=True, dtype="bf16", router_std=0.3),
    Workload("bf16_T33", T=33, d=256, E=4, k=2, I=192, renorm=False, dtype="bf16", router_std=0.3),
    Workload("bf16_T32_one_expert", T=32, d=128, E=1, k=1, I=320, renorm=True, dtype="bf16"),
]


@pytest.mark.parametrize("wl", EDGE, ids=[w.name for w in EDGE])
def test_edge_case(wl):
    inp, res, perm = run(wl, seed=3)
    check(wl, inp, res, perm)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_zero_router_ties_to_lower_index(dtype):
    wl = Workload("zero_router", T=70, d=128, E=6, k=3, I=128, renorm=True, dtype=dtype)
    inp = make_inputs(wl, "cuda", 5)
    inp.w_router.zero_()
    inp, res, perm = run(wl, inp)
    idx = res.topk_idx.cpu().numpy()
    assert (idx == np.arange(3)).all()
    np.testing.assert_allclose(res.topk_gate.cpu().numpy(), 1.0 / 3, rtol=1e-6)
    np.testing.assert_array_equal(res.counts.cpu().numpy(), [70, 70, 70, 0, 0, 0])
    assert abs(float(res.aux.cpu()[0]) - 1.0) < 1e-6
    check(wl, inp, res, perm)


def test_duplicate_router_rows_tie():
    wl = Workload("dup_rows", T=64, d=128, E=5, k=2, I=128, renorm=True, dtype="bf16")
    inp = make_inputs(wl, "cuda", 6)
    big = torch.sign(inp.x.float().mean(0)) * 0.5
    inp.w_router[3] = big.to(inp.w_router.dtype)
    inp.w_router[1] = inp.w_router[3]
    inp, res, perm = run(wl, inp)
    idx = res.topk_idx.cpu().numpy()
    probs_equal_top = [t for t in range(wl.T) if set(idx[t]) == {1, 3}]
    assert probs_equal_top, "the shared row should win for some tokens"
    for t in probs_equal_top:
        assert list(idx[t]) == [1, 3]
    check(wl, inp, res, perm)


def test_unused_experts():
    wl = Workload("unused", T=257, d=128, E=6, k=2, I=192, renorm=True, dtype="bf16")
    inp = make_inputs(wl, "cuda", 7)
    inp.b_router = torch.tensor([0, -40.0, 0, -40.0, 0, 0], device="cuda")
    inp, res, perm = run(wl, inp)
    counts = res.counts.cpu().numpy()
    assert counts[1] == 0 and counts[3] == 0
    check(wl, inp, res, perm)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_zero_tokens(dtype):
    wl = Workload("empty", T=0, d=128, E=4, k=2, I=128, renorm=True, dtype=dtype)
    inp = make_inputs(wl, "cuda", 0)
    res = moe_forward(inp.x, inp.w_router, None, inp.w_gate, inp.w_up, inp.w_down, 2, True)
    torch.cuda.synchronize()
    assert res.out.shape == (0, 128)
    np.testing.assert_array_equal(res.counts.cpu().numpy(), 0)
    assert float(res.aux.cpu()[0]) == 0.0
    assert int(res.status.cpu()[0]) == 0


def test_bit_deterministic():
    wl = Workload("determinism", T=777, d=256, E=8, k=2, I=384, renorm=True, dtype="bf16")
    inp = make_inputs(wl, "cuda", 8)
    a = moe_forward(inp.x, inp.w_router, None, inp.w_gate, inp.w_up, inp.w_down, 2, True)
    b = moe_forward(inp.x, inp.w_router, None, inp.w_gate, inp.w_up, inp.w_down, 2, True)
    torch.cuda.synchronize()
    assert torch.equal(a.out, b.out)
    assert torch.equal(a.topk_idx, b.topk_idx) and torch.equal(a.topk_gate, b.topk_gate)
    assert torch.equal(a.aux, b.aux)


def test_nonfinite_logit_sets_status_and_stays_in_bounds():
    wl = Workload("nonfinite", T=64, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16")
    inp = make_inputs(wl, "cuda", 9)
    inp.x[5, 3] = float("inf")
    inp.x[9, 0] = float("nan")
    res = moe_forward(inp.x, inp.w_router, None, inp.w_gate, inp.w_up, inp.w_down, 2, True)
    torch.cuda.synchronize()
    st = int(res.status.cpu()[0])
    assert st & B.MOE_DEV_NONFINITE
    assert not st & (B.MOE_DEV_TIMEOUT | B.MOE_DEV_INTERNAL)
    idx = res.topk_idx.cpu().numpy()
    assert ((idx >= 0) & (idx < 4)).all()
    assert int(res.counts.cpu().sum()) == 128
    # tokens without a non-finite value are unaffected
    good = [t for t in range(64) if t not in (5, 9)]
    assert torch.isfinite(res.out[good]).all()


# ---------------------------------------------------------------- workloads --

def test_tiny_f32_all_tokens():
    wl = WORKLOADS["tiny_f32"]
    inp, res, perm = run(wl)
    check(wl, inp, res, perm)


def test_small_bf16_all_tokens():
    wl = WORKLOADS["small_bf16"]
    inp, res, perm = run(wl)
    check(wl, inp, res, perm)


def test_mixtral_prefill_full_size_all_tokens():
    wl = WORKLOADS["mixtral_prefill"]
    inp, res, perm = run(wl)
    check(wl, inp, res, perm)


def test_fine_grained_full_size_all_tokens():
    wl = WORKLOADS["fine_grained"]
    inp, res, perm = run(wl)
    counts = res.counts.cpu().numpy()
    assert counts[0] > 2 * counts.mean(), "the Zipf-like bias should skew the load towards expert 0"
    check(wl, inp, res, perm)


def test_large_batch_all_tokens():
    """A batch far past the benchmark workloads: 131072 tokens (1024 router
    blocks, so the routing scan sums 8 blocks per slice over 128 slices, and
    about 1030 token tiles across the GEMM groups), every token compared."""
    wl = Workload("large_batch", T=131072, d=1024, E=8, k=2, I=128, renorm=True, dtype="bf16")
    inp, res, perm = run(wl, seed=12)
    check(wl, inp, res, perm)


@pytest.mark.parametrize("T,E,dtype,merged", [(65536, 8, "bf16", True), (65664, 8, "bf16", False),
                                              (4096, 32, "f32", True), (4128, 32, "f32", False)])
def test_routing_scan_in_permute_at_its_limit(T, E, dtype, merged):
    """The permute does the routing scan while router blocks x experts stay
    at most 4096 (bf16: 512 blocks of 128 tokens x 8 experts; fp32: 128
    blocks of 32 tokens x 32 experts) and the scan kernel runs one block
    later: both sides of the limit give every token's output, the counts
    and the permutation of the oracle."""
    from sparse_mixture_experts_renorm_b200 import launch_plan

    wl = Workload(f"scan_limit_{T}_{E}_{dtype}", T=T, d=256 if dtype == "bf16" else 64, E=E, k=2,
                  I=128 if dtype == "bf16" else 64, renorm=True, dtype=dtype)
    plan = launch_plan(wl.T, wl.d, wl.E, wl.k, wl.I, wl.torch_dtype)
    assert bool(plan & B.MOE_PLAN_PERMUTE_SCAN) == merged
    inp, res, perm = run(wl, seed=14)
    check(wl, inp, res, perm)


@pytest.mark.parametrize("T", [6016, 6144])
def test_down_projection_forms_at_their_switch(T):
    """The down GEMM (k = 2, combine folded in) runs token-major while its
    grid has at most three tiles per CTA pair (6016 tokens: 220 tiles upper
    bound on 148 SMs) and weight-major above (6144 tokens: 224): every token
    of both compared with the oracle."""
    wl = Workload(f"down_forms_{T}", T=T, d=1024, E=8, k=2, I=256, renorm=True, dtype="bf16")
    inp, res, perm = run(wl, seed=15)
    check(wl, inp, res, perm)


@pytest.mark.parametrize("T", [255, 256])
def test_gateup_forms_at_their_switch(T):
    """The gate/up GEMM runs token-major once the batch averages 64 rows per
    expert (R = 512 with E = 8) and weight-major (narrow) below."""
    wl = Workload(f"gateup_forms_{T}", T=T, d=256, E=8, k=2, I=256, renorm=False, dtype="bf16")
    inp, res, perm = run(wl, seed=16)
    check(wl, inp, res, perm)


def test_most_experts_with_many_tokens():
    """The largest expert count (256) and top-k (8) at 2048 tokens: 256 GEMM
    groups of about 64 rows, the router's shared-memory path and a scan over
    four slices of 256 experts."""
    wl = Workload("max_experts", T=2048, d=256, E=256, k=8, I=128, renorm=True, dtype="bf16", router_std=0.3)
    inp, res, perm = run(wl, seed=13)
    check(wl, inp, res, perm)


def test_mixtral_decode_all_tokens():
    wl = WORKLOADS["mixtral_decode"]
    inp, res, perm = run(wl)
    check(wl, inp, res, perm)


# ------------------------------------------------------- router logit error --

@pytest.mark.parametrize("name", ["mixtral_prefill", "small_bf16", "tiny_f32"])
def test_router_logit_error_pin(name):
    """Measures the router's logit error against fp64 and holds it to the bar
    the gate tolerance is derived from. With k = E and no renormalisation the
    gates are the whole softmax, so log(g_j) - log(g_0) = l_j - l_0: the GPU's
    logit differences, read back through the C ABI, against the oracle's
    fp64 logits of the same stored x and W_r (the workload's first two draws;
    the experts are shrunk to I = 64 since only the router matters here).
    The read-back adds the fp32 rounding of the exponential and of the gate,
    a few 1e-7 at most."""
    base = WORKLOADS[name]
    wl = base.replace(name=name + "_logits", k=base.E, renorm=False, I=64)
    inp, res, _ = run(wl)
    import oracle

    l_o = oracle.router_logits(inp.x.cpu(), inp.w_router.cpu(), None if inp.b_router is None else inp.b_router.cpu())
    idx = res.topk_idx.cpu().numpy().astype(np.int64)
    g = res.topk_gate.cpu().numpy().astype(np.float64)
    assert (g > 0).all()
    lg = np.log(g)
    d_gpu = lg[:, 1:] - lg[:, :1]
    lo = np.take_along_axis(l_o, idx, axis=1)
    d_ora = lo[:, 1:] - lo[:, :1]
    err = float(np.abs(d_gpu - d_ora).max())
    # each difference carries two logits' errors
    logit_err = err / 2
    print(f"\n[{name}] router logit error (half the max error of a logit difference): {logit_err:.3e}")
    assert logit_err <= parity.LOGIT_TOL[base.dtype], (logit_err, parity.LOGIT_TOL[base.dtype])
    assert parity.GATE_TOL[base.dtype] >= parity.LOGIT_TOL[base.dtype] / 2


# ---------------------------------------------------------- failure handling --

def test_bounded_wait_gives_up_and_reports():
    """A barrier wait that can never complete gives up after its limit and sets
    MOE_DEV_TIMEOUT; the context stays usable (a forward runs afterwards)."""
    import ctypes
    import time

    lib = B.load_library()
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    st = lib.moe_selftest_wait_timeout(ctypes.c_void_p(status.data_ptr()), 50_000_000,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.MOE_OK
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(status.item()) & B.MOE_DEV_TIMEOUT
    wl = Workload("after_timeout", T=40, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16", router_std=0.3)
    inp, res, perm = run(wl, seed=11)
    check(wl, inp, res, perm)


# ------------------------------------------------------------- CUDA graphs --

@pytest.mark.parametrize("name", ["mixtral_decode", "small_bf16"])
def test_layer_replays_from_a_cuda_graph(name):
    """The whole call (its kernels chained by programmatic dependent launch)
    can be captured once and replayed: the replay gives bit-identical outputs
    to the eager call, also on a second batch copied into the captured input
    buffer. The layer's status word is OR-ed by every call and never cleared
    here, so the final check covers the warm-up, the capture and both
    replays."""
    from sparse_mixture_experts_renorm_b200 import MoELayer
    from sparse_mixture_experts_renorm_b200.workloads import make_tokens

    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda", 0)
    layer = MoELayer(inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm, wl.T)
    x = inp.x.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # x and the weights were written on the current stream
    with torch.cuda.stream(s):
        for _ in range(2):  # warm-up outside the capture (attributes, occupancy queries)
            layer(x, stream=s.cuda_stream)
    torch.cuda.synchronize()
    eager = layer.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer(x, stream=s.cuda_stream)
    layer.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.out, eager)
    x2 = make_tokens(wl, wl.T, "cuda", seed=7)
    ref2 = moe_forward(x2, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.out, ref2.out) and torch.equal(layer.topk_idx, ref2.topk_idx)
    assert int(layer.status.item()) == 0


# ------------------------------------------------------- host-memory path --

@pytest.mark.parametrize("name", ["small_bf16", "tiny_f32", "mixtral_decode"])
def test_host_pipeline_matches_device_calls(name):
    """The end-to-end path (pinned host batches in, copies on their own
    streams overlapped with the compute of neighbouring batches, fp32 output
    and statistic back to pinned host memory) returns, for every batch, the
    bit-identical output and statistic of a plain device call on the same
    batch, also when batches reuse the two device buffers in turn."""
    from sparse_mixture_experts_renorm_b200 import HostPipeline, MoELayer
    from sparse_mixture_experts_renorm_b200.workloads import make_tokens

    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda", 0)
    layer = MoELayer(inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm, wl.T)
    pipe = HostPipeline(layer)
    n = 5
    xs = [make_tokens(wl, wl.T, "cpu", seed=100 + i).pin_memory() for i in range(n)]
    outs = [torch.empty((wl.T, wl.d), dtype=torch.float32).pin_memory() for _ in range(n)]
    auxs = [torch.empty((1,), dtype=torch.float32).pin_memory() for _ in range(n)]
    for i in range(n):
        pipe.submit(xs[i], outs[i], auxs[i])
    pipe.synchronize()
    assert int(layer.status.item()) == 0
    for i in range(n):
        ref = moe_forward(xs[i].cuda(), inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k,
                          wl.renorm)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref.out.cpu()), f"batch {i}"
        assert torch.equal(auxs[i], ref.aux.cpu()), f"batch {i}"
