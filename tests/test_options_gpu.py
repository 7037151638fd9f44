"""GPU parity of the layer's options against the fp64 oracle: the pre-MoE
RMSNorm (both forms), the router z-loss, capacity-factor dropping and shared
experts, alone and together, on both dtypes, through the C ABI
(moe_forward_ex)."""
import numpy as np
import pytest
import torch

import parity
from sparse_mixture_experts_renorm_b200 import MoEOptions, get_permutation, moe_forward
from sparse_mixture_experts_renorm_b200.workloads import WORKLOADS, Workload, make_inputs, make_option_inputs

pytestmark = pytest.mark.gpu

# (workload, norm_form, norm_weight, n_shared, capacity_factor, z_loss)
CASES = [
    (Workload("bf16_norm_torch_w", T=300, d=512, E=8, k=2, I=512, renorm=True, dtype="bf16", x_std=3.0,
              router_std=0.05), 1, True, 0, 0.0, True),
    (Workload("bf16_norm_page_now", T=257, d=256, E=6, k=3, I=320, renorm=True, dtype="bf16", x_std=0.5,
              router_std=0.1), 2, False, 0, 0.0, True),
    (Workload("bf16_norm_E64_split", T=700, d=384, E=64, k=6, I=128, renorm=False, dtype="bf16", x_std=2.0,
              router_std=0.1, zipf_bias=True), 1, True, 0, 0.0, True),
    (Workload("bf16_norm_E100_smem", T=200, d=192, E=100, k=4, I=64, renorm=True, dtype="bf16", x_std=2.0,
              router_std=0.2), 1, True, 0, 0.0, True),
    (Workload("f32_norm_torch_w", T=150, d=96, E=5, k=2, I=64, renorm=True, dtype="f32", x_std=3.0,
              router_std=0.5), 1, True, 0, 0.0, True),
    (Workload("f32_norm_page_w", T=70, d=64, E=4, k=1, I=48, renorm=False, dtype="f32", x_std=0.3,
              router_std=0.5), 2, True, 0, 0.0, False),
    (Workload("bf16_capacity_fused_k2", T=600, d=256, E=8, k=2, I=256, renorm=True, dtype="bf16",
              router_std=0.05, zipf_bias=True), 0, False, 0, 1.0, False),
    (Workload("bf16_capacity_k3", T=333, d=128, E=6, k=3, I=192, renorm=True, dtype="bf16", router_std=0.1,
              zipf_bias=True), 0, False, 0, 0.5, True),
    (Workload("f32_capacity", T=200, d=64, E=4, k=2, I=64, renorm=True, dtype="f32", router_std=0.5,
              zipf_bias=True), 0, False, 0, 0.75, False),
    (Workload("bf16_shared1_k2", T=300, d=256, E=8, k=2, I=256, renorm=True, dtype="bf16", router_std=0.1), 0,
     False, 1, 0.0, False),
    (Workload("bf16_shared2_tails", T=129, d=192, E=4, k=1, I=320, renorm=True, dtype="bf16", router_std=0.1), 0,
     False, 2, 0.0, False),
    (Workload("f32_shared1", T=90, d=64, E=4, k=2, I=96, renorm=True, dtype="f32", router_std=0.5), 0, False, 1,
     0.0, True),
    (Workload("bf16_all_options", T=1000, d=256, E=16, k=4, I=256, renorm=True, dtype="bf16", x_std=2.0,
              router_std=0.1, zipf_bias=True), 1, True, 2, 1.25, True),
    (Workload("f32_all_options", T=100, d=64, E=6, k=2, I=64, renorm=False, dtype="f32", x_std=2.0, router_std=0.5,
              zipf_bias=True), 2, True, 1, 1.0, True),
    (Workload("bf16_decode_all_options", T=32, d=512, E=8, k=2, I=512, renorm=True, dtype="bf16", x_std=2.0,
              router_std=0.1, zipf_bias=True), 1, True, 1, 1.0, True),
]


def make_options(wl, norm_form, norm_weight, n_shared, cf, z, seed=3):
    oi = make_option_inputs(wl, "cuda", seed, n_shared=n_shared, norm_weight=norm_weight)
    return MoEOptions(norm_form=norm_form, norm_eps=1e-5, norm_weight=oi.norm_weight, shared_gate=oi.shared_gate,
                      shared_up=oi.shared_up, shared_down=oi.shared_down, capacity_factor=cf, z_loss=z)


def run(wl, options, seed=3, inp=None):
    if inp is None:
        inp = make_inputs(wl, "cuda", seed)
    res = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                      options=options)
    torch.cuda.synchronize()
    perm = get_permutation(res, wl.T, wl.d, wl.E, wl.k, wl.I, inp.x.dtype)
    torch.cuda.synchronize()
    return inp, res, perm


@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_option_parity(case):
    wl, form, nw, ns, cf, z = case
    opts = make_options(wl, form, nw, ns, cf, z)
    inp, res, perm = run(wl, opts)
    rep = parity.check(inp, res, perm, wl.k, wl.renorm, wl.dtype, options=opts)
    print(f"\n[{wl.name}] {rep}")
    if cf > 0:
        assert rep["dropped"] > 0, "the capacity case should drop assignments"


def test_plain_options_are_bit_identical_to_moe_forward():
    """A default options struct runs exactly the plain layer."""
    wl = Workload("plain", T=300, d=256, E=8, k=2, I=256, renorm=True, dtype="bf16", router_std=0.1)
    inp = make_inputs(wl, "cuda", 5)
    a = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    b = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                    options=MoEOptions())
    torch.cuda.synchronize()
    assert torch.equal(a.out, b.out) and torch.equal(a.topk_idx, b.topk_idx) and torch.equal(a.topk_gate, b.topk_gate)


def test_options_are_deterministic():
    wl, form, nw, ns, cf, z = CASES[12]
    opts = make_options(wl, form, nw, ns, cf, z)
    inp, r1, _ = run(wl, opts)
    out1, zl1, dr1 = r1.out.clone(), r1.z_loss.clone(), r1.dropped.clone()
    _, r2, _ = run(wl, opts, inp=inp)
    assert torch.equal(out1, r2.out) and torch.equal(zl1, r2.z_loss) and torch.equal(dr1, r2.dropped)


def test_capacity_large_factor_drops_nothing():
    wl = Workload("cap_large", T=256, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16", router_std=0.1)
    inp = make_inputs(wl, "cuda", 9)
    plain = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    capped = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                         options=MoEOptions(capacity_factor=float(wl.E)))
    torch.cuda.synchronize()
    assert int(capped.dropped.item()) == 0
    assert torch.equal(plain.out, capped.out)


def test_t0_with_options():
    wl = Workload("t0", T=0, d=128, E=4, k=2, I=128, renorm=True, dtype="bf16")
    inp = make_inputs(wl, "cuda", 1)
    opts = make_options(wl, 1, True, 1, 1.0, True)
    res = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                      options=opts)
    torch.cuda.synchronize()
    assert float(res.z_loss.item()) == 0.0 and int(res.dropped.item()) == 0
    assert int(res.counts.sum().item()) == 0


@pytest.mark.parametrize("name", ["mixtral_prefill", "fine_grained"])
def test_full_size_with_all_options(name):
    """Full-size workload with the norm, shared experts (one at the Mixtral
    shape, two at the fine-grained one), a capacity of 1.25 and the z-loss;
    every token's output row is compared."""
    wl = WORKLOADS[name]
    opts = make_options(wl, 1, True, 2 if name == "fine_grained" else 1, 1.25, True)
    inp, res, perm = run(wl, opts, seed=0)
    rep = parity.check(inp, res, perm, wl.k, wl.renorm, wl.dtype, options=opts)
    print(f"\n[{wl.name}+options] {rep}")
    assert np.isfinite(rep["max_abs"])


# fold_combine: the combine done by the down GEMM's epilogue for every top-k
# (fp32 atomic adds into the zeroed output): the same parity bars, and at full
# size the output of the combine kernel up to the order of a token's adds.
FOLD_CASES = [
    (Workload("bf16_fold_k6_E64", T=700, d=256, E=64, k=6, I=128, renorm=False, dtype="bf16", router_std=0.1,
              zipf_bias=True), 0.0),
    (Workload("bf16_fold_k3_capacity", T=333, d=128, E=6, k=3, I=192, renorm=True, dtype="bf16", router_std=0.1,
              zipf_bias=True), 0.5),
    (Workload("bf16_fold_k1", T=200, d=128, E=4, k=1, I=256, renorm=True, dtype="bf16", router_std=0.3), 0.0),
    (Workload("bf16_fold_k4_decode", T=24, d=256, E=8, k=4, I=256, renorm=True, dtype="bf16", router_std=0.3), 0.0),
]


@pytest.mark.parametrize("case", FOLD_CASES, ids=[c[0].name for c in FOLD_CASES])
def test_fold_combine_parity(case):
    wl, cf = case
    opts = MoEOptions(capacity_factor=cf, fold_combine=True)
    inp, res, perm = run(wl, opts)
    rep = parity.check(inp, res, perm, wl.k, wl.renorm, wl.dtype, options=opts)
    print(f"\n[{wl.name}] {rep}")
    if cf > 0:
        assert rep["dropped"] > 0, "the capacity case should drop assignments"


def test_fold_combine_full_size_matches_the_combine_kernel():
    """fine_grained (k = 6) with the folded combine against the default
    path on the same inputs: identical routing and dispatch, and outputs
    equal up to fp32 rounding of a different order of six additions."""
    wl = WORKLOADS["fine_grained"]
    inp = make_inputs(wl, "cuda", 0)
    a = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    b = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                    options=MoEOptions(fold_combine=True))
    torch.cuda.synchronize()
    assert int(a.status.item()) == 0 and int(b.status.item()) == 0
    assert torch.equal(a.topk_idx, b.topk_idx) and torch.equal(a.topk_gate, b.topk_gate)
    assert torch.equal(a.counts, b.counts)
    scale = a.out.abs().max().item()
    diff = (a.out - b.out).abs().max().item()
    print(f"\n[fine_grained fold] max |out| {scale:.4g}, max-abs difference {diff:.3g}")
    assert diff <= 1e-5 * scale


def test_host_pipeline_with_options_matches_device_calls():
    """The library's host-memory pipeline carries the options (a copy taken
    at creation): every batch's output and statistic equal those of a plain
    device call with the same options, bit for bit."""
    from sparse_mixture_experts_renorm_b200 import HostPipeline, MoELayer
    from sparse_mixture_experts_renorm_b200.workloads import make_tokens

    wl, form, nw, ns, cf, z = CASES[12]
    opts = make_options(wl, form, nw, ns, cf, z)
    inp = make_inputs(wl, "cuda", 3)
    layer = MoELayer(inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm, wl.T,
                     options=opts)
    pipe = HostPipeline(layer)
    n = 4
    xs = [make_tokens(wl, wl.T, "cpu", seed=200 + i).pin_memory() for i in range(n)]
    outs = [torch.empty((wl.T, wl.d), dtype=torch.float32).pin_memory() for _ in range(n)]
    auxs = [torch.empty((1,), dtype=torch.float32).pin_memory() for _ in range(n)]
    for i in range(n):
        pipe.submit(xs[i], outs[i], auxs[i])
    pipe.synchronize()
    pipe.close()
    assert int(layer.status.item()) == 0
    for i in range(n):
        ref = moe_forward(xs[i].cuda(), inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k,
                          wl.renorm, options=opts)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref.out.cpu()), f"batch {i}"
        assert torch.equal(auxs[i], ref.aux.cpu()), f"batch {i}"
