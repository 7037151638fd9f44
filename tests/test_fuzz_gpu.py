"""GPU parity on seeded random shapes: T, d, E, k, I, renorm, the dtype, the
router bias and the layer's options drawn together, so that combinations the
hand-picked cases do not name (an odd expert count with the norm and a
capacity, k = E with shared experts, a ragged tail in every GEMM tile) are
compared with the fp64 oracle too. The draws are fixed by one numpy seed;
every case is run through the C ABI exactly like the named cases. Every
even-numbered case also sets fold_combine (the combine in the down GEMM's
epilogue for every top-k), so both combine paths meet the random shapes."""
import numpy as np
import pytest
import torch

import parity
from sparse_mixture_experts_renorm_b200 import MoEOptions, get_permutation, moe_forward
from sparse_mixture_experts_renorm_b200.workloads import Workload, make_inputs, make_option_inputs

N_CASES = 40
E_CHOICES = [1, 2, 3, 4, 5, 7, 8, 12, 16, 17, 24, 32, 33, 48, 64, 65, 100, 128, 200, 256]


def draw_cases(n=N_CASES, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        bf16 = rng.random() < 0.7
        if rng.random() < 0.3:
            T = int(rng.integers(1, 41))
        else:
            T = int(rng.integers(41, 401))
        d = 64 * int(rng.integers(1, 7)) if bf16 else 4 * int(rng.integers(1, 49))
        I = 64 * int(rng.integers(1, 7)) if bf16 else int(rng.integers(1, 201))
        E = int(rng.choice(E_CHOICES))
        k = int(rng.integers(1, min(E, 8) + 1))
        renorm = bool(rng.random() < 0.6)
        router_std = float(rng.choice([0.05, 0.2, 0.5]))
        zipf = bool(rng.random() < 0.3)
        norm_form = int(rng.choice([1, 2])) if rng.random() < 0.3 else 0
        norm_w = bool(norm_form and rng.random() < 0.7)
        n_shared = int(rng.integers(1, 3)) if rng.random() < 0.25 else 0
        cf = float(rng.uniform(0.5, 2.0)) if rng.random() < 0.3 else 0.0
        z = bool(rng.random() < 0.4)
        x_std = float(rng.choice([1.0, 2.0])) if norm_form else 1.0
        wl = Workload(f"fz{i:02d}", T=T, d=d, E=E, k=k, I=I, renorm=renorm, dtype="bf16" if bf16 else "f32",
                      x_std=x_std, router_std=router_std, zipf_bias=zipf)
        cases.append((wl, norm_form, norm_w, n_shared, cf, z))
    return cases


CASES = draw_cases()


def folds(wl) -> bool:
    """Even-numbered cases run with fold_combine (the draws stay the same)."""
    return int(wl.name[2:]) % 2 == 0


def case_id(c):
    wl, form, nw, ns, cf, z = c
    opts = "".join([f"n{form}" if form else "", "w" if nw else "", f"s{ns}" if ns else "",
                    f"c{cf:.2f}" if cf else "", "z" if z else "", "f" if folds(wl) else ""])
    return (f"{wl.name}-{wl.dtype}-T{wl.T}-d{wl.d}-E{wl.E}-k{wl.k}-I{wl.I}-{'r' if wl.renorm else 'nr'}"
            + (f"-{opts}" if opts else ""))


def test_draws_cover_the_options_and_shapes():
    """The fixed draw reaches every option, both dtypes, both renorm
    settings, the register and shared-memory router paths (E <= 16 and
    E > 16) and the short-batch GEMM configuration (T <= 32)."""
    wls = [c[0] for c in CASES]
    assert {w.dtype for w in wls} == {"bf16", "f32"}
    assert {w.renorm for w in wls} == {True, False}
    assert any(w.E <= 16 for w in wls) and any(w.E > 16 for w in wls)
    assert any(w.T <= 32 and w.dtype == "bf16" for w in wls)
    assert any(c[1] == 1 for c in CASES) and any(c[1] == 2 for c in CASES)
    assert any(c[3] for c in CASES) and any(c[4] for c in CASES) and any(c[5] for c in CASES)
    # the folded combine on the bf16 path with k != 2 and no shared experts, where it changes the plan
    assert any(folds(c[0]) and c[0].dtype == "bf16" and c[0].k != 2 and not c[3] for c in CASES)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[case_id(c) for c in CASES])
def test_random_shape_parity(case):
    wl, form, nw, ns, cf, z = case
    inp = make_inputs(wl, "cuda", 17)
    opts = None
    if form or ns or cf or z or folds(wl):
        oi = make_option_inputs(wl, "cuda", 17, n_shared=ns, norm_weight=nw)
        opts = MoEOptions(norm_form=form, norm_eps=1e-5, norm_weight=oi.norm_weight, shared_gate=oi.shared_gate,
                          shared_up=oi.shared_up, shared_down=oi.shared_down, capacity_factor=cf, z_loss=z,
                          fold_combine=folds(wl))
    res = moe_forward(inp.x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm,
                      options=opts)
    torch.cuda.synchronize()
    perm = get_permutation(res, wl.T, wl.d, wl.E, wl.k, wl.I, inp.x.dtype)
    torch.cuda.synchronize()
    assert int(res.status.item()) == 0
    rep = parity.check(inp, res, perm, wl.k, wl.renorm, wl.dtype, options=opts)
    print(f"\n[{case_id(case)}] {rep}")
