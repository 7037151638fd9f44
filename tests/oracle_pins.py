"""Pins that tie the fp64 oracle to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
an independent fact: a brute-force per-token formulation written with plain
loops, a dense SwiGLU computed by torch in fp64 (a library routine), closed
forms, the tie rule on exact ties, the uniform-routing value of the
load-balancing statistic, a stable library sort for the dispatch order, and
the structural facts printed on the pages. ``tests/test_oracle.py`` runs them
against the oracle; ``tests/test_oracle_mutants.py`` runs them against copies
of the oracle with planted mistakes and requires that some pin fails.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# helpers (input construction only; no layer arithmetic)
# ---------------------------------------------------------------------------

def _rand_case(T, d, E, k, I, dtype, seed, router_std=0.7, bias=False):
    g = torch.Generator().manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn((T, d), generator=g).to(dt)
    wr = (torch.randn((E, d), generator=g) * router_std).to(dt)
    wg = (torch.randn((E, I, d), generator=g) * 0.3).to(dt)
    wu = (torch.randn((E, I, d), generator=g) * 0.3).to(dt)
    wd = (torch.randn((E, d, I), generator=g) * 0.3).to(dt)
    b = (torch.randn((E,), generator=g) * 0.5) if bias else None
    return x, wr, b, wg, wu, wd


def _f64(t):
    return t.detach().to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def brute_force(x, wr, b, wg, wu, wd, k, renorm):
    """Second formulation: per token, a literal softmax, top-k by k passes of a
    strict-greater arg-max scan in ascending expert order (so an exact tie
    keeps the lower index), then every expert evaluated densely and weighted
    by its gate if selected, zero otherwise. No sort, no dispatch."""
    X, WR, WG, WU, WD = (_f64(a) for a in (x, wr, wg, wu, wd))
    B = np.zeros(WR.shape[0]) if b is None else _f64(b)
    T, d = X.shape
    E = WR.shape[0]
    probs = np.zeros((T, E))
    idx = np.zeros((T, k), dtype=np.int64)
    gates = np.zeros((T, k))
    out = np.zeros((T, d))
    for t in range(T):
        logits = []
        for e in range(E):
            s = 0.0
            for c in range(d):
                s += X[t, c] * WR[e, c]
            logits.append(s + B[e])
        m = max(logits)
        ex = [math.exp(v - m) for v in logits]
        z = sum(ex)
        p = [v / z for v in ex]
        probs[t] = p
        chosen = []
        for _ in range(k):
            best = -1
            for e in range(E):
                if e in chosen:
                    continue
                if best < 0 or p[e] > p[best]:
                    best = e
            chosen.append(best)
        w = [p[e] for e in chosen]
        if renorm:
            sw = sum(w)
            w = [v / sw for v in w] if sw > 0 else [1.0 / k] * k
        idx[t] = chosen
        gates[t] = w
        for e in range(E):
            mult = w[chosen.index(e)] if e in chosen else 0.0
            gpre = WG[e] @ X[t]
            upre = WU[e] @ X[t]
            h = gpre / (1.0 + np.exp(-gpre)) * upre
            out[t] += mult * (WD[e] @ h)
    return probs, idx, gates, out


def dense_swiglu_torch(x, wg, wu, wd):
    """torch fp64 SwiGLU MLP of one expert: down(silu(gate x) * up x)."""
    X, G, U, D = (torch.as_tensor(_f64(a)) for a in (x, wg, wu, wd))
    return (F.silu(X @ G.T) * (X @ U.T)) @ D.T


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

BRUTE_CASES = [
    # T, d, E, k, I, dtype, renorm, bias, seed
    (9, 16, 4, 2, 24, "f32", True, False, 1),
    (11, 24, 5, 3, 40, "bf16", True, True, 2),
    (7, 16, 6, 2, 20, "f32", False, True, 3),
    (5, 8, 3, 1, 12, "bf16", False, False, 4),
    (6, 12, 4, 4, 10, "f32", True, False, 5),
]


def pin_brute_force():
    for (T, d, E, k, I, dt, renorm, bias, seed) in BRUTE_CASES:
        x, wr, b, wg, wu, wd = _rand_case(T, d, E, k, I, dt, seed, bias=bias)
        bp, bidx, bg, bout = brute_force(x, wr, b, wg, wu, wd, k, renorm)
        r = oracle.forward(x, wr, b, wg, wu, wd, k, renorm)
        np.testing.assert_allclose(r.probs, bp, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(r.topk_idx, bidx)
        np.testing.assert_allclose(r.topk_gate, bg, rtol=0, atol=1e-13)
        scale = max(1.0, float(np.abs(bout).max()))
        np.testing.assert_allclose(r.out, bout, rtol=0, atol=1e-11 * scale)


def pin_gates_sum_to_one():
    x, wr, b, wg, wu, wd = _rand_case(64, 16, 8, 3, 8, "bf16", 11, router_std=0.2)
    probs = oracle.router_probs(x, wr, b)
    _, gate, _ = oracle.topk(probs, 3, renorm=True)
    np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # without renorm the gates are the raw probabilities, which sum to < 1
    _, raw, _ = oracle.topk(probs, 3, renorm=False)
    assert np.all(raw.sum(axis=1) < 1.0)


def pin_dense_E1_k1():
    """E=1, k=1: the layer is one dense SwiGLU MLP."""
    x, wr, b, wg, wu, wd = _rand_case(13, 24, 1, 1, 40, "bf16", 7)
    r = oracle.forward(x, wr, b, wg, wu, wd, 1, renorm=True)
    ref = dense_swiglu_torch(x, wg[0], wu[0], wd[0]).numpy()
    np.testing.assert_array_equal(r.topk_idx, 0)
    np.testing.assert_allclose(r.topk_gate, 1.0, rtol=0, atol=0)
    np.testing.assert_allclose(r.out, ref, rtol=0, atol=1e-11 * max(1.0, np.abs(ref).max()))
    # without renorm the single gate is p = 1 as well
    r0 = oracle.forward(x, wr, b, wg, wu, wd, 1, renorm=False)
    np.testing.assert_allclose(r0.out, ref, rtol=0, atol=1e-11 * max(1.0, np.abs(ref).max()))


def pin_soft_mixture_k_eq_E():
    """k = E with renorm: out = sum_e p_e * SwiGLU_e(x), a dense soft mixture."""
    T, d, E, I = 10, 16, 4, 24
    x, wr, b, wg, wu, wd = _rand_case(T, d, E, E, I, "f32", 8, bias=True)
    r = oracle.forward(x, wr, b, wg, wu, wd, E, renorm=True)
    logits = torch.as_tensor(_f64(x)) @ torch.as_tensor(_f64(wr)).T + torch.as_tensor(_f64(b))
    p = torch.softmax(logits, dim=-1)
    ref = sum(p[:, e:e + 1] * dense_swiglu_torch(x, wg[e], wu[e], wd[e]) for e in range(E)).numpy()
    np.testing.assert_allclose(r.probs, p.numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(r.out, ref, rtol=0, atol=1e-11 * max(1.0, np.abs(ref).max()))


def pin_zero_router():
    """W_r = 0: every p = 1/E exactly, so the tie rule selects experts 0..k-1
    in order; the gates are 1/k (renorm) or 1/E; aux = 1 (uniform P)."""
    T, d, E, k, I = 12, 16, 6, 3, 8
    x, wr, b, wg, wu, wd = _rand_case(T, d, E, k, I, "bf16", 9)
    wr = torch.zeros_like(wr)
    for renorm, g in ((True, 1.0 / k), (False, 1.0 / E)):
        r = oracle.forward(x, wr, None, wg, wu, wd, k, renorm)
        np.testing.assert_array_equal(r.topk_idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
        np.testing.assert_allclose(r.topk_gate, g, rtol=1e-15, atol=0)
        np.testing.assert_array_equal(r.counts, [T] * k + [0] * (E - k))
        assert abs(r.aux - 1.0) < 1e-14
        np.testing.assert_array_equal(r.gap, 0.0)


def pin_uniform_counts_aux():
    """Uniform f (every expert receives T*k/E assignments): aux = sum_e P_e = 1
    whatever the probabilities are."""
    E, k, T, d = 4, 2, 16, 4
    x = torch.zeros((T, d))
    for t in range(T):
        x[t, t % E] = 3.0 + 0.1 * (t % 3)
        x[t, (t + 1) % E] = 1.5
    wr = torch.eye(E, d)
    wg = torch.zeros((E, 3, d))
    wd = torch.zeros((E, d, 3))
    r = oracle.forward(x, wr, None, wg, wg, wd, k, renorm=True)
    np.testing.assert_array_equal(r.counts, [T * k // E] * E)
    assert abs(r.aux - 1.0) < 1e-14
    # the statistic is E * sum_e f_e * P_e with sum_e f_e = 1; the page's own
    # normalisation by T alone is k times larger
    assert abs(r.counts.sum() / T - k) == 0


def pin_aux_closed_form():
    """A hand-sized case: E=2, k=1, logits (a, 0) for every token, with
    f = (1, 0) when a > 0: aux = 2 * sigmoid(a)."""
    a = 0.75  # exact in fp32
    T = 5
    x = torch.ones((T, 1))
    wr = torch.tensor([[a], [0.0]])
    w3 = torch.zeros((2, 1, 1))
    r = oracle.forward(x, wr, None, w3, w3, w3, 1, renorm=False)
    sig = 1.0 / (1.0 + math.exp(-a))
    np.testing.assert_allclose(r.probs[:, 0], sig, rtol=1e-15)
    np.testing.assert_array_equal(r.counts, [T, 0])
    assert abs(r.aux - 2.0 * sig) < 1e-15
    np.testing.assert_allclose(r.topk_gate[:, 0], sig, rtol=1e-15)
    np.testing.assert_allclose(r.gap, sig - (1 - sig), rtol=1e-14)


def pin_expert_closed_form():
    """d=2, I=3 with small integer weights, worked by hand:
    gate pre-activations g_i = sum_c Wg[i,c] x_c, up u_i likewise,
    h_i = g_i / (1 + e^{-g_i}) * u_i, y_o = sum_i Wd[o,i] h_i."""
    x = torch.tensor([[1.0, -2.0]])
    wg = torch.tensor([[[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]]])   # g = (1, -2, -1)
    wu = torch.tensor([[[2.0, 1.0], [1.0, 0.0], [0.0, -1.0]]])  # u = (0, 1, 2)
    wd = torch.tensor([[[1.0, 2.0, 3.0], [-1.0, 0.0, 1.0]]])
    h = [1.0 / (1 + math.exp(-1.0)) * 0.0, -2.0 / (1 + math.exp(2.0)) * 1.0, -1.0 / (1 + math.exp(1.0)) * 2.0]
    y = [1.0 * h[0] + 2.0 * h[1] + 3.0 * h[2], -1.0 * h[0] + 0.0 * h[1] + 1.0 * h[2]]
    got = oracle.expert_rows(x, wg, wu, wd, [0], [0])
    np.testing.assert_allclose(got[0], y, rtol=1e-15, atol=1e-15)


def pin_duplicate_logit_tie():
    """Two identical router rows give bit-identical probabilities: the lower
    expert index must come first."""
    E, d, k = 5, 8, 2
    g = torch.Generator().manual_seed(21)
    x = torch.randn((20, d), generator=g)
    wr = torch.randn((E, d), generator=g) * 0.1
    wr[3] = 2.0 * torch.sign(x.mean(0))  # large and shared
    wr[1] = wr[3]
    w3 = torch.zeros((E, 2, d))
    wd3 = torch.zeros((E, d, 2))
    r = oracle.forward(x, wr, None, w3, w3, wd3, k, renorm=True)
    p = r.probs
    both = p[:, 1] == p[:, 3]
    assert both.all()
    top = (p[:, 1] >= p.max(axis=1))
    assert top.any()
    for t in np.nonzero(top)[0]:
        assert list(r.topk_idx[t]) == [1, 3]
        assert r.gap[t] > 0


def pin_dispatch_stable_sort():
    """The dispatch order equals a stable library sort of the flattened
    (token, slot) assignments by expert id; every token appears k times; the
    permutation and its inverse agree; segments ascend in token order."""
    T, E, k = 37, 6, 3
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    offsets, perm, inv, _ = oracle.dispatch(idx, E)
    order = np.argsort(idx.reshape(-1), kind="stable")
    np.testing.assert_array_equal(perm, order // k)
    expect_inv = np.empty(T * k, dtype=np.int64)
    expect_inv[order] = np.arange(T * k)
    np.testing.assert_array_equal(inv.reshape(-1), expect_inv)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(idx.reshape(-1), minlength=E))]))
    np.testing.assert_array_equal(np.bincount(perm, minlength=T), k)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
    for t in range(T):
        for j in range(k):
            assert perm[inv[t, j]] == t
            assert offsets[idx[t, j]] <= inv[t, j] < offsets[idx[t, j] + 1]


def pin_axonml_unit_tests():
    """The facts the axonml-nn moe.rs tests check, on the same shapes:
    constant input 0.1, d=64, I=256, E=8 or 4, k=2: gates sum to 1 within
    1e-5, indices < E, the statistic is > 0, and the counts sum to T*k."""
    g = torch.Generator().manual_seed(0)
    x = torch.full((4, 64), 0.1)
    wr = torch.randn((8, 64), generator=g) * 0.125
    probs = oracle.router_probs(x, wr)
    idx, gate, _ = oracle.topk(probs, 2, renorm=True)
    assert gate.shape == (4, 2) and idx.shape == (4, 2)
    assert np.all(np.abs(gate.sum(1) - 1) < 1e-5)
    assert np.all(idx < 8)
    x10 = torch.full((10, 64), 0.1)
    wr4 = torch.randn((4, 64), generator=g) * 0.125
    wg = torch.randn((4, 256, 64), generator=g) * 0.1
    wu = torch.randn((4, 256, 64), generator=g) * 0.1
    wd = torch.randn((4, 64, 256), generator=g) * 0.1
    r = oracle.forward(x10, wr4, None, wg, wu, wd, 2, renorm=True)
    assert r.out.shape == (10, 64)
    assert r.aux > 0
    assert int(r.counts.sum()) == 20


def pin_mixtral_parameter_count():
    """The Mixtral MoE Block page prints 1.45B parameters for its block; with
    three projection matrices per expert (gate, up, down) the count is
    1,451,270,144, and with the two-matrix Sequential it would be ~0.98B, so
    the printed figure fixes the gated expert structure the oracle uses."""
    with open(os.path.join(GOLDEN, "mixtral_block_params.json")) as f:
        gold = json.load(f)
    d, I, E = gold["d"], gold["I"], gold["E"]
    attn = d * d + 2 * d * gold["kv_dim"] + d * d
    norms = 2 * d
    router = E * d
    gated = attn + norms + router + E * 3 * d * I
    ungated = attn + norms + router + E * 2 * d * I
    assert gated == gold["gated_count"]
    assert round(gated / 1e9, 2) == gold["printed_billions"]
    assert round(ungated / 1e9, 2) != gold["printed_billions"]
    # the oracle's expert takes exactly the three matrices: a change to any one
    # of them changes its output
    x, wr, b, wg, wu, wd = _rand_case(3, 8, 1, 1, 6, "f32", 13)
    base = oracle.expert_rows(x, wg, wu, wd, [0, 1, 2], [0, 0, 0])
    for which in range(3):
        mats = [wg.clone(), wu.clone(), wd.clone()]
        mats[which] = mats[which] * 1.5
        got = oracle.expert_rows(x, *mats, [0, 1, 2], [0, 0, 0])
        assert np.abs(got - base).max() > 1e-6


def pin_gap_definition():
    """gap = p_(k) - p_(k+1), +inf when k = E."""
    x, wr, b, wg, wu, wd = _rand_case(20, 8, 5, 2, 4, "f32", 17)
    probs = oracle.router_probs(x, wr, b)
    _, _, gap = oracle.topk(probs, 2, renorm=True)
    srt = -np.sort(-probs, axis=1)
    np.testing.assert_allclose(gap, srt[:, 1] - srt[:, 2], rtol=0, atol=0)
    _, _, gapE = oracle.topk(probs, 5, renorm=True)
    assert np.all(np.isinf(gapE))


# ---------------------------------------------------------------------------
# pins of the layer's options: pre-MoE RMSNorm, z-loss, capacity, shared experts
# ---------------------------------------------------------------------------

def pin_rmsnorm_torch_form():
    """Form 1 is torch's nn.RMSNorm: against torch.nn.functional.rms_norm in
    fp64 (a library routine), with and without a weight, two eps values."""
    g = torch.Generator().manual_seed(31)
    x = torch.randn((9, 24), generator=g).to(torch.bfloat16)
    w = (1.0 + 0.3 * torch.randn((24,), generator=g)).to(torch.bfloat16)
    for eps in (1e-5, 0.5):
        ref = F.rms_norm(x.double(), (24,), w.double(), eps).numpy()
        np.testing.assert_allclose(oracle.rmsnorm(x, w, eps, form=1), ref, rtol=0, atol=1e-14)
        ref1 = F.rms_norm(x.double(), (24,), None, eps).numpy()
        np.testing.assert_allclose(oracle.rmsnorm(x, None, eps, form=1), ref1, rtol=0, atol=1e-14)


def pin_rmsnorm_worked_values():
    """x = (3, 4), w = (1, 2), eps = 0.5, worked by hand.
    Form 2 (eps outside the root, as printed under Model Architecture
    Patterns): rms = 5/sqrt(2) = 3.5355..., x_hat = w*x / 4.0355... =
    (0.74339..., 1.98238...). Form 1 (torch): 1/sqrt(12.5 + 0.5) = 0.27735...,
    x_hat = (0.83205..., 2.21880...). With eps = 0 and unit weight both forms
    give mean(x_hat^2) = 1 and are invariant to scaling x."""
    x = torch.tensor([[3.0, 4.0]])
    w = torch.tensor([1.0, 2.0])
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 0.5, form=2)[0], [0.7433960585957724, 1.9823894895887266],
                               rtol=1e-15)
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 0.5, form=1)[0], [0.8320502943378437, 2.2188007849009166],
                               rtol=1e-15)
    g = torch.Generator().manual_seed(32)
    xr = torch.randn((5, 16), generator=g)
    for form in (1, 2):
        a = oracle.rmsnorm(xr, None, 0.0, form=form)
        np.testing.assert_allclose((a * a).mean(axis=1), 1.0, rtol=1e-14)
        np.testing.assert_allclose(oracle.rmsnorm(xr * 4.0, None, 0.0, form=form), a, rtol=1e-14)


def pin_norm_feeds_router_and_experts():
    """With the norm on, the whole layer equals the brute-force layer applied
    to torch's rms_norm(x) (fp64), router and experts alike."""
    T, d, E, k, I = 8, 16, 4, 2, 12
    x, wr, b, wg, wu, wd = _rand_case(T, d, E, k, I, "bf16", 33, bias=True)
    w = (1.0 + 0.2 * torch.randn((d,), generator=torch.Generator().manual_seed(34))).to(torch.bfloat16)
    xh = F.rms_norm(x.double(), (d,), w.double(), 1e-5)
    bp, bidx, bg, bout = brute_force(xh, wr, b, wg, wu, wd, k, True)
    r = oracle.forward(x, wr, b, wg, wu, wd, k, True, norm_form=1, norm_weight=w, norm_eps=1e-5)
    np.testing.assert_allclose(r.probs, bp, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(r.topk_idx, bidx)
    np.testing.assert_allclose(r.out, bout, rtol=0, atol=1e-11 * max(1.0, float(np.abs(bout).max())))


def pin_z_loss_closed_forms():
    """Zero logits: (ln E)^2. Router weights zero and bias (0, ln 3): every
    token's logsumexp is ln 4, so z = (ln 4)^2. Two tokens with logits
    (a, a, a, a) and (L, L, L, L): z = ((a + ln 4)^2 + (L + ln 4)^2) / 2, a mean
    over tokens, not a sum."""
    np.testing.assert_allclose(oracle.z_loss(np.zeros((7, 8))), 4.324077125263812, rtol=1e-15)
    x = torch.randn((6, 4), generator=torch.Generator().manual_seed(35))
    wr = torch.zeros((2, 4))
    b = torch.tensor([0.0, math.log(3.0)])
    w3 = torch.zeros((2, 1, 4))
    wd3 = torch.zeros((2, 4, 1))
    r = oracle.forward(x, wr, b, w3, w3, wd3, 1, True)
    np.testing.assert_allclose(r.z_loss, 1.9218120556728056, rtol=1e-7)  # b is stored in fp32
    a, L = -1.5, 30.0
    lg = np.array([[a] * 4, [L] * 4])
    np.testing.assert_allclose(oracle.z_loss(lg), ((a + math.log(4)) ** 2 + (L + math.log(4)) ** 2) / 2, rtol=1e-15)
    assert oracle.z_loss(np.zeros((0, 3))) == 0.0


def pin_z_loss_scipy():
    """Against scipy.special.logsumexp on random logits with a bias."""
    from scipy.special import logsumexp

    x, wr, b, *_ = _rand_case(33, 12, 6, 2, 4, "f32", 36, bias=True)
    lg = oracle.router_logits(x, wr, b)
    ref = _f64(x) @ _f64(wr).T + _f64(b)
    np.testing.assert_allclose(lg, ref, rtol=0, atol=1e-12)
    lse = logsumexp(ref, axis=1)
    np.testing.assert_allclose(oracle.z_loss(lg), np.mean(lse * lse), rtol=1e-14)


def pin_capacity_values():
    """C = ceil(cf * T * k / E): 10 tokens, k = 1, E = 4, cf = 1 gives 3 (2.5
    rounded up); cf = 1.25 at T = 4096, k = 2, E = 8 gives 1280; cf = 0.5 at
    T = 7, k = 2, E = 3 gives 3 (2.33 rounded up); cf = 0 means no limit."""
    assert oracle.capacity(1.0, 10, 1, 4) == 3
    assert oracle.capacity(1.25, 4096, 2, 8) == 1280
    assert oracle.capacity(0.5, 7, 2, 3) == 3
    assert oracle.capacity(0.0, 10, 1, 4) == -1


def pin_capacity_dispatch_worked():
    """A hand-worked drop with C = 2. Assignments per expert in token order:
    e0: t0 t1 t2 t3 t5 -> keeps t0 t1; e1: t0 t2 t4 t5 -> keeps t0 t2;
    e2: t1 t3 t4 -> keeps t1 t3. Six slots are dropped."""
    idx = np.array([[0, 1], [0, 2], [1, 0], [2, 0], [1, 2], [0, 1]], dtype=np.int32)
    offsets, perm, inv, dropped = oracle.dispatch(idx, 3, cap=2)
    np.testing.assert_array_equal(offsets, [0, 2, 4, 6])
    np.testing.assert_array_equal(perm, [0, 1, 0, 2, 1, 3])
    np.testing.assert_array_equal(inv, [[0, 2], [1, 4], [3, -1], [5, -1], [-1, -1], [-1, -1]])
    assert dropped == 6
    # no limit: the plain dispatch
    offsets, perm, inv, dropped = oracle.dispatch(idx, 3)
    np.testing.assert_array_equal(offsets, [0, 5, 9, 12])
    assert dropped == 0 and inv.min() == 0


def pin_capacity_layer():
    """Every token routed to expert 0 (bias), k = 1, cf = 1 over E = 4 with
    T = 10: C = 3, so tokens 0-2 get gate * SwiGLU_0(x) (dense torch) and the
    other 7 get zero; counts and the statistic are those before dropping.
    A factor large enough to keep everything gives the plain layer."""
    T, d, E, I = 10, 8, 4, 6
    x, wr, _, wg, wu, wd = _rand_case(T, d, E, 1, I, "f32", 37, router_std=0.01)
    b = torch.tensor([20.0, 0.0, 0.0, 0.0])
    r = oracle.forward(x, wr, b, wg, wu, wd, 1, False, capacity_factor=1.0)
    assert r.capacity == 3 and r.dropped == 7
    np.testing.assert_array_equal(r.counts, [10, 0, 0, 0])
    dense = dense_swiglu_torch(x, wg[0], wu[0], wd[0]).numpy() * r.topk_gate[:, :1]
    np.testing.assert_allclose(r.out[:3], dense[:3], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(r.out[3:], 0.0)
    np.testing.assert_array_equal(r.inv[:, 0], [0, 1, 2] + [-1] * 7)
    plain = oracle.forward(x, wr, b, wg, wu, wd, 1, False)
    big = oracle.forward(x, wr, b, wg, wu, wd, 1, False, capacity_factor=4.0)
    assert big.dropped == 0
    np.testing.assert_array_equal(big.out, plain.out)


def pin_shared_experts():
    """Shared experts add sum_s SwiGLU_s(x) (dense torch, fp64) to every
    token, with weight 1, on top of the routed output."""
    T, d, E, k, I, S = 9, 12, 4, 2, 10, 2
    x, wr, b, wg, wu, wd = _rand_case(T, d, E, k, I, "bf16", 38, bias=True)
    g = torch.Generator().manual_seed(39)
    sg = (torch.randn((S, I, d), generator=g) * 0.3).to(torch.bfloat16)
    su = (torch.randn((S, I, d), generator=g) * 0.3).to(torch.bfloat16)
    sd = (torch.randn((S, d, I), generator=g) * 0.3).to(torch.bfloat16)
    plain = oracle.forward(x, wr, b, wg, wu, wd, k, True)
    r = oracle.forward(x, wr, b, wg, wu, wd, k, True, shared=(sg, su, sd))
    extra = sum(dense_swiglu_torch(x, sg[s], su[s], sd[s]) for s in range(S)).numpy()
    np.testing.assert_allclose(r.out - plain.out, extra, rtol=0, atol=1e-11 * max(1.0, float(np.abs(extra).max())))
    np.testing.assert_array_equal(r.topk_idx, plain.topk_idx)


def pin_round_bf16_matches_torch():
    """The diagnostic bf16 rounding equals torch's fp32 -> bf16 conversion
    (round to nearest, ties to even), including exact ties."""
    g = torch.Generator().manual_seed(40)
    v = torch.randn((4096,), generator=g) * 3.0
    ties = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 + 2.0 ** -7, 0.0, -0.0])
    v = torch.cat([v, ties])
    got = oracle.round_bf16(v.double().numpy())
    ref = v.to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got, ref)
    assert got[-6] == 1.0 and got[-5] == 1.0 + 2.0 ** -6


ALL_PINS = [
    pin_brute_force,
    pin_gates_sum_to_one,
    pin_dense_E1_k1,
    pin_soft_mixture_k_eq_E,
    pin_zero_router,
    pin_uniform_counts_aux,
    pin_aux_closed_form,
    pin_expert_closed_form,
    pin_duplicate_logit_tie,
    pin_dispatch_stable_sort,
    pin_axonml_unit_tests,
    pin_mixtral_parameter_count,
    pin_gap_definition,
    pin_rmsnorm_torch_form,
    pin_rmsnorm_worked_values,
    pin_norm_feeds_router_and_experts,
    pin_z_loss_closed_forms,
    pin_z_loss_scipy,
    pin_capacity_values,
    pin_capacity_dispatch_worked,
    pin_capacity_layer,
    pin_shared_experts,
    pin_round_bf16_matches_torch,
]
