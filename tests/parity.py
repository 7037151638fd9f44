"""Element-by-element comparison of the CUDA path with the fp64 oracle.

Rules:
  * Top-k indices and the dispatch order must match the oracle exactly on
    every token whose oracle gap p_(k) - p_(k+1) exceeds 1e-4; the count of
    excluded near-tie tokens is reported. For excluded tokens the GPU's choice
    must still be valid (k distinct experts whose oracle probabilities are
    within the gap threshold of the oracle's k-th), and every other output is
    checked against the oracle evaluated at the GPU's choice.
  * Counts and the dispatch order are checked exactly against the oracle's
    own dispatch of the GPU's indices (integer work is bit-exact).
  * Gates within 2e-6 absolute for fp32 and 2e-5 for bf16, the statistic
    within 1e-4 absolute. A gate is a softmax ratio of two or more logits,
    |dg| <= max|dl| / 2, and the bf16 router accumulates its d products on the
    tensor cores in fp32 (not round-to-nearest at every add), which leaves a
    logit error of a few 1e-5 at d = 4096 (a relative 1e-6 of sum |x_c w_c|).
  * Outputs: max-abs <= 2e-2 and relative Frobenius <= 1e-2 for bf16;
    both <= 1e-4 for fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

GAP_THRESHOLD = 1e-4
TOL = {"bf16": dict(max_abs=2e-2, rel_fro=1e-2), "f32": dict(max_abs=1e-4, rel_fro=1e-4)}
GATE_TOL = {"bf16": 2e-5, "f32": 2e-6}


def _np(t):
    return t.detach().cpu().numpy()


def check(inp, res, perm, k, renorm, dtype, tokens=None, h_round=False, report=None):
    """inp: workloads.Inputs (CUDA tensors); res: MoEOutputs; perm: (offsets,
    perm_tok, inv) from get_permutation; tokens: sample of tokens whose output
    rows are compared (None = all)."""
    x = inp.x.cpu()
    wr = inp.w_router.cpu()
    b = None if inp.b_router is None else inp.b_router.cpu()
    T, d = x.shape
    E = wr.shape[0]
    rep = {} if report is None else report

    probs = oracle.router_probs(x, wr, b)
    idx_o, gate_o, gap = oracle.topk(probs, k, renorm)
    counts_o, _, aux_o = oracle.stats(probs, idx_o)
    offs_o, perm_o, inv_o, _ = oracle.dispatch(idx_o, E)

    idx_g = _np(res.topk_idx).astype(np.int32)
    gate_g = _np(res.topk_gate).astype(np.float64)
    counts_g = _np(res.counts).astype(np.int64)
    aux_g = float(_np(res.aux)[0])
    offs_g, perm_g, inv_g = (_np(a).astype(np.int64) for a in perm)

    near = gap <= GAP_THRESHOLD
    rep["near_tie_tokens"] = int(near.sum())
    assert int(_np(res.status)[0]) == 0, f"device status word {int(_np(res.status)[0]):#x}"

    # --- routing ---------------------------------------------------------
    ok = ~near
    mism = np.nonzero((idx_g[ok] != idx_o[ok]).any(axis=1))[0]
    assert mism.size == 0, f"{mism.size} non-near-tie tokens routed differently, first {np.nonzero(ok)[0][mism[:5]]}"
    assert np.all((idx_g >= 0) & (idx_g < E))
    for t in np.nonzero(near)[0]:
        assert len(set(idx_g[t].tolist())) == k
        kth = np.sort(probs[t])[::-1][k - 1]
        assert np.all(probs[t, idx_g[t]] >= kth - GAP_THRESHOLD), f"token {t}: invalid near-tie choice"
    gate_ref = oracle.gates_for(probs, idx_g, renorm)
    gerr = float(np.abs(gate_g - gate_ref).max()) if T else 0.0
    rep["gate_max_abs"] = gerr
    assert gerr <= GATE_TOL[dtype], f"gate error {gerr}"

    # --- counts, statistic, dispatch order (exact) -------------------------
    counts_ref, _, aux_ref = oracle.stats(probs, idx_g)
    np.testing.assert_array_equal(counts_g, counts_ref)
    if not near.any():
        np.testing.assert_array_equal(counts_g, counts_o)
    rep["aux"] = aux_g
    rep["aux_oracle"] = aux_o
    assert abs(aux_g - aux_ref) <= 1e-4, f"aux {aux_g} vs {aux_ref}"
    offs_r, perm_r, inv_r, _ = oracle.dispatch(idx_g, E)
    np.testing.assert_array_equal(offs_g, offs_r)
    np.testing.assert_array_equal(perm_g, perm_r)
    np.testing.assert_array_equal(inv_g.reshape(T, k), inv_r)
    # the oracle's own order, restricted to tokens that are not near ties
    for e in range(E):
        mine = perm_g[offs_g[e]:offs_g[e + 1]]
        theirs = perm_o[offs_o[e]:offs_o[e + 1]]
        np.testing.assert_array_equal(mine[~near[mine]], theirs[~near[theirs]])

    # --- outputs -------------------------------------------------------------
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    rep["tokens_compared"] = int(tokens.size)
    if tokens.size:
        ref = oracle.moe_tokens(x, inp.w_gate.cpu(), inp.w_up.cpu(), inp.w_down.cpu(), tokens, idx_g[tokens],
                                gate_ref[tokens], h_round=h_round)
        got = _np(res.out)[tokens].astype(np.float64)
        diff = got - ref
        max_abs = float(np.abs(diff).max())
        rel_fro = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
        rep["max_abs"] = max_abs
        rep["rel_fro"] = rel_fro
        tol = TOL[dtype]
        assert np.isfinite(got).all()
        assert max_abs <= tol["max_abs"], f"max-abs {max_abs} > {tol['max_abs']}"
        assert rel_fro <= tol["rel_fro"], f"relative Frobenius {rel_fro} > {tol['rel_fro']}"
    return rep


def sample_tokens(perm, T, k, n_random=64, edge=4, seed=0, cap=None):
    """Tokens whose rows sit at the start and the ragged end of every expert's
    segment (and of every 128-row tile boundary nearby), plus random ones."""
    offs, perm_tok, _ = (_np(a) for a in perm)
    pick = set()
    rng = np.random.default_rng(seed)
    for e in range(len(offs) - 1):
        a, bnd = int(offs[e]), int(offs[e + 1])
        if bnd <= a:
            continue
        for r in list(range(a, min(bnd, a + edge))) + list(range(max(a, bnd - edge), bnd)):
            pick.add(int(perm_tok[r]))
        for r in range(a + 127, bnd, 128):
            pick.add(int(perm_tok[r]))
            if r + 1 < bnd:
                pick.add(int(perm_tok[r + 1]))
    pick.update(rng.choice(T, size=min(T, n_random), replace=False).tolist())
    pick.update([0, T - 1])
    out = np.array(sorted(pick), dtype=np.int32)
    if cap is not None and out.size > cap:
        out = np.sort(rng.choice(out, size=cap, replace=False)).astype(np.int32)
    return out
