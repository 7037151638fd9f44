"""Element-by-element comparison of the CUDA path with the fp64 oracle.

Rules:
  * Top-k indices (best first) and the dispatch order must match the oracle
    exactly on every token whose sorted oracle probabilities p_(1) >= ... >=
    p_(k+1) are all more than 1e-4 apart. Where only a gap inside the list is
    that small, the set must still match and the order may differ between
    the near-equal neighbours; where p_(k) - p_(k+1) is that small (a near
    tie), the set may differ. Both counts are reported. For excluded tokens the GPU's choice
    must still be valid (k distinct experts whose oracle probabilities are
    within the gap threshold of the oracle's k-th), and every other output is
    checked against the oracle evaluated at the GPU's choice.
  * Counts and the dispatch order are checked exactly against the oracle's
    own dispatch of the GPU's indices (integer work is bit-exact).
  * Gates within GATE_TOL absolute, the statistic within 1e-4 absolute. A
    gate is a softmax ratio of logits: with every logit off by at most dl,
    |dp_j| = p_j |dl_j - sum_i p_i dl_i| <= 2 dl p_j (1 - p_j) <= dl / 2 (and
    the same for a renormalised gate, a softmax over the k chosen logits).
    So the gate bar is half the router's logit error bar plus the fp32
    rounding of the softmax. The logit error bar of the bf16 router (fp32
    tensor-core accumulation of d bf16 products) is pinned by
    test_router_logit_error_pin, which reads the logits back from the gates
    of a k = E call at d = 4096; the fp32 router adds its d FFMA products in
    index order.
  * Outputs: max-abs <= 2e-2 and relative Frobenius <= 1e-2 for bf16;
    both <= 1e-4 for fp32; every token's output row is compared unless a
    test names a subset.
  * Options. RMSNorm: the oracle normalises in fp64 and routes and evaluates
    the experts on x_hat. Capacity: the kept rows, inv (-1 for a dropped
    slot) and the dropped count are compared exactly with the oracle's
    capacity dispatch of the GPU's indices. Shared experts: part of the
    output comparison. Every output bar is held against the pure fp64
    oracle: relative Frobenius <= 1e-2 unchanged; the bf16 max-abs bar is
    widened for the norm and the shared experts only by amounts the oracle
    computes by itself (option_max_abs_bar). z-loss: relative error <= 1e-4
    (each token's logsumexp carries the router's logit error and an fp32
    rounding; the per-block fp32 sums of at most 128 terms add at most
    128 * 2^-24 relative).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

GAP_THRESHOLD = 1e-4
TOL = {"bf16": dict(max_abs=2e-2, rel_fro=1e-2), "f32": dict(max_abs=1e-4, rel_fro=1e-4)}
# Router logit error bars, set from test_router_logit_error_pin's
# measurement against fp64 (largest of all tokens, read back through the
# gates of a k = E call): 4.3e-6 for the bf16 tensor-core router at the
# Mixtral prefill shape (d = 4096), 6.6e-7 at d = 1024, and 3.6e-6 for the
# fp32 router on the tiny workload, whose router std of 0.5 gives logits of
# std 5.7 (the read-back there includes the fp32 exponential of logit gaps
# of up to ~20). The bars leave about 2.5x room. The gate bars follow from
# them (module docstring) plus a few fp32 roundings of values <= 1.
LOGIT_TOL = {"bf16": 1e-5, "f32": 1e-5}
GATE_TOL = {dt: LOGIT_TOL[dt] / 2 + 5e-7 for dt in LOGIT_TOL}
Z_REL_TOL = 1e-4


def _np(t):
    return t.detach().cpu().numpy()


def check(inp, res, perm, k, renorm, dtype, tokens=None, report=None, options=None):
    """inp: workloads.Inputs (CUDA tensors); res: MoEOutputs; perm: (offsets,
    perm_tok, inv) from get_permutation; tokens: the tokens whose output rows
    are compared (None, the default, compares every token); options: the
    MoEOptions of the call."""
    x = inp.x.cpu()
    wr = inp.w_router.cpu()
    b = None if inp.b_router is None else inp.b_router.cpu()
    T, d = x.shape
    E = wr.shape[0]
    rep = {} if report is None else report

    xin = x
    if options is not None and options.norm_form:
        nw = None if options.norm_weight is None else options.norm_weight.cpu()
        xin = oracle.rmsnorm(x, nw, options.norm_eps, options.norm_form)
    cf = 0.0 if options is None else options.capacity_factor
    cap = oracle.capacity(cf, T, k, E)
    shared = None
    if options is not None and options.n_shared:
        shared = (options.shared_gate.cpu(), options.shared_up.cpu(), options.shared_down.cpu())

    logits = oracle.router_logits(xin, wr, b)
    probs = oracle.softmax(logits)
    idx_o, gate_o, gap = oracle.topk(probs, k, renorm)
    counts_o, _, aux_o = oracle.stats(probs, idx_o)
    offs_o, perm_o, inv_o, _ = oracle.dispatch(idx_o, E, cap)

    idx_g = _np(res.topk_idx).astype(np.int32)
    gate_g = _np(res.topk_gate).astype(np.float64)
    counts_g = _np(res.counts).astype(np.int64)
    aux_g = float(_np(res.aux)[0])
    offs_g, perm_g, inv_g = (_np(a).astype(np.int64) for a in perm)

    srt = -np.sort(-probs, axis=1)[:, :min(k + 1, E)]
    order_gap = (srt[:, :-1] - srt[:, 1:]).min(axis=1) if srt.shape[1] > 1 else np.full(T, np.inf)
    near = gap <= GAP_THRESHOLD
    near_order = ~near & (order_gap <= GAP_THRESHOLD)
    rep["near_tie_tokens"] = int(near.sum())
    rep["near_order_tokens"] = int(near_order.sum())
    assert int(_np(res.status)[0]) == 0, f"device status word {int(_np(res.status)[0]):#x}"

    # --- routing ---------------------------------------------------------
    ok = ~near & ~near_order
    for t in np.nonzero(near_order)[0]:
        assert sorted(idx_g[t].tolist()) == sorted(idx_o[t].tolist()), f"token {t}: different set, gap {gap[t]}"
        assert np.all(np.diff(probs[t, idx_g[t]]) <= GAP_THRESHOLD), f"token {t}: list out of order"
    mism = np.nonzero((idx_g[ok] != idx_o[ok]).any(axis=1))[0]
    if mism.size:
        t0 = int(np.nonzero(ok)[0][mism[0]])
        raise AssertionError(
            f"{mism.size} non-near-tie tokens routed differently, first {np.nonzero(ok)[0][mism[:5]]}; token {t0}: "
            f"gpu {idx_g[t0].tolist()} oracle {idx_o[t0].tolist()} p_gpu_choice {probs[t0, idx_g[t0]].tolist()} "
            f"p_oracle_choice {probs[t0, idx_o[t0]].tolist()} gap {gap[t0]} order_gap {order_gap[t0]}")
    assert np.all((idx_g >= 0) & (idx_g < E))
    for t in np.nonzero(near)[0]:
        assert len(set(idx_g[t].tolist())) == k
        kth = np.sort(probs[t])[::-1][k - 1]
        assert np.all(probs[t, idx_g[t]] >= kth - GAP_THRESHOLD), f"token {t}: invalid near-tie choice"
        # best first, up to near-equal neighbours
        assert np.all(np.diff(probs[t, idx_g[t]]) <= GAP_THRESHOLD), f"token {t}: near-tie choice out of order"
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
    offs_r, perm_r, inv_r, drop_r = oracle.dispatch(idx_g, E, cap)
    np.testing.assert_array_equal(offs_g, offs_r)
    np.testing.assert_array_equal(perm_g[:int(offs_r[E])], perm_r)
    np.testing.assert_array_equal(inv_g.reshape(T, k), inv_r)
    if cap >= 0:
        rep["dropped"] = drop_r
        assert res.dropped is not None and int(_np(res.dropped)[0]) == drop_r, "dropped count"
    # the oracle's own order, restricted to tokens that are not near ties (a
    # near-tie flip can move which tokens a capacity drops: compare then only
    # without near ties)
    if cap < 0 or not near.any():
        for e in range(E):
            mine = perm_g[offs_g[e]:offs_g[e + 1]]
            theirs = perm_o[offs_o[e]:offs_o[e + 1]]
            np.testing.assert_array_equal(mine[~near[mine]], theirs[~near[theirs]])
    if res.z_loss is not None:
        z_g = float(_np(res.z_loss)[0])
        z_o = oracle.z_loss(logits)
        rep["z_loss"] = z_g
        assert abs(z_g - z_o) <= Z_REL_TOL * abs(z_o) + 1e-7, f"z-loss {z_g} vs {z_o}"

    # --- outputs ---------------------------------------------------------------
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    rep["tokens_compared"] = int(tokens.size)
    if tokens.size:
        keep = (inv_r[tokens] >= 0) if cap >= 0 else None
        wts = (inp.w_gate.cpu(), inp.w_up.cpu(), inp.w_down.cpu())
        # the pure fp64 layer: routed part and shared part evaluated apart
        # (their sum is the layer's output up to the order of two fp64 adds)
        routed = oracle.moe_tokens(xin, *wts, tokens, idx_g[tokens], gate_ref[tokens], keep=keep)
        ref = routed
        shared_part = None
        if shared is not None:
            shared_part = oracle.moe_tokens(xin, *wts, tokens, idx_g[tokens][:, :0], gate_ref[tokens][:, :0],
                                            shared=shared)
            ref = routed + shared_part
        got = _np(res.out)[tokens].astype(np.float64)
        assert np.isfinite(got).all()
        diff = got - ref
        max_abs = float(np.abs(diff).max())
        rel_fro = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
        rep["max_abs"] = max_abs
        rep["rel_fro"] = rel_fro
        tol = TOL[dtype]
        bar = tol["max_abs"]
        if dtype == "bf16" and options is not None and (options.norm_form or options.n_shared):
            bar = option_max_abs_bar(rep, xin, wts, tokens, idx_g[tokens], gate_ref[tokens], keep, shared,
                                     routed, shared_part, options)
        assert max_abs <= bar, f"max-abs {max_abs} > {bar} ({rep})"
        assert rel_fro <= tol["rel_fro"], f"relative Frobenius {rel_fro} > {tol['rel_fro']} ({rep})"
    return rep


def option_max_abs_bar(rep, xin, wts, tokens, idx, gate, keep, shared, routed, shared_part, options):
    """Max-abs bar of the bf16 layer with the RMSNorm or shared experts,
    derived from the oracle alone (nothing here mirrors the kernels).

    The 2e-2 bar is stated for the plain layer, whose bf16 error comes from
    rounding the stored bf16 operands of the expert GEMMs. Two options change
    that error:
      * shared experts add full expert outputs of weight 1. The rounding
        error of an expert's output is relative to that output, and the
        routed and shared parts' errors are independent, so the plain bar is
        scaled by sqrt(1 + (rms shared / rms routed)^2), both RMS values taken
        from the pure oracle over the compared rows;
      * the normalised input x_hat of a bf16 layer is itself a bf16 tensor:
        its one rounding moves the output by at most
        A = max |oracle(bf16(x_hat)) - oracle(x_hat)| (same routing and gates,
        everything else exact), which is added to the bar (triangle
        inequality).
    """
    bar = TOL["bf16"]["max_abs"]
    if shared_part is not None:
        rr = float(np.sqrt(np.mean(routed ** 2)))
        rs = float(np.sqrt(np.mean(shared_part ** 2)))
        scale = float(np.sqrt(1.0 + (rs / max(rr, 1e-300)) ** 2))
        rep["shared_scale"] = scale
        bar *= scale
    if options.norm_form:
        xr = oracle.round_bf16(xin)
        ref_r = oracle.moe_tokens(xr, *wts, tokens, idx, gate, keep=keep, shared=shared)
        ref = routed if shared_part is None else routed + shared_part
        allow = float(np.abs(ref_r - ref).max())
        rep["xhat_allowance"] = allow
        bar += allow
    rep["max_abs_bar"] = bar
    return bar
