"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch every one: a dropped term, a wrong sign, a wrong index or
tie order, a transposed operand, a swapped projection, a wrong
normalisation."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = [
    ("swap_gate_up", "double silu = g / (1.0 + exp(-g));\n        h[i] = silu * u;",
     "double silu = u / (1.0 + exp(-u));\n        h[i] = silu * g;"),
    ("silu_sign", "double silu = g / (1.0 + exp(-g));", "double silu = g / (1.0 + exp(g));"),
    ("no_silu", "double silu = g / (1.0 + exp(-g));", "double silu = g;"),
    ("transposed_down", "acc += h[i] * load_elem(w_down, dtype, wrow + i);",
     "acc += h[i] * load_elem(w_down, dtype, e * d * I + i * d + o);"),
    ("drop_renorm", "gate[t * k + j] = pj / s;", "gate[t * k + j] = pj;"),
    ("renorm_always", "if (!renorm)\n        gate[t * k + j] = pj;", "if (0)\n        gate[t * k + j] = pj;"),
    ("tie_to_higher_index", "return (ra->e > rb->e) - (ra->e < rb->e);",
     "return (ra->e < rb->e) - (ra->e > rb->e);"),
    ("ascending_topk", "if (ra->p > rb->p) return -1;\n  if (ra->p < rb->p) return 1;",
     "if (ra->p < rb->p) return -1;\n  if (ra->p > rb->p) return 1;"),
    ("drop_bias", "if (b_router) acc += (double)b_router[e];", "(void)b_router;"),
    ("softmax_no_normalise", "for (int e = 0; e < E; ++e) p[e] /= s;", "(void)s;"),
    ("aux_page_literal_f", "((double)counts[e] / ((double)T * (double)k))", "((double)counts[e] / (double)T)"),
    ("aux_no_E", "*aux = (double)E * s;", "*aux = s;"),
    ("gap_wrong_slot", "gap[t] = (k < E) ? r[k - 1].p - r[k].p : INFINITY;",
     "gap[t] = (k < E) ? r[0].p - r[k].p : INFINITY;"),
    ("dispatch_token_descending", "if (topk_idx[t * k + j] == e) {", "if (topk_idx[t * k + j] == E - 1 - e) {"),
    ("combine_gate_sum", "if (!keep || keep[i * k + j]) acc += gate[i * k + j] * y[(i * k + j) * d + c];",
     "if (!keep || keep[i * k + j]) { double gs = 0.0; for (int jj = 0; jj < k; ++jj) gs += gate[i * k + jj];"
     " acc += gs * y[(i * k + j) * d + c]; }"),
    ("router_transposed", "load_elem(w_router, w_dtype, (int64_t)e * d + c)",
     "load_elem(w_router, w_dtype, c * E + e)"),
    # options: RMSNorm, z-loss, capacity, shared experts
    ("rms_eps_outside_in_torch_form", "form == 1 ? 1.0 / sqrt(ms + eps) : 1.0 / (sqrt(ms) + eps)",
     "form == 1 ? 1.0 / (sqrt(ms) + eps) : 1.0 / (sqrt(ms) + eps)"),
    ("rms_eps_inside_in_page_form", "form == 1 ? 1.0 / sqrt(ms + eps) : 1.0 / (sqrt(ms) + eps)",
     "form == 1 ? 1.0 / sqrt(ms + eps) : 1.0 / sqrt(ms + eps)"),
    ("rms_sum_not_mean", "const double ms = ss / (double)d;", "const double ms = ss;"),
    ("rms_no_weight", "const double w = weight ? load_elem(weight, w_dtype, c) : 1.0;", "const double w = 1.0;"),
    ("z_not_squared", "acc += lse * lse;", "acc += lse;"),
    ("z_max_not_lse", "const double lse = m + log(s);", "const double lse = m;"),
    ("z_sum_not_mean", "return acc / (double)T;", "return acc;"),
    ("capacity_floor", "return (int64_t)ceil(cf * (double)T * (double)k / (double)E);",
     "return (int64_t)floor(cf * (double)T * (double)k / (double)E);"),
    ("capacity_per_token_not_assignment", "return (int64_t)ceil(cf * (double)T * (double)k / (double)E);",
     "return (int64_t)ceil(cf * (double)T / (double)E);"),
    ("capacity_off_by_one", "if (capacity >= 0 && taken >= capacity) {", "if (capacity >= 0 && taken > capacity) {"),
    ("dropped_slot_still_combined", "if (!keep || keep[i * k + j]) acc", "if (1) acc"),
    ("shared_not_added", "acc += ys[(i * n_shared + s) * d + c];", "acc += 0.0 * ys[(i * n_shared + s) * d + c];"),
    ("bf16_round_toward_zero", "u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    ("shared_half_weight", "acc += ys[(i * n_shared + s) * d + c];", "acc += 0.5 * ys[(i * n_shared + s) * d + c];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = src.replace(old, new)
    csrc = tmp_path / f"{name}.c"
    csrc.write_text(mutated)
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(csrc), "-lm"], check=True)
    failed = []
    with oracle.use_library(str(lib)):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, IndexError, ValueError):
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
