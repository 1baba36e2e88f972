"""Plausible mistakes planted in a COPY of the oracle must fail at least one pin.

Each mutation edits the C source text in a temporary directory (the committed oracle
is untouched), builds it, swaps it in for the duration of the test, and runs the pins
of ``test_oracle_pins.py``.  A mutation that no pin catches fails this test.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "more_oracle.c")

MUTATIONS = {
    "tie_break_reversed": ("return (a->e < b->e) ? -1 : (a->e > b->e);",
                           "return (a->e > b->e) ? -1 : (a->e < b->e);"),
    "ascending_order": ("if (la > lb) return -1;\n  if (la < lb) return 1;",
                        "if (la < lb) return -1;\n  if (la > lb) return 1;"),
    "R1_transposed": ("s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);\n    z[i] = s;",
                      "s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)i * h + t]);\n    z[i] = s;"),
    "R2_transposed": ("for (int i = 0; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)i * M + e]);\n    logits[e] = s;",
                      "for (int i = 0; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)e * r + i]);\n    logits[e] = s;"),
    "dropped_rank_term": ("for (int i = 0; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)i * M + e]);\n    logits[e] = s;",
                          "for (int i = 1; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)i * M + e]);\n    logits[e] = s;"),
    "dropped_hidden_term": ("for (int t = 0; t < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);\n    z[i] = s;",
                            "for (int t = 0; t + 1 < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);\n    z[i] = s;"),
    "fullrank_W_transposed": ("const uint16_t* w = W + (size_t)t * M;\n    for (int e = 0; e < M; ++e) logits[e] += xt * oracle_bf16(w[e]);",
                              "for (int e = 0; e < M; ++e) logits[e] += xt * oracle_bf16(W[(size_t)e * h + t]);"),
    "fullrank_dropped_hidden_term": ("for (int t = 0; t < h; ++t) {\n    const double xt",
                                     "for (int t = 1; t < h; ++t) {\n    const double xt"),
    "softmax_sign": ("gate[j] = exp(sel_logit[j] - top) / denom;", "gate[j] = exp(top - sel_logit[j]) / denom;"),
    "softmax_missing_shift": ("denom += exp(sel_logit[j] - top);", "denom += exp(sel_logit[j]);"),
    "margin_wrong_runner_up": ("sel_logit[k - 1] - logits[scratch[k].e]",
                               "sel_logit[k - 1] - logits[scratch[k + 1 < M ? k + 1 : k].e]"),
    "counts_double_first": ("jb->counts[jb->idx[o + j]] += 1;", "jb->counts[jb->idx[o + j]] += (j == 0) ? 2 : 1;"),
    "rms_without_mean": ("*rms = sqrt(ss / (double)M);", "*rms = sqrt(ss);"),
    "stats_max_skips_expert_0": ("double mx = l[0];\n    for (int e = 1; e < jb->M; ++e)",
                                 "double mx = l[1];\n    for (int e = 2; e < jb->M; ++e)"),
    "stats_Z_without_shift": ("for (int e = 0; e < jb->M; ++e) sum += exp(l[e] - mx);",
                              "for (int e = 0; e < jb->M; ++e) sum += exp(l[e]);"),
    "stats_psum_unnormalised": ("jb->psum[e] += exp(l[e] - mx) / sum;", "jb->psum[e] += exp(l[e] - mx);"),
    "stats_psum_dropped_last_expert": ("for (int e = 0; e < jb->M; ++e) jb->psum[e] += exp(l[e] - mx) / sum;",
                                       "for (int e = 0; e + 1 < jb->M; ++e) jb->psum[e] += exp(l[e] - mx) / sum;"),
}

PINS = [
    pins.test_logits_equal_explicit_W_product,
    pins.test_projection_and_pairs_agree_with_matmul,
    lambda: pins.test_topk_matches_brute_force_random(13),
    lambda: pins.test_topk_matches_brute_force_tie_heavy(16),
    pins.test_golden_tie_order,
    pins.test_relabelling_equivariance,
    pins.test_k_equals_M_gives_full_softmax,
    pins.test_gate_special_cases,
    pins.test_margin_gaps_and_rms_against_sorted_logits,
    pins.test_counts_are_the_bincount_of_indices,
    pins.test_golden_jl_construction,
    pins.test_golden_hypercube_top1_is_sign_pattern,
    pins.test_train_stats_closed_forms,
    pins.test_train_stats_against_library_softmax,
    pins.test_train_stats_shift_and_relabelling,
    pins.test_fullrank_matches_the_factored_router_when_W_is_their_product,
    pins.test_fullrank_tie_order_and_brute_force_ranks,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))  # every occurrence
    lib_path = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o",
                           str(lib_path), str(mutated), "-lm", "-lpthread"])
    monkeypatch.setattr(oracle, "_lib", oracle._bind(ctypes.CDLL(str(lib_path))))
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught the planted mistake {name}"


PY_MUTATIONS = {
    # name: (oracle function, source anchor, replacement)
    "backward_g_sign": ("router_backward_f64", "ybar = P * (pbar[None, :] - g[:, None])",
                        "ybar = P * (pbar[None, :] + g[:, None])"),
    "backward_no_topk_scatter": ("router_backward_f64", "np.add.at(ybar,", "(lambda *a: None)(ybar,"),
    "backward_R1_grad_from_z": ("router_backward_f64", "X.T @ zbar, z.T @ ybar, g)",
                                "X.T @ (z * 0 + zbar.mean()), z.T @ ybar, g)"),
    "dispatch_within_expert_reversed": ("dispatch", 'order = np.argsort(flat, kind="stable")',
                                        'order = flat.size - 1 - np.argsort(flat[::-1], kind="stable")'),
    "dispatch_offsets_inclusive": ("dispatch", "offsets = np.concatenate([[0], np.cumsum(counts)])",
                                   "offsets = np.concatenate([np.cumsum(counts), [flat.size]])"),
    "dispatch_counts_drop_last_slot": ("dispatch", "counts = np.bincount(flat, minlength=M)",
                                       "counts = np.bincount(flat[:-1], minlength=M)"),
}
PY_PINS = {
    "router_backward_f64": [pins.test_backward_matches_finite_differences, pins.test_backward_matches_torch_autograd,
                            pins.test_backward_constant_pbar_and_bf16_entry],
    "dispatch": [lambda: pins.test_dispatch_matches_brute_force(50, 4, 16),
                 pins.test_dispatch_invariants_on_routing_output],
}


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_planted_python_mistake_is_caught(name, monkeypatch):
    """The same for the numpy parts of the oracle (backward, dispatch): a mutated copy of the
    module's source, with the mutated function put in place of the original."""
    import types

    func, old, new = PY_MUTATIONS[name]
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    mutant = types.ModuleType("oracle_mutant")
    mutant.__file__ = oracle.__file__
    exec(compile(src.replace(old, new), oracle.__file__, "exec"), mutant.__dict__)
    monkeypatch.setattr(oracle, func, getattr(mutant, func))
    caught = []
    for pin in PY_PINS[func]:
        try:
            pin()
        except AssertionError:
            caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught the planted mistake {name}"
