"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU;
the real oracle is untouched), compiles it, and checks that at least one pin
of tests/test_oracle_pins.py -- the hand-worked fixtures, the torch-CPU sort
recipe, the invariants -- rejects the mutant.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from mixture_experts_routed_non_b200 import synthetic
from test_oracle_backward import check_autograd, check_finite_differences
from test_oracle_pairs import check_pair_fixture, check_table_equivalence
from test_oracle_router import check_router_against_torch, check_router_fixture
from test_oracle_pins import (GOLDEN, _bf, _load, _num, _recipe_torch_cpu,
                              check_combine_direct_sum, check_metadata_invariants)

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = {
    "gate_up_swapped": ("h[j] = g / (1.0 + exp(-g)) * u;", "h[j] = u / (1.0 + exp(-u)) * g;"),
    "silu_sign": ("h[j] = g / (1.0 + exp(-g)) * u;", "h[j] = g / (1.0 + exp(g)) * u;"),
    "b1_dropped": ("z[j] = b1e ? bf16_value(b1e[j]) : 0.0;", "z[j] = 0.0;"),
    "b2_dropped": ("y[n] = b2e ? bf16_value(b2e[n]) : 0.0;", "y[n] = 0.0;"),
    "concat_wrong_up": ("else             { g = z[j];     u = z[I + j]; }",
                        "else             { g = z[j];     u = z[j + 1]; }"),
    "interleave_wrong": ("if (layout == 0) { g = z[2 * j]; u = z[2 * j + 1]; }",
                         "if (layout == 0) { g = z[j]; u = z[I + j]; }"),
    "score_ignored": ("for (int32_t n = 0; n < H; ++n) o[n] += w * y[n];",
                      "for (int32_t n = 0; n < H; ++n) o[n] += y[n];"),
    "w2_transposed_index": ("const uint16_t *wr = w2e + (size_t)j * H;\n        for (int32_t n = 0; n < H; ++n) y[n] += hv * bf16_value(wr[n]);",
                            "for (int32_t n = 0; n < H; ++n) y[n] += hv * bf16_value(w2e[(size_t)n * I + (j % I)]);"),
    "sort_unstable": ("for (int64_t i = 0; i < q; ++i) {\n        int32_t p = cursor[pair_expert[i]]++;",
                      "for (int64_t i = q - 1; i >= 0; --i) {\n        int32_t p = cursor[pair_expert[i]]++;"),
    "token_offset_late": ("        token_offset[t] = (int32_t)q;\n        for (int32_t k = 0; k < K; ++k) {",
                          "        for (int32_t k = 0; k < K; ++k) {"),
    "offsets_inclusive": ("off[e + 1] = off[e] + freq[e];", "off[e + 1] = off[e] + freq[e] + (e == 0);"),
    "invalid_counted": ("if (e >= 0 && e < E) {", "if (e < E) { if (e < 0) e = 0;"),
    "pairs_offset_inclusive": ("if (pair_token[j] < t) ++below;", "if (pair_token[j] <= t) ++below;"),
    "pairs_bad_token_kept": ("if (t >= 0 && t < N) {", "if (t >= 0) {"),
    "pairs_sort_unstable": ("for (int64_t j = 0; j < q; ++j) {\n        int32_t p = cursor[pair_expert[j]]++;",
                            "for (int64_t j = q - 1; j >= 0; --j) {\n        int32_t p = cursor[pair_expert[j]]++;"),
    "router_ties_to_higher_id": ("if (!taken[e] && (best < 0 || row[e] > row[best])) best = e;",
                                 "if (!taken[e] && (best < 0 || row[e] >= row[best])) best = e;"),
    "router_picks_smallest": ("if (!taken[e] && (best < 0 || row[e] > row[best])) best = e;",
                              "if (!taken[e] && (best < 0 || row[e] < row[best])) best = e;"),
    "router_topk_softmax_over_all": ("for (int32_t k = 0; k < K; ++k) s += exp(row[ix[k]] - top);",
                                     "for (int32_t e = 0; e < E; ++e) s += exp(row[e] - top);"),
    "router_no_renorm": ("if (mode == 2) {", "if (mode == 3) {"),
    "bwd_silu_derivative": ("dz[gi] = dh * u * sig * (1.0 + g * (1.0 - sig));", "dz[gi] = dh * u * sig;"),
    "bwd_gate_up_swapped": ("dz[ui] = dh * g * sig;", "dz[ui] = dh * u * sig;"),
    "bwd_score_dropped": ("dy[n] = s * dout[n];", "dy[n] = dout[n];"),
    "bwd_score_grad_of_dy": ("acc += dout[n] * y[n];", "acc += dy[n] * y[n];"),
    "bwd_w2_not_transposed": ("for (int32_t n = 0; n < H; ++n) dh += dy[n] * wr[n];",
                              "for (int32_t n = 0; n < H; ++n) dh += dy[n] * w2e[(size_t)n * I + j];"),
    "pairs_score_of_next": ("scores[q] = weights[i];", "scores[q] = weights[i + 1 < P_list ? i + 1 : i];"),
    "gather_holds_pair_index": ("x_gather_idx[p] = pair_token[i];", "x_gather_idx[p] = (int32_t)i;"),
    "reverse_scatter_identity": ("s_rev[i] = p;", "s_rev[i] = (int32_t)i;"),
    "score_of_next_slot": ("scores[q] = topk_w[t * K + k];", "scores[q] = topk_w[t * K + (k + 1) % K];"),
    "combine_reverse_index_ignored": ("const double *yr = ysorted + (size_t)s_rev[q] * H;",
                                      "const double *yr = ysorted + (size_t)q * H;"),
    "combine_score_ignored": ("const double w = (double)scores[q];", "const double w = 1.0;"),
}


def _mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert old in src, f"mutation anchor missing for {name}"
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src.replace(old, new, 1))
    so = str(tmp_path / f"mut_{name}.so")
    oracle.compile_source(str(path), so)
    return so


def _pins_pass(lib):
    """Run the library-level pins against one build; True when all agree."""
    try:
        # hand-worked metadata example
        g = _load("metadata_worked_example.json")
        idx = np.array(g["topk_idx"], np.int32)
        w = np.array([[_num(v) for v in r] for r in g["topk_w"]], np.float32)
        md = oracle.metadata(idx, w, g["E"], lib_path=lib)
        ex = g["expected"]
        if (md["off"].tolist() != ex["expert_frequency_offset"]
                or md["s_scatter_idx"].tolist() != ex["s_scatter_idx"]
                or md["token_offset"].tolist() != ex["num_activated_expert_per_token_offset"]
                or md["x_gather_idx"].tolist() != ex["x_gather_idx"]):
            return False
        check_metadata_invariants(idx, w, g["E"], md)
        # the combine against a per-slot sum
        check_combine_direct_sum(lib)
        # closed-form SwiGLU fixture, both layouts
        g = _load("swiglu_closed_form.json")
        x, w1, b1, w2, b2 = (_bf(g[k]) for k in ("x", "w1", "b1", "w2", "b2"))
        idx = np.array(g["topk_idx"], np.int32)
        w = np.array([[_num(v) for v in r] for r in g["topk_w"]], np.float32)
        wts = oracle.Weights(x, w1, b1, w2, b2)
        env = {"exp": math.exp}
        for layout, key in ((0, "interleaved"), (1, "concatenated")):
            out = oracle.forward_rows(wts, idx, w, layout=layout, lib_path=lib)
            out_ex = [eval(s, env) for s in g["expected_closed_form"][key]["out"]]
            if not np.allclose(out[0], out_ex, rtol=1e-12, atol=1e-12):
                return False
        # backward: finite differences, torch autograd through the recipe
        check_finite_differences(0, lib)
        check_autograd(1, lib)
        # router top-k: hand-worked closed forms, torch.topk / torch.softmax
        check_router_fixture(lib)
        check_router_against_torch(lib)
        # pair-list metadata: hand-worked fixture, table oracle on a flattened table
        check_pair_fixture(lib)
        wl = synthetic.WORKLOADS["tiny"]
        idx, w = synthetic.make_routing(wl, invalid_value=float("nan"))
        check_table_equivalence(idx, w, wl.E, lib)
        # torch-CPU sort recipe on the tiny workload
        inp = synthetic.make_inputs("tiny", device="cpu")
        wts = oracle.Weights(inp.x, inp.w1, inp.b1, inp.w2, inp.b2)
        for layout in (0, 1):
            out = oracle.forward_rows(wts, inp.topk_idx.numpy(), inp.topk_w.numpy(),
                                      layout=layout, lib_path=lib)
            if not np.allclose(out, _recipe_torch_cpu(inp, layout), rtol=1e-9, atol=1e-10):
                return False
        return True
    except AssertionError:
        return False


def test_unmutated_oracle_passes_pins():
    assert _pins_pass(None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_rejected(tmp_path, name):
    assert not _pins_pass(_mutant(tmp_path, name)), f"pins did not catch mutant {name}"
