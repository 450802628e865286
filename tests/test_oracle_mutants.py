"""Planted mistakes in the oracle must be caught by its pins.

Each case copies the oracle's C source, plants one plausible mistake (a
dropped term, a wrong index or sign, a transposed operand, a missed rule),
compiles the copy with gcc, and re-runs every pin in `pins.py` against it.
A mutant that passes every pin would mean the pins cannot tell that mistake
from the method, so the test fails. Nothing here touches a GPU, and no planted
mistake reads or writes outside its buffers.
"""
import os
import shutil
import tempfile

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fvattn_oracle.c")

MUTANTS = {
    "pool_divides_by_full_block": ("const double cnt = (double)(tv * yv * xv);",
                                   "const double cnt = (double)(g->bt * g->bh * g->bw);"),
    "extent_off_by_one": ("*tv = (g->T - *t0 < g->bt) ? g->T - *t0 : g->bt;",
                          "*tv = (g->T - *t0 < g->bt) ? g->T - *t0 : g->bt - 1;"),
    "q_k_transposed": ("const double *qi = qbar + r * D;", "const double *qi = kbar + r * D;"),
    "route_missing_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "probs_not_normalised": ("for (int j = 0; j < nb; ++j) P[j] /= z;", "(void)z;"),
    "rank_ascending": ("if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
                       "if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;"),
    "tie_to_higher_index": ("if (x->s < y->s) return 1;\n    return (x->j < y->j) ? -1 : (x->j > y->j);",
                            "if (x->s < y->s) return 1;\n    return (x->j > y->j) ? -1 : (x->j < y->j);"),
    "topp_count_off_by_one": ("{ m_p = q + 1; found = 1; }", "{ m_p = q; found = 1; }"),
    "floor_ignored": ("int m = m_p > k_min ? m_p : k_min;", "int m = m_p;"),
    "diagonal_not_kept": ("keep[i] = 1; /* repair", "(void)0; /* repair"),
    "nonfinite_not_repaired": ("if (!isfinite(s[j])) finite = 0;", "(void)0;"),
    "attn_ignores_lists": ("    if (kv_cnt) {\n                cnt", "    if (0) {\n                cnt"),
    "attn_missing_scale": ("logit[nk] = scale * dot;", "logit[nk] = dot;"),
    "attn_wrong_query_block": ("const int i = token_block(g, n);", "const int i = token_block(g, 0);"),
    "f16_exponent_bias": ("else v = ldexp((double)(1024 + m), e - 25);", "else v = ldexp((double)(1024 + m), e - 24);"),
    "f16_subnormal_scale": ("if (e == 0) v = ldexp((double)m, -24);", "if (e == 0) v = ldexp((double)m, -25);"),
    "order_store_shifted": ("if (order) order[r * (int64_t)nb + q] = rk[q].j;",
                            "if (order) order[r * (int64_t)nb + q] = rk[q > 0 ? q - 1 : 0].j;"),
    "probs_store_reversed": ("probs[r * (int64_t)nb + j] = P[j];", "probs[r * (int64_t)nb + j] = P[nb - 1 - j];"),
    "probs_store_unnormalised": ("probs[r * (int64_t)nb + j] = P[j];", "probs[r * (int64_t)nb + j] = P[j] * z;"),
    "augment_ascending": ("    if (x->p > y->p) return -1;\n    if (x->p < y->p) return 1;",
                          "    if (x->p < y->p) return -1;\n    if (x->p > y->p) return 1;"),
    "augment_skips_and_continues": ("if (spent + cost > budget) break;", "if (spent + cost > budget) continue;"),
    "augment_costs_query_tokens_only": ("const int64_t cost = (int64_t)size[i] * size[c[x].j];",
                                        "const int64_t cost = (int64_t)size[i];"),
    "augment_forgets_base_lists": ("for (int e = 0; e < kv_cnt[r]; ++e) keep[r * nb + kv_idx[r * (int64_t)nb + e]] = 1;",
                                   "for (int e = 0; e < 0; ++e) keep[r * nb + kv_idx[r * (int64_t)nb + e]] = 1;"),
    "f16_inputs_read_as_bf16": ("return g->fp16 ? f16_to_f64(h) : bf16_to_f64(h);", "return bf16_to_f64(h);"),
}


@pytest.fixture(scope="module")
def tmpdir_mod():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmpdir_mod):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path_c = os.path.join(tmpdir_mod, f"{name}.c")
    path_so = os.path.join(tmpdir_mod, f"{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    oracle.compile_oracle(path_c, path_so)
    orc = oracle.Oracle(path_so)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
