"""Plausible mistakes planted in copies of the oracle (on the CPU) must fail a pin.

Each entry alters one spot of oracle.c -- a dropped term, a wrong index, a
swapped operand, a reversed order -- compiles the copy, and runs the pins of
``pins.FAST_PINS`` against it until one fails.  A mutant that passes every pin
would mean the pins cannot tell that mistake from the correct oracle.  Every
alteration keeps memory accesses in bounds so that a mutant can only compute
wrong numbers, never crash.
"""
import os

import pytest

import oracle
import pins

# (name, text in oracle.c, replacement, which occurrence (0-based))
MUTANTS = [
    ("gqa_map_select", "const int j = h * G + g; /* contiguous GQA groups */",
     "const int j = g * Hkv + h;", 0),
    ("gqa_map_sparse", "const int j = h * G + g;\n        const size_t qoff",
     "const int j = g * Hkv + h;\n        const size_t qoff", 0),
    ("no_scale_select", "logit[t] = c * dot;", "logit[t] = dot;", 0),
    ("no_scale_sparse", "logit[t] = c * dot;", "logit[t] = dot;", 1),
    ("average_over_block_only", "mass[t] += p / (double)(B * G);",
     "mass[t] += p / (double)(B);", 0),
    ("tie_higher_index_wins", "return (a->page > b->page) - (a->page < b->page);",
     "return (a->page < b->page) - (a->page > b->page);", 0),
    ("smallest_scores_kept", "if (a->score > b->score) return -1;\n  if (a->score < b->score) return 1;",
     "if (a->score > b->score) return 1;\n  if (a->score < b->score) return -1;", 0),
    ("not_ascending", "qsort(chosen, (size_t)take, sizeof(int), by_int);", "", 0),
    ("block_tokens_dropped", "for (int u = 0; u < B; ++u) {", "for (int u = 0; u < 0; ++u) {", 0),
    ("tail_tokens_kept", "slot < P && lp * P + slot < n", "slot < P", 0),
    ("unnormalised_select_output", "const double p = exp(logit[t] - mx) / sum;\n          long pp",
     "const double p = exp(logit[t] - mx);\n          long pp", 0),
    ("values_are_keys_select", "cache_row(v, pp, h, t % P, Hkv, P, d)",
     "cache_row(k, pp, h, t % P, Hkv, P, d)", 0),
    ("values_are_keys_sparse", "vrow[nk] = cache_row(v, pp, h, slot, Hkv, P, d);",
     "vrow[nk] = cache_row(k, pp, h, slot, Hkv, P, d);", 0),
    ("block_values_are_keys", "vrow[nk] = blk_v + off;", "vrow[nk] = blk_k + off;", 0),
    ("page_score_last_token", "sc += mass[t];", "sc = mass[t];", 0),
    ("bad_widening", "((uint32_t)bits) << 16", "((uint32_t)bits) << 15", 0),
    ("first_slot_only_sparse", "krow[nk] = cache_row(k, pp, h, slot, Hkv, P, d);",
     "krow[nk] = cache_row(k, pp, h, 0, Hkv, P, d);", 0),
    ("lse_missing_max", "lse_out[((size_t)s * B + b) * Hq + j] = mx + log(sum);",
     "lse_out[((size_t)s * B + b) * Hq + j] = log(sum);", 0),
    ("kv_head_ignored", "(((size_t)phys * Hkv + h) * P + slot)", "(((size_t)phys * Hkv + 0) * P + slot)", 0),
    ("query_row_ignored", "const size_t qoff = (((size_t)s * B + b) * Hq + j) * (size_t)d;",
     "const size_t qoff = (((size_t)s * B + 0) * Hq + j) * (size_t)d;", 0),
    ("max_not_subtracted_sparse", "sum += exp(logit[t] - mx);", "sum += exp(logit[t]);", 1),
    ("global_budget_per_head", "const long budget = (long)Hkv * (topk[s] / P);",
     "const long budget = (long)(topk[s] / P);", 0),
    ("global_items_head_ignored", "items[h * np + lp].score = score[((size_t)s * Hkv + h) * max_pages + lp];",
     "items[h * np + lp].score = score[((size_t)s * Hkv + 0) * max_pages + lp];", 0),
    ("losa_cache_for_active", "const int act = active[(size_t)s * B + b] != 0;",
     "const int act = active[(size_t)s * B + b] == 0;", 0),
    ("losa_block_dropped", "const double wb = exp(lse_b - top);", "const double wb = 0.0 * exp(lse_b - top);", 0),
    ("losa_cache_lse_ignored", "lse_p = cache_lse_in[ro];", "lse_p = 0.0;", 0),
    ("global_pages_unsorted", "qsort(chosen, (size_t)take, sizeof(int), by_int); /* head-major",
     "(void)by_int; /* head-major", 0),
]


def _mutate(src: str, old: str, new: str, occurrence: int) -> str:
    pos = -1
    for _ in range(occurrence + 1):
        pos = src.find(old, pos + 1)
        assert pos >= 0, f"mutation anchor not found: {old!r} (occurrence {occurrence})"
    return src[:pos] + new + src[pos + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, occ):
    with open(oracle.SOURCE) as f:
        src = f.read()
    path = tmp_path / f"{name}.c"
    path.write_text(_mutate(src, old, new, occ))
    lib = oracle.compile_source(str(path), str(tmp_path / f"lib{name}.so"))
    mutant = oracle.Oracle(lib)
    for pin in pins.FAST_PINS:
        try:
            pin(mutant)
        except (AssertionError, oracle.OracleError, ValueError, FloatingPointError):
            return  # caught
    pytest.fail(f"mutant {name} passed every pin")


def test_unaltered_copy_passes(tmp_path):
    """Control: a verbatim copy compiled the same way passes every pin."""
    lib = oracle.compile_source(oracle.SOURCE, str(tmp_path / "libcopy.so"))
    copy = oracle.Oracle(lib)
    for pin in pins.FAST_PINS:
        pin(copy)
    assert os.path.exists(lib)
