"""Plant one plausible mistake at a time in a copy of the oracle and check that
at least one pin fails for each. This shows the pins constrain every step of
the oracle: probe order, Bloom test (and its OR over alternative masks), inner
product, list range, top-k order and padding. The mutants are built from the oracle source into a temporary folder;
the real oracle is never modified."""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle.build import SRC, build
from oracle_pins import PINS

MUTANTS = {
    "tie_higher_id_first": ("return a->id < b->id ? -1 : 1;", "return a->id > b->id ? -1 : 1;"),
    "ascending_scores": ("return a->score > b->score ? -1 : 1;",
                         "return a->score < b->score ? -1 : 1;"),
    "bloom_any_bit": ("if ((sig[w] & mask[w]) != mask[w]) return 0;",
                      "if (mask[w] && (sig[w] & mask[w]) == 0) return 0;"),
    "bloom_first_word_only": ("for (int32_t w = 0; w < W; ++w)\n        if ((sig[w]",
                              "for (int32_t w = 0; w < 1; ++w)\n        if ((sig[w]"),
    "bloom_transposed": ("if ((sig[w] & mask[w]) != mask[w]) return 0;",
                         "if ((sig[w] & mask[w]) != sig[w]) return 0;"),
    "dot_drops_last_term": ("for (int32_t j = 0; j < d; ++j) s +=", "for (int32_t j = 0; j < d - 1; ++j) s +="),
    "dot_unsigned_operand": ("s += (int32_t)a[j] * (int32_t)b[j];", "s += (int32_t)(uint8_t)a[j] * (int32_t)b[j];"),
    "probe_row_stride": ("oracle_dot(q, cent + (int64_t)c * d, d)", "oracle_dot(q, cent + (int64_t)c, d)"),
    "probe_off_by_one": ("out_lists[p] = (int32_t)cs[p].id;", "out_lists[p] = (int32_t)cs[p + (p + 1 < nlist)].id;"),
    "list_drops_last_item": ("for (int64_t i = off[c]; i < off[c + 1]; ++i)",
                             "for (int64_t i = off[c]; i + 1 < off[c + 1]; ++i)"),
    "item_row_stride": ("oracle_dot(q, items + i * d, d)", "oracle_dot(q, items + i, d)"),
    "pad_id_zero": ("out_ids[r] = -1;", "out_ids[r] = 0;"),
    "pad_score_zero": ("out_scores[r] = INT32_MIN;", "out_scores[r] = 0;"),
    "filter_after_topk": ("if (!bloom_pass_any(sigs + i * W, m, A, W)) continue;", ""),
    "or_needs_every_mask": ("if (oracle_bloom_pass(sig, m + (int64_t)a * W, W)) return 1;\n    return 0;",
                            "if (!oracle_bloom_pass(sig, m + (int64_t)a * W, W)) return 0;\n    return 1;"),
    "or_first_mask_only": ("for (int32_t a = 0; a < A; ++a)\n        if (oracle_bloom_pass",
                           "for (int32_t a = 0; a < 1; ++a)\n        if (oracle_bloom_pass"),
    "or_mask_stride": ("m + (int64_t)a * W, W)", "m + (int64_t)a, W)"),
    "or_query_stride": ("masks + (int64_t)b * A * W;", "masks + (int64_t)b * W;"),
    "row_ids_ignored": ("cand[n].id = row_ids ? row_ids[i] : i;", "cand[n].id = i;"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique for {name}"
    msrc = os.path.join(mutant_dir, f"{name}.c")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(mutant_dir, f"{name}.so")
    build(msrc, so, extra=("-Wno-error",))
    lib = oracle.load(so)
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches mutant {name}"
