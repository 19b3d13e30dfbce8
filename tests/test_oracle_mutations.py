"""Plant plausible mistakes in the oracle (on the CPU) and check that at least
one pin of test_oracle_pins.py fails for each.  This is what makes the pins
meaningful: a dropped term, a wrong index or a wrong tie-break in the oracle
cannot pass silently."""
import math

import numpy as np
import pytest

from oracle import hga_oracle as ho
import test_oracle_pins as pins

ALL_PINS = [pins.pin_golden_routing, pins.pin_golden_attention,
            pins.pin_bf16_rounding, pins.pin_summaries_exact,
            lambda: pins.pin_bruteforce_routing(3, True),
            lambda: pins.pin_bruteforce_routing(5, False),
            lambda: pins.pin_dense_equivalence(0, 200),
            lambda: pins.pin_dense_equivalence(48, 200),
            pins.pin_invariants]


def _some_pin_fails():
    for pin in ALL_PINS:
        try:
            pin()
        except (AssertionError, KeyError, IndexError, ValueError):
            return True
    return False


def _cand_off_by_one(b0, p):            # lets the first local chunk in
    lo = p.sink // p.chunk
    hi = (b0 - p.local) // p.chunk + 1
    return list(range(lo, max(lo, hi)))


def _cand_with_sink(b0, p):              # forgets to exclude the sink chunk
    hi = (b0 - p.local) // p.chunk if b0 - p.local > 0 else 0
    return list(range(0, max(0, hi)))


def _cand_drop_last(b0, p):              # loses the chunk next to the window
    lo = p.sink // p.chunk
    hi = (b0 - p.local) // p.chunk - 1
    return list(range(lo, hi)) if hi > lo else []


def _select_high_index_ties(cands, scores, k):
    n = len(cands)
    k_eff = n if k <= 0 else min(k, n)
    order = sorted(range(n), key=lambda i: (-scores[i], -cands[i]))
    chosen = sorted(cands[i] for i in order[:k_eff])
    margin = math.inf if k_eff in (0, n) else float(
        scores[order[k_eff - 1]] - scores[order[k_eff]])
    return chosen, margin


def _scores_mean(rows, summaries):        # mean over rows instead of max
    if summaries.shape[0] == 0:
        return np.zeros(0)
    return (rows @ summaries.T / math.sqrt(rows.shape[1])).mean(axis=0)


def _scores_unscaled(rows, summaries):    # drops the 1/sqrt(d)
    if summaries.shape[0] == 0:
        return np.zeros(0)
    return (rows @ summaries.T).max(axis=0)


def _set_no_diag(b0, pos, groups, p):
    toks = set(range(0, min(p.sink, pos + 1)))
    for j in groups:
        toks.update(range(j * p.group, (j + 1) * p.group))
    toks.update(range(max(0, b0 - p.local), b0))
    return np.array(sorted(toks) or [0], dtype=np.int64)


def _set_future(b0, pos, groups, p):      # whole block, ignoring causality
    toks = set(range(0, p.sink))
    for j in groups:
        toks.update(range(j * p.group, (j + 1) * p.group))
    toks.update(range(max(0, b0 - p.local), b0 + p.qblock))
    return np.array(sorted(toks), dtype=np.int64)


def _round_truncate(x):                  # chops instead of rounding to even
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)


def _group_per_chunk_quota(q, q0, T, gsum_h, chunks, p, b, h, q_route=None):
    # best groups chosen per chunk instead of over all chosen chunks
    rows, _, _ = ho.routing_rows(q, q0, T, p, b, h, q_route)
    per = p.chunk // p.group
    out = []
    for c in chunks:
        cands = [c * per + i for c in [c] for i in range(per)]
        S = np.stack([gsum_h[j] for j in cands])
        ch, _ = ho.select_top(cands, ho.block_scores(rows, S),
                              max(1, p.top_groups // max(1, len(chunks))))
        out += ch
    return sorted(out), math.inf


MUTATIONS = {
    "candidates_off_by_one": ("chunk_candidates", _cand_off_by_one),
    "candidates_include_sink": ("chunk_candidates", _cand_with_sink),
    "candidates_drop_last": ("chunk_candidates", _cand_drop_last),
    "ties_to_high_index": ("select_top", _select_high_index_ties),
    "score_mean_not_max": ("block_scores", _scores_mean),
    "score_unscaled": ("block_scores", _scores_unscaled),
    "attention_no_diagonal": ("attention_set", _set_no_diag),
    "attention_sees_future": ("attention_set", _set_future),
    "rounding_truncates": ("round_bf16", _round_truncate),
    "group_quota_per_chunk": ("route_groups_unit", _group_per_chunk_quota),
}


def test_unmutated_oracle_passes_all_pins():
    assert not _some_pin_fails()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(ho, attr, fn)
    assert _some_pin_fails(), f"planted mistake {name} passed every pin"
