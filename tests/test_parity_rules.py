"""The set checks used by the GPU parity tests of the selection rules (CPU
only): they accept the oracle's own sets and reject sets that are clearly
wrong in size or content."""
import numpy as np
import pytest

import oracle as O
from tests import parity as P

RULES = [O.Selection(O.RULE_RATIO, ratio=(1, 8)), O.Selection(O.RULE_BLOCK_TOPK, block=16),
         O.Selection(O.RULE_TOPP, p=0.6), O.Selection(O.RULE_THRESHOLD, tau=2e-3)]


def keys_with_heavy_hitters(seed, n=700):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n)
    x[rng.choice(n, 40, replace=False)] += 5.0
    return x


@pytest.mark.parametrize("sel", RULES, ids=lambda s: f"rule{s.rule}")
def test_oracle_sets_accepted(sel):
    for seed in range(5):
        x = keys_with_heavy_hitters(seed)
        S = O.select(x, 256, sel)
        P.check_set_rule(S, x, 256, sel, "oracle set")


@pytest.mark.parametrize("sel", RULES, ids=lambda s: f"rule{s.rule}")
def test_wrong_sets_rejected(sel):
    x = keys_with_heavy_hitters(7)
    S = O.select(x, 256, sel)
    m = int((S >= 0).sum())
    # one row fewer (a whole block fewer for block selection)
    drop = sel.block if sel.rule == O.RULE_BLOCK_TOPK else 1
    short = np.concatenate([S[:m - drop], np.full(256 - m + drop, -1, np.int32)])
    with pytest.raises(AssertionError):
        P.check_set_rule(short, x, 256, sel, "short set")
    # the largest key swapped for the smallest unselected one
    swapped = S.copy()
    best = int(np.argmax(x))
    worst = int(np.argmin(x))
    if best in S[:m] and worst not in S[:m]:
        v = S[:m].tolist()
        v[v.index(best)] = worst
        swapped[:m] = np.sort(v)
        with pytest.raises(AssertionError):
            P.check_set_rule(swapped, x, 256, sel, "swapped set")
    # entries after the padding
    if m + 2 <= 256:
        bad = S.copy()
        bad[m:m + 2] = [-1, 5]
        with pytest.raises(AssertionError):
            P.check_set_rule(bad, x, 256, sel, "entry after padding")
