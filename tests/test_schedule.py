"""The launchers' static schedule of work items (fa_schedule_items; host only, no GPU):
a valid partition, each list heaviest first, never worse than longest-processing-time
first, within LPT's 4/3 bound of the optimum found by brute force on small cases, and
errors for bad arguments."""
import itertools
import math

import numpy as np
import pytest

from exact_io_aware_60_b200 import fa


def loads(cost, off, ids):
    return [sum(cost[i] for i in ids[off[c]:off[c + 1]]) for c in range(len(off) - 1)]


def lpt_max(cost, lists):
    """Longest processing time first onto the least loaded list (plain reference)."""
    load = [0.0] * lists
    for x in sorted(cost, reverse=True):
        load[load.index(min(load))] += x
    return max(load)


def check_valid(cost, lists, off, ids):
    n = len(cost)
    assert off[0] == 0 and off[lists] == n
    assert all(off[c] <= off[c + 1] for c in range(lists))
    assert sorted(ids.tolist()) == list(range(n))
    for c in range(lists):
        cs = [cost[i] for i in ids[off[c]:off[c + 1]]]
        assert cs == sorted(cs, reverse=True)


def gpt2_costs(kind):
    """Item costs of the GPT-2-shaped causal launch (B8 H12 N1024): forward items in
    64-key blocks plus 1.8, backward items in query tiles plus 0.9."""
    if kind == "fwd":
        return [2.0 * (8 - u // 96) + 1.8 for u in range(768)]
    return [float(8 - u // 96) + 0.9 for u in range(768)]


@pytest.mark.parametrize("kind,lists", [("fwd", 296), ("bwd", 148)])
def test_gpt2_shaped_schedule(kind, lists):
    cost = gpt2_costs(kind)
    off, ids = fa.fa_schedule_items(cost, lists)
    check_valid(cost, lists, off, ids)
    mx = max(loads(cost, off, ids))
    lower = max(sum(cost) / lists, max(cost))
    assert mx <= lpt_max(cost, lists) + 1e-4
    assert lower - 1e-4 <= mx <= 1.06 * lower


def test_small_cases_against_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(60):
        n = int(rng.integers(1, 8))
        lists = int(rng.integers(1, 4))
        cost = [float(x) for x in rng.integers(1, 10, size=n)]
        off, ids = fa.fa_schedule_items(cost, lists)
        check_valid(cost, lists, off, ids)
        got = max(loads(cost, off, ids))
        best = min(max(sum(cost[i] for i in range(n) if a[i] == c) for c in range(lists))
                   for a in itertools.product(range(lists), repeat=n))
        assert got <= lpt_max(cost, lists) + 1e-6
        assert got <= (4.0 / 3.0 - 1.0 / (3 * lists)) * best + 1e-6


def test_deterministic_and_equal_costs_spread_evenly():
    cost = [1.0] * 1000
    a = fa.fa_schedule_items(cost, 148)
    b = fa.fa_schedule_items(cost, 148)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    sizes = np.diff(a[0].astype(np.int64))
    assert sizes.max() - sizes.min() <= 1


@pytest.mark.parametrize("cost,lists", [
    ([], 4), ([1.0] * 2049, 4), ([1.0], 0), ([1.0], 513), ([1.0, 0.0], 2),
    ([1.0, -1.0], 2), ([1.0, math.nan], 2), ([1.0, math.inf], 2)])
def test_bad_arguments(cost, lists):
    with pytest.raises(fa.FAError) as e:
        fa.fa_schedule_items(cost, lists)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
