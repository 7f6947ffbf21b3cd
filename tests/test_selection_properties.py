"""Property-based checks (hypothesis) of both oracles' selection rules against brute force on
random tiny rows with many exact ties: the kept set is the unique subset of the right size that
dominates every dropped candidate in (value desc, index asc) order."""

import itertools

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import fasa_oracle as fo
from oracle import prism_oracle as po


def _dominates(a, ia, b, ib):
    return a > b or (a == b and ia < ib)


def _brute(vals, cand, n):
    found = [set(S) for S in itertools.combinations(cand, n)
             if all(_dominates(vals[a], a, vals[b], b) for a in S for b in set(cand) - set(S))]
    assert len(found) == 1
    return found[0]


@settings(max_examples=150, deadline=None)
@given(st.lists(st.integers(0, 4), min_size=1, max_size=9), st.integers(0, 10), st.booleans())
def test_prism_topk_selection(levels, k, sink):
    nb = len(levels)
    p = np.array(levels, dtype=np.float64) / 16.0
    i = nb - 1
    flags = po.FLAG_KEEP_SINK if sink else 0
    r = po.select_row(p, i, flags, k=k)
    forced = {0, i} if sink else {i}
    cand = [j for j in range(i + 1) if j not in forced]
    want = _brute(p, cand, min(k, len(cand))) | forced
    assert set(r.kept.tolist()) == want
    assert list(r.kept) == sorted(r.kept)


@settings(max_examples=150, deadline=None)
@given(st.lists(st.integers(0, 4), min_size=1, max_size=9), st.integers(1, 64))
def test_prism_mass_selection(levels, m):
    nb = len(levels)
    p = np.array(levels, dtype=np.float64) / 16.0   # dyadic: every partial sum is exact
    mass = m / 64.0
    i = nb - 1
    r = po.select_row(p, i, 0, mass=mass)
    cand = [j for j in range(i + 1) if j != i]
    base = p[i]
    # the smallest n whose dominant prefix reaches the mass (all candidates if none does)
    order = sorted(cand, key=lambda j: (-p[j], j))
    n = len(order)
    for t in range(len(order) + 1):
        if base + sum(p[j] for j in order[:t]) >= mass:
            n = t
            break
    assert set(r.kept.tolist()) == set(order[:n]) | {i}


@settings(max_examples=150, deadline=None)
@given(st.lists(st.integers(-3, 3), min_size=1, max_size=9), st.integers(1, 11))
def test_fasa_topk_selection(levels, k):
    keys = np.array(levels, dtype=np.float32) / 4.0
    got = fo.select_row(keys, k)
    want = _brute(keys, list(range(keys.size)), min(k, keys.size))
    assert set(got.tolist()) == want
    assert list(got) == sorted(got)
