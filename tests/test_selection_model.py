"""A host model of the decode selection strategy (chunked bound -> candidates -> exact merge),
checked against the oracle's top-k on adversarial key distributions.

The kernels split the cache into chunks; per chunk and head they take a lower bound LB of the
chunk's k-th largest key (any value with at least k of the chunk's 4-key group maxima at or above
it; the bisection may stop early, so any such value is allowed), keep the tokens with key >= LB in
token order, and a merge picks the first k of the candidates by (key desc, index asc).  This model
checks that the strategy never drops a token of the exact top k, for exact and deliberately loose
bounds, including the distributions that send every token to the merge (identical keys)."""

import numpy as np
import pytest

from oracle import fasa_oracle as fo


def _valid_bounds(keys, k):
    """The exact bound (k-th largest group maximum) and a looser valid one (halfway to the minimum)."""
    gm = np.array([keys[g:g + 4].max() for g in range(0, keys.size, 4)])
    if gm.size < k:
        return [keys.min()]
    exact = np.sort(gm)[::-1][k - 1]
    loose = gm.min() + (exact - gm.min()) // 2
    assert (gm >= loose).sum() >= k
    return [exact, loose]


def model_select(keys, k, chunk, loose=False):
    cand = []
    for c0 in range(0, keys.size, chunk):
        kc = keys[c0:c0 + chunk]
        bounds = _valid_bounds(kc, k)
        lb = bounds[-1] if loose else bounds[0]
        cand += [c0 + i for i in range(kc.size) if kc[i] >= lb]
    # merge: first k of the candidates by (key desc, index asc), output ascending
    order = sorted(cand, key=lambda t: (-int(keys[t]), t))
    return np.sort(np.asarray(order[:k], dtype=np.int64)), len(cand)


def _as_float_keys(u):
    """Order-preserving map of uint keys back to float32 scores, for the oracle's ranking."""
    return u.astype(np.float64).astype(np.float32)


DISTS = {
    "random": lambda rng, n: rng.integers(0, 1 << 20, n),
    "identical": lambda rng, n: np.full(n, 7),
    "two-values": lambda rng, n: rng.integers(0, 2, n),
    "ascending": lambda rng, n: np.arange(n),
    "descending": lambda rng, n: np.arange(n)[::-1].copy(),
    "plateau-top": lambda rng, n: np.where(rng.random(n) < 0.1, 1000, rng.integers(0, 1000, n)),
    "needles": lambda rng, n: np.where(rng.random(n) < 0.01, 5000 + rng.integers(0, 3, n), rng.integers(0, 50, n)),
}


@pytest.mark.parametrize("dist", sorted(DISTS))
@pytest.mark.parametrize("k,chunk,n", [(5, 32, 301), (16, 64, 1000), (40, 64, 700), (1, 16, 37), (300, 64, 250)])
def test_chunked_bound_never_drops_a_top_k_token(dist, k, chunk, n):
    rng = np.random.default_rng(k * 1000 + n)
    keys = DISTS[dist](rng, n).astype(np.int64)
    want = fo.select_row(_as_float_keys(keys), k)
    for loose in (False, True):
        got, ncand = model_select(keys, k, chunk, loose)
        np.testing.assert_array_equal(got, want)
        assert ncand >= min(k, n)
    if dist == "identical":
        # every token ties with every bound: all of them reach the merge
        assert model_select(keys, k, chunk)[1] == n
