"""A host model of the decode selection strategy (chunked bound -> candidates -> exact merge),
checked against the oracle's top-k on adversarial key distributions.

The kernels split the cache into chunks; per chunk and head they take a lower bound LB of the
chunk's k-th largest key (any value with at least k of the chunk's 4-key group maxima at or above
it; the bisection may stop early, so any such value is allowed), keep the tokens with key >= LB in
token order, and a merge picks the first k of the candidates by (key desc, index asc).  This model
checks that the strategy never drops a token of the exact top k, for exact and deliberately loose
bounds, including the distributions that send every token to the merge (identical keys).  The
merge's own bound (the least of its threads' candidate maxima) is modelled too, with 256 threads as
in the kernel and with 8 so that it cuts deep."""

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


def model_merge(keys, cand, k, threads=256):
    """The merge: with k <= threads, the least of the threads' maxima (thread t holds candidates
    t, t + threads, ...; a thread without one contributes 0, below every key) bounds the k-th largest
    from below, so only candidates at or above it go on to the exact selection; then the first k by
    (key desc, index asc), output ascending."""
    if k < len(cand) and k <= threads:
        lb2 = min(max((int(keys[c]) for c in cand[t::threads]), default=0) for t in range(threads))
        cand = [c for c in cand if keys[c] >= lb2]
    order = sorted(cand, key=lambda t: (-int(keys[t]), t))
    return np.sort(np.asarray(order[:k], dtype=np.int64))


def model_select(keys, k, chunk, loose=False, threads=256):
    cand = []
    for c0 in range(0, keys.size, chunk):
        kc = keys[c0:c0 + chunk]
        bounds = _valid_bounds(kc, k)
        lb = bounds[-1] if loose else bounds[0]
        cand += [c0 + i for i in range(kc.size) if kc[i] >= lb]
    return model_merge(keys, cand, k, threads), len(cand)


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
        for threads in (256, 8):   # 8 threads: the merge's own bound cuts deep into the candidates
            got, ncand = model_select(keys, k, chunk, loose, threads)
            np.testing.assert_array_equal(got, want)
            assert ncand >= min(k, n)
    if dist == "identical":
        # every token ties with every bound: all of them reach the merge
        assert model_select(keys, k, chunk)[1] == n
