"""Pins of the decode-side oracle ("FASA: Frequency-aware Sparse Attention", §2)
against closed forms, torch routines, brute force and RoPE invariants."""

import itertools
import math

import numpy as np
import pytest
import torch

from oracle import fasa_oracle as fo


def _rope_torch(x, pos, base, d):
    """Rotate-half RoPE at integer positions ``pos`` through transformers' rotate_half (float64)."""
    from transformers.models.llama.modeling_llama import rotate_half
    theta = base ** (-2.0 * torch.arange(d // 2, dtype=torch.float64) / d)
    ang = torch.as_tensor(pos, dtype=torch.float64)[..., None] * theta
    c = torch.cat([ang.cos(), ang.cos()], -1)
    s = torch.cat([ang.sin(), ang.sin()], -1)
    x = torch.as_tensor(x, dtype=torch.float64)
    return x * c + rotate_half(x) * s


def _inputs(B=2, Hq=4, Hkv=2, L=40, d=16, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(B, Hq, d)), rng.normal(size=(B, Hkv, L, d)), rng.normal(size=(B, Hkv, L, d)))


def test_all_pairs_dominant_is_full_dot_product():
    q, K, _ = _inputs()
    d = q.shape[-1]
    fc = np.tile(np.arange(d // 2), (K.shape[1], 1))
    s = fo.tip_scores(q, K, fc)
    Kq = torch.repeat_interleave(torch.from_numpy(K), q.shape[1] // K.shape[1], dim=1)
    ref = torch.einsum("bhd,bhtd->bht", torch.from_numpy(q), Kq).numpy()
    np.testing.assert_allclose(s, ref, rtol=0, atol=1e-12)


def test_subset_score_is_sum_over_chosen_pairs_only():
    """Zeroing every dim outside the chosen pairs leaves the full dot product equal to the TIP score."""
    q, K, _ = _inputs(seed=1)
    d = q.shape[-1]
    fc = np.array([[1, 5, 6], [0, 2, 7]])
    s = fo.tip_scores(q, K, fc)
    group = q.shape[1] // K.shape[1]
    for h in range(q.shape[1]):
        g = h // group
        keep = np.zeros(d, dtype=bool)
        keep[fc[g]] = True
        keep[fc[g] + d // 2] = True
        qm = torch.from_numpy(np.where(keep, q[:, h], 0.0))
        ref = torch.einsum("bd,btd->bt", qm, torch.from_numpy(K[:, g])).numpy()
        np.testing.assert_allclose(s[:, h], ref, rtol=0, atol=1e-12)


def test_tip_scores_invariant_under_common_position_shift():
    """Each rotary pair's dot product depends on the position difference only, so any subset of
    pairs gives scores invariant under shifting the query and all keys by the same offset."""
    B, Hq, Hkv, L, d, base = 1, 2, 1, 24, 16, 1e4
    rng = np.random.default_rng(2)
    q0, K0 = rng.normal(size=(B, Hq, d)), rng.normal(size=(B, Hkv, L, d))
    fc = np.array([[0, 3, 6]])
    out = []
    for shift in (0, 37, 1000):
        pos_k = np.arange(L) + shift
        pos_q = np.full((B, Hq), L - 1 + shift)
        q = _rope_torch(q0, pos_q, base, d).numpy()
        K = _rope_torch(K0, pos_k, base, d).numpy()
        out.append(fo.tip_scores(q, K, fc))
    np.testing.assert_allclose(out[1], out[0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(out[2], out[0], rtol=0, atol=1e-10)
    # the invariance is a property of the true pairs: mixing dims across pairs breaks it
    bad = []
    for shift in (0, 37):
        pos_k = np.arange(L) + shift
        q = _rope_torch(q0, np.full((B, Hq), L - 1 + shift), base, d).numpy()
        K = _rope_torch(K0, pos_k, base, d).numpy()
        dims = np.array([0, 1])  # halves of two different pairs
        bad.append(np.einsum("bhd,btd->bht", q[..., dims], K[:, 0][..., dims]))
    assert np.abs(bad[1] - bad[0]).max() > 1e-3


def test_gather_fc_layout_gives_the_same_scores():
    q, K, _ = _inputs(seed=3)
    d = q.shape[-1]
    fc = np.array([[2, 4, 0, 7], [1, 3, 5, 6]])
    Kfc = fo.gather_fc(K, fc)
    assert Kfc.shape == K.shape[:3] + (8,)
    np.testing.assert_array_equal(Kfc[:, 1, :, 0], K[:, 1, :, 1])
    np.testing.assert_array_equal(Kfc[:, 1, :, 4], K[:, 1, :, 1 + d // 2])
    group = q.shape[1] // K.shape[1]
    for h in range(q.shape[1]):
        g = h // group
        qd = q[:, h][:, fo.fc_dims(fc[g], d)]
        np.testing.assert_allclose(np.einsum("bc,btc->bt", qd, Kfc[:, g]), fo.tip_scores(q, K, fc)[:, h],
                                   rtol=0, atol=1e-12)


def _dominates(a, ia, b, ib):
    return a > b or (a == b and ia < ib)


@pytest.mark.parametrize("seed", range(5))
def test_selection_matches_bruteforce(seed):
    rng = np.random.default_rng(seed)
    L = 9
    keys = (rng.integers(0, 5, size=L).astype(np.float32) - 2.0) / 4.0   # many exact ties, negatives
    for k in range(0, L + 2):
        got = fo.select_row(keys, k)
        n = min(k, L)
        found = [set(S) for S in itertools.combinations(range(L), n)
                 if all(_dominates(keys[a], a, keys[b], b) for a in S for b in set(range(L)) - set(S))]
        assert len(found) == 1
        assert set(got.tolist()) == found[0]
        assert list(got) == sorted(got)
        best = max(sum(float(keys[t]) for t in S) for S in itertools.combinations(range(L), n)) if n else 0.0
        assert sum(float(keys[t]) for t in got) == best
    idx = fo.select_tokens(keys[None, None], L + 3)
    assert list(idx[0, 0, :L]) == list(range(L)) and np.all(idx[0, 0, L:] == -1)


def test_all_tokens_kept_is_dense_single_query_attention():
    q, K, V = _inputs(seed=4)
    B, Hq, d = q.shape
    L = K.shape[2]
    idx = np.tile(np.arange(L), (B, Hq, 1))
    o, lse = fo.focused_attention(q, K, V, idx)
    group = Hq // K.shape[1]
    Kq = torch.repeat_interleave(torch.from_numpy(K), group, dim=1)
    Vq = torch.repeat_interleave(torch.from_numpy(V), group, dim=1)
    qt = torch.from_numpy(q)[:, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, Kq, Vq)[:, :, 0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    lse_ref = torch.logsumexp(torch.einsum("bhd,bhtd->bht", torch.from_numpy(q), Kq) / math.sqrt(d), -1)
    np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=0, atol=1e-12)


def test_single_kept_token_returns_its_value():
    q, K, V = _inputs(seed=5)
    B, Hq, d = q.shape
    idx = -np.ones((B, Hq, 3), dtype=np.int64)
    idx[..., 0] = 7
    o, lse = fo.focused_attention(q, K, V, idx, scale=0.3)
    group = Hq // K.shape[1]
    for h in range(Hq):
        np.testing.assert_array_equal(o[:, h], V[:, h // group, 7])
        np.testing.assert_allclose(lse[:, h], 0.3 * np.einsum("bd,bd->b", q[:, h], K[:, h // group, 7]),
                                   rtol=0, atol=1e-12)
    # no kept token: zero output, lse = -inf
    o0, lse0 = fo.focused_attention(q, K, V, -np.ones((B, Hq, 2), dtype=np.int64))
    assert np.all(o0 == 0) and np.all(np.isneginf(lse0))


def test_decode_step_top1_picks_planted_key():
    """A key equal to a large multiple of the query in the dominant pairs wins the TIP, and FAC over
    that single token returns its value."""
    q, K, V = _inputs(B=1, Hq=2, Hkv=1, L=30, d=16, seed=6)
    fc = np.array([[1, 4]])
    d = 16
    dims = fo.fc_dims(fc[0], d)
    K[0, 0, 11, dims] = 50.0 * q[0, 0, dims]
    _, idx, o, _ = fo.decode_step(q, K, V, fc, 1)
    assert idx[0, 0, 0] == 11
    np.testing.assert_array_equal(o[0, 0], V[0, 0, 11])


def test_ranked_float32_score_is_within_the_recursive_summation_bound():
    """|fl32 running sum - exact sum| <= (n u / (1 - n u)) sum |q_c k_c| with u = 2**-24, n = 2 nfc
    terms (products exact for bf16 inputs); and an all-dyadic case where the float32 sum is exact."""
    q, K, _ = _inputs(seed=8)
    qb = torch.from_numpy(q).to(torch.bfloat16).to(torch.float64).numpy()
    Kb = torch.from_numpy(K).to(torch.bfloat16).to(torch.float64).numpy()
    fc = np.array([[1, 5, 6, 7], [0, 2, 3, 4]])
    keys = fo.tip_keys(qb, Kb, fc).astype(np.float64)
    exact = fo.tip_scores(qb, Kb, fc)
    n, u = 8, 2.0 ** -24
    group = q.shape[1] // K.shape[1]
    for h in range(q.shape[1]):
        dims = fo.fc_dims(fc[h // group], q.shape[-1])
        mag = np.einsum("bd,btd->bt", np.abs(qb[:, h][:, dims]), np.abs(Kb[:, h // group][..., dims]))
        assert np.all(np.abs(keys[:, h] - exact[:, h]) <= n * u / (1 - n * u) * mag)
    qi = np.round(q * 4) / 4
    Ki = np.round(K * 4) / 4
    np.testing.assert_array_equal(fo.tip_keys(qi, Ki, fc).astype(np.float64), fo.tip_scores(qi, Ki, fc))


def test_float32_diagnostic_is_the_left_to_right_sum():
    """The float32 diagnostic (not ranked): products 2^24, 1, -2^24 in column order give 2^24 + 1 ->
    2^24 (ties to even), then 0, where the exact sum is 1; with the cancellation first it is exact."""
    d = 16
    fc = np.array([[0, 1, 2, 3]])          # columns: dims 0, 1, 2, 3, then 8, 9, 10, 11
    q = np.zeros((1, 1, d))
    K = np.zeros((1, 1, 1, d))
    q[0, 0, [0, 1, 2]] = 1.0
    K[0, 0, 0, [0, 1, 2]] = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    assert fo.tip_scores(q, K, fc)[0, 0, 0] == 1.0
    assert fo.tip_keys(q, K, fc)[0, 0, 0] == 0.0
    K[0, 0, 0, [0, 1, 2]] = [1.0, 2.0 ** 24, -(2.0 ** 24)]   # 1 + 2^24 -> 2^24 as well
    assert fo.tip_keys(q, K, fc)[0, 0, 0] == 0.0
    K[0, 0, 0, [0, 1, 2]] = [2.0 ** 24, -(2.0 ** 24), 1.0]   # cancellation first: exact
    assert fo.tip_keys(q, K, fc)[0, 0, 0] == 1.0


def test_ranked_score_is_the_exact_dot_product():
    """The selection ranks the dot product itself, not a float32 running sum: token 0's products
    2^24, 1, -2^24 sum to 1 (a float32 column-order sum gives 0), token 1's to 1/2, token 2's to
    -1; top-1 is token 0 and top-2 is {0, 1}."""
    d = 16
    fc = np.array([[0, 1, 2, 3]])
    q = np.zeros((1, 1, d))
    q[0, 0, [0, 1, 2]] = 1.0
    K = np.zeros((1, 1, 3, d))
    V = np.arange(3 * d, dtype=np.float64).reshape(1, 1, 3, d)
    K[0, 0, 0, [0, 1, 2]] = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    K[0, 0, 1, 1] = 0.5
    K[0, 0, 2, 0] = -1.0
    s, idx, o, _ = fo.decode_step(q, K, V, fc, 1)
    np.testing.assert_array_equal(s[0, 0], [1.0, 0.5, -1.0])
    assert idx[0, 0].tolist() == [0]
    np.testing.assert_array_equal(o[0, 0], V[0, 0, 0])
    assert fo.decode_step(q, K, V, fc, 2)[1][0, 0].tolist() == [0, 1]


def test_scores_of_bf16_inputs_equal_the_exact_rational_sum():
    """bf16 x bf16 products and their sum over a few dozen columns are exact in float64 when the
    magnitudes stay within a few binades: the float64 score equals the exact rational dot product
    (fractions), so the ranked value carries no summation-order rounding."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    d, L = 32, 25
    q = torch.from_numpy(rng.normal(size=(1, 2, d))).to(torch.bfloat16).double().numpy()
    K = torch.from_numpy(rng.uniform(0.25, 4.0, size=(1, 1, L, d)) * rng.choice([-1, 1], size=(1, 1, L, d))
                         ).to(torch.bfloat16).double().numpy()
    q = np.where(np.abs(q) < 0.25, 0.25, q)                  # keep every product within 2^-4 .. 2^4
    fc = np.array([[0, 3, 5, 6, 9, 12, 14, 15]])
    s = fo.tip_scores(q, K, fc)
    dims = fo.fc_dims(fc[0], d)
    for h in range(2):
        for t in range(L):
            exact = sum(Fraction(float(q[0, h, c])) * Fraction(float(K[0, 0, t, c])) for c in dims)
            assert s[0, h, t] == float(exact)


def test_power_of_two_query_scaling_scales_the_keys_exactly():
    """Scaling q by 2^e scales every float32 product and partial sum by 2^e exactly (no overflow or
    underflow here), so the ranked keys scale exactly and the kept tokens do not change; negating q
    reverses the ranking of distinct keys."""
    q, K, _ = _inputs(seed=9)
    fc = np.array([[1, 5, 6, 7], [0, 2, 3, 4]])
    k = 5
    base = fo.tip_keys(q, K, fc)
    for e in (-3, 1, 4):
        scaled = fo.tip_keys(q * 2.0 ** e, K, fc)
        np.testing.assert_array_equal(scaled, base * np.float32(2.0 ** e))
        np.testing.assert_array_equal(fo.select_tokens(scaled, k), fo.select_tokens(base, k))
    neg = fo.tip_keys(-q, K, fc)
    np.testing.assert_array_equal(neg, -base)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            row = base[b, h].astype(np.float64)
            if np.unique(row).size == row.size:
                lowest = np.sort(np.argsort(row, kind="stable")[:k])
                np.testing.assert_array_equal(fo.select_row(neg[b, h], k), lowest)
