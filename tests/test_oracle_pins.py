"""Pins of the CPU oracle against things other than itself.

Each test ties one step of the oracle to a closed form, a library routine, a
brute-force search or an invariant of "Prism: Spectral-Aware Block-Sparse
Attention", so that a dropped term, a wrong sign, a wrong index or a
transposed operand in the oracle fails at least one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dirichlet_factors.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            base, d, m, beta, theta, D = line.split()
            rows.append((float(base), int(d), int(m), int(beta), float(theta), float(D)))
    return rows


# ---------------------------------------------------------------------------
# §2: amplitude collapse of mean pooling under RoPE (closed-form Dirichlet factor)
# ---------------------------------------------------------------------------
def test_golden_file_is_what_its_generator_writes():
    """The stored Dirichlet factors come from tests/golden/make_golden.py (closed form, standard
    library only) and nothing else has edited them."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(os.path.dirname(GOLDEN),
                                                                              "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(GOLDEN) as f:
        assert f.read() == mod.render()


@pytest.mark.parametrize("row", _golden_rows())
def test_pooled_pair_amplitude_is_dirichlet_factor(row):
    base, d, m, beta, theta, D = row
    L = 4 * beta
    cos, sin = po.rope_tables(base, L, d)
    x = np.zeros((L, d))
    x[:, m] = 1.0                       # constant pair (1, 0) rotated at theta_m
    xr = po.apply_rope(x, cos, sin)
    xbar = po.pool_blocks(xr, beta)
    amp = np.hypot(xbar[:, m], xbar[:, m + d // 2])
    # every block keeps the same amplitude (a block offset only rotates the mean)
    np.testing.assert_allclose(amp, D, rtol=0, atol=3e-6)
    # and the oracle's frequency formula gives the golden theta
    assert po.rope_frequencies(base, d)[m] == pytest.approx(theta, rel=1e-15)


def test_retained_amplitude_closed_form_multi_pair():
    base, d, beta, L, bs = 1e4, 32, 16, 128, 5
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(7)
    vec = rng.normal(size=d)
    xr = po.apply_rope(np.broadcast_to(vec, (L, d)).copy(), cos, sin)
    xbar = po.pool_blocks(xr, beta)
    theta = po.rope_frequencies(base, d)
    Dm = np.abs(np.sin(beta * theta / 2)) / (beta * np.abs(np.sin(theta / 2)))
    pair_e = vec[: d // 2] ** 2 + vec[d // 2:] ** 2
    high, low = po.band_masks(d, bs)
    for band, pairs in ((high, np.arange(bs)), (low, np.arange(bs, d // 2))):
        expect = math.sqrt((pair_e[pairs] * Dm[pairs] ** 2).sum() / pair_e[pairs].sum())
        got = po.retained_amplitude(xr, xbar, band)
        assert got == pytest.approx(expect, rel=2e-6)


# ---------------------------------------------------------------------------
# §3.2: the energy temperature undoes the pooling attenuation exactly for a
# single rotary pair: calibrated block logit == token logit at block starts.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("beta,rtol", [(8, 2e-6), (16, 2e-5)])
def test_single_pair_calibration_identity(beta, rtol):
    d, L, base = 16, 8 * beta, 1e4
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(3)
    q = np.zeros(d)
    k = np.zeros(d)
    q[[0, d // 2]] = rng.normal(size=2)
    k[[0, d // 2]] = rng.normal(size=2)
    Q = np.broadcast_to(q, (1, 1, L, d)).copy()
    K = np.broadcast_to(k, (1, 1, L, d)).copy()
    sc = po.prism_scores(Q, K, beta, band_split=1, flags=0, rope=(cos, sin))
    qr = po.apply_rope(Q, cos, sin)[0, 0]
    kr = po.apply_rope(K, cos, sin)[0, 0]
    nb = L // beta
    tok = np.array([[qr[i * beta] @ kr[j * beta] for j in range(nb)] for i in range(nb)]) / math.sqrt(d)
    scale = np.abs(q).max() * np.abs(k).max() * 2 / math.sqrt(d)
    np.testing.assert_allclose(sc.logits[0, 0], tok, rtol=0, atol=rtol * scale * 10)
    # the same logits without calibration are attenuated by D^2
    raw = po.prism_scores(Q, K, beta, band_split=1, flags=po.FLAG_NO_CALIB, rope=(cos, sin))
    D = abs(math.sin(beta / 2)) / (beta * abs(math.sin(0.5)))
    np.testing.assert_allclose(raw.logits[0, 0], tok * D * D, rtol=0, atol=rtol * scale * 10)
    assert sc.tau[0, 0, 0] == pytest.approx(D * D, rel=1e-5)


def test_tau_is_product_of_q_and_k_ratios_gqa():
    base, d, beta, L, bs = 1e4, 16, 8, 64, 3
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(11)
    qv = rng.normal(size=(1, 4, 1, d))
    kv = rng.normal(size=(1, 2, 1, d))
    Q = np.broadcast_to(qv, (1, 4, L, d)).copy()
    K = np.broadcast_to(kv, (1, 2, L, d)).copy()
    sc = po.prism_scores(Q, K, beta, bs, 0, (cos, sin))
    theta = po.rope_frequencies(base, d)
    Dm = np.abs(np.sin(beta * theta / 2)) / (beta * np.abs(np.sin(theta / 2)))

    def rho(v, pairs):
        e = v[pairs] ** 2 + v[pairs + d // 2] ** 2
        return math.sqrt((e * Dm[pairs] ** 2).sum() / e.sum())

    for h in range(4):
        g = h // 2
        for bi, pairs in enumerate((np.arange(bs), np.arange(bs, d // 2))):
            expect = rho(qv[0, h, 0], pairs) * rho(kv[0, g, 0], pairs)
            assert sc.tau[0, h, bi] == pytest.approx(expect, rel=5e-6)


# ---------------------------------------------------------------------------
# RoPE convention against the transformers Llama rotary routine.
# ---------------------------------------------------------------------------
def test_rope_matches_transformers_llama_rotary():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    L, d = 37, 16
    cos, sin = po.rope_tables(5e5, L, d)
    rng = np.random.default_rng(0)
    q = rng.normal(size=(1, 2, L, d))
    k = rng.normal(size=(1, 1, L, d))
    c = torch.from_numpy(np.concatenate([cos, cos], -1).astype(np.float64))[None]
    s = torch.from_numpy(np.concatenate([sin, sin], -1).astype(np.float64))[None]
    qe, ke = apply_rotary_pos_emb(torch.from_numpy(q), torch.from_numpy(k), c, s)
    np.testing.assert_allclose(po.apply_rope(q, cos, sin), qe.numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(po.apply_rope(k, cos, sin), ke.numpy(), rtol=0, atol=1e-14)


def test_rope_invariants():
    L, d = 300, 32
    cos, sin = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(1)
    x = rng.normal(size=(L, d))
    xr = po.apply_rope(x, cos, sin)
    np.testing.assert_array_equal(xr[0], x[0])                 # position 0 is the identity
    n0 = x[:, : d // 2] ** 2 + x[:, d // 2:] ** 2
    n1 = xr[:, : d // 2] ** 2 + xr[:, d // 2:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=3e-7)              # pair norms kept (fp32 table)
    q = np.broadcast_to(rng.normal(size=d), (L, d)).copy()
    k = np.broadcast_to(rng.normal(size=d), (L, d)).copy()
    qr = po.apply_rope(q, cos, sin)
    kr = po.apply_rope(k, cos, sin)
    for a, b, delta in [(5, 2, 100), (40, 40, 17), (10, 90, 150)]:
        assert qr[a] @ kr[b] == pytest.approx(qr[a + delta] @ kr[b + delta], abs=2e-5)
    # energies per band are the same before and after rotation
    e_pre = po.block_token_energy(x[None], 10, 5, 0)
    e_post = po.block_token_energy(xr[None], 10, 5, 0)
    np.testing.assert_allclose(e_post, e_pre, rtol=3e-7)


# ---------------------------------------------------------------------------
# Block size 1: pooling is the identity, tau == 1, probabilities are the
# token-level causal softmax (computed here with torch's rotary + softmax).
# ---------------------------------------------------------------------------
def _torch_rotate(x, cos, sin):
    from transformers.models.llama.modeling_llama import rotate_half
    c = torch.from_numpy(np.concatenate([cos, cos], -1).astype(np.float64))
    s = torch.from_numpy(np.concatenate([sin, sin], -1).astype(np.float64))
    t = torch.from_numpy(np.asarray(x, dtype=np.float64))
    return t * c + rotate_half(t) * s


def test_block_one_equals_token_causal_softmax():
    B, Hq, Hkv, L, d = 2, 4, 2, 12, 8
    cos, sin = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(5)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    sc = po.prism_scores(Q, K, 1, 2, 0, (cos, sin))
    np.testing.assert_allclose(sc.tau, 1.0, rtol=1e-12)
    qt = _torch_rotate(Q, cos, sin)
    kt = torch.repeat_interleave(_torch_rotate(K, cos, sin), Hq // Hkv, dim=1)
    logits = qt @ kt.transpose(-1, -2) / math.sqrt(d)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    ref = torch.softmax(logits.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(sc.probs, ref.numpy(), rtol=0, atol=1e-12)


def test_no_calib_is_plain_mean_pool_matmul():
    B, Hq, Hkv, L, d, beta = 1, 4, 1, 96, 16, 8
    cos, sin = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(9)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    sc = po.prism_scores(Q, K, beta, 4, po.FLAG_NO_CALIB, (cos, sin))
    pool = torch.nn.functional.avg_pool1d
    qt = _torch_rotate(Q, cos, sin).reshape(B * Hq, L, d).transpose(1, 2)
    kt = _torch_rotate(K, cos, sin).reshape(B * Hkv, L, d).transpose(1, 2)
    qb = pool(qt, beta).transpose(1, 2).reshape(B, Hq, L // beta, d)
    kb = pool(kt, beta).transpose(1, 2).reshape(B, Hkv, L // beta, d)
    kb = torch.repeat_interleave(kb, Hq // Hkv, dim=1)
    s = qb @ kb.transpose(-1, -2) / math.sqrt(d)
    nb = L // beta
    mask = torch.ones(nb, nb, dtype=torch.bool).tril()
    ref = torch.softmax(s.masked_fill(~mask, float("-inf")), -1)
    np.testing.assert_allclose(sc.qbar, qb.numpy(), rtol=0, atol=1e-13)
    np.testing.assert_allclose(sc.probs, ref.numpy(), rtol=0, atol=1e-12)


def test_estimate_scale_invariances():
    """R4/R5: rho is a ratio of energies, so scaling Q (or K) by c leaves tau unchanged and scales
    every calibrated block logit by c."""
    B, Hq, Hkv, L, d, beta = 1, 2, 1, 96, 16, 8
    rope = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(18)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    for flags in (0, po.FLAG_RELATIVE_CALIB, po.FLAG_SINGLE_BAND):
        a = po.prism_scores(Q, K, beta, 3, flags, rope)
        b = po.prism_scores(2.5 * Q, K, beta, 3, flags, rope)
        c = po.prism_scores(Q, -0.75 * K, beta, 3, flags, rope)
        np.testing.assert_allclose(b.tau, a.tau, rtol=1e-12)
        np.testing.assert_allclose(c.tau, a.tau, rtol=1e-12)
        np.testing.assert_allclose(b.logits, 2.5 * a.logits, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(c.logits, -0.75 * a.logits, rtol=1e-10, atol=1e-12)


def test_rows_see_later_key_blocks_only_through_tau():
    """R5/R6: row i's probabilities use key blocks j <= i; later keys enter only through the
    sequence-wide temperature (reading R4), so with tau held fixed (or SFA_NO_CALIB) the first rows
    do not change when the later key blocks do."""
    B, Hq, Hkv, L, d, beta, bs = 1, 2, 1, 96, 16, 8, 3
    rope = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(19)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    K2 = K.copy()
    i = 5
    K2[:, :, (i + 1) * beta:] = 3.0 * rng.normal(size=K2[:, :, (i + 1) * beta:].shape)
    a = po.prism_scores(Q, K, beta, bs, po.FLAG_NO_CALIB, rope)
    b = po.prism_scores(Q, K2, beta, bs, po.FLAG_NO_CALIB, rope)
    np.testing.assert_array_equal(b.probs[..., :i + 1, :], a.probs[..., :i + 1, :])
    a = po.prism_scores(Q, K, beta, bs, 0, rope)
    b = po.prism_scores(Q, K2, beta, bs, 0, rope)
    assert not np.allclose(b.tau, a.tau)                  # the temperature is sequence-wide
    s_fixed = po.block_logits(b.qbar, b.kbar, a.tau, bs, 0, Hq // Hkv)
    np.testing.assert_array_equal(po.causal_block_softmax(s_fixed)[..., :i + 1, :], a.probs[..., :i + 1, :])


def test_band_bookkeeping_equivalences():
    B, Hq, Hkv, L, d, beta = 1, 2, 1, 64, 16, 8
    cos, sin = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(2)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    single = po.prism_scores(Q, K, beta, 3, po.FLAG_SINGLE_BAND, (cos, sin))
    all_low = po.prism_scores(Q, K, beta, 0, 0, (cos, sin))      # band H empty
    all_high = po.prism_scores(Q, K, beta, d // 2, 0, (cos, sin))  # band L empty
    np.testing.assert_allclose(all_low.probs, single.probs, rtol=0, atol=1e-13)
    np.testing.assert_allclose(all_high.probs, single.probs, rtol=0, atol=1e-13)
    # a real split differs from the single band (the two temperatures differ)
    split = po.prism_scores(Q, K, beta, 3, 0, (cos, sin))
    assert not np.allclose(split.tau[..., 0], split.tau[..., 1])
    assert np.abs(split.probs - single.probs).max() > 1e-6
    # high-band dims are pairs m < bs and their partners m + d/2
    hm = po.high_band_mask(d, 3)
    assert list(np.nonzero(hm)[0]) == [0, 1, 2, 8, 9, 10]


# ---------------------------------------------------------------------------
# Selection: brute force over subsets on tiny rows.
# ---------------------------------------------------------------------------
def _dominates(pa, a, pb, b):
    return pa > pb or (pa == pb and a < b)


def _brute_topk(p, cand, n):
    found = []
    for S in itertools.combinations(cand, n):
        rest = [c for c in cand if c not in S]
        if all(_dominates(p[a], a, p[b], b) for a in S for b in rest):
            found.append(set(S))
    assert len(found) == 1
    best = max(sum(p[j] for j in S) for S in itertools.combinations(cand, n)) if n else 0.0
    assert sum(p[j] for j in found[0]) == best
    return found[0]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("flags", [0, po.FLAG_KEEP_SINK])
def test_selection_matches_bruteforce(seed, flags):
    rng = np.random.default_rng(seed)
    nb = 9
    # dyadic values with many exact ties: sums are exact in float64
    P = rng.integers(0, 6, size=(nb, nb)).astype(np.float64) / 64.0
    for i in range(nb):
        # reading R7: the diagonal is always kept, and block 0 too with KEEP_SINK
        forced = (0, i) if (flags & po.FLAG_KEEP_SINK) and i > 0 else (i,)
        assert set(po.forced_blocks(i, flags)) == set(forced)
        cand = [j for j in range(i + 1) if j not in forced]
        for k in range(0, nb + 1):
            r = po.select_row(P[i], i, flags, k=k)
            S = _brute_topk(P[i], cand, min(k, len(cand)))
            assert set(r.kept.tolist()) == S | set(forced)
            assert list(r.kept) == sorted(r.kept)
        for mass in (0.0, 3 / 64, 0.25, 0.5, 0.9, 1.0, 5.0):
            r = po.select_row(P[i], i, flags, mass=mass)
            base = sum(P[i][j] for j in forced)
            n_need = len(cand)
            for n in range(len(cand) + 1):
                best = max(sum(P[i][j] for j in S) for S in itertools.combinations(cand, n)) if n else 0.0
                if base + best >= mass:
                    n_need = n
                    break
            S = _brute_topk(P[i], cand, n_need)
            assert r.n_taken == n_need
            assert set(r.kept.tolist()) == S | set(forced)


def test_selection_invariants_on_softmax_rows():
    rng = np.random.default_rng(4)
    nb = 20
    s = rng.normal(size=(1, 1, nb, nb)) * 3
    p = po.causal_block_softmax(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-12)
    assert np.all(np.triu(p[0, 0], 1) == 0)
    for flags in (0, po.FLAG_KEEP_SINK):
        sel0 = po.select_blocks(p, flags, k=0)
        all1 = po.select_blocks(p, flags, mass=1.0)
        for i in range(nb):
            forced = {0, i} if flags & po.FLAG_KEEP_SINK else {i}
            assert set(sel0[0][0][i].kept.tolist()) == forced
            assert list(all1[0][0][i].kept) == list(range(i + 1))
            for kk in (1, 3, 50):
                r = po.select_row(p[0, 0, i], i, flags, k=kk)
                assert i in r.kept
                assert len(r.kept) == min(i + 1, kk + len(forced))


# ---------------------------------------------------------------------------
# Attention: exact over kept blocks (§1) against torch SDPA and brute force.
# ---------------------------------------------------------------------------
def _sdpa(Q, K, V, causal):
    group = Q.shape[1] // K.shape[1]
    k = torch.repeat_interleave(torch.from_numpy(K), group, dim=1)
    v = torch.repeat_interleave(torch.from_numpy(V), group, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), k, v, is_causal=causal).numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_all_blocks_kept_equals_dense_attention(causal):
    B, Hq, Hkv, L, d, beta = 1, 4, 2, 64, 8, 16
    rng = np.random.default_rng(6)
    Q, K, V = (rng.normal(size=(B, h, L, d)) for h in (Hq, Hkv, Hkv))
    nb = L // beta
    kept = [[[np.arange(nb if not causal else i + 1) for i in range(nb)] for _ in range(Hq)]
            for _ in range(B)]
    O, lse = po.sparse_attention(Q, K, V, kept, beta, causal=causal)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, causal), rtol=0, atol=1e-12)
    if causal:
        np.testing.assert_allclose(O, po.dense_causal_attention_bruteforce(Q, K, V), rtol=0, atol=1e-12)
    from scipy.special import logsumexp
    g = Hq // Hkv
    for h in range(Hq):
        s = Q[0, h] @ K[0, h // g].T / math.sqrt(d)
        if causal:
            s = np.where(np.tril(np.ones((L, L), bool)), s, -np.inf)
        np.testing.assert_allclose(lse[0, h], logsumexp(s, axis=1), rtol=0, atol=1e-12)


def test_diagonal_only_is_blockwise_local_attention():
    B, Hq, Hkv, L, d, beta = 1, 2, 1, 48, 8, 16
    rng = np.random.default_rng(8)
    Q, K, V = (rng.normal(size=(B, h, L, d)) for h in (Hq, Hkv, Hkv))
    nb = L // beta
    kept = [[[np.array([i]) for i in range(nb)] for _ in range(Hq)]]
    O, _ = po.sparse_attention(Q, K, V, kept, beta)
    for i in range(nb):
        sl = slice(i * beta, (i + 1) * beta)
        ref = po.dense_causal_attention_bruteforce(Q[:, :, sl], K[:, :, sl], V[:, :, sl])
        np.testing.assert_allclose(O[:, :, sl], ref, rtol=0, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(10)
    Q, K, V = (rng.normal(size=(1, 1, 1, 4)) for _ in range(3))
    O, lse = po.sparse_attention(Q, K, V, [[[np.array([0])]]], 1)
    np.testing.assert_allclose(O[0, 0, 0], V[0, 0, 0], rtol=0, atol=0)   # a single key: o = v0
    Q, K, V = (rng.normal(size=(1, 1, 8, 4)) for _ in range(3))
    O, lse = po.sparse_attention(Q, K, V, [[[np.array([], dtype=np.int64), np.array([0, 1])]]], 4)
    assert np.all(O[0, 0, :4] == 0) and np.all(np.isneginf(lse[0, 0, :4]))
    np.testing.assert_allclose(O[0, 0, 0 + 4 * 0], 0.0)
    O2, _ = po.sparse_attention(Q, K, V, [[[np.array([0]), np.array([0, 1])]]], 4)
    np.testing.assert_allclose(O2[0, 0, 0], V[0, 0, 0], atol=1e-15)       # first token sees itself


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    x = (rng.normal(size=100000) * np.exp(rng.normal(size=100000) * 4)).astype(np.float32)
    ours = po.round_to_bf16(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_tiny_path_structure():
    from block_sparse_long_dual_b200.workloads import TINY
    from block_sparse_long_dual_b200.synthetic import make_inputs
    w = TINY.scaled(seq_len=512)
    Q, K, V = (t.numpy() for t in make_inputs(w))
    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    r = po.prism_path(Q, K, V, block=w.block, band_split=w.band_split, flags=w.flags, k=w.k,
                      rope=(cos, sin), dtype="f32")
    nb = w.nb
    for i in range(nb):
        kept = r.selection[0][0][i].kept
        assert i in kept and (i == 0 or 0 in kept)
        assert len(kept) == min(i + 1, w.k + (2 if i else 1))
    assert np.all(np.isfinite(r.out))


def test_f32_rounding_matches_torch():
    rng = np.random.default_rng(13)
    x = rng.normal(size=20000) * np.exp(rng.normal(size=20000) * 4)
    ref = torch.from_numpy(x).to(torch.float32).to(torch.float64).numpy()
    np.testing.assert_array_equal(po.round_to_dtype(x, "f32"), ref)


def test_rope_tables_are_float32_roundings_of_the_exact_angles():
    """R1: the tables hold cos/sin of the float64 angle, each rounded once to float32 (checked
    against the standard library's cos/sin at a sample of entries, to half a float32 ulp)."""
    base, L, d = 5e5, 4096, 128
    cos, sin = po.rope_tables(base, L, d)
    assert cos.dtype == np.float32 and sin.dtype == np.float32 and cos.shape == (L, d // 2)
    rng = np.random.default_rng(14)
    for p, m in zip(rng.integers(0, L, 200), rng.integers(0, d // 2, 200)):
        ang = float(p) * base ** (-2.0 * float(m) / d)
        for table, exact in ((cos, math.cos(ang)), (sin, math.sin(ang))):
            v = float(table[p, m])
            assert abs(v - exact) <= 0.5 * float(np.spacing(np.float32(abs(v)))) * (1 + 1e-9)


def test_selection_arrays_layout():
    """The array form of a selection: counts = number kept, idx = the kept ids ascending, then -1."""
    rng = np.random.default_rng(15)
    nb = 7
    p = po.causal_block_softmax(rng.normal(size=(1, 2, nb, nb)))
    for flags in (0, po.FLAG_KEEP_SINK):
        sel = po.select_blocks(p, flags, k=2)
        counts, idx = po.selection_to_arrays(sel, kmax=5)
        for h in range(2):
            for i in range(nb):
                kept = sorted(set(sel[0][h][i].kept.tolist()))
                assert counts[0, h, i] == len(kept)
                assert idx[0, h, i].tolist() == kept + [-1] * (5 - len(kept))


def test_zero_energy_band_has_unit_temperature():
    """R4: a band with no energy anywhere retains nothing to restore, so its tau is exactly 1
    (and its logits are 0, so the other band alone decides)."""
    rng = np.random.default_rng(16)
    d, bs, L, beta = 16, 3, 64, 8
    Q = rng.normal(size=(1, 2, L, d))
    K = rng.normal(size=(1, 1, L, d))
    hmask = np.zeros(d, dtype=bool)
    hmask[:bs] = True
    hmask[d // 2:d // 2 + bs] = True
    Q[..., hmask] = 0.0
    K[..., hmask] = 0.0
    sc = po.prism_scores(Q, K, beta, bs, 0, rope=po.rope_tables(1e4, L, d))
    assert np.all(sc.tau[..., 0] == 1.0)
    assert np.all(sc.tau[..., 1] < 1.0)


def test_block_token_energy_closed_form():
    """R3/R4 energies: a constant vector under RoPE keeps each pair's norm, so every block holds
    beta times the vector's squared norm in each band."""
    d, bs, L, beta = 16, 3, 64, 8
    rng = np.random.default_rng(17)
    x = rng.normal(size=d)
    X = np.broadcast_to(x, (1, 1, L, d)).copy()
    xr = po.apply_rope(X, *po.rope_tables(1e4, L, d))
    e = po.block_token_energy(xr, beta, bs, 0)
    h = np.r_[x[:bs], x[d // 2:d // 2 + bs]]
    lo = np.r_[x[bs:d // 2], x[d // 2 + bs:]]
    # the float32 tables give c^2 + s^2 = 1 only to about 2^-23
    np.testing.assert_allclose(e[0, 0, :, 0], beta * np.sum(h ** 2), rtol=1e-7)
    np.testing.assert_allclose(e[0, 0, :, 1], beta * np.sum(lo ** 2), rtol=1e-7)


def test_path_attention_reads_the_rounded_rotated_values():
    """R1/R8: the attention step reads Q_r, K_r rounded to the input dtype, as the GPU stores them."""
    from block_sparse_long_dual_b200.workloads import TINY
    from block_sparse_long_dual_b200.synthetic import make_inputs
    w = TINY.scaled(seq_len=256)
    Q, K, V = (t.numpy() for t in make_inputs(w))
    rope = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    for dtype, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        r = po.prism_path(Q, K, V, block=w.block, band_split=w.band_split, flags=w.flags, k=w.k,
                          rope=rope, dtype=dtype)
        for got, exact in ((r.q_attn, r.scores.q_rot), (r.k_attn, r.scores.k_rot)):
            ref = torch.from_numpy(exact).to(tdt).to(torch.float64).numpy()
            np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------------------
# Alternative reading R4b (RELATIVE_CALIB): band H restored relative to band L.
# ---------------------------------------------------------------------------
def test_relative_calibration_closed_form_and_low_band_untouched():
    base, d, beta, L, bs = 1e4, 16, 8, 64, 3
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(21)
    qv, kv = rng.normal(size=d), rng.normal(size=d)
    Q = np.broadcast_to(qv, (1, 1, L, d)).copy()
    K = np.broadcast_to(kv, (1, 1, L, d)).copy()
    rel = po.prism_scores(Q, K, beta, bs, po.FLAG_RELATIVE_CALIB, (cos, sin))
    theta = po.rope_frequencies(base, d)
    Dm = np.abs(np.sin(beta * theta / 2)) / (beta * np.abs(np.sin(theta / 2)))

    def rho(v, pairs):
        e = v[pairs] ** 2 + v[pairs + d // 2] ** 2
        return math.sqrt((e * Dm[pairs] ** 2).sum() / e.sum())

    hi, lo = np.arange(bs), np.arange(bs, d // 2)
    want = (rho(qv, hi) * rho(kv, hi)) / (rho(qv, lo) * rho(kv, lo))
    assert rel.tau[0, 0, 0] == pytest.approx(want, rel=1e-5)
    assert rel.tau[0, 0, 1] == 1.0
    # Q, K with no high-band energy: identical to plain mean pooling
    rng = np.random.default_rng(22)
    Qr_, Kr_ = rng.normal(size=(1, 2, 96, d)), rng.normal(size=(1, 1, 96, d))
    hm = po.high_band_mask(d, bs)
    Qr_[..., hm] = 0.0
    Kr_[..., hm] = 0.0
    cos2, sin2 = po.rope_tables(base, 96, d)
    a = po.prism_scores(Qr_, Kr_, beta, bs, po.FLAG_RELATIVE_CALIB, (cos2, sin2))
    b = po.prism_scores(Qr_, Kr_, beta, bs, po.FLAG_NO_CALIB, (cos2, sin2))
    np.testing.assert_allclose(a.probs, b.probs, rtol=0, atol=1e-13)
    # one band relative to itself: no calibration
    c = po.prism_scores(Qr_, Kr_, beta, bs, po.FLAG_RELATIVE_CALIB | po.FLAG_SINGLE_BAND, (cos2, sin2))
    np.testing.assert_allclose(c.tau, 1.0)


# ---------------------------------------------------------------------------
# Alternative readings of §3: per-block temperature (BLOCK_TAU) and the two
# spectral branches combined by their maximum (BAND_MAX).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("row", _golden_rows()[:2])
def test_block_tau_rho_is_dirichlet_factor_per_block(row):
    """A constant vector in one rotary pair: every block's own retained amplitude is the
    Dirichlet factor of that pair (golden), and a band without energy gets rho = 1."""
    base, d, m, beta, theta, D = row
    L = 5 * beta
    cos, sin = po.rope_tables(base, L, d)
    x = np.zeros((1, 1, L, d))
    x[..., m] = 1.0
    xr = po.apply_rope(x, cos, sin)
    xbar = po.pool_blocks(xr, beta)
    h, l = po.band_masks(d, m + 1)
    np.testing.assert_allclose(po.block_retained_amplitude(xr, xbar, h), D, rtol=0, atol=3e-6)
    np.testing.assert_allclose(po.block_retained_amplitude(xr, xbar, l), 1.0)
    # a block with no energy: rho = 1
    assert po.block_retained_amplitude(xr * 0.0, xbar * 0.0, h).min() == 1.0


def test_block_tau_rho_floor_on_full_turn():
    """theta = 2 pi / beta: each block holds one full turn of the pair, its mean cancels (to the
    float32 table's rounding) and rho is floored at 1e-3."""
    beta, d, L = 8, 4, 32
    base = (beta / (2 * math.pi)) ** 2          # theta_1 = base**(-2/4) = 2 pi / beta
    cos, sin = po.rope_tables(base, L, d)
    x = np.zeros((1, 1, L, d))
    x[..., 1] = 1.0
    xr = po.apply_rope(x, cos, sin)
    xbar = po.pool_blocks(xr, beta)
    assert np.abs(xbar).max() < 1e-6
    h, _ = po.band_masks(d, 2)
    np.testing.assert_array_equal(po.block_retained_amplitude(xr, xbar, h), po.BLOCK_RHO_FLOOR)


def test_block_tau_restores_each_block_to_its_token_rms():
    """Dividing a block mean by its own rho gives a vector whose squared norm is the block's
    mean token energy in that band (checked against the rotated tokens with torch)."""
    base, d, beta, L, bs = 1e4, 16, 8, 64, 3
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(31)
    X = rng.normal(size=(1, 2, L, d))
    xr = po.apply_rope(X, cos, sin)
    xbar = po.pool_blocks(xr, beta)
    for band in po.band_masks(d, bs):
        rho = po.block_retained_amplitude(xr, xbar, band)
        lhs = ((xbar[..., band] / rho[..., None]) ** 2).sum(-1)
        t = _torch_rotate(X, cos, sin)[..., torch.from_numpy(band)]
        rms2 = (t ** 2).sum(-1).reshape(1, 2, L // beta, beta).mean(-1).numpy()
        np.testing.assert_allclose(lhs, rms2, rtol=1e-12)


def test_block_tau_block_one_equals_token_causal_softmax():
    B, Hq, Hkv, L, d = 1, 4, 2, 10, 8
    cos, sin = po.rope_tables(1e4, L, d)
    rng = np.random.default_rng(32)
    Q = rng.normal(size=(B, Hq, L, d))
    K = rng.normal(size=(B, Hkv, L, d))
    sc = po.prism_scores(Q, K, 1, 2, po.FLAG_BLOCK_TAU, (cos, sin))
    qt = _torch_rotate(Q, cos, sin)
    kt = torch.repeat_interleave(_torch_rotate(K, cos, sin), Hq // Hkv, dim=1)
    logits = qt @ kt.transpose(-1, -2) / math.sqrt(d)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    ref = torch.softmax(logits.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(sc.probs, ref.numpy(), rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        po.prism_scores(Q, K, 1, 2, po.FLAG_BLOCK_TAU | po.FLAG_NO_CALIB, (cos, sin))


def test_band_max_mirrored_bands_is_half_logit_softmax():
    """Identical bands: both branches give softmax(s^H), while the sum reading gives softmax(2 s^H)."""
    L, d = 9, 4
    rng = np.random.default_rng(33)
    q = rng.normal(size=(1, 1, L, 2))
    k = rng.normal(size=(1, 1, L, 2))
    Q = np.stack([q[..., 0], q[..., 0], q[..., 1], q[..., 1]], -1)   # dims (0, 2) = band H, (1, 3) = band L
    K = np.stack([k[..., 0], k[..., 0], k[..., 1], k[..., 1]], -1)
    mx = po.prism_scores(Q, K, 1, 1, po.FLAG_BAND_MAX, None)
    sm = po.prism_scores(Q, K, 1, 1, 0, None)
    sH = torch.from_numpy(q[0, 0] @ k[0, 0].T / math.sqrt(d))
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    np.testing.assert_allclose(mx.probs[0, 0], torch.softmax(sH.masked_fill(~mask, -math.inf), -1).numpy(),
                               rtol=0, atol=1e-13)
    np.testing.assert_allclose(sm.probs[0, 0], torch.softmax((2 * sH).masked_fill(~mask, -math.inf), -1).numpy(),
                               rtol=0, atol=1e-13)


def test_band_max_one_hot_branch_against_uniform_branch():
    """Band H one-hot at block j* (huge logit), band L uniform (zero logits): row i >= j* keeps
    (i+1)/(2i+1) on j* and 1/(2i+1) elsewhere; rows i < j* stay uniform."""
    L, d, js, A = 8, 4, 3, 12.0
    Q = np.zeros((1, 1, L, d))
    K = np.zeros((1, 1, L, d))
    Q[..., 0] = A
    K[0, 0, js, 0] = A
    p = po.prism_scores(Q, K, 1, 1, po.FLAG_BAND_MAX, None).probs[0, 0]
    for i in range(L):
        want = np.zeros(L)
        if i < js:
            want[:i + 1] = 1.0 / (i + 1)
        else:
            want[:i + 1] = 1.0 / (2 * i + 1)
            want[js] = (i + 1) / (2 * i + 1)
        np.testing.assert_allclose(p[i], want, rtol=0, atol=1e-12)


def test_band_max_single_band_is_default():
    base, d, beta, L = 1e4, 16, 8, 64
    cos, sin = po.rope_tables(base, L, d)
    rng = np.random.default_rng(34)
    Q, K = rng.normal(size=(1, 2, L, d)), rng.normal(size=(1, 1, L, d))
    for flags, bs in ((po.FLAG_SINGLE_BAND, 3), (0, 0), (0, d // 2)):
        a = po.prism_scores(Q, K, beta, bs, flags | po.FLAG_BAND_MAX, (cos, sin))
        b = po.prism_scores(Q, K, beta, bs, flags, (cos, sin))
        np.testing.assert_array_equal(a.probs, b.probs)


def test_block_tau_logit_closed_form_with_different_q_and_k_amplitudes():
    """Constant Q in rotary pair 0 only; constant K in pairs 0 and 8 (one band).  Every block of Q
    keeps rho_Q = D_0 and every block of K rho_K = sqrt((D_0^2 b^2 + D_8^2 c^2) / (b^2 + c^2))
    (golden Dirichlet factors, beta = 64, base 1e4, d = 64), and only pair 0 meets in the dot
    product, so s_ij = D_0 a b cos(64 (i - j)) / (rho_K sqrt(d))."""
    rows = {(r[2], r[3]): r for r in _golden_rows() if r[0] == 1e4 and r[1] == 64}
    D0, D8 = rows[(0, 64)][5], rows[(8, 64)][5]
    beta, d, L, a, b, c = 64, 64, 64 * 6, 1.3, 0.7, 2.1
    cos, sin = po.rope_tables(1e4, L, d)
    Q = np.zeros((1, 1, L, d))
    K = np.zeros((1, 1, L, d))
    Q[..., 0] = a
    K[..., 0] = b
    K[..., 8] = c
    sc = po.prism_scores(Q, K, beta, 0, po.FLAG_BLOCK_TAU | po.FLAG_SINGLE_BAND, (cos, sin))
    rho_k = math.sqrt((D0 ** 2 * b ** 2 + D8 ** 2 * c ** 2) / (b ** 2 + c ** 2))
    nb = L // beta
    i, j = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    want = D0 * a * b * np.cos(64.0 * (i - j)) / (rho_k * math.sqrt(d))
    np.testing.assert_allclose(sc.logits[0, 0], want, rtol=0, atol=2e-5)
