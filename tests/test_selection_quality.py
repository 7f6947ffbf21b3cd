"""Pins of the selection-quality measurement (CPU)."""

import math

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200.workloads import Workload
from oracle import prism_oracle as po
from tests import selection_quality as sq


def _rand(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


def test_token_mass_recall_extremes_and_brute_force():
    B, H, L, d, beta = 1, 1, 96, 8, 16
    qa, ka = _rand((B, H, L, d), 1), _rand((B, H, L, d), 2)
    i = 4
    # all causal blocks kept: every token keeps all of its mass
    assert sq.token_mass_recall(qa, ka, range(i + 1), beta, 0, 0, 0, i) == pytest.approx(1.0, abs=1e-12)
    # nothing kept: no mass
    assert sq.token_mass_recall(qa, ka, [], beta, 0, 0, 0, i) == 0.0
    # brute force with torch's softmax for a subset
    kept = [0, 2, 4]
    tq = torch.arange(i * beta, (i + 1) * beta)
    s = torch.from_numpy(qa[0, 0]) @ torch.from_numpy(ka[0, 0]).T / math.sqrt(d)
    s = s[tq][:, :(i + 1) * beta]
    s = s.masked_fill(torch.arange((i + 1) * beta)[None, :] > tq[:, None], float("-inf"))
    p = torch.softmax(s, dim=-1)
    cols = torch.cat([torch.arange(j * beta, (j + 1) * beta) for j in kept])
    want = p[:, cols].sum(-1).mean().item()
    assert sq.token_mass_recall(qa, ka, kept, beta, 0, 0, 0, i) == pytest.approx(want, abs=1e-12)


def test_recall_is_monotone_in_k():
    w = Workload(name="q", batch=1, heads_q=2, heads_kv=1, seq_len=1024, head_dim=32, dtype="bf16", block=64,
                 rope_base=1e4, band_split=8, k=2, planted_frac=0.1)
    res = {k: sq.measure(w.scaled(k=k), n_rows=6, rules=(("top-k", "k"),)) for k in (0, 2, 6, 100)}
    for v, _ in sq.VARIANTS:
        r = [res[k][(v, "top-k")][0] for k in (0, 2, 6, 100)]
        assert all(a <= b + 1e-12 for a, b in zip(r, r[1:]))
        assert r[-1] == pytest.approx(1.0, abs=1e-9)   # every block kept
