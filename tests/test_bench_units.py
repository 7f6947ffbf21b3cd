"""The bench's algorithmic units (what the roofline numbers divide by), checked on CPU against
direct counts: attention FLOPs over kept blocks, the density-to-k rule, scoring and decode bytes."""

import importlib.util
import os

import numpy as np
import pytest

from block_sparse_long_dual_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_attention_flops_counts_kept_pairs(bench):
    """4 d per (query, key) pair actually attended: full blocks off the diagonal, the causal
    triangle (with its diagonal) on it; brute-force pair count on a tiny layout."""
    block, d = 4, 8
    counts = np.array([[[1, 2, 3]]])  # rows i = 0, 1, 2 keep i + 1 blocks (diagonal included)
    pairs = 0
    for i, n in enumerate(counts[0, 0]):
        kept = list(range(i - n + 1, i + 1))
        for j in kept:
            for tq in range(block):
                for tk in range(block):
                    if j < i or tk <= tq:
                        pairs += 1
    assert bench.attention_flops(counts, block, d) == 4 * d * pairs


def test_k_for_density_is_the_smallest_k(bench):
    for nb, rho in ((256, 0.10), (1024, 0.05), (512, 0.01), (512, 1.0)):
        k = wl.k_for_density(nb, rho)
        assert wl.kept_blocks_topk(nb, k) >= rho * nb * (nb + 1) / 2 - 1e-9
        if k > 0:
            assert wl.kept_blocks_topk(nb, k - 1) < rho * nb * (nb + 1) / 2
    assert wl.LLAMA_32K.k == 13 and wl.LLAMA_128K.k == 25


def test_scoring_and_decode_bytes(bench):
    w = wl.LLAMA_128K
    qk = (32 + 8) * 131072 * 128 * 2
    want = 2 * qk + 2 * 131072 * 64 * 4 + (32 + 8) * 1024 * 128 * 8 + 32 * 1024 * 1024 * 4
    assert bench.scoring_bytes(w) == want
    dw = wl.FASA_DECODE_128K_B4
    sel, att, total = bench.decode_bytes(dw)
    assert sel == 4 * 8 * 131072 * 24 * 2 + 4 * 32 * 128 * 2       # compact keys + q
    assert att == 4 * 32 * (256 * 2 * 128 * 2 + 2 * 128 * 2 + 256 * 4)
    assert total > sel + att


def test_scoring_bytes_without_stored_q_rot_or_probs(bench):
    """RoPE on load drops the Q_rot write (K_rot is still written); a fused selection drops the
    probabilities; counted directly for the 128K layer."""
    w = wl.LLAMA_128K
    q = 32 * 131072 * 128 * 2
    k = 8 * 131072 * 128 * 2
    table = 2 * 131072 * 64 * 4
    means = (32 + 8) * 1024 * 128 * 8
    probs = 32 * 1024 * 1024 * 4
    assert bench.scoring_bytes(w, True, False) == (q + k) + k + table + means + probs
    assert bench.scoring_bytes(w, False, True) == 2 * (q + k) + table + means
    assert bench.scoring_bytes(w, False, False) == (q + k) + k + table + means
