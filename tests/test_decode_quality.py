"""The decode estimate on the oracle: when a few frequency pairs carry the scores (the page's
premise), ranking by those pairs keeps nearly all the attention mass exact top-k keeps, while as
many other pairs or recency keep little."""

from tests import decode_quality as dq
from block_sparse_long_dual_b200.workloads import DecodeWorkload


def test_dominant_pairs_recover_exact_top_k_mass():
    w = DecodeWorkload(name="q", batch=1, heads_q=4, heads_kv=1, seq_len=4096, head_dim=64, nfc=8, k=64,
                       dominant_gain=3.0)
    r = dq.measure(w)
    exact, dom = r["all pairs (exact top-k)"], r["dominant pairs"]
    assert dom >= 0.9 * exact
    assert r["other pairs"] < 0.5 * dom
    assert r["most recent k (no estimate)"] < 0.5 * dom
    assert exact <= 1.0 + 1e-12
