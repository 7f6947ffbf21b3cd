"""Decode selection quality (test infrastructure): the exact softmax attention mass of one query
token that its kept tokens capture ("FASA: Frequency-aware Sparse Attention" §2B: the estimate
should pick the tokens that matter), on the float64 oracle.

Rankings compared for the same cache and budget k: all 64 rotary pairs (the exact top-k by
q.k: the best any subset of size k can do for these scores), the dominant pairs the synthetic
inputs were built around (the offline calibration the page describes is out of scope), the same
number of other pairs, and no estimate at all (the most recent k tokens).  Caches: the bench's
inputs (N(0, 1) with 1% needles), noise only, and the same with the dominant pairs' amplitude
tripled (scores carried mostly by a few frequency pairs, the premise of the page's §2A).

Run: python tests/decode_quality.py  (prints a markdown table)
"""

from __future__ import annotations

import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_long_dual_b200.synthetic import make_decode_inputs  # noqa: E402
from block_sparse_long_dual_b200.workloads import DecodeWorkload  # noqa: E402
from oracle import fasa_oracle as fo  # noqa: E402


def mass_recall(q, K, kept):
    """Exact softmax(q.k / sqrt(d)) mass over the kept tokens, per (b, h), averaged."""
    B, Hq, d = q.shape
    group = Hq // K.shape[1]
    out = []
    for b in range(B):
        for h in range(Hq):
            s = K[b, h // group] @ q[b, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            idx = kept[b, h][kept[b, h] >= 0]
            out.append(p[idx].sum())
    return float(np.mean(out))


def measure(w: DecodeWorkload, seed=0):
    qt, Kt, _, fc = make_decode_inputs(w, seed=seed)
    q, K = qt.double().numpy(), Kt.double().numpy()
    half = w.head_dim // 2
    rng = np.random.default_rng(seed + 9)
    other = np.stack([np.sort(rng.choice(np.setdiff1d(np.arange(half), fc[g]), w.nfc, replace=False))
                      for g in range(w.heads_kv)])
    allp = np.tile(np.arange(half), (w.heads_kv, 1))
    res = {}
    for name, pairs in (("all pairs (exact top-k)", allp), ("dominant pairs", fc), ("other pairs", other)):
        idx = fo.select_tokens(fo.tip_scores(q, K, pairs), w.k)
        res[name] = mass_recall(q, K, idx)
    recent = np.tile(np.arange(w.seq_len - w.k, w.seq_len), (w.batch, w.heads_q, 1))
    res["most recent k (no estimate)"] = mass_recall(q, K, recent)
    return res


def quality_workloads():
    base = dict(batch=1, heads_q=8, heads_kv=2, seq_len=16384, head_dim=128, nfc=12, k=256)
    return [DecodeWorkload(name="1% needles (bench inputs)", **base),
            DecodeWorkload(name="noise only", needle_frac=0.0, **base),
            DecodeWorkload(name="1% needles, dominant pairs x3", dominant_gain=3.0, **base),
            DecodeWorkload(name="noise only, dominant pairs x3", needle_frac=0.0, dominant_gain=3.0, **base)]


def main():
    print("| cache | ranking | exact attention mass kept (k = 256 of 16384) |")
    print("|---|---|---|")
    for w in quality_workloads():
        for name, v in measure(w).items():
            print(f"| {w.name} | {name} | {v:.3f} |")


if __name__ == "__main__":
    main()
