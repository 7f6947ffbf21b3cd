"""Selection quality of the block estimate, measured against exact attention (test infrastructure).

For sampled query tokens, the fraction of each token's exact causal softmax
attention mass that falls inside its query block's kept key blocks; also how
often the planted semantic blocks and the previous (most recent) block are
kept.  Variants: the calibrated dual-band estimate ("Prism: Spectral-Aware
Block-Sparse Attention" §3), plain mean pooling (the baseline the page
improves on, §1-§2: NO_CALIB), one band (SINGLE_BAND) and the alternative
reading that restores the high band only relative to the low band
(RELATIVE_CALIB).  Everything runs on
the CPU oracle in float64.

Run: python tests/selection_quality.py  (prints a markdown table)
"""

from __future__ import annotations

import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_long_dual_b200.synthetic import make_inputs, planted_blocks  # noqa: E402
from block_sparse_long_dual_b200.workloads import (BAND_MAX, BLOCK_TAU, NO_CALIB, RELATIVE_CALIB,  # noqa: E402
                                                   SINGLE_BAND, Workload)
from oracle import prism_oracle as po  # noqa: E402

VARIANTS = (("calibrated dual band", 0), ("plain mean pooling", NO_CALIB), ("single band", SINGLE_BAND),
            ("relative calibration", RELATIVE_CALIB), ("band max", BAND_MAX),
            ("band max + relative calibration", BAND_MAX | RELATIVE_CALIB), ("per-block temperature", BLOCK_TAU))


def token_mass_recall(qa, ka, kept, block, b, h, g, i, causal=True, scale=None):
    """Mean over the tokens of query block i of the exact softmax mass on the kept blocks."""
    d = qa.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    tq = np.arange(i * block, (i + 1) * block)
    nk = (i + 1) * block if causal else ka.shape[-2]
    s = (qa[b, h, tq] @ ka[b, g, :nk].T) * scale
    if causal:
        s = np.where(np.arange(nk)[None, :] <= tq[:, None], s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    mask = np.zeros(nk, dtype=bool)
    for j in kept:
        mask[j * block:(j + 1) * block] = True
    return float(p[:, mask].sum(axis=1).mean())


def measure(w: Workload, n_rows: int = 24, seed: int = 0, rules=(("top-k", "k"), ("mass", "mass"))):
    """{(variant, rule): (token-mass recall, mean kept blocks, planted recall, previous-block recall)}."""
    Q, K, _ = make_inputs(w, seed=seed)
    Qn, Kn = Q.double().numpy(), K.double().numpy()
    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    rng = np.random.default_rng(seed + 17)
    rows = [(int(rng.integers(w.batch)), int(rng.integers(w.heads_q)), int(rng.integers(8, w.nb)))
            for _ in range(n_rows)]
    planted = set(planted_blocks(w).tolist())
    out = {}
    for vname, flags in VARIANTS:
        sc = po.prism_scores(Qn, Kn, w.block, w.band_split, flags | w.flags, (cos, sin))
        qa = po.round_to_dtype(sc.q_rot, w.dtype)
        ka = po.round_to_dtype(sc.k_rot, w.dtype)
        for rname, kind in rules:
            if kind == "k":
                sel = po.select_blocks(sc.probs, flags | w.flags, k=w.k if w.k is not None else 4)
            else:
                sel = po.select_blocks(sc.probs, flags | w.flags, mass=float(np.float32(w.mass or 0.9)))
            rec, nk, pl_hit, pl_tot, prev = [], [], 0, 0, []
            for b, h, i in rows:
                kept = sel[b][h][i].kept
                rec.append(token_mass_recall(qa, ka, kept, w.block, b, h, h // w.group, i))
                nk.append(kept.size)
                cand = [j for j in planted if j < i]
                pl_tot += len(cand)
                pl_hit += sum(1 for j in cand if j in set(kept.tolist()))
                prev.append(1.0 if (i - 1) in set(kept.tolist()) else 0.0)
            out[(vname, rname)] = (float(np.mean(rec)), float(np.mean(nk)),
                                   (pl_hit / pl_tot) if pl_tot else float("nan"), float(np.mean(prev)))
    return out


def quality_workloads():
    base = dict(batch=1, heads_q=4, heads_kv=1, seq_len=8192, head_dim=128, dtype="bf16", block=128,
                band_split=32, k=4, mass=0.9)
    return [
        Workload(name="slash + 5% semantic, base 1e6", rope_base=1e6, slash=True, planted_frac=0.05, **base),
        Workload(name="5% semantic, base 5e5", rope_base=5e5, planted_frac=0.05, **base),
        Workload(name="noise only, base 5e5", rope_base=5e5, **base),
    ]


def main():
    print("| workload | variant | rule | token-mass recall | kept blocks / row | planted recall | previous-block recall |")
    print("|---|---|---|---|---|---|---|")
    for w in quality_workloads():
        res = measure(w)
        for (v, r), (rec, nk, pl, prev) in res.items():
            rule = f"top-{w.k} + diagonal" if r == "top-k" else f"mass {w.mass}"
            print(f"| {w.name} | {v} | {rule} | {rec:.3f} | {nk:.1f} | {pl:.3f} | {prev:.3f} |")


if __name__ == "__main__":
    main()
