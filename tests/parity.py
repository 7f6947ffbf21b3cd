"""Helpers for the GPU-vs-oracle parity tests (test infrastructure)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import prism_oracle as po

NEAR_TIE_REL = 1e-6   # block masks: candidates within 1e-6 relative of the row threshold are not compared


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy() if t.dtype in (torch.bfloat16, torch.float16) \
        else t.detach().cpu().numpy()


def uncertain_candidates(sel: po.RowSelection, p_row: np.ndarray, mass: float | None, rel=NEAR_TIE_REL):
    """Candidates whose membership may legitimately differ between float32 and float64 scores."""
    order, n = sel.order, sel.n_taken
    U = set()
    if order.size == 0:
        return U
    if n > 0:
        t = p_row[order[n - 1]]
        for c in order:
            if abs(p_row[c] - t) <= rel * t:
                U.add(int(c))
    if mass is not None:
        near = False
        if n == 0:
            near = abs(sum(p_row[j] for j in sel.forced) - mass) <= rel
        else:
            near = abs(sel.cum_before_last - mass) <= rel or abs(sel.cum_final - mass) <= rel
        if near:
            U.update(int(c) for c in order[max(0, n - 1):n + 1])
    return U


def threshold_alone(sel: po.RowSelection, p_row: np.ndarray, mass: float | None, rel=NEAR_TIE_REL) -> bool:
    """True when the only candidate the near-tie rule excuses is the threshold candidate itself (no
    other candidate within the window and, in mass mode, no running sum near the target): the
    literal rule still excuses that candidate, but no float32/float64 difference can move it."""
    order, n = sel.order, sel.n_taken
    if order.size == 0 or n == 0:
        return False
    t = p_row[order[n - 1]]
    if sum(1 for c in order if abs(p_row[c] - t) <= rel * t) > 1:
        return False
    if mass is not None and (abs(sel.cum_before_last - mass) <= rel or abs(sel.cum_final - mass) <= rel):
        return False
    return True


def compare_masks(sel, probs_oracle, counts, idx, mass=None):
    """Row-by-row comparison of the GPU's kept sets with the oracle's.

    Returns (stats, exact) where exact[b][h][i] is True when the GPU row equals
    the oracle row exactly (those rows are the ones whose outputs are compared).
    stats["threshold_only_rows"] counts rows excused only because the rule, read
    literally, excuses the threshold candidate itself (see threshold_alone)."""
    counts = counts.cpu().numpy()
    idx = idx.cpu().numpy()
    B, H, nb = counts.shape
    stats = dict(rows=0, uncertain_rows=0, mismatches=0, bad_rows=[], threshold_only_rows=0)
    exact = np.zeros((B, H, nb), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                r = sel[b][h][i]
                n = int(counts[b, h, i])
                g = idx[b, h, i, :n]
                assert np.all(idx[b, h, i, n:] == -1), "padding must be -1"
                assert np.all(np.diff(g) > 0), "kept list must be ascending"
                gs, os_ = set(g.tolist()), set(r.kept.tolist())
                stats["rows"] += 1
                if gs == os_:
                    exact[b, h, i] = True
                    continue
                U = uncertain_candidates(r, probs_oracle[b, h, i], mass)
                if U:
                    stats["uncertain_rows"] += 1
                if (gs - U) != (os_ - U):
                    stats["mismatches"] += 1
                    stats["bad_rows"].append((b, h, i, sorted(gs ^ os_)))
                elif threshold_alone(r, probs_oracle[b, h, i], mass):
                    stats["threshold_only_rows"] += 1
    return stats, exact


def rel_err(a: np.ndarray, b: np.ndarray, floor=1e-30):
    m = np.abs(b) > floor
    return float(np.max(np.abs(a[m] - b[m]) / np.abs(b[m]))) if m.any() else 0.0


def random_index_lists(rng, B, H, nb, kmax, causal=True, p_keep=0.3, empty_rows=(), diag_only_rows=()):
    """Seeded synthetic kept lists (ascending, -1 padded) for attention-stage tests."""
    counts = np.zeros((B, H, nb), dtype=np.int32)
    idx = np.full((B, H, nb, kmax), -1, dtype=np.int32)
    kept = [[[None] * nb for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                hi = i + 1 if causal else nb
                cand = np.arange(hi)
                sel = cand[rng.random(hi) < p_keep]
                if causal:
                    sel = np.union1d(sel, [i])
                sel = np.sort(sel)[:kmax]
                if (b, h, i) in empty_rows:
                    sel = np.zeros(0, dtype=np.int64)
                if (b, h, i) in diag_only_rows:
                    sel = np.array([i])
                kept[b][h][i] = sel.astype(np.int64)
                counts[b, h, i] = sel.size
                idx[b, h, i, :sel.size] = sel
    return counts, idx, kept
