"""Helpers for the GPU-vs-oracle parity tests (test infrastructure)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import prism_oracle as po

NEAR_TIE_REL = 1e-6   # block masks: candidates within 1e-6 relative of the row threshold are not compared


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy() if t.dtype in (torch.bfloat16, torch.float16) \
        else t.detach().cpu().numpy()


def _window(order, p_row, ref, rel):
    """Candidates whose probability lies within ``rel`` (relative) of ``ref``."""
    return {int(c) for c in order if abs(p_row[c] - ref) <= rel * ref}


def allowed_selection(sel: po.RowSelection, p_row: np.ndarray, mass: float | None, rel=NEAR_TIE_REL):
    """What a GPU row may keep, beyond the forced blocks, when its probabilities differ from the
    float64 oracle's by float32 rounding.

    Returns (must, may, deltas): the GPU's kept candidates G must satisfy must <= G <= may and
    |G| - n in deltas, n = the oracle's number of kept candidates.
      * Near-ties: W = the candidates within ``rel`` of the oracle's threshold probability (that of
        the last candidate it keeps).  Which members of W are kept may differ; how many may not,
        unless the running mass allows it below.  A threshold with no other candidate in its window
        excuses nothing: the GPU must then keep exactly the oracle's candidates.
      * Mass rule: one candidate fewer only if the running sum before the oracle's last add is
        within ``rel`` of the target (a float32 sum may already reach it there); one more only if
        the final running sum is within ``rel`` of the target (a float32 sum may still fall short),
        the extra one being the next candidate or one within ``rel`` of it."""
    order, n = sel.order, sel.n_taken
    top = {int(c) for c in order[:n]}
    W = _window(order, p_row, p_row[order[n - 1]], rel) if n > 0 else set()
    if len(W) == 1:
        W = set()
    must = top - W
    may = top | W
    deltas = {0}
    if mass is not None:
        if n > 0 and abs(sel.cum_before_last - mass) <= rel:
            deltas.add(-1)
            must -= {int(order[n - 1])} | W
        if n < order.size and abs(sel.cum_final - mass) <= rel:
            deltas.add(1)
            nxt = p_row[order[n]]
            may |= _window(order, p_row, nxt, rel) | {int(order[n])}
    return must, may, deltas


def threshold_alone(sel: po.RowSelection, p_row: np.ndarray, mass: float | None, rel=NEAR_TIE_REL) -> bool:
    """True when, read literally, the near-tie rule would excuse only the threshold candidate itself:
    no other candidate within the window and, in mass mode, no running sum near the target.  No
    float32/float64 difference can move such a row, so allowed_selection excuses nothing there."""
    order, n = sel.order, sel.n_taken
    if order.size == 0 or n == 0:
        return False
    if len(_window(order, p_row, p_row[order[n - 1]], rel)) > 1:
        return False
    if mass is not None and (abs(sel.cum_before_last - mass) <= rel or abs(sel.cum_final - mass) <= rel):
        return False
    return True


def compare_masks(sel, probs_oracle, counts, idx, mass=None):
    """Row-by-row comparison of the GPU's kept sets with the oracle's (see allowed_selection).

    Returns (stats, exact) where exact[b][h][i] is True when the GPU row equals the oracle row
    exactly (those rows are the ones whose outputs are compared).  stats: rows; excused_rows (kept
    sets that differ within the near-tie rule); count_diff_rows (of those, rows whose count differs,
    possible only in mass mode); mismatches and bad_rows (everything else);
    threshold_only_rows (mismatching rows where the literal rule would have excused the threshold
    candidate alone: always also counted in mismatches)."""
    counts = counts.cpu().numpy()
    idx = idx.cpu().numpy()
    B, H, nb = counts.shape
    stats = dict(rows=0, excused_rows=0, count_diff_rows=0, mismatches=0, bad_rows=[], threshold_only_rows=0)
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
                p_row = probs_oracle[b, h, i]
                forced = set(int(j) for j in r.forced)
                G = gs - forced
                must, may, deltas = allowed_selection(r, p_row, mass)
                if forced <= gs and must <= G and G <= may and (len(G) - r.n_taken) in deltas:
                    stats["excused_rows"] += 1
                    if len(G) != r.n_taken:
                        stats["count_diff_rows"] += 1
                    continue
                stats["mismatches"] += 1
                stats["bad_rows"].append((b, h, i, sorted(gs ^ os_)))
                if threshold_alone(r, p_row, mass) and (gs ^ os_) <= {int(r.order[r.n_taken - 1])}:
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


def compare_token_lists(idx_gpu: np.ndarray, scores: np.ndarray, k: int, rel=NEAR_TIE_REL):
    """Decode selection: the GPU's kept token lists [B, H, k] against the oracle's first min(k, L)
    tokens by (float64 score desc, index asc).  Tokens whose score lies within ``rel`` (relative)
    of the row's k-th score are interchangeable when at least two lie there; the number kept is
    always min(k, L).  Returns stats (rows, excused_rows, mismatches, bad_rows)."""
    B, H, L = scores.shape
    n = min(k, L)
    stats = dict(rows=0, excused_rows=0, mismatches=0, bad_rows=[])
    for b in range(B):
        for h in range(H):
            row = idx_gpu[b, h]
            assert np.all(row[n:] == -1), "padding must be -1"
            got = row[:n]
            assert np.all(np.diff(got) > 0) and np.all(got >= 0), "kept list must be ascending"
            s = scores[b, h]
            order = np.lexsort((np.arange(L), -s))
            want = set(order[:n].tolist())
            gs = set(got.tolist())
            stats["rows"] += 1
            if gs == want:
                continue
            T = s[order[n - 1]]
            W = set(np.nonzero(np.abs(s - T) <= rel * abs(T))[0].tolist())
            if len(W) < 2:
                W = set()
            if (want - W) <= gs <= (want | W):
                stats["excused_rows"] += 1
            else:
                stats["mismatches"] += 1
                stats["bad_rows"].append((b, h, sorted(gs ^ want)[:8]))
    return stats
