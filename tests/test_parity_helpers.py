"""The mask comparison the GPU parity tests rely on, checked on the CPU: it must accept an exact
match, excuse only near-ties (another candidate within 1e-6 relative of the row threshold, or a
running mass within 1e-6 of the target), and count every other difference, a missing or an extra
block included."""

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po
from tests.parity import compare_masks


def _arrays(kept_rows, nb, kmax):
    counts = torch.zeros((1, 1, nb), dtype=torch.int32)
    idx = torch.full((1, 1, nb, kmax), -1, dtype=torch.int32)
    for i, kept in enumerate(kept_rows):
        counts[0, 0, i] = len(kept)
        idx[0, 0, i, :len(kept)] = torch.tensor(sorted(kept), dtype=torch.int32)
    return counts, idx


def _probs(rows):
    nb = len(rows)
    p = np.zeros((1, 1, nb, nb))
    for i, r in enumerate(rows):
        p[0, 0, i, :len(r)] = r
    return p


def test_exact_match_and_a_clear_difference():
    p = _probs([[1.0], [0.3, 0.7], [0.5, 0.2, 0.3], [0.1, 0.4, 0.2, 0.3]])
    sel = po.select_blocks(p, 0, k=1)
    kept = [sel[0][0][i].kept.tolist() for i in range(4)]
    stats, exact = compare_masks(sel, p, *_arrays(kept, 4, 2))
    assert stats["mismatches"] == 0 and exact.all()
    wrong = [list(k) for k in kept]
    wrong[3] = [2, 3]                                 # row 3 keeps block 1 (0.4), not block 2 (0.2)
    stats, exact = compare_masks(sel, p, *_arrays(wrong, 4, 2))
    assert stats["mismatches"] == 1 and not exact[0, 0, 3] and exact[0, 0, :3].all()


def test_near_tie_at_the_threshold_is_excused_and_only_that():
    p = _probs([[1.0], [0.5, 0.5], [0.1, 0.5, 0.4]])
    sel = po.select_blocks(p, 0, k=1)
    assert sel[0][0][2].kept.tolist() == [1, 2]
    swapped = [[0], [0, 1], [0, 2]]                   # block 0 (0.1) instead of block 1 (0.5)
    stats, _ = compare_masks(sel, p, *_arrays(swapped, 3, 2))
    assert stats["mismatches"] == 1
    p2 = _probs([[1.0], [0.5, 0.5], [0.3, 0.3 * (1 + 5e-7), 0.4]])
    sel2 = po.select_blocks(p2, 0, k=1)
    assert sel2[0][0][2].kept.tolist() == [1, 2]
    tie = [[0], [0, 1], [0, 2]]                       # the other side of a 5e-7 near-tie: excused
    stats, exact = compare_masks(sel2, p2, *_arrays(tie, 3, 2))
    assert stats["mismatches"] == 0 and stats["excused_rows"] == 1 and not exact[0, 0, 2]
    assert stats["threshold_only_rows"] == 0 and stats["count_diff_rows"] == 0
    # the near-tie excuses the choice between the two tied blocks, not their number
    stats, _ = compare_masks(sel2, p2, *_arrays([[0], [0, 1], [2]], 3, 2))
    assert stats["mismatches"] == 1
    stats, _ = compare_masks(sel2, p2, *_arrays([[0], [0, 1], [0, 1, 2]], 3, 3))
    assert stats["mismatches"] == 1


def test_top_k_row_missing_its_threshold_block_is_a_mismatch():
    p = _probs([[1.0], [0.3, 0.7], [0.5, 0.2, 0.3], [0.1, 0.4, 0.2, 0.3]])
    sel = po.select_blocks(p, 0, k=2)
    assert sel[0][0][3].kept.tolist() == [1, 2, 3]
    short = [sel[0][0][i].kept.tolist() for i in range(3)] + [[1, 3]]   # block 2 (0.2) dropped
    stats, exact = compare_masks(sel, p, *_arrays(short, 4, 3))
    assert stats["mismatches"] == 1 and stats["threshold_only_rows"] == 1 and not exact[0, 0, 3]


def test_running_mass_at_the_target_is_excused():
    # row 1: forced diagonal 0.5; adding block 0 (0.5) reaches exactly 1.0; target within 1e-6 of 0.5
    p = _probs([[1.0], [0.5, 0.5]])
    mass = 0.5 + 5e-7
    sel = po.select_blocks(p, 0, mass=mass)
    assert sel[0][0][1].kept.tolist() == [0, 1]
    kept = [[0], [1]]                                 # a float32 running sum may stop at the diagonal
    stats, _ = compare_masks(sel, p, *_arrays(kept, 2, 2), mass)
    assert stats["mismatches"] == 0 and stats["count_diff_rows"] == 1
    assert stats["threshold_only_rows"] == 0
    # far from the target, stopping one block early is a mismatch (the literal window, which always
    # holds the threshold candidate, would have excused it: counted as such)
    sel75 = po.select_blocks(p, 0, mass=0.75)
    stats, _ = compare_masks(sel75, p, *_arrays(kept, 2, 2), 0.75)
    assert stats["mismatches"] == 1 and stats["threshold_only_rows"] == 1


def test_running_mass_just_above_the_target_allows_one_more_block():
    # row 2: diagonal 0.3 + block 1 (0.6) = 0.9 reaches the target 0.9 - 4e-7; a float32 sum may
    # fall short and add block 0 (0.1) as well
    p = _probs([[1.0], [0.5, 0.5], [0.1, 0.6, 0.3]])
    mass = 0.9 - 4e-7
    sel = po.select_blocks(p, 0, mass=mass)
    assert sel[0][0][2].kept.tolist() == [1, 2]
    rows = [[0], [0, 1], [0, 1, 2]]
    stats, _ = compare_masks(sel, p, *_arrays(rows, 3, 3), mass)
    assert stats["mismatches"] == 0 and stats["count_diff_rows"] == 1
    # far from the target the extra block is a mismatch
    sel8 = po.select_blocks(p, 0, mass=0.8)
    stats, _ = compare_masks(sel8, p, *_arrays(rows, 3, 3), 0.8)
    assert stats["mismatches"] == 1
    # a wrong block in its place is counted
    p3 = _probs([[1.0], [0.5, 0.5], [0.1, 0.6, 0.3]])
    sel3 = po.select_blocks(p3, 0, mass=0.75)
    assert sel3[0][0][2].kept.tolist() == [1, 2]
    stats, _ = compare_masks(sel3, p3, *_arrays([[0], [0, 1], [0, 2]], 3, 2), 0.75)
    assert stats["mismatches"] == 1


def test_malformed_gpu_rows_are_rejected():
    p = _probs([[1.0], [0.5, 0.5]])
    sel = po.select_blocks(p, 0, k=1)
    counts, idx = _arrays([[0], [0, 1]], 2, 3)
    idx[0, 0, 0, 2] = 0                               # padding that is not -1
    with pytest.raises(AssertionError, match="padding"):
        compare_masks(sel, p, counts, idx)
    counts, idx = _arrays([[0], [0, 1]], 2, 2)
    idx[0, 0, 1] = torch.tensor([1, 0], dtype=torch.int32)   # not ascending
    with pytest.raises(AssertionError, match="ascending"):
        compare_masks(sel, p, counts, idx)


def test_token_list_comparison_excuses_only_true_near_ties():
    from tests.parity import compare_token_lists
    s = np.array([[[5.0, 3.0, 3.0 * (1 + 5e-7), 1.0, 4.0]]])   # tokens 1 and 2 tie within 1e-6
    k = 3                                                      # oracle: {0, 4, 2}
    ok = compare_token_lists(np.array([[[0, 2, 4]]]), s, k)
    assert ok["mismatches"] == 0 and ok["excused_rows"] == 0
    tie = compare_token_lists(np.array([[[0, 1, 4]]]), s, k)
    assert tie["mismatches"] == 0 and tie["excused_rows"] == 1
    wrong = compare_token_lists(np.array([[[0, 3, 4]]]), s, k)
    assert wrong["mismatches"] == 1
    s2 = np.array([[[5.0, 3.0, 2.0, 1.0, 4.0]]])               # no tie: the threshold token is not excused
    assert compare_token_lists(np.array([[[0, 1, 4]]]), s2, k)["mismatches"] == 0
    assert compare_token_lists(np.array([[[0, 2, 4]]]), s2, k)["mismatches"] == 1
    with pytest.raises(AssertionError, match="padding"):
        compare_token_lists(np.array([[[0, 1, 4, 2]]]), s2, k)
