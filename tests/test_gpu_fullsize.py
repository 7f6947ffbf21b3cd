"""Full-size workloads (the shapes the benchmark times), checked on sampled heads.

The GPU runs the whole layer exactly as bench.py launches it; the oracle
recomputes the estimate, the masks and selected output blocks for a few
(batch, head) pairs, which it can do one by one.  Properties that hold at any
size (diagonal kept, counts, ascending lists) are checked on every row.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import LLAMA_32K, LLAMA_128K, QWEN_64K_B2, sweep
from oracle import prism_oracle as po
from tests.parity import compare_masks, rel_err, to_np

pytestmark = pytest.mark.gpu

FULL = [LLAMA_32K, LLAMA_128K, QWEN_64K_B2, sweep(0.01)]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled(w):
    dev = torch.device("cuda")
    Q, K, V = make_inputs(w, seed=0)
    model = sfa.PrismAttention(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                               head_dim=w.head_dim, dtype=w.dtype, block=w.block, rope_base=w.rope_base,
                               band_split=w.band_split, k=w.k, mass=w.mass, flags=w.flags, device=dev,
                               with_lse=True)
    model(Q.to(dev), K.to(dev), V.to(dev))
    torch.cuda.synchronize()
    assert int(model.status.item()) == 0
    nb = w.nb
    counts = model.counts.cpu().numpy()
    idx = model.idx.cpu().numpy()
    # any-size properties on every row
    ar = np.arange(nb)
    for b in range(w.batch):
        for h in range(w.heads_q):
            for i in (0, 1, nb // 3, nb - 1):
                n = counts[b, h, i]
                row = idx[b, h, i, :n]
                assert row[-1] == i and np.all(np.diff(row) > 0) and np.all(idx[b, h, i, n:] == -1)
    last = idx[np.arange(w.batch)[:, None, None], np.arange(w.heads_q)[None, :, None], ar[None, None, :],
                counts - 1]
    assert np.all(last == ar[None, None, :])
    if w.k is not None:
        assert np.all(counts == np.minimum(ar + 1, w.k + 1)[None, None, :])

    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    mass = None if w.mass is None else float(np.float32(w.mass))
    samples = [(0, 0), (w.batch - 1, w.heads_q - 1)]
    for b, h in samples:
        g = h // w.group
        Qh = to_np(Q[b:b + 1, h:h + 1])
        Kh = to_np(K[b:b + 1, g:g + 1])
        Vh = to_np(V[b:b + 1, g:g + 1])
        sc = po.prism_scores(Qh, Kh, w.block, w.band_split, w.flags, (cos, sin))
        P = model.probs[b, h].cpu().numpy()
        err = rel_err(np.tril(P).reshape(-1), np.tril(sc.probs[0, 0]).reshape(-1), floor=1e-35)
        print(f"{w.name} b={b} h={h}: max relative error of block probabilities {err:.3e}")
        assert err < 1e-6, f"block probabilities: max relative error {err:.3e}"
        sel = po.select_blocks(sc.probs, w.flags, k=w.k, mass=mass)
        stats, exact = compare_masks(sel, sc.probs, model.counts[b:b + 1, h:h + 1], model.idx[b:b + 1, h:h + 1],
                                     mass)
        print(f"{w.name} b={b} h={h}: near-tie rows {stats['uncertain_rows']}, "
              f"threshold-only excusals {stats['threshold_only_rows']}")
        assert stats["mismatches"] == 0, stats["bad_rows"][:5]
        # outputs of a few query blocks whose masks agree exactly
        want = [i for i in (0, 1, nb // 2, nb - 1) if exact[0, 0, i]]
        assert len(want) >= 3
        kept = [[[sel[0][0][i].kept if i in want else np.zeros(0, np.int64) for i in range(nb)]]]
        qa = po.round_to_dtype(po.apply_rope(Qh, cos, sin), w.dtype)
        ka = po.round_to_dtype(po.apply_rope(Kh, cos, sin), w.dtype)
        Oref, lref = po.sparse_attention(qa, ka, Vh, kept, w.block)
        Og = to_np(model.O[b, h]).astype(np.float64)
        lg = model.lse[b, h].cpu().numpy()
        for i in want:
            sl = slice(i * w.block, (i + 1) * w.block)
            np.testing.assert_allclose(Og[sl], Oref[0, 0, sl], rtol=0, atol=2e-2)
            np.testing.assert_allclose(lg[sl], lref[0, 0, sl], rtol=0, atol=2e-2)
