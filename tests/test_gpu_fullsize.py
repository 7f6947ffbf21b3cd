"""Full-size workloads (the shapes the benchmark times), checked on sampled heads.

The GPU runs the whole layer exactly as bench.py launches it; the oracle
recomputes the estimate, the masks and selected output blocks for a few
(batch, head) pairs, which it can do one by one.  Properties that hold at any
size (diagonal kept, counts, ascending lists) are checked on every row.  The
100% density point of the sweep is also checked against dense causal attention
written out here (softmax over every earlier token), independently of the
oracle's block-sparse routine.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import LLAMA_32K, LLAMA_128K, QWEN_64K_B2, Workload, sweep
from oracle import prism_oracle as po
from tests.parity import compare_masks, rel_err, to_np

pytestmark = pytest.mark.gpu

FULL = [LLAMA_32K, LLAMA_128K, QWEN_64K_B2, sweep(0.01), sweep(0.25), sweep(1.0)]

# (batch, Q head) pairs the oracle recomputes, and query blocks whose outputs it compares
HEADS = {LLAMA_128K.name: [(0, h) for h in (0, 5, 10, 15, 20, 25, 30, 31)]}


def query_blocks(w: Workload) -> list:
    nb = w.nb
    if w.name == LLAMA_128K.name:
        mid = np.linspace(2, nb - 5, 10).astype(int).tolist()
        return sorted(set([0, 1] + mid + list(range(nb - 4, nb))))
    return sorted(set([0, 1, nb // 2, nb - 2, nb - 1]))


def check_any_size(w: Workload, counts: np.ndarray, idx: np.ndarray):
    """Every row: ascending, diagonal last, -1 padding; top-k counts are min(i + 1, k + 1)."""
    nb = w.nb
    ar = np.arange(nb)
    kmax = idx.shape[-1]
    pos = np.arange(kmax)[None, None, None, :]
    valid = pos < counts[..., None]
    assert np.all(np.where(valid, idx >= 0, idx == -1)), "entries past the count must be -1"
    d = np.diff(idx, axis=-1)
    assert np.all(np.where(valid[..., 1:], d > 0, True)), "kept lists must be ascending"
    last = np.take_along_axis(idx, (counts - 1)[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(last == ar[None, None, :]), "the diagonal block must be the last kept entry"
    if w.k is not None:
        assert np.all(counts == np.minimum(ar + 1, w.k + 1)[None, None, :])


def dense_causal_block(qa, ka, v, i, block, scale):
    """Dense causal softmax attention of query block i over every earlier token (float64)."""
    tq = np.arange(i * block, (i + 1) * block)
    s = (qa[tq] @ ka[:(i + 1) * block].T) * scale
    s = np.where(np.arange((i + 1) * block)[None, :] <= tq[:, None], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    den = e.sum(axis=1, keepdims=True)
    return (e @ v[:(i + 1) * block]) / den, (m + np.log(den))[:, 0]


def run_model(w: Workload, fused=False):
    dev = torch.device("cuda")
    Q, K, V = make_inputs(w, seed=0)
    model = sfa.PrismAttention(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                               head_dim=w.head_dim, dtype=w.dtype, block=w.block, rope_base=w.rope_base,
                               band_split=w.band_split, k=w.k, mass=w.mass, flags=w.flags, device=dev,
                               with_lse=True, fused=fused)
    model(Q.to(dev), K.to(dev), V.to(dev))
    torch.cuda.synchronize()
    assert int(model.status.item()) == 0
    return model, Q, K, V


def check_heads(w: Workload, model, Q, K, V, samples, blocks, dense=False):
    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    mass = None if w.mass is None else float(np.float32(w.mass))
    scale = 1.0 / math.sqrt(w.head_dim)
    for b, h in samples:
        g = h // w.group
        Qh = to_np(Q[b:b + 1, h:h + 1])
        Kh = to_np(K[b:b + 1, g:g + 1])
        Vh = to_np(V[b:b + 1, g:g + 1])
        sc = po.prism_scores(Qh, Kh, w.block, w.band_split, w.flags, (cos, sin))
        if model.probs is not None:
            P = model.probs[b, h].cpu().numpy()
            err = rel_err(np.tril(P).reshape(-1), np.tril(sc.probs[0, 0]).reshape(-1), floor=1e-35)
            print(f"{w.name} b={b} h={h}: max relative error of block probabilities {err:.3e}")
            assert err < 1e-6, f"block probabilities: max relative error {err:.3e}"
        sel = po.select_blocks(sc.probs, w.flags, k=w.k, mass=mass)
        stats, exact = compare_masks(sel, sc.probs, model.counts[b:b + 1, h:h + 1], model.idx[b:b + 1, h:h + 1],
                                     mass)
        print(f"{w.name} b={b} h={h}: near-tie rows excused {stats['excused_rows']} "
              f"(count differs {stats['count_diff_rows']})")
        assert stats["mismatches"] == 0, stats["bad_rows"][:5]
        assert stats["threshold_only_rows"] == 0
        # outputs of the sampled query blocks whose masks agree exactly
        want = [i for i in blocks if exact[0, 0, i]]
        assert len(want) >= len(blocks) - 1
        kept = [[[sel[0][0][i].kept if i in want else np.zeros(0, np.int64) for i in range(w.nb)]]]
        qa = po.round_to_dtype(po.apply_rope(Qh, cos, sin), w.dtype)
        ka = po.round_to_dtype(po.apply_rope(Kh, cos, sin), w.dtype)
        Oref, lref = po.sparse_attention(qa, ka, Vh, kept, w.block)
        Og = to_np(model.O[b, h]).astype(np.float64)
        lg = model.lse[b, h].cpu().numpy()
        for i in want:
            sl = slice(i * w.block, (i + 1) * w.block)
            np.testing.assert_allclose(Og[sl], Oref[0, 0, sl], rtol=0, atol=2e-2)
            np.testing.assert_allclose(lg[sl], lref[0, 0, sl], rtol=0, atol=2e-2)
            if dense:
                od, ld = dense_causal_block(qa[0, 0], ka[0, 0], Vh[0, 0], i, w.block, scale)
                np.testing.assert_allclose(Og[sl], od, rtol=0, atol=2e-2)
                np.testing.assert_allclose(lg[sl], ld, rtol=0, atol=2e-2)


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled(w):
    model, Q, K, V = run_model(w)
    check_any_size(w, model.counts.cpu().numpy(), model.idx.cpu().numpy())
    samples = HEADS.get(w.name, [(0, 0), (w.batch - 1, w.heads_q - 1)])
    dense = w.density is not None and w.density >= 1.0
    if dense:
        assert np.all(model.counts.cpu().numpy() == np.arange(1, w.nb + 1)[None, None, :])
    check_heads(w, model, Q, K, V, samples, query_blocks(w), dense=dense)


# The longest sequence the prefill calls accept at block 128 (nb = 2048): one head, so the 8-row
# instantiations of the block-score kernel (unfused, and fused with 64 probabilities per lane) run.
LONGEST = Workload(name="1h-256k-nb2048", batch=1, heads_q=1, heads_kv=1, seq_len=262144, head_dim=128,
                   dtype="bf16", block=128, rope_base=5e5, band_split=32, k=25, planted_frac=0.05)


@pytest.mark.parametrize("fused,mass", [(False, None), (True, None), (True, 0.9)],
                         ids=["unfused-topk", "fused-topk", "fused-mass"])
def test_longest_sequence_one_head(fused, mass):
    w = LONGEST if mass is None else LONGEST.scaled(k=None, mass=mass)
    model, Q, K, V = run_model(w, fused=fused)
    assert (model.probs is None) == fused
    check_any_size(w, model.counts.cpu().numpy(), model.idx.cpu().numpy())
    check_heads(w, model, Q, K, V, [(0, 0)], [0, 1, 700, 1500, w.nb - 2, w.nb - 1])
