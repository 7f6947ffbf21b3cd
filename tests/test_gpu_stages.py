"""Stage-level parity: sfa_select and sfa_block_sparse_attn on shared seeded inputs.

The selection is integer output decided by float32 comparisons, so both sides
take the same float32 probabilities as input and must agree bit for bit.  The
attention takes seeded Q/K/V and seeded index lists.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from oracle import prism_oracle as po
from tests.parity import random_index_lists, to_np

pytestmark = pytest.mark.gpu


def synthetic_probs(B, H, nb, seed, quantize=None):
    """Causal row-softmax matrices in float32 (seeded); optional quantisation creates exact ties."""
    g = torch.Generator().manual_seed(seed)
    s = torch.randn((B, H, nb, nb), generator=g, dtype=torch.float64) * 2.0
    mask = torch.ones(nb, nb, dtype=torch.bool).tril()
    p = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
    if quantize:
        p = torch.round(p * quantize) / quantize
    return p.to(torch.float32)


SEL_CASES = [
    # (B, H, nb, k, mass, flags, quantize)
    (1, 2, 37, 5, None, 0, None),
    (1, 2, 37, 0, None, 1, None),
    (2, 1, 64, 3, None, 1, 64.0),
    (1, 3, 50, 100, None, 0, None),
    (1, 2, 40, None, 0.9, 0, None),
    (1, 2, 40, None, 0.5, 1, 32.0),
    (1, 1, 33, None, 1.0, 0, None),
    (1, 1, 2048, 25, None, 0, None),
    (1, 1, 1024, None, 0.9, 1, None),
]


@pytest.mark.parametrize("case", SEL_CASES, ids=lambda c: f"nb{c[2]}-k{c[3]}-m{c[4]}-f{c[5]}-q{c[6]}")
def test_select_bit_exact(case):
    B, H, nb, k, mass, flags, quant = case
    P = synthetic_probs(B, H, nb, seed=nb * 7 + H, quantize=quant)
    block = 128
    shape = sfa.Shape(B, H, H, nb * block, 128, sfa.BF16)
    counts, idx = sfa.select(P.cuda(), shape, block=block, k=k, mass=mass, flags=flags)
    torch.cuda.synchronize()
    m32 = None if mass is None else float(np.float32(mass))
    P64 = P.numpy().astype(np.float64)
    sel = po.select_blocks(P64, flags, k=k, mass=m32)
    counts = counts.cpu().numpy()
    idx = idx.cpu().numpy()
    kmax = idx.shape[-1]
    skipped = 0
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                r = sel[b][h][i]
                if (quant is None and mass is not None and r.n_taken > 0
                        and (abs(r.cum_before_last - m32) < 1e-12 or abs(r.cum_final - m32) < 1e-12)):
                    # non-dyadic values: float64 sums in another order may land on either side of mass
                    skipped += 1
                    continue
                n = counts[b, h, i]
                assert n == r.kept.size, (b, h, i)
                assert list(idx[b, h, i, :n]) == list(r.kept), (b, h, i)
                assert np.all(idx[b, h, i, n:] == -1)
    assert skipped <= 2


ATT_CASES = [
    # (dtype, B, Hq, Hkv, nb, block, d, causal)
    ("bf16", 1, 4, 2, 9, 128, 128, True),
    ("bf16", 2, 2, 1, 5, 128, 128, False),
    ("f32", 1, 2, 1, 7, 64, 64, True),
    ("f32", 1, 2, 2, 5, 128, 128, True),
    ("bf16", 1, 2, 1, 6, 64, 128, True),
    ("bf16", 1, 1, 1, 7, 128, 128, True),     # odd number of query tiles, no GQA
    ("bf16", 1, 3, 1, 3, 128, 128, False),    # group of 3: tile pairs straddle query blocks
]


@pytest.mark.parametrize("case", ATT_CASES, ids=lambda c: "-".join(map(str, c)))
def test_attention_stage(case):
    dt, B, Hq, Hkv, nb, block, d, causal = case
    L = nb * block
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    g = torch.Generator().manual_seed(123 + nb)
    Q, K, V = (torch.randn((B, h, L, d), generator=g).to(tdt) for h in (Hq, Hkv, Hkv))
    rng = np.random.default_rng(nb)
    kmax = nb + 2
    counts, idx, kept = random_index_lists(rng, B, Hq, nb, kmax, causal=causal, p_keep=0.4,
                                           empty_rows={(0, 0, 2)}, diag_only_rows={(0, 1, nb - 1)})
    dev = torch.device("cuda")
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    O = sfa.block_sparse_attn(Q.to(dev), K.to(dev), V.to(dev), torch.from_numpy(counts).to(dev),
                              torch.from_numpy(idx).to(dev), block=block, causal=causal, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Oref, lref = po.sparse_attention(to_np(Q), to_np(K), to_np(V), kept, block, causal=causal)
    tol = 2e-2 if dt == "bf16" else 1e-4
    np.testing.assert_allclose(to_np(O), Oref, rtol=0, atol=tol)
    lg = lse.cpu().numpy()
    fin = np.isfinite(lref)
    np.testing.assert_array_equal(np.isfinite(lg), fin)
    np.testing.assert_allclose(lg[fin], lref[fin], rtol=0, atol=tol)
    # the empty row is exactly zero
    assert np.all(to_np(O)[0, 0, 2 * block:3 * block] == 0)


@pytest.mark.parametrize("dt,block,d", [("bf16", 128, 128), ("f32", 64, 64)])
def test_attention_rejects_bad_index_lists(dt, block, d):
    """Lists that are not ascending / out of range / above the diagonal set SFA_ERR_INDEX; the tile is zero."""
    B, H, nb = 1, 1, 4
    L = nb * block
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(5)
    Q, K, V = (torch.randn((B, H, L, d), generator=g).to(tdt).to(dev) for _ in range(3))
    kmax = 3
    idx = torch.full((B, H, nb, kmax), -1, dtype=torch.int32)
    counts = torch.ones((B, H, nb), dtype=torch.int32)
    for i in range(nb):
        idx[0, 0, i, 0] = i
    idx[0, 0, 1, :2] = torch.tensor([1, 0])      # descending
    counts[0, 0, 1] = 2
    idx[0, 0, 2, 0] = 3                           # above the diagonal (causal)
    idx[0, 0, 3, :2] = torch.tensor([0, 9])      # out of range
    counts[0, 0, 3] = 2
    counts[0, 0, 0] = 5                           # count > kmax
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    O = sfa.block_sparse_attn(Q, K, V, counts.to(dev), idx.to(dev), block=block, causal=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 8
    assert torch.all(O.float() == 0).item()


def test_attention_bad_list_beside_a_good_one_two_tile_layout():
    """kmax above the short-list cut: two query tiles per CTA (two Q heads of a GQA group at one
    query block).  A tile whose list is invalid is zeroed and flagged while its CTA partner is
    computed exactly as in a call where the bad list is simply empty."""
    B, Hq, Hkv, nb, block, d = 1, 2, 1, 4, 128, 128
    L = nb * block
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(11)
    Q = torch.randn((B, Hq, L, d), generator=g).to(torch.bfloat16).to(dev)
    K, V = (torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16).to(dev) for _ in range(2))
    kmax = 16
    idx = torch.full((B, Hq, nb, kmax), -1, dtype=torch.int32)
    counts = torch.zeros((B, Hq, nb), dtype=torch.int32)
    for h in range(Hq):
        for i in range(nb):
            idx[0, h, i, :i + 1] = torch.arange(i + 1, dtype=torch.int32)
            counts[0, h, i] = i + 1
    bad_idx, bad_counts = idx.clone(), counts.clone()
    bad_idx[0, 0, 2, :3] = torch.tensor([1, 0, 2], dtype=torch.int32)  # head 0, block 2: not ascending
    bad_idx[0, 1, 3, 1] = 7                                             # head 1, block 3: out of range
    good_counts = counts.clone()
    good_counts[0, 0, 2] = 0
    good_counts[0, 1, 3] = 0
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    O_bad = sfa.block_sparse_attn(Q, K, V, bad_counts.to(dev), bad_idx.to(dev), block=block, causal=True,
                                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 8
    status.zero_()
    O_good = sfa.block_sparse_attn(Q, K, V, good_counts.to(dev), idx.to(dev), block=block, causal=True,
                                   status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = lambda i: slice(i * block, (i + 1) * block)
    assert torch.all(O_bad[0, 0, rows(2)].float() == 0).item()
    assert torch.all(O_bad[0, 1, rows(3)].float() == 0).item()
    assert torch.equal(O_bad, O_good)
    assert O_good[0, 0, rows(3)].float().abs().sum().item() > 0  # a partner tile was computed
