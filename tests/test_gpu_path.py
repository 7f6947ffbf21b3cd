"""GPU path vs the CPU oracle on small seeded workloads (several tiles, ragged tails).

Every call goes through the C-ABI library (via the ctypes binding).  The same
seeded host tensors feed both sides; nothing the GPU computes is fed back into
the oracle.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import (BAND_MAX, BLOCK_TAU, KEEP_SINK, NO_CALIB, RELATIVE_CALIB,
                                                   SINGLE_BAND, TINY, Workload)
from oracle import prism_oracle as po
from tests.parity import compare_masks, rel_err, to_np

pytestmark = pytest.mark.gpu

TOL_O = {"bf16": 2e-2, "f32": 1e-4}


def W(name, **kw):
    base = dict(batch=1, heads_q=4, heads_kv=2, seq_len=2048, head_dim=128, dtype="bf16", block=128,
                rope_base=5e5, band_split=32, k=3, planted_frac=0.25)
    base.update(kw)
    return Workload(name=name, **base)


CASES = [
    TINY,
    W("bf16-topk-b2", batch=2),
    W("bf16-mass-ragged", heads_q=4, heads_kv=1, seq_len=21 * 128, k=None, mass=0.9, slash=True, rope_base=1e6),
    W("bf16-sink-nocalib", seq_len=19 * 128, k=2, flags=KEEP_SINK | NO_CALIB),
    W("bf16-single-band-k0", k=0, flags=SINGLE_BAND),
    W("bf16-topk-all", seq_len=8 * 128, k=100),
    W("bf16-mass-one", seq_len=9 * 128, k=None, mass=1.0),
    W("f32-d128-b128", dtype="f32", seq_len=10 * 128, k=2),
    W("bf16-d64-b64", head_dim=64, block=64, band_split=16, seq_len=33 * 64, k=4, flags=KEEP_SINK),
    W("f32-d128-b64-mass", dtype="f32", block=64, seq_len=24 * 64, k=None, mass=0.5, slash=True),
    W("bf16-one-block", seq_len=128, k=1),
    W("bf16-relative-calib-mass", seq_len=12 * 128, k=None, mass=0.9, slash=True, flags=RELATIVE_CALIB),
    W("bf16-relative-calib-single", seq_len=6 * 128, k=2, flags=RELATIVE_CALIB | SINGLE_BAND | KEEP_SINK),
    W("bf16-band-max-mass", seq_len=14 * 128, k=None, mass=0.9, slash=True, flags=BAND_MAX),
    W("bf16-band-max-topk-sink", seq_len=11 * 128, k=3, flags=BAND_MAX | KEEP_SINK),
    W("bf16-block-tau-topk", seq_len=12 * 128, k=3, flags=BLOCK_TAU),
    W("bf16-block-tau-band-max-mass", seq_len=10 * 128, k=None, mass=0.8, slash=True, flags=BLOCK_TAU | BAND_MAX),
    W("f32-d64-b64-band-max-block-tau", dtype="f32", head_dim=64, block=64, band_split=16, seq_len=20 * 64, k=2,
      flags=BAND_MAX | BLOCK_TAU),
    W("bf16-band-max-single-band", seq_len=5 * 128, k=1, flags=BAND_MAX | SINGLE_BAND),
]


def run_both(w: Workload, seed=0):
    Q, K, V = make_inputs(w, seed=seed)
    dev = torch.device("cuda")
    model = sfa.PrismAttention(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                               head_dim=w.head_dim, dtype=w.dtype, block=w.block, rope_base=w.rope_base,
                               band_split=w.band_split, k=w.k, mass=w.mass, flags=w.flags, device=dev,
                               with_lse=True)
    model(Q.to(dev), K.to(dev), V.to(dev))
    torch.cuda.synchronize()
    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    mass = None if w.mass is None else float(np.float32(w.mass))
    ref = po.prism_path(to_np(Q), to_np(K), to_np(V), block=w.block, band_split=w.band_split, flags=w.flags,
                        k=w.k, mass=mass, rope=(cos, sin), dtype=w.dtype)
    return model, ref, mass


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_path_matches_oracle(w):
    model, ref, mass = run_both(w)
    assert int(model.status.item()) == 0
    sc = ref.scores

    # a1: rotated Q/K as stored for the attention (rounded to the input dtype)
    for got, want in ((model.Q_rot, ref.q_attn), (model.K_rot, ref.k_attn)):
        g = to_np(got).astype(np.float64)
        if w.dtype == "bf16":
            # one bf16 ulp of the value, plus the float32 rounding of x*c - y*s when it cancels
            ulp = np.abs(want) * 2.0 ** -7 * 1.01 + 2e-6
            diff = np.abs(g - want)
            assert np.all(diff <= ulp), "rotated values differ by more than one bf16 ulp"
            assert np.mean(diff > 0) < 1e-3
        else:
            np.testing.assert_allclose(g, want, rtol=0, atol=2e-6)

    # a2/a3: block means, energies, temperatures (diagnostic tolerances at float32 rounding)
    qbar, kbar, energy, tau = sfa.workspace_views(model.workspace, model.shape, w.block)
    np.testing.assert_allclose(to_np(qbar), sc.qbar, rtol=0, atol=1e-7)
    np.testing.assert_allclose(to_np(kbar), sc.kbar, rtol=0, atol=1e-7)
    e = to_np(energy)
    np.testing.assert_allclose(e[:, :w.heads_q, :, :2], sc.tok_energy_q, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(e[:, w.heads_q:, :, :2], sc.tok_energy_k, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(to_np(tau), sc.tau, rtol=1e-7, atol=0)

    # a4: probabilities (relative error of the float32 output vs float64)
    P = to_np(model.probs)
    assert np.all(np.triu(P, 1) == 0)
    err = rel_err(np.tril(P).reshape(-1), np.tril(sc.probs).reshape(-1), floor=1e-35)
    print(f"{w.name}: max relative error of block probabilities {err:.3e}")
    assert err < 1e-6, f"max relative error of block probabilities {err:.3e}"

    # a5: masks identical except near-ties at the row threshold
    stats, exact = compare_masks(ref.selection, sc.probs, model.counts, model.idx, mass)
    print(f"{w.name}: rows {stats['rows']}, near-tie rows excused {stats['excused_rows']} "
          f"(count differs {stats['count_diff_rows']})")
    assert stats["mismatches"] == 0, stats["bad_rows"][:5]
    assert stats["threshold_only_rows"] == 0
    if w.k is not None:
        assert stats["count_diff_rows"] == 0

    # a6: outputs on rows whose kept set equals the oracle's
    O = to_np(model.O).astype(np.float64)
    lse = to_np(model.lse)
    nb = w.nb
    rows = np.repeat(exact, w.block, axis=-1)  # [B, H, L]
    assert rows.mean() > 0.9
    np.testing.assert_allclose(O[rows], ref.out[rows], rtol=0, atol=TOL_O[w.dtype])
    np.testing.assert_allclose(lse[rows], ref.lse[rows], rtol=0, atol=TOL_O[w.dtype])


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fused_scores_select_matches(w):
    """sfa_block_scores_select: the same index lists as sfa_block_scores + sfa_select (bit for
    bit), with and without the probabilities stored, and the oracle's masks."""
    Q, K, V = make_inputs(w, seed=1)
    dev = torch.device("cuda")
    kw = dict(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len, head_dim=w.head_dim,
              dtype=w.dtype, block=w.block, rope_base=w.rope_base, band_split=w.band_split, k=w.k, mass=w.mass,
              flags=w.flags, device=dev)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    sep = sfa.PrismAttention(**kw)
    fused = sfa.PrismAttention(**kw, fused=True)
    assert fused.probs is None
    sep(Qd, Kd, Vd)
    fused.idx.fill_(-7)
    fused(Qd, Kd, Vd)
    torch.cuda.synchronize()
    assert torch.equal(sep.counts, fused.counts)
    assert torch.equal(sep.idx, fused.idx)
    assert torch.equal(sep.Q_rot, fused.Q_rot) and torch.equal(sep.K_rot, fused.K_rot)
    assert torch.equal(sep.O, fused.O)
    assert int(fused.status.item()) == 0

    # probabilities requested from the fused call: identical to sfa_block_scores'
    mass = None if w.mass is None else float(np.float32(w.mass))
    _, _, P, counts, idx, _ = sfa.block_scores_select(Qd, Kd, sep.cos, sep.sin, band_split=w.band_split,
                                                      block=w.block, k=w.k, mass=w.mass, flags=w.flags,
                                                      want_probs=True)
    torch.cuda.synchronize()
    assert torch.equal(P, sep.probs)
    assert torch.equal(counts, sep.counts) and torch.equal(idx, sep.idx)

    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    sc = po.prism_scores(to_np(Q), to_np(K), w.block, w.band_split, w.flags, (cos, sin))
    sel = po.select_blocks(sc.probs, w.flags, k=w.k, mass=mass)
    stats, _ = compare_masks(sel, sc.probs, fused.counts, fused.idx, mass)
    assert stats["mismatches"] == 0, stats["bad_rows"][:5]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_rope_on_load_matches(w):
    """sfa_block_sparse_attn_rope on pre-RoPE Q (Q_rot never stored) gives the same O and lse,
    bit for bit, as sfa_block_sparse_attn on the stored Q_rot; alone and with the fused selection."""
    Q, K, V = make_inputs(w, seed=2)
    dev = torch.device("cuda")
    kw = dict(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len, head_dim=w.head_dim,
              dtype=w.dtype, block=w.block, rope_base=w.rope_base, band_split=w.band_split, k=w.k, mass=w.mass,
              flags=w.flags, device=dev, with_lse=True)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    for fused in (False, True):
        ref = sfa.PrismAttention(**kw, fused=fused)
        ref(Qd, Kd, Vd)
        rol = sfa.PrismAttention(**kw, rope_on_load=True, fused=fused)
        assert rol.Q_rot is None
        rol.O.fill_(7)
        rol(Qd, Kd, Vd)
        torch.cuda.synchronize()
        assert int(rol.status.item()) == 0
        assert torch.equal(ref.K_rot, rol.K_rot)
        assert torch.equal(ref.counts, rol.counts) and torch.equal(ref.idx, rol.idx)
        assert torch.equal(ref.O, rol.O), f"fused={fused}: O differs"
        assert torch.equal(ref.lse, rol.lse), f"fused={fused}: lse differs"
