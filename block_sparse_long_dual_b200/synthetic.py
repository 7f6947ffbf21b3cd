"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This module generates input tensors only; it holds none of the method's
arithmetic.  Recipe (pre-RoPE Q, K, V, layout [B, H, L, d]):

* ``torch.Generator().manual_seed(seed)``; Q, K, V drawn N(0, 1) in float32,
  head by head, then cast to the workload dtype (bf16 is round-to-nearest-even).
* Semantic component (low band, "global semantics" of
  "Prism: Spectral-Aware Block-Sparse Attention" §3.1): u ~ N(0, 1) from seed 1
  on the low-band dims only; 0.5 * u is added to every Q token and to every
  token of a planted key-block set P drawn uniformly from blocks 1..nb-1 with
  seed 2.  |P| = round(planted_frac * nb).  Shared by all heads.
* Slash component (high band, "local relative position", same §3.1): a
  constant c ~ N(0, 1) from seed 3 on the high-band dims, added to every Q and
  K token.  After RoPE, q.k gains sum_m |c_m|^2 cos((p_q - p_k) theta_m): a
  recency diagonal that block mean pooling attenuates (§2).

Decode inputs (``make_decode_inputs``; "FASA: Frequency-aware Sparse
Attention" §2B): q [B, Hq, d], K, V [B, Hkv, L, d] drawn N(0, 1) from
``seed`` and cast to bf16 (K and q stand for already-rotated values: a random
vector's rotation is again random).  Dominant pairs ``fc`` [Hkv, nfc]: nfc
distinct pairs per KV head drawn with seed 5 (a stand-in for the offline
calibration the page describes).  Needles: round(needle_frac * L) tokens per
(b, KV head), drawn with seed 6, get 2 x the group's mean query added on that
head's dominant dims, so the estimate has real winners to find.  With
``dominant_gain`` != 1 the dominant dims of q and K are scaled by it (a cache
whose attention scores are carried mostly by a few frequency pairs, the
premise of the page's §2A); the bench inputs use 1.
"""

from __future__ import annotations

import torch

from .workloads import DecodeWorkload, Workload


def _band_dims(head_dim: int, band_split: int):
    half = head_dim // 2
    high = torch.zeros(head_dim, dtype=torch.bool)
    high[:band_split] = True
    high[half:half + band_split] = True
    return high, ~high


def planted_blocks(w: Workload) -> torch.Tensor:
    n = int(round(w.planted_frac * w.nb))
    if n == 0 or w.nb < 2:
        return torch.zeros(0, dtype=torch.long)
    g = torch.Generator().manual_seed(2)
    perm = torch.randperm(w.nb - 1, generator=g)[:n] + 1
    return torch.sort(perm).values


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu"):
    """Q [B,Hq,L,d], K [B,Hkv,L,d], V [B,Hkv,L,d] in the workload dtype on ``device``."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(seed)
    high, low = _band_dims(w.head_dim, w.band_split)
    sem = torch.zeros(w.head_dim)
    if w.planted_frac > 0:
        gu = torch.Generator().manual_seed(1)
        sem = torch.randn(w.head_dim, generator=gu) * low
    slash = torch.zeros(w.head_dim)
    if w.slash:
        gc = torch.Generator().manual_seed(3)
        slash = torch.randn(w.head_dim, generator=gc) * high
    P = planted_blocks(w)
    tokmask = torch.zeros(w.seq_len, dtype=torch.bool)
    for j in P.tolist():
        tokmask[j * w.block:(j + 1) * w.block] = True

    def draw(heads, add_all, add_planted):
        out = torch.empty((w.batch, heads, w.seq_len, w.head_dim), dtype=dt, device=device)
        for b in range(w.batch):
            for h in range(heads):
                x = torch.randn((w.seq_len, w.head_dim), generator=g)
                if add_all is not None:
                    x += add_all
                if add_planted is not None and P.numel():
                    x[tokmask] += add_planted
                out[b, h].copy_(x.to(dt))
        return out

    q_add = 0.5 * sem + slash if (w.planted_frac > 0 or w.slash) else None
    k_all = slash if w.slash else None
    k_pl = 0.5 * sem if w.planted_frac > 0 else None
    Q = draw(w.heads_q, q_add, None)
    K = draw(w.heads_kv, k_all, k_pl)
    V = draw(w.heads_kv, None, None)
    return Q, K, V


def decode_fc(w: DecodeWorkload):
    """Dominant pair lists [Hkv, nfc] (int64, sorted per head)."""
    g = torch.Generator().manual_seed(5)
    rows = [torch.sort(torch.randperm(w.head_dim // 2, generator=g)[:w.nfc]).values for _ in range(w.heads_kv)]
    return torch.stack(rows).numpy()


def make_decode_inputs(w: DecodeWorkload, seed: int = 0, device: str | torch.device = "cpu"):
    """q [B,Hq,d], K [B,Hkv,L,d], V [B,Hkv,L,d] bf16 on ``device``, and fc [Hkv, nfc]."""
    g = torch.Generator().manual_seed(seed)
    fc = decode_fc(w)
    q = torch.randn((w.batch, w.heads_q, w.head_dim), generator=g)
    half = w.head_dim // 2
    if w.dominant_gain != 1.0:
        for h in range(w.heads_q):
            dims = torch.cat([torch.as_tensor(fc[h // w.group]), torch.as_tensor(fc[h // w.group]) + half])
            q[:, h, dims] *= w.dominant_gain
    K = torch.empty((w.batch, w.heads_kv, w.seq_len, w.head_dim), dtype=torch.bfloat16, device=device)
    V = torch.empty_like(K)
    gn = torch.Generator().manual_seed(6)
    nneedle = int(round(w.needle_frac * w.seq_len))
    for b in range(w.batch):
        for h in range(w.heads_kv):
            x = torch.randn((w.seq_len, w.head_dim), generator=g)
            if w.dominant_gain != 1.0:
                x[:, torch.cat([torch.as_tensor(fc[h]), torch.as_tensor(fc[h]) + half])] *= w.dominant_gain
            if nneedle:
                dims = torch.cat([torch.as_tensor(fc[h]), torch.as_tensor(fc[h]) + half])
                qm = q[b, h * w.group:(h + 1) * w.group].mean(0)
                pos = torch.randperm(w.seq_len, generator=gn)[:nneedle]
                x[pos[:, None], dims[None, :]] += 2.0 * qm[dims]
            K[b, h].copy_(x.to(torch.bfloat16))
            V[b, h].copy_(torch.randn((w.seq_len, w.head_dim), generator=g).to(torch.bfloat16))
    return q.to(torch.bfloat16).to(device), K, V, fc
