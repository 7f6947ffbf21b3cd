"""CPU oracle for the decode-side analogue of the estimate -> exact-attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library and computes in float64 from
the same seeded host arrays the GPU receives.

What it restates (source: "FASA: Frequency-aware Sparse Attention", §2):

* §2A: RoPE splits each head into frequency chunks; a few "dominant" chunks
  carry the head's context selection, and which ones is fixed per head by a
  one-time offline calibration.
* §2B.1 Token Importance Predictor (TIP): the attention score of the current
  query against every cached key is estimated from the dominant chunks only;
  the highest-scoring tokens form the subset T_t.
* §2B.2 Focused Attention Computation (FAC): full-dimension attention of the
  query over T_t only, with the tokens' original (absolute) positions, i.e.
  the cached rotated keys as they are.
* §2C FASA-C: everything stays on the GPU and only the dominant part of the
  keys is read for the estimate.

Readings (the page gives no formulas; listed with reasons in the design notes):

D1  A frequency chunk is one rotary pair (m, m + d/2) of the rotate-half
    convention; ``fc`` [Hkv, nfc] lists each KV head's dominant pairs (the
    calibration itself is out of scope: the list is an input).  The Q heads of a
    GQA group share their KV head's list, so one compact key copy serves the group.
D2  TIP score of Q head h for cached token t:
        s_t = sum_{m in fc[g(h)]} q_m k_{t,m} + q_{m+d/2} k_{t,m+d/2}
    from the rotated query (at the newest position) and the rotated cache.
    The page fixes no precision and no summation order, so the ranked value
    is the dot product itself: ``tip_scores`` in float64 (each bf16 x bf16
    product is exact there, and so is the sum of the few dozen products
    unless their magnitudes span more than ~30 binades).  ``tip_keys``, a
    float32 running sum in column order, is a diagnostic only (the error a
    float32 estimate makes), not what is ranked.
D3  T_t = the first min(k, L) tokens in the order (score desc, index asc),
    output ascending, padded with -1.  No forced tokens (the page names none).
D4  FAC: o = sum_{t in T_t} softmax_t(scale * q . k_t) v_t over all d dims,
    lse = log sum_t exp(scale * q . k_t); scale = 1/sqrt(d) by default.
D5  The compact key copy K_fc [B, Hkv, L, 2 nfc] holds, per token, the low
    dims fc[c] (c < nfc) then the high dims fc[c] + d/2 (FASA-C's "only the
    dominant part of the keys is read").

Pins (tests/test_fasa_oracle_pins.py): all pairs dominant equals the full q.k
(torch), all tokens kept equals dense single-query attention (torch SDPA), one
kept token gives o = v exactly, TIP scores invariant under a common shift of
positions (RoPE through transformers' rotate_half), brute-force subset
selection on tiny caches, and the K_fc layout against the full-cache TIP.
"""

from __future__ import annotations

import math

import numpy as np


def fc_dims(fc_row: np.ndarray, head_dim: int) -> np.ndarray:
    """D1/D5: dims of a dominant-pair list, low halves first then their partners."""
    fc_row = np.asarray(fc_row, dtype=np.int64)
    return np.concatenate([fc_row, fc_row + head_dim // 2])


def gather_fc(K: np.ndarray, fc: np.ndarray) -> np.ndarray:
    """D5: compact dominant-dims copy K_fc [B, Hkv, L, 2 nfc] of K [B, Hkv, L, d]."""
    K = np.asarray(K)
    d = K.shape[-1]
    return np.stack([K[:, g][..., fc_dims(fc[g], d)] for g in range(K.shape[1])], axis=1)


def tip_scores(q: np.ndarray, K: np.ndarray, fc: np.ndarray) -> np.ndarray:
    """D2: float64 TIP scores [B, Hq, L] of q [B, Hq, d] against the full cache K [B, Hkv, L, d]."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    group = Hq // Hkv
    out = np.zeros((B, Hq, K.shape[2]))
    for h in range(Hq):
        g = h // group
        dims = fc_dims(fc[g], d)
        out[:, h] = np.einsum("bd,btd->bt", q[:, h][:, dims], K[:, g][..., dims])
    return out


def tip_keys(q: np.ndarray, K: np.ndarray, fc: np.ndarray) -> np.ndarray:
    """Diagnostic, not ranked: the TIP score as a float32 running sum over the compact columns in
    order [B, Hq, L], starting from 0, each step rounding (sum + q_c * k_c) once."""
    q = np.asarray(q, dtype=np.float32)
    K = np.asarray(K, dtype=np.float32)
    B, Hq, d = q.shape
    group = Hq // K.shape[1]
    out = np.zeros((B, Hq, K.shape[2]), dtype=np.float32)
    for h in range(Hq):
        g = h // group
        acc = np.zeros((B, K.shape[2]), dtype=np.float32)
        for dim in fc_dims(fc[g], d):
            prod = q[:, h, dim][:, None] * K[:, g, :, dim]   # float32 product, exact for bf16 inputs
            acc = acc + prod                                 # float32 add: one rounding per step
        out[:, h] = acc
    return out


def select_row(keys: np.ndarray, k: int) -> np.ndarray:
    """D3 for one row: ascending indices of the first min(k, L) tokens by (score desc, index asc)."""
    L = keys.shape[0]
    n = min(k, L)
    order = sorted(range(L), key=lambda t: (-float(keys[t]), t))
    return np.sort(np.asarray(order[:n], dtype=np.int64))


def select_tokens(keys: np.ndarray, k: int) -> np.ndarray:
    """D3: idx [B, Hq, k] int, ascending, -1 padded."""
    B, H, L = keys.shape
    idx = -np.ones((B, H, k), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            kept = select_row(keys[b, h], k)
            idx[b, h, :kept.size] = kept
    return idx


def focused_attention(q, K, V, idx, scale=None):
    """D4: o [B, Hq, d], lse [B, Hq] over the kept tokens (float64)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, d = q.shape
    group = Hq // K.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            kept = idx[b, h][idx[b, h] >= 0]
            if kept.size == 0:
                continue
            s = (K[b, g, kept] @ q[b, h]) * scale
            mx = s.max()
            e = np.exp(s - mx)
            o[b, h] = (e @ V[b, g, kept]) / e.sum()
            lse[b, h] = mx + math.log(e.sum())
    return o, lse


def decode_step(q, K, V, fc, k, scale=None):
    """TIP -> select -> FAC for one decode step: (scores, idx, o, lse), scores float64 [B, Hq, L]."""
    s = tip_scores(q, K, fc)
    idx = select_tokens(s, k)
    o, lse = focused_attention(q, K, V, idx, scale)
    return s, idx, o, lse
