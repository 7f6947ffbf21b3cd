"""CPU oracle for the Prism block-sparse attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library: no kernels, headers, tables,
helpers or pre/post-processing.  It reads plain NumPy arrays (the same seeded
host inputs the GPU path receives) and computes everything in float64.

What it restates (source: "Prism: Spectral-Aware Block-Sparse Attention"):

* §1 (the problem): importance of a key block is estimated from mean-pooled
  block vectors; attention is then computed exactly, but only over a chosen
  subset of blocks.
* §2 (mean pooling and RoPE): RoPE rotates each pair of dimensions at its own
  frequency; averaging a block of fast-rotating pairs cancels them
  (destructive interference), so the pooled amplitude collapses in the high
  band.
* §3.1 (dual-band estimation): the head dimension is split into a
  high-frequency band and a low-frequency band, each pooled on its own.
* §3.2 (energy-based temperature): a temperature tau built from the energy
  (RMS norm) of the vectors restores the logit amplitude lost by pooling, so
  block selection needs block-level matrix products only.
* §5 (results): the estimate is "block-level matrix multiplications only".

The page gives no formulas, so every open step takes the plainest reading that
the rest supports.  The readings (all enforced here, and listed with their
reasons in the design notes of the repository):

R1  RoPE: rotate-half pairing (m, m + d/2), theta_m = base**(-2m/d), position
    p = token index, no rope scaling; cos/sin computed in float64 and rounded
    to float32 (the table both sides use); the rotation itself in float64.
R2  Band split: ``band_split`` = number of highest-frequency rotary pairs in
    the high band H, i.e. dims {0..bs-1} U {d/2..d/2+bs-1}; band L = the rest.
R3  Pool: block mean of the *unrounded* rotated vectors.
R4  Energy and tau, per (batch, Q head, band):
        E_tok  = mean over tokens of ||x_t^b||^2
        E_pool = mean over blocks of ||xbar_j^b||^2
        rho    = sqrt(E_pool / E_tok)            (rho = 1 if E_tok == 0)
        tau    = max(rho(Q_h) * rho(K_g), 1e-6)
    NO_CALIB sets tau = 1; SINGLE_BAND treats all d dims as one band.
R4b (alternative reading, flag RELATIVE_CALIB): restore the high band's
    amplitude relative to the low band only: tau^H <- tau^H / tau^L,
    tau^L <- 1 (the low band keeps its plain mean-pooling scale).
R4c (alternative reading, flag BLOCK_TAU): the temperature is per block pair,
    tau^b_ij = rho^b_i(Q_h) * rho^b_j(K_g), with each block's own retained
    amplitude rho^b_i(X) = sqrt(||xbar_i^b||^2 / ((1/block) sum_{t in i}
    ||x_t^b||^2)), floored at 1e-3 (so tau >= 1e-6 as in R4) and 1 when the
    block's band energy is 0.  Exclusive with NO_CALIB and RELATIVE_CALIB.
R5  Logits: s_ij = (1/sqrt(d)) * sum_b (qbar_i^b . kbar_j^b) / tau^b, j <= i.
R6  Probabilities: causal row softmax over j <= i; p_ij = 0 for j > i.
R5b (alternative reading, flag BAND_MAX; §3 "two parallel branches"): each
    band's calibrated logits s^b_ij = (qbar_i^b . kbar_j^b) / (tau^b sqrt(d))
    get their own causal softmax p^b; the branches combine by the elementwise
    maximum, renormalised over j <= i:
        p_ij = max_b p^b_ij / sum_{j' <= i} max_b p^b_ij'.
    A band with no dims has no branch (then p is the R5/R6 result).
R7  Selection: forced F_i = {i} (and {0} with KEEP_SINK); candidates ordered
    by (p desc, index asc); top-k keeps F_i plus the first min(k, |C_i|);
    mass keeps F_i and adds candidates in order while the running sum
    (forced blocks included) is below ``mass``.  Output ascending.
R8  Attention: plain softmax attention of each query token over the tokens of
    its kept blocks (s <= t when causal), from the bf16/fp32-rounded Q_r, K_r
    and V values; empty key set gives o = 0, lse = -inf.
R9  Layout [B, H, L, d]; GQA maps Q head h to KV head h // (Hq // Hkv); scores
    and masks are per Q head.

Pins (tests/test_oracle_pins.py): the Dirichlet amplitude-collapse closed form
(§2), the exact single-pair calibration identity (§3.2), block size 1 reducing
to token-level causal softmax, mean pooling cross-checked with torch's
avg_pool1d, RoPE against the transformers Llama rotary routine, brute-force
selection, and all-blocks-kept attention against brute-force dense causal
attention.  R4c: per-block rho equal to the golden Dirichlet factor for a
constant pair, the 1e-3 floor on a full turn per block, restoration of each
block's token RMS, block size 1 giving token softmax.  R5b: mirrored bands
giving the half-logit softmax, a one-hot branch against a uniform branch in
closed form, and a single band reducing to R5/R6.  Also: the RoPE tables as
float32 roundings of the exact angles, per-block band energies of a rotated
constant vector, tau = 1 for a band with no energy, the array form of a
selection, and the attention reading the rounded Q_r / K_r.  Every pin's power
is itself checked: tests/test_oracle_mutations.py plants mistakes in a copy of
this module and requires a pin to fail for each.  Parity of the *selection
rule itself* with the pages' own selections is unpinned: the pages print no
worked example.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

FLAG_KEEP_SINK = 1
FLAG_NO_CALIB = 2
FLAG_SINGLE_BAND = 4
FLAG_RELATIVE_CALIB = 8
FLAG_BAND_MAX = 16
FLAG_BLOCK_TAU = 32

TAU_FLOOR = 1e-6
BLOCK_RHO_FLOOR = 1e-3


# ---------------------------------------------------------------------------
# R1: RoPE (Prism §2 names RoPE; the convention is the rotate-half one used by
# the Llama / Qwen models the page evaluates on, §5).
# ---------------------------------------------------------------------------
def rope_tables(base: float, seq_len: int, head_dim: int):
    """cos/sin tables [L, d/2]: angle p * base**(-2m/d) in float64, rounded to float32."""
    half = head_dim // 2
    m = np.arange(half, dtype=np.float64)
    theta = np.power(np.float64(base), -2.0 * m / head_dim)
    p = np.arange(seq_len, dtype=np.float64)
    ang = p[:, None] * theta[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope_frequencies(base: float, head_dim: int) -> np.ndarray:
    half = head_dim // 2
    return np.power(np.float64(base), -2.0 * np.arange(half, dtype=np.float64) / head_dim)


def apply_rope(x: np.ndarray, cos32: np.ndarray, sin32: np.ndarray) -> np.ndarray:
    """Rotate pairs (m, m+d/2) of x [..., L, d] by the table angle of each position (float64)."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    c = cos32.astype(np.float64)
    s = sin32.astype(np.float64)
    lo = x[..., :half]
    hi = x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = lo * c - hi * s
    out[..., half:] = hi * c + lo * s
    return out


# ---------------------------------------------------------------------------
# R2: band split (Prism §3.1).
# ---------------------------------------------------------------------------
def high_band_mask(head_dim: int, band_split: int, single_band: bool = False) -> np.ndarray:
    """Boolean [d]: True for dims in the high-frequency band H.

    With ``single_band`` every dim belongs to one band (reported as H)."""
    half = head_dim // 2
    mask = np.zeros(head_dim, dtype=bool)
    if single_band:
        mask[:] = True
        return mask
    mask[:band_split] = True
    mask[half:half + band_split] = True
    return mask


def band_masks(head_dim: int, band_split: int, single_band: bool = False):
    h = high_band_mask(head_dim, band_split, single_band)
    return h, ~h


# ---------------------------------------------------------------------------
# R3: block mean pooling (Prism §1, §3.1).
# ---------------------------------------------------------------------------
def pool_blocks(xr: np.ndarray, block: int) -> np.ndarray:
    """Mean over each block of ``block`` consecutive tokens: [..., L, d] -> [..., L/block, d]."""
    L, d = xr.shape[-2], xr.shape[-1]
    nb = L // block
    return xr.reshape(*xr.shape[:-2], nb, block, d).mean(axis=-2)


# ---------------------------------------------------------------------------
# R4: energy-based temperature (Prism §3.2).
# ---------------------------------------------------------------------------
def retained_amplitude(xr: np.ndarray, xbar: np.ndarray, band: np.ndarray) -> np.ndarray:
    """rho = sqrt(E_pool / E_tok) of one band, for every leading index of xr [..., L, d]."""
    e_tok = (xr[..., band] ** 2).sum(axis=-1).mean(axis=-1)
    e_pool = (xbar[..., band] ** 2).sum(axis=-1).mean(axis=-1)
    rho = np.ones_like(e_tok)
    nz = e_tok > 0
    rho[nz] = np.sqrt(e_pool[nz] / e_tok[nz])
    return rho


def block_retained_amplitude(xr: np.ndarray, xbar: np.ndarray, band: np.ndarray) -> np.ndarray:
    """R4c: rho of every block [..., nb] for one band: sqrt(||xbar_j||^2 / mean_{t in j} ||x_t||^2),
    floored at BLOCK_RHO_FLOOR; 1 where the block's band energy is 0."""
    nb = xbar.shape[-2]
    block = xr.shape[-2] // nb
    e_tok = (xr[..., band] ** 2).sum(axis=-1).reshape(*xr.shape[:-2], nb, block).mean(axis=-1)
    e_pool = (xbar[..., band] ** 2).sum(axis=-1)
    rho = np.ones_like(e_tok)
    nz = e_tok > 0
    rho[nz] = np.maximum(np.sqrt(e_pool[nz] / e_tok[nz]), BLOCK_RHO_FLOOR)
    return rho


def temperatures(qr, kr, qbar, kbar, band_split, flags, group):
    """tau [B, Hq, 2] (index 0 = band H, 1 = band L); band L is all ones with SINGLE_BAND."""
    B, Hq = qr.shape[0], qr.shape[1]
    tau = np.ones((B, Hq, 2), dtype=np.float64)
    if flags & FLAG_NO_CALIB:
        return tau
    d = qr.shape[-1]
    single = bool(flags & FLAG_SINGLE_BAND)
    bands = band_masks(d, band_split, single)
    for bi, band in enumerate(bands):
        if single and bi == 1:
            break
        rq = retained_amplitude(qr, qbar, band)            # [B, Hq]
        rk = retained_amplitude(kr, kbar, band)            # [B, Hkv]
        rk_per_q = np.repeat(rk, group, axis=1)            # Q head h -> KV head h // group
        tau[:, :, bi] = np.maximum(rq * rk_per_q, TAU_FLOOR)
    if flags & FLAG_RELATIVE_CALIB:
        if single:
            tau[:] = 1.0
        else:
            tau[:, :, 0] = tau[:, :, 0] / tau[:, :, 1]
            tau[:, :, 1] = 1.0
    return tau


# ---------------------------------------------------------------------------
# R5/R6: calibrated block logits and causal block softmax (Prism §3.2, §5).
# ---------------------------------------------------------------------------
def band_logits(qbar, kbar, tau, band_split, flags, group, qr=None, kr=None):
    """Per-band calibrated logits [(band index, s^b [B, Hq, nb, nb])] for the bands that have dims.

    R5 divides band b by tau^b [B, Hq, 2]; with BLOCK_TAU (R4c) by rho^b_i(Q) rho^b_j(K)
    from the rotated tokens ``qr``, ``kr``."""
    d = qbar.shape[-1]
    single = bool(flags & FLAG_SINGLE_BAND)
    kq = np.repeat(kbar, group, axis=1)
    out = []
    for bi, band in enumerate(band_masks(d, band_split, single)):
        if single and bi == 1:
            break
        if not band.any():
            continue
        part = qbar[..., band] @ np.swapaxes(kq[..., band], -1, -2)
        if flags & FLAG_BLOCK_TAU:
            rq = block_retained_amplitude(qr, qbar, band)                                 # [B, Hq, nb]
            rk = np.repeat(block_retained_amplitude(kr, kbar, band), group, axis=1)      # [B, Hq, nb]
            part = part / (rq[..., :, None] * rk[..., None, :])
        else:
            part = part / tau[:, :, bi][:, :, None, None]
        out.append((bi, part / math.sqrt(d)))
    return out


def block_logits(qbar, kbar, tau, band_split, flags, group, qr=None, kr=None):
    """s [B, Hq, nb, nb] = sum of the band logits (all entries; the caller masks j > i)."""
    s = np.zeros(qbar.shape[:-1] + (kbar.shape[-2],), dtype=np.float64)
    for _, part in band_logits(qbar, kbar, tau, band_split, flags, group, qr, kr):
        s = s + part
    return s


def band_max_probs(band_probs):
    """R5b: elementwise maximum of the per-band causal softmaxes, renormalised per row."""
    c = band_probs[0]
    for q in band_probs[1:]:
        c = np.maximum(c, q)
    return c / c.sum(axis=-1, keepdims=True)


def causal_block_softmax(s: np.ndarray) -> np.ndarray:
    nb = s.shape[-1]
    allowed = np.tril(np.ones((nb, nb), dtype=bool))
    z = np.where(allowed, s, -np.inf)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.where(allowed, np.exp(z), 0.0)
    return e / e.sum(axis=-1, keepdims=True)


@dataclass
class ScoreResult:
    q_rot: np.ndarray          # float64, unrounded rotated Q
    k_rot: np.ndarray
    qbar: np.ndarray           # [B, Hq, nb, d]
    kbar: np.ndarray           # [B, Hkv, nb, d]
    tok_energy_q: np.ndarray   # [B, Hq, nb, 2] per-block sum of ||x_t^b||^2
    tok_energy_k: np.ndarray
    tau: np.ndarray            # [B, Hq, 2]
    logits: np.ndarray         # [B, Hq, nb, nb]
    probs: np.ndarray          # [B, Hq, nb, nb], zero above the diagonal


def block_token_energy(xr, block, band_split, flags):
    d = xr.shape[-1]
    single = bool(flags & FLAG_SINGLE_BAND)
    hmask, lmask = band_masks(d, band_split, single)
    L = xr.shape[-2]
    nb = L // block
    sq = (xr ** 2).reshape(*xr.shape[:-2], nb, block, d).sum(axis=-2)
    out = np.zeros(xr.shape[:-2] + (nb, 2))
    out[..., 0] = sq[..., hmask].sum(axis=-1)
    if not single:
        out[..., 1] = sq[..., lmask].sum(axis=-1)
    return out


def prism_scores(Q, K, block, band_split, flags=0, rope=None) -> ScoreResult:
    """Steps R1-R6 for Q [B, Hq, L, d] and K [B, Hkv, L, d] (pre-RoPE values).

    ``rope`` is (cos32, sin32) tables or None when Q, K are already rotated."""
    if (flags & FLAG_BLOCK_TAU) and (flags & (FLAG_NO_CALIB | FLAG_RELATIVE_CALIB)):
        raise ValueError("BLOCK_TAU excludes NO_CALIB and RELATIVE_CALIB")
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    group = Q.shape[1] // K.shape[1]
    if rope is not None:
        qr = apply_rope(Q, *rope)
        kr = apply_rope(K, *rope)
    else:
        qr, kr = Q, K
    qbar = pool_blocks(qr, block)
    kbar = pool_blocks(kr, block)
    tau = temperatures(qr, kr, qbar, kbar, band_split, flags, group)
    parts = band_logits(qbar, kbar, tau, band_split, flags, group, qr, kr)
    s = np.zeros(qbar.shape[:-1] + (kbar.shape[-2],), dtype=np.float64)
    for _, part in parts:
        s = s + part
    if (flags & FLAG_BAND_MAX) and len(parts) == 2:
        p = band_max_probs([causal_block_softmax(part) for _, part in parts])
    else:
        p = causal_block_softmax(s)
    return ScoreResult(qr, kr, qbar, kbar,
                       block_token_energy(qr, block, band_split, flags),
                       block_token_energy(kr, block, band_split, flags),
                       tau, s, p)


# ---------------------------------------------------------------------------
# R7: block selection (Prism §1: "a subset of relevant blocks").
# ---------------------------------------------------------------------------
@dataclass
class RowSelection:
    kept: np.ndarray           # ascending kept block indices
    order: np.ndarray          # candidates in (p desc, index asc) order
    n_taken: int               # how many of ``order`` were kept
    forced: tuple = field(default_factory=tuple)
    cum_before_last: float = float("nan")   # mass mode: running sum before the last add
    cum_final: float = float("nan")


def forced_blocks(i: int, flags: int) -> tuple:
    if (flags & FLAG_KEEP_SINK) and i != 0:
        return (0, i)
    return (i,)


def candidate_order(p_row: np.ndarray, i: int, forced: tuple) -> np.ndarray:
    cand = np.array([j for j in range(i + 1) if j not in forced], dtype=np.int64)
    if cand.size == 0:
        return cand
    # np.lexsort sorts by the last key first: primary -p (descending p), then index.
    return cand[np.lexsort((cand, -p_row[cand]))]


def select_row(p_row, i, flags, k=None, mass=None) -> RowSelection:
    forced = forced_blocks(i, flags)
    order = candidate_order(p_row, i, forced)
    cum_before = float("nan")
    if k is not None:
        n = min(int(k), order.size)
        cum = float("nan")
    else:
        cum = float(sum(p_row[j] for j in forced))
        n = 0
        while n < order.size and cum < mass:
            cum_before = cum
            cum += float(p_row[order[n]])
            n += 1
    kept = np.sort(np.concatenate([np.array(forced, dtype=np.int64), order[:n]]))
    return RowSelection(kept, order, n, forced, cum_before, cum)


def select_blocks(probs, flags=0, k=None, mass=None):
    """Selection for every (b, h, i) row of probs [B, H, nb, nb]; nested lists of RowSelection."""
    if (k is None) == (mass is None):
        raise ValueError("exactly one of k / mass")
    B, H, nb = probs.shape[0], probs.shape[1], probs.shape[2]
    return [[[select_row(probs[b, h, i], i, flags, k=k, mass=mass) for i in range(nb)]
             for h in range(H)] for b in range(B)]


def selection_to_arrays(sel, kmax):
    """counts [B, H, nb] int32 and idx [B, H, nb, kmax] int32 (ascending, -1 padded)."""
    B, H, nb = len(sel), len(sel[0]), len(sel[0][0])
    counts = np.zeros((B, H, nb), dtype=np.int32)
    idx = np.full((B, H, nb, kmax), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                kept = sel[b][h][i].kept
                counts[b, h, i] = kept.size
                idx[b, h, i, :kept.size] = kept
    return counts, idx


# ---------------------------------------------------------------------------
# R8: exact attention over the kept blocks (Prism §1).
# ---------------------------------------------------------------------------
def sparse_attention(Qr, Kr, V, kept_lists, block, causal=True, scale=None):
    """O [B, Hq, L, d] and lse [B, Hq, L] (natural log) for kept_lists[b][h][i] = kept block ids.

    Q/K/V are the rounded values the attention reads (bf16 or fp32), as float64."""
    Qr = np.asarray(Qr, dtype=np.float64)
    Kr = np.asarray(Kr, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, L, d = Qr.shape
    group = Hq // Kr.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros_like(Qr)
    lse = np.full((B, Hq, L), -np.inf)
    nb = L // block
    for b in range(B):
        for h in range(Hq):
            g = h // group
            for i in range(nb):
                kept = np.asarray(kept_lists[b][h][i], dtype=np.int64)
                if kept.size == 0:
                    continue
                tq = np.arange(i * block, (i + 1) * block)
                tk = (kept[:, None] * block + np.arange(block)[None, :]).reshape(-1)
                s = (Qr[b, h, tq] @ Kr[b, g, tk].T) * scale
                if causal:
                    s = np.where(tk[None, :] <= tq[:, None], s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                has = np.isfinite(m[:, 0])
                m_safe = np.where(np.isfinite(m), m, 0.0)
                e = np.exp(s - m_safe)
                den = e.sum(axis=1, keepdims=True)
                o = (e @ V[b, g, tk]) / np.where(den > 0, den, 1.0)
                O[b, h, tq] = np.where(has[:, None], o, 0.0)
                lse[b, h, tq] = np.where(has, m_safe[:, 0] + np.log(np.where(den[:, 0] > 0, den[:, 0], 1.0)), -np.inf)
    return O, lse


def dense_causal_attention_bruteforce(Qr, Kr, V, scale=None):
    """Token-by-token dense causal softmax attention (pure loops; small inputs only)."""
    Qr = np.asarray(Qr, dtype=np.float64)
    Kr = np.asarray(Kr, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, L, d = Qr.shape
    group = Hq // Kr.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros_like(Qr)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            for t in range(L):
                w = [math.exp(float(np.dot(Qr[b, h, t], Kr[b, g, s])) * scale) for s in range(t + 1)]
                tot = sum(w)
                acc = np.zeros(d)
                for s in range(t + 1):
                    acc += (w[s] / tot) * V[b, g, s]
                O[b, h, t] = acc
    return O


# ---------------------------------------------------------------------------
# Rounding helpers: the attention reads Q_r / K_r rounded to the input dtype.
# ---------------------------------------------------------------------------
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (round to nearest even), returned as float64.

    Two steps: float64 -> float32 is itself RNE, then float32 -> bf16 RNE by the
    bit pattern.  Double rounding can differ from a direct float64 -> bf16 RNE
    only when the float64 value sits within 2^-24 relative of a bf16 midpoint."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    r = r.astype(np.uint32)
    nan = np.isnan(f)
    out = r.view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# The whole path.
# ---------------------------------------------------------------------------
@dataclass
class PathResult:
    scores: ScoreResult
    selection: list
    q_attn: np.ndarray
    k_attn: np.ndarray
    out: np.ndarray
    lse: np.ndarray


def prism_path(Q, K, V, *, block, band_split, flags=0, k=None, mass=None, rope=None,
               dtype="bf16", causal=True):
    sc = prism_scores(Q, K, block, band_split, flags, rope)
    sel = select_blocks(sc.probs, flags, k=k, mass=mass)
    qa = round_to_dtype(sc.q_rot, dtype)
    ka = round_to_dtype(sc.k_rot, dtype)
    kept = [[[r.kept for r in row] for row in hb] for hb in sel]
    O, lse = sparse_attention(qa, ka, np.asarray(V, dtype=np.float64), kept, block, causal)
    return PathResult(sc, sel, qa, ka, O, lse)
