"""Mutation check of the oracle pins.

Each case plants one plausible mistake in a fresh copy of an oracle module's source (on the CPU;
the installed module is only patched for the duration of the case) and requires that at least one
pin test fails against the mutated oracle.  A mistake that no pin catches is either equivalent to
the original or a hole in the pins; both make this test fail, so every entry below is known to be
caught.  Each ``old`` snippet must occur exactly once in the oracle, so an edit to the oracle that
moves a snippet fails here loudly instead of silently dropping the case.

Three mutants tried are equivalent and so are not listed: skipping the single-band early exit in the
temperatures (the empty band L then gets rho = 1, so tau_L = 1 all the same), not zeroing the output
of a query row with no keys (its weights are already all 0, so o = 0), and dropping the explicit NaN
case of the bf16 rounding (a quiet NaN rounds to a NaN by the bit rule already).
"""

from __future__ import annotations

import inspect
import itertools
import sys
import types

import pytest

from oracle import fasa_oracle as fo
from oracle import prism_oracle as po
from tests import test_fasa_oracle_pins, test_oracle_pins, test_selection_properties

# (what is wrong, the oracle source snippet, the mutated snippet)
PRISM_MUTANTS = [
    ("rope: sign of the sine term", "lo * c - hi * s", "lo * c + hi * s"),
    ("rope: frequency exponent -m/d instead of -2m/d",
     "theta = np.power(np.float64(base), -2.0 * m / head_dim)",
     "theta = np.power(np.float64(base), -1.0 * m / head_dim)"),
    ("band: partner dims shifted by one",
     "mask[half:half + band_split] = True", "mask[half + 1:half + 1 + band_split] = True"),
    ("band: one pair too many in band H", "mask[:band_split] = True", "mask[:band_split + 1] = True"),
    ("pool: block sum instead of block mean",
     "return xr.reshape(*xr.shape[:-2], nb, block, d).mean(axis=-2)",
     "return xr.reshape(*xr.shape[:-2], nb, block, d).sum(axis=-2)"),
    ("rho: no square root", "rho[nz] = np.sqrt(e_pool[nz] / e_tok[nz])", "rho[nz] = e_pool[nz] / e_tok[nz]"),
    ("rho: token energy averaged over dims instead of summed",
     "e_tok = (xr[..., band] ** 2).sum(axis=-1).mean(axis=-1)\n    e_pool",
     "e_tok = (xr[..., band] ** 2).mean(axis=-1).mean(axis=-1)\n    e_pool"),
    ("tau: rho_Q^2 instead of rho_Q rho_K",
     "np.maximum(rq * rk_per_q, TAU_FLOOR)", "np.maximum(rq * rq, TAU_FLOOR)"),
    ("tau: KV head of a Q head tiled instead of repeated",
     "rk_per_q = np.repeat(rk, group, axis=1)", "rk_per_q = np.tile(rk, (1, group))"),
    ("relative calibration: product instead of quotient",
     "tau[:, :, 0] = tau[:, :, 0] / tau[:, :, 1]", "tau[:, :, 0] = tau[:, :, 0] * tau[:, :, 1]"),
    ("logits: multiplied by tau", "part = part / tau[:, :, bi][:, :, None, None]",
     "part = part * tau[:, :, bi][:, :, None, None]"),
    ("logits: 1/d instead of 1/sqrt(d)", "out.append((bi, part / math.sqrt(d)))",
     "out.append((bi, part / d))"),
    ("logits: KV blocks tiled instead of repeated over the group",
     "kq = np.repeat(kbar, group, axis=1)", "kq = np.tile(kbar, (1, group, 1, 1))"),
    ("block tau: rho without the square root",
     "np.maximum(np.sqrt(e_pool[nz] / e_tok[nz]), BLOCK_RHO_FLOOR)",
     "np.maximum(e_pool[nz] / e_tok[nz], BLOCK_RHO_FLOOR)"),
    ("block tau: floor taken as a ceiling",
     "np.maximum(np.sqrt(e_pool[nz] / e_tok[nz]), BLOCK_RHO_FLOOR)",
     "np.minimum(np.sqrt(e_pool[nz] / e_tok[nz]), BLOCK_RHO_FLOOR)"),
    ("block tau: block energies summed instead of averaged",
     "nb, block).mean(axis=-1)", "nb, block).sum(axis=-1)"),
    ("block tau: rho_i(Q) rho_j(Q) instead of rho_i(Q) rho_j(K)",
     "part = part / (rq[..., :, None] * rk[..., None, :])",
     "part = part / (rq[..., :, None] * rq[..., None, :])"),
    ("block tau: product instead of quotient",
     "part = part / (rq[..., :, None] * rk[..., None, :])",
     "part = part * (rq[..., :, None] * rk[..., None, :])"),
    ("band max: minimum instead of maximum", "c = np.maximum(c, q)", "c = np.minimum(c, q)"),
    ("band max: no renormalisation", "return c / c.sum(axis=-1, keepdims=True)", "return c"),
    ("softmax: not causal", "allowed = np.tril(np.ones((nb, nb), dtype=bool))",
     "allowed = np.ones((nb, nb), dtype=bool)"),
    ("select: sink flag ignored", "return (0, i)", "return (i,)"),
    ("select: reversed tie-break", "cand[np.lexsort((cand, -p_row[cand]))]",
     "cand[np.lexsort((-cand, -p_row[cand]))]"),
    ("select: k + 1 candidates", "n = min(int(k), order.size)", "n = min(int(k) + 1, order.size)"),
    ("select: <= instead of < in the mass rule", "while n < order.size and cum < mass:",
     "while n < order.size and cum <= mass:"),
    ("select: forced blocks not counted toward the mass",
     "cum = float(sum(p_row[j] for j in forced))", "cum = 0.0"),
    ("attention: strict causal mask", "s = np.where(tk[None, :] <= tq[:, None], s, -np.inf)",
     "s = np.where(tk[None, :] < tq[:, None], s, -np.inf)"),
    ("attention: 1/d scale", "scale = 1.0 / math.sqrt(d)\n    O = np.zeros_like(Qr)\n    lse",
     "scale = 1.0 / d\n    O = np.zeros_like(Qr)\n    lse"),
    ("attention: Q head mapped to KV head h % Hkv",
     "g = h // group\n            for i in range(nb):",
     "g = h % Kr.shape[1]\n            for i in range(nb):"),
    ("attention: lse without the running maximum",
     "np.where(has, m_safe[:, 0] + np.log(", "np.where(has, np.log("),
    ("rounding: bf16 by truncation", "r = ((u + 0x7FFF + lsb) >> 16) << 16", "r = (u >> 16) << 16"),
    ("rope: sign of the second row", "out[..., half:] = hi * c + lo * s", "out[..., half:] = hi * c - lo * s"),
    ("rope: positions counted from 1", "p = np.arange(seq_len, dtype=np.float64)",
     "p = np.arange(1, seq_len + 1, dtype=np.float64)"),
    ("rope: tables kept in float64", "return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)",
     "return np.cos(ang), np.sin(ang)"),
    ("rho: 0 instead of 1 for a band without energy",
     "    rho = np.ones_like(e_tok)\n    nz = e_tok > 0\n    rho[nz] = np.sqrt",
     "    rho = np.zeros_like(e_tok)\n    nz = e_tok > 0\n    rho[nz] = np.sqrt"),
    ("tau: floor taken as a ceiling", "np.maximum(rq * rk_per_q, TAU_FLOOR)", "np.minimum(rq * rk_per_q, TAU_FLOOR)"),
    ("relative calibration: single band left uncalibrated to 1",
     "        if single:\n            tau[:] = 1.0", "        if single:\n            pass"),
    ("band max: flag ignored", "if (flags & FLAG_BAND_MAX) and len(parts) == 2:", "if False:"),
    ("energy: band L summed over the band H dims", "out[..., 1] = sq[..., lmask].sum(axis=-1)",
     "out[..., 1] = sq[..., hmask].sum(axis=-1)"),
    ("energy: block mean instead of block sum",
     "sq = (xr ** 2).reshape(*xr.shape[:-2], nb, block, d).sum(axis=-2)",
     "sq = (xr ** 2).reshape(*xr.shape[:-2], nb, block, d).mean(axis=-2)"),
    ("select: sink forced on row 0 too", "if (flags & FLAG_KEEP_SINK) and i != 0:", "if (flags & FLAG_KEEP_SINK):"),
    ("select arrays: padded with 0", "idx = np.full((B, H, nb, kmax), -1, dtype=np.int32)",
     "idx = np.full((B, H, nb, kmax), 0, dtype=np.int32)"),
    ("select arrays: count off by one", "counts[b, h, i] = kept.size", "counts[b, h, i] = kept.size - 1"),
    ("rounding: float32 rounding skipped",
     "return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)",
     "return np.asarray(x, dtype=np.float64)"),
    ("path: attention reads the unrounded Q_r", "qa = round_to_dtype(sc.q_rot, dtype)", "qa = sc.q_rot"),
    ("path: attention reads the unrounded K_r", "ka = round_to_dtype(sc.k_rot, dtype)", "ka = sc.k_rot"),
]

FASA_MUTANTS = [
    ("fc: rotary partner shifted by one", "return np.concatenate([fc_row, fc_row + head_dim // 2])",
     "return np.concatenate([fc_row, fc_row + head_dim // 2 - 1])"),
    ("fc: partner dims dropped", "return np.concatenate([fc_row, fc_row + head_dim // 2])",
     "return np.concatenate([fc_row, fc_row])"),
    ("gather: KV head 0's cache for every head", "K[:, g][..., fc_dims(fc[g], d)]",
     "K[:, 0][..., fc_dims(fc[g], d)]"),
    ("tip: one pair list for every KV head", "dims = fc_dims(fc[g], d)", "dims = fc_dims(fc[0], d)"),
    ("tip: Q head mapped to KV head h % Hkv",
     "g = h // group\n        dims = fc_dims", "g = h % K.shape[1]\n        dims = fc_dims"),
    ("tip keys: one pair list for every KV head", "for dim in fc_dims(fc[g], d):",
     "for dim in fc_dims(fc[0], d):"),
    ("tip keys: float64 running sum", "acc = np.zeros((B, K.shape[2]), dtype=np.float32)",
     "acc = np.zeros((B, K.shape[2]), dtype=np.float64)"),
    ("select: reversed tie-break", "key=lambda t: (-float(keys[t]), t)", "key=lambda t: (-float(keys[t]), -t)"),
    ("select: k + 1 tokens", "n = min(k, L)", "n = min(k + 1, L)"),
    ("fac: no softmax scale", "s = (K[b, g, kept] @ q[b, h]) * scale", "s = (K[b, g, kept] @ q[b, h])"),
    ("fac: lse without the maximum", "lse[b, h] = mx + math.log(e.sum())", "lse[b, h] = math.log(e.sum())"),
    ("fac: 1/d scale", "scale = 1.0 / math.sqrt(d) if scale is None", "scale = 1.0 / d if scale is None"),
    ("fac: Q head mapped to KV head h % Hkv", "            g = h // group\n            kept = idx",
     "            g = h % K.shape[1]\n            kept = idx"),
    ("fac: empty row lse 0", "lse = np.full((B, Hq), -np.inf)", "lse = np.zeros((B, Hq))"),
    ("tip keys: Q head mapped to KV head h % Hkv", "        g = h // group\n        acc",
     "        g = h % K.shape[1]\n        acc"),
    ("tip keys: columns summed in reverse", "for dim in fc_dims(fc[g], d):", "for dim in fc_dims(fc[g], d)[::-1]:"),
    ("gather: head 0's pair list for every head", "K[:, g][..., fc_dims(fc[g], d)]",
     "K[:, g][..., fc_dims(fc[0], d)]"),
    ("select: padded with 0", "idx = -np.ones((B, H, k), dtype=np.int64)", "idx = np.zeros((B, H, k), dtype=np.int64)"),
    ("select: output in rank order", "return np.sort(np.asarray(order[:n], dtype=np.int64))",
     "return np.asarray(order[:n], dtype=np.int64)"),
    ("decode step: ranks the float32 running sum", "idx = select_tokens(s, k)",
     "idx = select_tokens(tip_keys(q, K, fc), k)"),
    ("tip: float32 dot product", "out[:, h] = np.einsum(\"bd,btd->bt\", q[:, h][:, dims], K[:, g][..., dims])",
     "out[:, h] = np.einsum(\"bd,btd->bt\", q[:, h][:, dims].astype(np.float32), K[:, g][..., dims].astype(np.float32))"),
]

PIN_MODULES = [test_oracle_pins, test_fasa_oracle_pins, test_selection_properties]


def _pin_cases():
    """Every (name, function, kwargs) of the pin modules, parametrizations expanded."""
    cases = []
    for mod in PIN_MODULES:
        for name, fn in vars(mod).items():
            if not name.startswith("test_") or not callable(fn):
                continue
            grids = []
            for mark in getattr(fn, "pytestmark", []):
                if mark.name != "parametrize":
                    continue
                names = [s.strip() for s in mark.args[0].split(",")]
                grid = []
                for v in mark.args[1]:
                    vals = v.values if type(v).__name__ == "ParameterSet" else (v,) if len(names) == 1 else v
                    grid.append(dict(zip(names, vals)))
                grids.append(grid)
            for combo in itertools.product(*grids):
                kw = {}
                for part in combo:
                    kw.update(part)
                cases.append((f"{mod.__name__}.{name}{kw or ''}", fn, kw))
    return cases


def _mutant_module(module, old, new):
    src = inspect.getsource(module)
    assert src.count(old) == 1, f"snippet not unique in {module.__name__}: {old!r}"
    name = module.__name__ + "__mutant"
    mut = types.ModuleType(name)
    mut.__file__ = module.__file__
    sys.modules[name] = mut          # dataclasses look the defining module up while decorating
    try:
        exec(compile(src.replace(old, new), module.__file__, "exec"), mut.__dict__)
    finally:
        del sys.modules[name]
    return mut


def _first_failing_pin(cases):
    for label, fn, kw in cases:
        try:
            fn(**kw)
        except Exception as exc:     # an assertion, or the mutant crashing on a pin input
            return f"{label}: {type(exc).__name__}"
    return None


def _patch_with(module, mut, monkeypatch):
    for name, obj in vars(mut).items():
        if inspect.isfunction(obj) and obj.__module__ == mut.__name__:
            monkeypatch.setattr(module, name, obj)


@pytest.mark.parametrize("module,old,new", [pytest.param(po, o, n, id=d) for d, o, n in PRISM_MUTANTS]
                         + [pytest.param(fo, o, n, id="fasa " + d) for d, o, n in FASA_MUTANTS])
def test_planted_mistake_fails_a_pin(module, old, new, monkeypatch):
    _patch_with(module, _mutant_module(module, old, new), monkeypatch)
    caught = _first_failing_pin(_pin_cases())
    assert caught is not None, "no pin fails with this mistake planted"


def test_unplanted_copy_passes_every_pin(monkeypatch):
    """The harness itself: with both oracles replaced by unchanged copies made the same way, every
    pin case passes when called this way, so a failure above comes from the planted mistake."""
    for module, (_, old, _) in ((po, PRISM_MUTANTS[0]), (fo, FASA_MUTANTS[0])):
        _patch_with(module, _mutant_module(module, old, old), monkeypatch)
    assert _first_failing_pin(_pin_cases()) is None
