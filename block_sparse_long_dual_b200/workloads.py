"""Named workloads: the layer shapes, budgets and planted structure of each case.

The shapes stand in for the attention layers of the models that
"Prism: Spectral-Aware Block-Sparse Attention" (§5) evaluates on
(Llama-3.1-8B: 32 Q / 8 KV heads, head dim 128, RoPE base 5e5; Qwen3-8B: the
same head shape, RoPE base 1e6).  No weights or datasets are used: inputs are
seeded synthetic tensors (``synthetic.py``).  This module holds configuration
only, none of the method's arithmetic.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

KEEP_SINK = 1
NO_CALIB = 2
SINGLE_BAND = 4
RELATIVE_CALIB = 8
BAND_MAX = 16
BLOCK_TAU = 32


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seq_len: int
    head_dim: int
    dtype: str            # "bf16" | "f32"
    block: int
    rope_base: float
    band_split: int       # highest-frequency rotary pairs in the high band
    k: int | None = None  # top-k extra blocks beyond the forced ones
    mass: float | None = None
    flags: int = 0
    planted_frac: float = 0.0   # fraction of key blocks carrying the semantic component
    slash: bool = False         # constant high-band component on every Q/K token
    density: float | None = None

    @property
    def nb(self) -> int:
        return self.seq_len // self.block

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv

    def kmax(self) -> int:
        """Largest kept count a row can have (the idx row length)."""
        if self.mass is not None:
            return self.nb
        nforced = 2 if self.flags & KEEP_SINK else 1
        return min(self.nb, self.k + nforced)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


def k_for_density(nb: int, density: float, nforced: int = 1) -> int:
    """Smallest k with sum_i min(i+1, k+nforced) >= density * nb(nb+1)/2."""
    target = density * nb * (nb + 1) / 2.0
    for k in range(nb + 1):
        kept = sum(min(i + 1, k + nforced) for i in range(nb))
        if kept >= target - 1e-9:
            return k
    return nb


def kept_blocks_topk(nb: int, k: int, nforced: int = 1) -> int:
    return sum(min(i + 1, k + nforced) for i in range(nb))


def _llama(L: int, density: float) -> Workload:
    nb = L // 128
    return Workload(name=f"llama3.1-8b-{L // 1024}k-d{int(round(density * 100))}", batch=1,
                    heads_q=32, heads_kv=8, seq_len=L, head_dim=128, dtype="bf16", block=128,
                    rope_base=5e5, band_split=32, k=k_for_density(nb, density),
                    planted_frac=0.05, density=density)


TINY = Workload(name="tiny-1h-1k-d64-f32", batch=1, heads_q=1, heads_kv=1, seq_len=1024,
                head_dim=64, dtype="f32", block=64, rope_base=1e4, band_split=16, k=4,
                flags=KEEP_SINK)

LLAMA_32K = _llama(32768, 0.10)
LLAMA_128K = _llama(131072, 0.05)

QWEN_64K_B2 = Workload(name="qwen3-8b-64k-b2-mass0.9", batch=2, heads_q=32, heads_kv=8,
                       seq_len=65536, head_dim=128, dtype="bf16", block=128, rope_base=1e6,
                       band_split=32, mass=0.9, planted_frac=0.05, slash=True)


def sweep(density: float) -> Workload:
    nb = 65536 // 128
    return Workload(name=f"sweep-64k-d{density:g}", batch=1, heads_q=32, heads_kv=8,
                    seq_len=65536, head_dim=128, dtype="bf16", block=128, rope_base=5e5,
                    band_split=32, k=k_for_density(nb, density), planted_frac=0.02,
                    density=density)


SWEEP_DENSITIES = (0.01, 0.02, 0.05, 0.10, 0.25, 1.0)

ALL = {w.name: w for w in [TINY, LLAMA_32K, LLAMA_128K, QWEN_64K_B2]
       + [sweep(x) for x in SWEEP_DENSITIES]}


# ---------------------------------------------------------------------------
# Decode step ("FASA: Frequency-aware Sparse Attention" §2B): one query token
# per (batch, Q head) against a KV cache.  nfc = 12 of 64 rotary pairs is
# 18.75% of the key dims, the share of the cache the page's FASA-C reads
# (18.9%, §4); k = 256 is the page's extreme token budget (§4, LongBench).
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seq_len: int      # cache length L
    head_dim: int
    nfc: int          # dominant rotary pairs per KV head
    k: int            # token budget
    needle_frac: float = 0.01   # fraction of cache tokens aligned with the query on the dominant pairs
    dominant_gain: float = 1.0  # amplitude of q and K on the dominant pairs' dims (1: plain N(0, 1))

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv

    def scaled(self, **kw) -> "DecodeWorkload":
        return replace(self, **kw)


FASA_DECODE_128K_B4 = DecodeWorkload(name="fasa-decode-llama3.1-8b-128k-b4", batch=4, heads_q=32, heads_kv=8,
                                     seq_len=131072, head_dim=128, nfc=12, k=256)
FASA_DECODE_32K_B16 = DecodeWorkload(name="fasa-decode-llama3.1-8b-32k-b16", batch=16, heads_q=32, heads_kv=8,
                                     seq_len=32768, head_dim=128, nfc=12, k=256)
DECODE = {w.name: w for w in [FASA_DECODE_128K_B4, FASA_DECODE_32K_B16]}
