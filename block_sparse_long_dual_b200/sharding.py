"""How the path splits across processes (one per GPU).

Every quantity of the path is per (batch element, KV head group): the block
means, temperatures and scores of a Q head use only that head and its KV head,
the selection is per Q head, and attention reads only the group's K and V
("Prism: Spectral-Aware Block-Sparse Attention" §1, §3: per-head block
importance).  So the units (b, g) are independent and can be given to
different ranks with no exchange on the data path; only the timing is
reduced across ranks (max), and outputs are gathered only if a caller wants
them in one place.

The decode step splits the same way ("FASA: Frequency-aware Sparse
Attention" §2B): the compact keys, token scores, selection and focused
attention of a Q head read only its sequence's cache of its KV head, so the
(b, g) units of a decode batch are independent too.
"""

from __future__ import annotations


def units(batch: int, heads_kv: int) -> list[tuple[int, int]]:
    """All (batch, kv head) units of a layer, in a fixed order."""
    return [(b, g) for b in range(batch) for g in range(heads_kv)]


def shard(all_units: list, world: int, rank: int) -> list:
    """Round-robin share of ``all_units`` for ``rank`` of ``world`` (disjoint, covering)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return all_units[rank::world]


def q_heads(g: int, heads_q: int, heads_kv: int) -> range:
    """Q heads that read KV head ``g`` (grouped-query attention)."""
    group = heads_q // heads_kv
    return range(g * group, (g + 1) * group)
