"""The (batch, KV group) split of the path across ranks, on CPU with gloo.

Two processes each run the oracle on their share of the units of one small
layer and gather the outputs; rank 0 checks that the gathered result equals
one process running the whole layer, and that the shares are disjoint and
cover every unit.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_dual_b200 import sharding
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import Workload
from oracle import prism_oracle as po

W = Workload(name="shard-test", batch=2, heads_q=4, heads_kv=2, seq_len=256, head_dim=16, dtype="bf16", block=32,
             rope_base=1e4, band_split=4, k=2, planted_frac=0.25)


def run_units(us, Q, K, V):
    cos, sin = po.rope_tables(W.rope_base, W.seq_len, W.head_dim)
    out = {}
    for b, g in us:
        hs = list(sharding.q_heads(g, W.heads_q, W.heads_kv))
        r = po.prism_path(Q[b:b + 1, hs].double().numpy(), K[b:b + 1, g:g + 1].double().numpy(),
                          V[b:b + 1, g:g + 1].double().numpy(), block=W.block, band_split=W.band_split,
                          flags=W.flags, k=W.k, rope=(cos, sin), dtype=W.dtype)
        out[(b, g)] = r.out[0]
    return out


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Q, K, V = make_inputs(W, seed=0)
        mine = sharding.shard(sharding.units(W.batch, W.heads_kv), world, rank)
        res = run_units(mine, Q, K, V)
        gathered = [None] * world
        dist.all_gather_object(gathered, res)
        t = torch.tensor([float(rank + 1)])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)          # the bench's max-over-ranks timing reduction
        if rank == 0:
            merged = {}
            for part in gathered:
                assert not (set(part) & set(merged))
                merged.update(part)
            q.put((sorted(merged), {k: v for k, v in merged.items()}, float(t.item())))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_shards_are_disjoint_and_cover():
    us = sharding.units(3, 8)
    for world in (1, 2, 3, 4, 8):
        parts = [sharding.shard(us, world, r) for r in range(world)]
        flat = [u for p in parts for u in p]
        assert sorted(flat) == sorted(us) and len(flat) == len(set(flat))
    with pytest.raises(ValueError):
        sharding.shard(us, 2, 2)


def test_two_rank_gloo_split_equals_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    keys, merged, tmax = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert keys == sorted(sharding.units(W.batch, W.heads_kv))
    assert tmax == 2.0
    Q, K, V = make_inputs(W, seed=0)
    full = run_units(sharding.units(W.batch, W.heads_kv), Q, K, V)
    for u in keys:
        np.testing.assert_array_equal(merged[u], full[u])


# ---------------------------------------------------------------------------
# Decode step: the same (batch, KV group) split
# ---------------------------------------------------------------------------
from block_sparse_long_dual_b200.synthetic import make_decode_inputs  # noqa: E402
from block_sparse_long_dual_b200.workloads import DecodeWorkload  # noqa: E402
from oracle import fasa_oracle as fo  # noqa: E402

DW = DecodeWorkload(name="shard-decode", batch=2, heads_q=4, heads_kv=2, seq_len=300, head_dim=16, nfc=4, k=20)


def run_decode_units(us, q, K, V, fc):
    out = {}
    for b, g in us:
        hs = list(sharding.q_heads(g, DW.heads_q, DW.heads_kv))
        _, idx, o, _ = fo.decode_step(q[b:b + 1, hs].double().numpy(), K[b:b + 1, g:g + 1].double().numpy(),
                                         V[b:b + 1, g:g + 1].double().numpy(), fc[g:g + 1], DW.k)
        out[(b, g)] = (idx[0], o[0])
    return out


def _decode_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        qq, K, V, fc = make_decode_inputs(DW, seed=0)
        mine = sharding.shard(sharding.units(DW.batch, DW.heads_kv), world, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, run_decode_units(mine, qq, K, V, fc))
        if rank == 0:
            merged = {}
            for part in gathered:
                assert not (set(part) & set(merged))
                merged.update(part)
            q.put(merged)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_decode_split_equals_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    qq, K, V, fc = make_decode_inputs(DW, seed=0)
    _, idx, o, _ = fo.decode_step(qq.double().numpy(), K.double().numpy(), V.double().numpy(), fc, DW.k)
    assert sorted(merged) == sharding.units(DW.batch, DW.heads_kv)
    for (b, g), (ii, oo) in merged.items():
        hs = list(sharding.q_heads(g, DW.heads_q, DW.heads_kv))
        np.testing.assert_array_equal(ii, idx[b, hs])
        np.testing.assert_array_equal(oo, o[b, hs])
