"""Host side of context-parallel decode: shard bounds, the record exchange (gloo, 2 ranks on CPU), and the
record format's merge against the oracle's attention over the whole cache.

The records here are computed in fp64 by this test from the definition the C header gives (normalised output
and base-2 log-sum-exp over a rank's keys); the GPU test checks the kernels' records against the same oracle.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from full_gqa_attention_spark2_b200.context_parallel import gather_records, owner_of, shard_of
from oracle import spark_oracle as O

LOG2E = 1.0 / np.log(2.0)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("total", [8, 9, 100, 4097, 1 << 20])
def test_shards_cover_positions_once(world, total):
    bounds = [shard_of(r, world, total) for r in range(world)]
    assert bounds[0][0] == 0
    for (lo, n), (lo2, _) in zip(bounds, bounds[1:]):
        assert n >= 1 and lo + n == lo2
    assert sum(bounds[-1]) == total
    assert max(n for _, n in bounds) - min(n for _, n in bounds) <= 1
    probe = sorted({0, 1, total // 3, total // 2, total - 2, total - 1} | {lo for lo, _ in bounds})
    for p in probe:
        r = owner_of(p, world, total)
        lo, n = bounds[r]
        assert lo <= p < lo + n


def test_shard_rejects_more_ranks_than_positions():
    with pytest.raises(ValueError):
        shard_of(0, 4, 3)
    with pytest.raises(ValueError):
        owner_of(10, 2, 10)


def _record(qr, k, v):
    """One rank's record for one sequence: o [16, 256] normalised over its keys, lse [16] in base 2."""
    o = np.zeros((16, 256))
    lse = np.full(16, -np.inf)
    if len(k) == 0:
        return o, lse
    for h in range(16):
        s = (k[:, h // 4, :] @ qr[h]) / 16.0
        m = s.max()
        e = np.exp(s - m)
        o[h] = (e @ v[:, h // 4, :]) / e.sum()
        lse[h] = (m + np.log(e.sum())) * LOG2E
    return o, lse


def _merge(records, gate):
    """out [16, 256] from [(o, lse)] of every rank: the base-2 log-sum-exp weighted mean, gated."""
    lse = np.stack([r[1] for r in records])                  # [G, 16]
    M = lse.max(axis=0)
    w = np.where(np.isneginf(lse), 0.0, np.exp2(lse - M))
    o = np.einsum("gh,ghd->hd", w, np.stack([r[0] for r in records])) / w.sum(axis=0)[:, None]
    return o * O.sigmoid(gate)[:, None]


def _problem(B=2, total=300, seed=7):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, total, 4, 256))
    v = rng.standard_normal((B, total, 4, 256))
    q = rng.standard_normal((B, 16, 256))
    g = rng.standard_normal((B, 16)) * 2
    pos = np.array([total - 1, 137])[:B]
    return q, k, v, g, pos


def _flat(recs):
    """The header's record layout for B sequences: o [B][16][256] then lse [B][16]."""
    return np.concatenate([np.stack([r[0] for r in recs]).ravel(), np.stack([r[1] for r in recs]).ravel()])


def _unflat(x, B):
    o = x[:B * 16 * 256].reshape(B, 16, 256)
    lse = x[B * 16 * 256:].reshape(B, 16)
    return [(o[b], lse[b]) for b in range(B)]


def _reference(q, k, v, g, pos):
    out = []
    for b, p in enumerate(pos):
        qr = O.rope(q[b][None], np.array([p]), O.FULL)
        out.append(O.attention(qr, k[b, :p + 1], v[b, :p + 1], g[b][None], np.array([p]), np.arange(p + 1),
                               O.FULL)[0])
    return np.stack(out)


def _rank_record(q, k, v, pos, rank, world):
    total = k.shape[1]
    lo, n = shard_of(rank, world, total)
    recs = []
    for b, p in enumerate(pos):
        qr = O.rope(q[b][None], np.array([p]), O.FULL)[0]
        hi = min(p + 1, lo + n)
        recs.append(_record(qr, k[b, lo:hi], v[b, lo:hi]) if hi > lo else _record(qr, k[b, :0], v[b, :0]))
    return _flat(recs)


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_merge_of_shard_records_is_whole_cache_attention(world):
    q, k, v, g, pos = _problem()
    B = len(pos)
    recs = [_unflat(_rank_record(q, k, v, pos, r, world), B) for r in range(world)]
    got = np.stack([_merge([recs[r][b] for r in range(world)], g[b]) for b in range(B)])
    np.testing.assert_allclose(got, _reference(q, k, v, g, pos), rtol=1e-12, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, g, pos = _problem()
        mine = torch.from_numpy(_rank_record(q, k, v, pos, rank, world))
        gathered = gather_records(mine).numpy()               # [world, n], rank order
        B = len(pos)
        recs = [_unflat(gathered[r], B) for r in range(world)]
        res = np.stack([_merge([recs[r][b] for r in range(world)], g[b]) for b in range(B)])
        out[rank] = (res, gathered[rank].tobytes() == mine.numpy().tobytes())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_record_exchange_two_ranks_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    q, k, v, g, pos = _problem()
    ref = _reference(q, k, v, g, pos)
    for rank in range(world):
        res, own_row = out[rank]
        assert own_row                                   # row r of the gather is rank r's record
        np.testing.assert_allclose(res, ref, rtol=1e-12, atol=1e-12)
