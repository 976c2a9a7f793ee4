"""Context-parallel decode of full layers: one cache split by position across ranks.

One process per GPU (``torch.distributed``, NCCL between GPUs).  A full
layer's cache of ``total`` positions is cut into ``world`` contiguous shards;
rank r keeps positions ``key_off .. key_off + rows - 1`` in its own
``[B, 4, rows, 256]`` K and V.  A decode step of that layer:

  1. ``spark_kv_append_cp`` on every rank (the rank holding ``pos[b]`` writes
     token b, the others skip it);
  2. ``spark_attn_decode_cp_partial`` on every rank: its record (normalised
     output and base-2 log-sum-exp per sequence and query head, over its keys);
  3. an all-gather of the records (the one exchange of the step);
  4. ``spark_attn_decode_cp_merge``: the log-sum-exp weighted mean, gated.

Sliding layers are not sharded: every rank keeps the 512-row ring and calls
``spark_attn_decode``.  This module is plumbing (shard bounds, buffers, the
collective); the arithmetic runs in libspark_attn.so's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (SPARK_FULL, SparkLayerCfg, spark_attn_decode_cp_merge, spark_attn_decode_cp_partial,
               spark_decode_cp_record_bytes, spark_decode_workspace_bytes, spark_kv_append_cp)


def shard_of(rank: int, world: int, total: int) -> tuple[int, int]:
    """(key_off, rows) of rank's shard of positions 0 .. total-1: contiguous, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if total < world:
        raise ValueError(f"{total} positions cannot give each of {world} ranks a row")
    lo = rank * total // world
    hi = (rank + 1) * total // world
    return lo, hi - lo


def owner_of(pos: int, world: int, total: int) -> int:
    """The rank whose shard holds position pos (0 <= pos < total)."""
    if not 0 <= pos < total:
        raise ValueError(f"position {pos} outside 0..{total - 1}")
    r = min(world - 1, pos * world // total)
    while shard_of(r, world, total)[0] > pos:
        r -= 1
    while sum(shard_of(r, world, total)) <= pos:
        r += 1
    return r


def gather_records(record: torch.Tensor, out: torch.Tensor | None = None, group=None) -> torch.Tensor:
    """All-gather of one record per rank into [world, n], rank r's in row r."""
    world = dist.get_world_size(group)
    flat = record.reshape(-1)
    if out is None:
        out = torch.empty((world, flat.numel()), dtype=flat.dtype, device=flat.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, flat, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), flat, group=group)
    return out


class FullLayerShard:
    """This rank's shard of one full layer's cache for B sequences, and its decode step."""

    def __init__(self, B: int, total: int, cfg: SparkLayerCfg, group=None, device=None):
        if cfg.kind != SPARK_FULL:
            raise ValueError("only full layers are sharded; sliding layers keep the whole ring on every rank")
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.B, self.total, self.cfg = B, total, cfg
        self.key_off, self.rows = shard_of(self.rank, self.world, total)
        dev = torch.device("cuda") if device is None else device
        self.k_cache = torch.zeros(B, 4, self.rows, 256, dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.zeros_like(self.k_cache)
        n = spark_decode_cp_record_bytes(B) // 4
        self.record = torch.empty(n, dtype=torch.float32, device=dev)
        self.records = torch.empty(self.world, n, dtype=torch.float32, device=dev)
        self.workspace = torch.empty(spark_decode_workspace_bytes(B, self.rows, cfg), dtype=torch.uint8, device=dev)

    def append(self, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor, flags: int = 0) -> None:
        """k, v [B, 4, 256] of the new tokens at pos[b]; only the rank holding pos[b] stores token b."""
        spark_kv_append_cp(self.k_cache, self.v_cache, self.key_off, k, v, pos, self.cfg, flags)

    def attend(self, out: torch.Tensor, q: torch.Tensor, gate: torch.Tensor, pos: torch.Tensor,
               flags: int = 0) -> None:
        """out [B, 16, 256] on every rank: attention of q at pos[b] over all ranks' shards, gated."""
        spark_attn_decode_cp_partial(self.record, q, self.k_cache, self.v_cache, self.key_off, pos, self.cfg,
                                     self.workspace, flags)
        if self.world > 1:
            gather_records(self.record, self.records, self.group)
        else:
            self.records[0].copy_(self.record)
        spark_attn_decode_cp_merge(out, gate, self.records)
