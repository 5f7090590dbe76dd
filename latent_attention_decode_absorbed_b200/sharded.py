"""KV-sharded decode: the cached rows of each sequence split across GPUs.

The softmax sum over a sequence's rows ("DeepSeek-V2: MLA Explained", "MLA
Full Formulas" part 3) decomposes exactly over disjoint row ranges, so GPU g
can attend over its own range of every sequence's rows and report one
normalised fp32 output and log-normaliser per (query row, head): 513 floats.
One exchange follows: the GPUs all-gather those results, and every GPU merges
the shards with ``mla_combine_shards``.  Nothing else crosses GPUs; the query
projection (``mla_absorb_q``) and the value up-projection (``mla_out_uv``)
run replicated on every GPU.

Row ranges are whole 64-row pages.  The new rows of a step (the last q_len
rows) always lie in one shard, the last, so the causal rule only bites there:
every row of an earlier shard is visible to every query token.  On GPU g each
query token becomes its own sequence of the attention call (q_len 1), whose
length is the number of the shard's rows that token sees and whose block
table is the shard's pages of its sequence.

Host planning and the exchange are here; the arithmetic is in the library's
kernels (``mla_decode_fwd``, ``mla_combine``, ``mla_combine_shards``).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple

import numpy as np

from . import (MLA_BF16, MLA_F32, PAGE, mla_combine, mla_combine_shards, mla_decode_fwd)


@dataclass(frozen=True)
class ShardPlan:
    """Row ranges [lo, hi) of every sequence on every shard (GPU).

    ranges[g][b] = (lo, hi): sequence b's rows held by shard g; lo and hi are
    multiples of the page size except hi = L_b on the last shard."""
    seq_lens: Tuple[int, ...]
    q_len: int
    world: int
    ranges: Tuple[Tuple[Tuple[int, int], ...], ...]


def plan_shards(seq_lens: Sequence[int], q_len: int, world: int) -> ShardPlan:
    """Split each sequence's pages into `world` contiguous, non-empty runs.

    Pages are dealt out as evenly as possible (the last shards take the extra
    pages, so the last shard's part-filled page has company); the boundary
    before the last shard is then moved down, if needed, so that the last
    shard holds all q_len new rows.  Every sequence needs at least `world`
    pages."""
    if world < 1 or q_len < 1:
        raise ValueError("world and q_len must be >= 1")
    ranges: List[List[Tuple[int, int]]] = [[] for _ in range(world)]
    for L in seq_lens:
        L = int(L)
        if L < q_len:
            raise ValueError(f"sequence length {L} below q_len {q_len}")
        pages = -(-L // PAGE)
        if pages < world:
            raise ValueError(f"a sequence of {L} rows has {pages} pages, fewer than {world} shards")
        base, extra = divmod(pages, world)
        bounds = [0]
        for g in range(world):
            bounds.append(bounds[-1] + base + (1 if g >= world - extra else 0))
        rows = [min(p * PAGE, L) for p in bounds]
        # the last shard must start at or before the first new row
        first_new = L - q_len
        if rows[world - 1] > first_new:
            rows[world - 1] = (first_new // PAGE) * PAGE
            if world >= 2 and rows[world - 1] <= rows[world - 2]:
                raise ValueError(f"sequence of {L} rows: the {q_len} new rows do not fit one shard "
                                 f"with {world} non-empty shards")
        for g in range(world):
            ranges[g].append((rows[g], rows[g + 1]))
    return ShardPlan(tuple(int(x) for x in seq_lens), int(q_len), int(world),
                     tuple(tuple(r) for r in ranges))


def visible_rows(plan: ShardPlan, g: int, b: int, t: int) -> int:
    """How many of shard g's rows of sequence b query token t sees: the
    shard's rows at positions <= L_b - q_len + t (a prefix of the shard)."""
    lo, hi = plan.ranges[g][b]
    last_visible = plan.seq_lens[b] - plan.q_len + t          # inclusive position
    return max(0, min(hi, last_visible + 1) - lo)


def shard_inputs(plan: ShardPlan, g: int, block_table: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Block table and lengths of the attention call on shard g.

    block_table: the full table [batch, max_pages] (page ids of every
    sequence's pages in order).  Returns (table [batch*q_len, P_g], lens
    [batch*q_len]) int32, one row per query token (row b*q_len + t), P_g the
    most pages any sequence has on shard g; unused entries are -1."""
    B, T = len(plan.seq_lens), plan.q_len
    spans = [(lo // PAGE, -(-hi // PAGE)) for lo, hi in plan.ranges[g]]
    P = max(p1 - p0 for p0, p1 in spans)
    table = np.full((B * T, P), -1, np.int32)
    lens = np.zeros(B * T, np.int32)
    for b, (p0, p1) in enumerate(spans):
        for t in range(T):
            r = b * T + t
            table[r, :p1 - p0] = block_table[b, p0:p1]
            lens[r] = visible_rows(plan, g, b, t)
    return table, lens


def decode_shard(q_abs, cache, cache_scale, cache_dtype: int, num_pages: int, table, lens, n_heads: int,
                 split_tokens: int, softmax_scale: float, o_part, lse_part, o_shard, lse_shard, err=None,
                 stream=None):
    """Shard g's part of the attention: ``mla_decode_fwd`` over its rows (one
    sequence per query token, from ``shard_inputs``) and ``mla_combine`` of
    its splits into o_shard [rows, n_heads, 512] fp32 and lse_shard
    [rows, n_heads].  o_part / lse_part: workspace [rows, n_heads, S, 512] and
    [rows, n_heads, S] with S = ceil(table.shape[1] * 64 / split_tokens)."""
    rows, max_pages = table.shape[0], table.shape[1]
    S = -(-max_pages * PAGE // split_tokens)
    mla_decode_fwd(q_abs, MLA_BF16 if cache_dtype != MLA_F32 else MLA_F32, cache, cache_scale, cache_dtype,
                   num_pages, table, max_pages, PAGE, lens, rows, 1, n_heads, S, split_tokens, softmax_scale,
                   o_part, lse_part, err, stream)
    mla_combine(o_part, lse_part, rows, n_heads, S, o_shard, MLA_F32, lse_shard, stream)


def gather_shards(o_shard, lse_shard, group=None):
    """All-gather every GPU's shard result in rank order: returns
    (o_all [world, rows, n_heads, 512], lse_all [world, rows, n_heads]).
    One NCCL all-gather per tensor on GPUs; other backends (gloo on the host)
    gather through a list."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return o_shard.unsqueeze(0), lse_shard.unsqueeze(0)
    world = dist.get_world_size(group)
    o_all = o_shard.new_empty((world,) + tuple(o_shard.shape))
    l_all = lse_shard.new_empty((world,) + tuple(lse_shard.shape))
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(o_all, o_shard.contiguous(), group=group)
        dist.all_gather_into_tensor(l_all, lse_shard.contiguous(), group=group)
    else:
        dist.all_gather(list(o_all.unbind(0)), o_shard.contiguous(), group=group)
        dist.all_gather(list(l_all.unbind(0)), lse_shard.contiguous(), group=group)
    return o_all, l_all


def merge_shards(o_all, lse_all, o_lat, o_dtype: int, lse_out=None, stream=None):
    """Every GPU's merge of the gathered shard results (``mla_combine_shards``)."""
    G, rows, n_heads = lse_all.shape
    mla_combine_shards(o_all, lse_all, G, rows, n_heads, o_lat, o_dtype, lse_out, stream)
