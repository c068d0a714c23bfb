"""Decode context parallel: one decode step over a KV cache sharded by
sequence position across the ranks of a process group.

Every rank holds, for every sequence, a contiguous page-aligned range of its
keys (its own pool pages and page-table columns). One step is:

  1. the local call, ``paged_decode_attn`` over the rank's shard, giving the
     rank's attention state (out_r, lse_r) for every row: a softmax over a
     disjoint key set, exactly what a split of the single-GPU call is;
  2. an all-gather of (out_r, lse_r) across the group (NCCL over NVLink on
     GPUs);
  3. the log-sum-exp merge of the gathered states (``pda_merge_states``),
     where an attention sink, if any, is added once.

Sources: "b12x 0.30.0, Kernel inventory, Attention table, Paged attention
row" (split-KV partials and their persistent merge) and "sglang profiler
skill, fuse-overlap catalog" (``merge_attn_states``; decode context parallel
rows). Reading taken: the shards are page-aligned contiguous token ranges,
and DCP applies to calls where every cached key is visible to every query
row (causal off, no window: the decode step over the whole context), since a
shard's local positions do not carry the global ones a causal or window
mask would need.

Steps 1 and 3 run in this library's CUDA kernels; this module only slices
the page table, moves the states between ranks and calls them. ``local_fn``
and ``merge_fn`` exist so the exchange logic can be tested on CPU ranks
(gloo) with the test suite's own stand-ins; the default is the library.
"""

from __future__ import annotations

from typing import Callable, Optional, Tuple

from . import binding as B


def shard_pages(num_pages_seq: int, rank: int, world: int) -> Tuple[int, int]:
    """Page range [p0, p1) of a sequence with num_pages_seq pages on `rank`:
    balanced contiguous blocks, rank 0 first."""
    p0 = num_pages_seq * rank // world
    p1 = num_pages_seq * (rank + 1) // world
    return p0, p1


def shard_sequences(page_table, kv_lens, page_size: int, rank: int, world: int):
    """The rank's view of a global (page table, kv_lens): page-table columns
    of its page range (left-aligned, -1 after) and its shard's key counts.

    page_table: int32 [B, max_pages]; kv_lens: int32 [B] (torch tensors, any
    device). Returns (local_page_table, local_kv_lens) on the same device."""
    import torch
    B_, max_pages = page_table.shape
    lens = kv_lens.to("cpu").tolist()
    local_pt = torch.full_like(page_table, -1)
    local_len = torch.zeros_like(kv_lens)
    for b in range(B_):
        n = (lens[b] + page_size - 1) // page_size
        p0, p1 = shard_pages(n, rank, world)
        if p1 > p0:
            local_pt[b, : p1 - p0] = page_table[b, p0:p1]
        local_len[b] = max(0, min(lens[b], p1 * page_size) - p0 * page_size)
    return local_pt, local_len


def _all_gather(t, world: int, group):
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def dcp_paged_decode_attn(q, k_pages, v_pages, page_table, kv_lens, *, num_kv_heads: int,
                          scale: float, kv_scale: float = 1.0, sinks=None, group=None,
                          local_fn: Optional[Callable] = None,
                          merge_fn: Optional[Callable] = None, **local_kw):
    """One decode step under decode context parallel.

    q                 [B, q_len, Hq, D] bf16, the same on every rank.
    k/v_pages         this rank's pools; page_table / kv_lens this rank's
                      shard (see shard_sequences).
    sinks             optional fp32 [Hq] attention-sink logits (merged once).
    Returns (out [B, q_len, Hq, D] fp32, lse [B, q_len, Hq] fp32), identical
    on every rank.
    """
    import torch.distributed as dist
    if local_kw.get("causal_offset", B.PDA_CAUSAL_OFF) != B.PDA_CAUSAL_OFF or \
            local_kw.get("window", 0) > 0:
        raise ValueError("decode context parallel takes calls that see every cached key "
                         "(causal off, no window)")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    Bsz, Lq, Hq, D = q.shape
    rows = Bsz * Lq * Hq
    local = local_fn or B.paged_decode_attn
    out_r, lse_r, _ = local(q, k_pages, v_pages, page_table, kv_lens, num_kv_heads=num_kv_heads,
                            scale=scale, kv_scale=kv_scale, **local_kw)
    out_r = out_r.reshape(rows, D)
    lse_r = lse_r.reshape(rows)
    if world > 1:
        o_parts = _all_gather(out_r, world, group)       # [world, rows, D]
        l_parts = _all_gather(lse_r, world, group)       # [world, rows]
    else:
        o_parts, l_parts = out_r.unsqueeze(0), lse_r.unsqueeze(0)
    merge = merge_fn or B.merge_states
    out, lse = merge(o_parts.contiguous(), l_parts.contiguous(), sinks=sinks)
    return out.reshape(Bsz, Lq, Hq, D), lse.reshape(Bsz, Lq, Hq)
