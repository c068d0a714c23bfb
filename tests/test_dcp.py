"""Decode context parallel: the exchange on CPU ranks (gloo, world size 2)
with oracle stand-ins for the local call and the merge, and the shard
arithmetic. The GPU path (library kernels) is in test_dcp_gpu.py."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shards_cover_each_sequence_once():
    from paged_kv_decode_30_b200 import dcp
    from paged_kv_decode_30_b200 import workloads as W
    wl = W.Workload(name="dcp_shards", batch=4, num_q_heads=4, num_kv_heads=2, head_dim=16,
                    page_size=8, kv_lens=("fixed", [0, 5, 64, 203]), seed=3)
    inp = W.generate(wl)
    for world in (1, 2, 3, 5):
        lens = torch.zeros(wl.batch, dtype=torch.int64)
        pages = [[] for _ in range(wl.batch)]
        for r in range(world):
            pt, kl = dcp.shard_sequences(inp["page_table"], inp["kv_lens"], 8, r, world)
            lens += kl.to(torch.int64)
            for b in range(wl.batch):
                n = (int(kl[b]) + 7) // 8
                pages[b] += pt[b, :n].tolist()
        assert lens.tolist() == inp["kv_lens"].tolist()
        for b in range(wl.batch):
            n = (int(inp["kv_lens"][b]) + 7) // 8
            assert pages[b] == inp["page_table"][b, :n].tolist()


def _oracle_local(q, k_pages, v_pages, page_table, kv_lens, *, num_kv_heads, scale, kv_scale,
                  page_size, kv_dtype, **kw):
    from oracle import oracle as orc
    from paged_kv_decode_30_b200 import workloads as W
    out, lse = orc.paged_decode_attn(
        W.to_bits(q), W.to_bits(k_pages), W.to_bits(v_pages), page_table.numpy(),
        kv_lens.numpy(), num_kv_heads=num_kv_heads, page_size=page_size, scale=scale,
        kv_dtype=kv_dtype, kv_scale=kv_scale)
    return torch.from_numpy(out), torch.from_numpy(lse), 1


def _oracle_merge(o_parts, l_parts, sinks=None):
    from oracle import oracle as orc
    o, l = o_parts.numpy(), l_parts.numpy()
    if sinks is not None:  # the sink is one more part with lse = sink, o = 0
        Hq = sinks.numel()
        rows = l.shape[1]
        l = np.concatenate([l, np.tile(sinks.numpy().astype(np.float64), rows // Hq)[None]], 0)
        o = np.concatenate([o, np.zeros((1,) + o.shape[1:])], 0)
    out, lse = orc.merge_states(o, l)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _worker(rank, world, port, kv_dtype, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from oracle import oracle as orc
    from paged_kv_decode_30_b200 import dcp
    from paged_kv_decode_30_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.Workload(name="dcp_cpu", batch=3, q_len=2, num_q_heads=8, num_kv_heads=2,
                        head_dim=32, page_size=8, kv_dtype=kv_dtype,
                        kv_lens=("fixed", [3, 40, 97]), seed=44)
        inp = W.generate(wl)
        pt, kl = dcp.shard_sequences(inp["page_table"], inp["kv_lens"], 8, rank, world)
        sinks = torch.tensor([0.5, -1.0, 3.0, float("-inf"), 0.0, 1.0, 2.0, -2.0])
        out, lse = dcp.dcp_paged_decode_attn(
            inp["q"], inp["k_pages"], inp["v_pages"], pt, kl, num_kv_heads=2,
            scale=W.scale_of(wl), kv_scale=inp["kv_scale"], sinks=sinks,
            local_fn=lambda *a, **k: _oracle_local(*a, page_size=8, kv_dtype=kv_dtype, **k),
            merge_fn=_oracle_merge)
        ref_out, ref_lse = orc.paged_decode_attn(
            W.to_bits(inp["q"]), W.to_bits(inp["k_pages"]), W.to_bits(inp["v_pages"]),
            inp["page_table"].numpy(), inp["kv_lens"].numpy(), num_kv_heads=2, page_size=8,
            scale=W.scale_of(wl), kv_dtype=kv_dtype, kv_scale=inp["kv_scale"],
            sinks=sinks.numpy())
        e_out = float(np.abs(out.numpy() - ref_out).max())
        both_inf = np.isinf(lse.numpy()) & np.isinf(ref_lse)
        e_lse = float(np.where(both_inf, 0.0, np.abs(lse.numpy() - ref_lse)).max())
        q_out.put((rank, e_out, e_lse))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["bf16", "fp8"])
def test_dcp_exchange_on_two_cpu_ranks(kv_dtype):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, kv_dtype, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, e_out, e_lse in res:
        assert e_out <= 1e-10 and e_lse <= 1e-10, (rank, e_out, e_lse)


def test_dcp_rejects_masked_calls():
    from paged_kv_decode_30_b200 import dcp
    with pytest.raises(ValueError):
        dcp.dcp_paged_decode_attn(torch.zeros(1, 1, 1, 64), None, None, None, None,
                                  num_kv_heads=1, scale=1.0, causal_offset=-2)
    with pytest.raises(ValueError):
        dcp.dcp_paged_decode_attn(torch.zeros(1, 1, 1, 64), None, None, None, None,
                                  num_kv_heads=1, scale=1.0, window=16)
