"""Decode context parallel on one GPU: the ranks' local calls and the merge
through the library's kernels (the NCCL all-gather between them is replaced
by stacking the states in one process), against the oracle."""

import pytest
import torch

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import dcp
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8_E4M3], ids=["bf16", "fp8"])
@pytest.mark.parametrize("world", [2, 3, 8])
def test_dcp_kernels_match_oracle(kv_dtype, world):
    wl = W.Workload(name="dcp_gpu", batch=6, q_len=2, num_q_heads=32, num_kv_heads=4,
                    head_dim=128, page_size=16, kv_dtype=kv_dtype,
                    kv_lens=("fixed", [1, 17, 300, 1000, 4096, 64]), seed=91)
    inp = W.generate(wl)
    d = U.to_device(inp)
    g = torch.Generator().manual_seed(5)
    sinks = (torch.randn(wl.num_q_heads, generator=g) * 2).cuda()
    rows = wl.batch * wl.q_len * wl.num_q_heads
    outs, lses = [], []
    for r in range(world):
        pt, kl = dcp.shard_sequences(d["page_table"], d["kv_lens"], wl.page_size, r, world)
        o, l, _ = B.paged_decode_attn(d["q"], d["k_pages"], d["v_pages"], pt.contiguous(),
                                      kl.contiguous(), num_kv_heads=wl.num_kv_heads,
                                      scale=W.scale_of(wl), kv_scale=inp["kv_scale"])
        outs.append(o.reshape(rows, wl.head_dim))
        lses.append(l.reshape(rows))
    out, lse = B.merge_states(torch.stack(outs).contiguous(), torch.stack(lses).contiguous(),
                              sinks=sinks)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    ref_out, ref_lse = U.run_oracle(inp, sinks=sinks.cpu().numpy())
    U.assert_parity(out.reshape(ref_out.shape).double().cpu().numpy(),
                    lse.reshape(ref_lse.shape).double().cpu().numpy(), ref_out, ref_lse,
                    kv_dtype, f"dcp world {world}")


def test_dcp_function_single_rank():
    """dcp_paged_decode_attn without a process group: one shard, the
    library's call then its merge (one part, plus the sink)."""
    wl = W.Workload(name="dcp_one", batch=3, num_q_heads=16, num_kv_heads=2, head_dim=128,
                    page_size=16, kv_lens=("fixed", [5, 200, 33]), seed=92)
    inp = W.generate(wl)
    d = U.to_device(inp)
    sinks = torch.tensor([1.0] * 16).cuda()
    out, lse = dcp.dcp_paged_decode_attn(d["q"], d["k_pages"], d["v_pages"], d["page_table"],
                                         d["kv_lens"], num_kv_heads=2, scale=W.scale_of(wl),
                                         sinks=sinks)
    torch.cuda.synchronize()
    ref_out, ref_lse = U.run_oracle(inp, sinks=sinks.cpu().numpy())
    U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse,
                    W.KV_BF16, "dcp single rank")
