"""paged_decode_attn_no_alloc: the entry point for callers that cannot
allocate device memory (for example an engine that has reserved nearly all
of HBM for its own KV-cache pool, or a latency-critical path where
cudaMalloc / cudaFree may synchronise the device). Its split partials live in
a fixed array inside the library; its results must match the regular entry
point's. This file is named so that pytest collects it last."""

import pytest
import torch

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

CASE_A = W.Workload(name="no_alloc_bf16", batch=6, num_q_heads=32, num_kv_heads=8,
                    head_dim=128, page_size=16, kv_lens=("fixed", [1000, 517, 33, 2048, 0, 700]),
                    extra_pages=3, seed=41)
CASE_B = W.Workload(name="no_alloc_longctx", batch=2, num_q_heads=16, num_kv_heads=4,
                    head_dim=256, page_size=128, scale=1 / 16,
                    kv_lens=("fixed", [9000, 4000]), seed=42)


def _both(inp, splits):
    wl = inp["workload"]
    t = U.to_device(inp)
    kw = dict(num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl),
              causal_offset=wl.causal_offset, window=wl.window, kv_scale=inp["kv_scale"],
              num_splits=splits)
    ref_out, ref_lse, ref_used = B.paged_decode_attn(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], **kw)
    out, lse, used = B.paged_decode_attn_no_alloc(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], **kw)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    assert used == ref_used
    return (out.double().cpu().numpy(), lse.double().cpu().numpy(),
            ref_out.double().cpu().numpy(), ref_lse.double().cpu().numpy(), used)


def test_no_alloc_matches_regular_entry_point_two_calls_in_a_row():
    tol = U.TOL[W.KV_BF16]
    # two calls in a row on different inputs and split counts: the second
    # call must not see anything the first left in the shared array
    for case, splits in ((CASE_A, 5), (CASE_B, 0)):
        out, lse, ref_out, ref_lse, used = _both(W.generate(case), splits)
        assert used > 1, "the case must exercise the split partials"
        assert U.max_err(out, ref_out) <= tol["out"]
        assert U.max_err(lse, ref_lse) <= tol["lse"]


def test_no_alloc_rejects_partials_beyond_its_limit():
    inp = W.generate(CASE_A)
    t = U.to_device(inp)
    # 16 splits of 128 * 32 rows of 129 floats (about 34 MB) do not fit (the
    # CUDA-core kernel splits 256 keys 16 ways; 128-key tiles would not)
    big = W.Workload(name="no_alloc_big", batch=128, num_q_heads=32, num_kv_heads=8,
                     head_dim=128, page_size=16, kv_lens=("const", 256), seed=43)
    binp = W.generate(big)
    bt = U.to_device(binp)
    need = B.workspace_bytes(B.make_params(
        batch=128, q_len=1, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
        max_pages_per_seq=bt["page_table"].shape[1], num_pages=bt["k_pages"].shape[0],
        scale=W.scale_of(big), num_splits=16, flags=B.PDA_FLAG_CUDA_CORES))
    assert need > B.PDA_NO_ALLOC_WORKSPACE_BYTES
    with pytest.raises(B.PdaError) as e:
        B.paged_decode_attn_no_alloc(bt["q"], bt["k_pages"], bt["v_pages"], bt["page_table"],
                                     bt["kv_lens"], num_kv_heads=8, scale=W.scale_of(big),
                                     num_splits=16, flags=B.PDA_FLAG_CUDA_CORES)
    assert e.value.status == 4  # PDA_ERR_WORKSPACE
    # the small case still works afterwards
    out, lse, _ = B.paged_decode_attn_no_alloc(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], num_kv_heads=8,
        scale=W.scale_of(CASE_A), num_splits=3)
    ref_out, ref_lse = U.run_oracle(inp)
    U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse,
                    W.KV_BF16, "no_alloc after a rejected call")
