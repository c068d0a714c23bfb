"""paged_decode_attn_no_alloc: the entry point for callers that cannot
allocate device memory (for example an engine that has reserved nearly all
of HBM for its own KV-cache pool, or a latency-critical path where
cudaMalloc / cudaFree may synchronise the device). The call's whole
workspace lives in a fixed array inside the library; with the same split
count its results must equal the regular entry point's bit for bit, and
match the oracle. This file is named so that pytest collects it last."""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASE_A = W.Workload(name="no_alloc_bf16", batch=6, num_q_heads=32, num_kv_heads=8,
                    head_dim=128, page_size=16, kv_lens=("fixed", [1000, 517, 33, 2048, 0, 700]),
                    extra_pages=3, seed=41)
CASE_B = W.Workload(name="no_alloc_longctx", batch=2, num_q_heads=16, num_kv_heads=4,
                    head_dim=256, page_size=128, scale=1 / 16,
                    kv_lens=("fixed", [9000, 4000]), seed=42)
# two tensor-core calls that differ in batch, rows, split count and flags
CASE_TC_BF16 = W.Workload(name="no_alloc_tc_bf16", batch=5, num_q_heads=16, num_kv_heads=4,
                          head_dim=128, page_size=32, kv_lens=("fixed", [3000, 1, 700, 0, 1500]),
                          extra_pages=2, seed=44)
CASE_TC_FP8 = W.Workload(name="no_alloc_tc_fp8_verify", batch=3, q_len=4, num_q_heads=64,
                         num_kv_heads=8, head_dim=128, page_size=128, kv_dtype=W.KV_FP8_E4M3,
                         causal_offset=W.CAUSAL_BOTTOM_RIGHT, window=700,
                         kv_lens=("fixed", [2500, 130, 900]), poison_invisible=True, seed=45)


def _both(inp, splits, flags=0):
    """The regular entry point, then the no-alloc one, on the same inputs;
    returns host float64 (out, lse) of each and the split count."""
    wl = inp["workload"]
    t = U.to_device(inp)
    kw = dict(num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl),
              causal_offset=wl.causal_offset, window=wl.window, kv_scale=inp["kv_scale"],
              num_splits=splits, flags=flags)
    ref_out, ref_lse, ref_used = B.paged_decode_attn(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], **kw)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    # out / lse start as NaN: every element must be written by the call
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    _, _, used = B.paged_decode_attn_no_alloc(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], out=out, lse=lse, **kw)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    assert used == ref_used
    return (out.double().cpu().numpy(), lse.double().cpu().numpy(),
            ref_out.double().cpu().numpy(), ref_lse.double().cpu().numpy(), used)


def _check(case, splits, flags=0, expect_kernel=None):
    inp = W.generate(case)
    if expect_kernel is not None:
        wl = inp["workload"]
        p = B.make_params(batch=wl.batch, q_len=wl.q_len, num_q_heads=wl.num_q_heads,
                          num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                          page_size=wl.page_size, max_pages_per_seq=inp["page_table"].shape[1],
                          num_pages=inp["k_pages"].shape[0], scale=W.scale_of(wl),
                          kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"], num_splits=splits,
                          flags=flags)
        assert B.plan_kernel(p) == expect_kernel
    out, lse, ref_out, ref_lse, used = _both(inp, splits, flags)
    assert used > 1, "the case must exercise the split partials"
    # same kernels, same split count: identical bits
    assert np.array_equal(out, ref_out, equal_nan=True)
    assert np.array_equal(lse, ref_lse, equal_nan=True)
    o_out, o_lse = U.run_oracle(inp)
    U.assert_parity(out, lse, o_out, o_lse, case.kv_dtype, f"{case.name}/no_alloc/s={used}")


def test_no_alloc_matches_regular_entry_point_two_calls_in_a_row():
    # two calls in a row on different inputs, kernels and split counts: the
    # second call must not see anything the first left in the shared array
    _check(CASE_A, 5, expect_kernel=B.PDA_KERNEL_SPLIT_TMA)
    _check(CASE_B, 0, expect_kernel=B.PDA_KERNEL_SPLIT_FMA)


def test_no_alloc_tensor_core_calls_back_to_back():
    """Two tensor-core calls in a row on the shared array: its counter
    header, queue order and (FP8) Q operand images are rewritten by the
    second call's prologue, and the in-kernel merge counts from zero."""
    _check(CASE_TC_BF16, 3, flags=B.PDA_FLAG_TENSOR_CORES, expect_kernel=B.PDA_KERNEL_SPLIT_TMA)
    _check(CASE_TC_FP8, 2, flags=B.PDA_FLAG_FUSED_MERGE, expect_kernel=B.PDA_KERNEL_SPLIT_TMA)
    _check(CASE_TC_BF16, 4, flags=B.PDA_FLAG_TENSOR_CORES | B.PDA_FLAG_FUSED_MERGE)


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


def _fresh_process_body():
    """Run in a new process: no_alloc calls come before any regular call, and
    the device's free memory does not move across a call whose workspace is
    larger than every earlier call's (a cudaMalloc, or the library-owned
    buffer of the regular entry point, would take at least 2 MiB)."""
    torch.cuda.set_device(0)
    B.load()
    wl = W.Workload(name="no_alloc_fresh", batch=64, num_q_heads=32, num_kv_heads=8,
                    head_dim=128, page_size=16, kv_lens=("uniform", 200, 900), seed=46)
    inp = W.generate(wl, device="cuda")
    t = U.to_device(inp)
    out = torch.empty((64, 1, 32, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((64, 1, 32), dtype=torch.float32, device="cuda")
    kw = dict(num_kv_heads=8, scale=W.scale_of(wl), out=out, lse=lse,
              flags=B.PDA_FLAG_TENSOR_CORES)

    def need(splits):
        return B.workspace_bytes(B.make_params(
            batch=64, q_len=1, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
            max_pages_per_seq=t["page_table"].shape[1], num_pages=t["k_pages"].shape[0],
            scale=W.scale_of(wl), num_splits=splits, flags=B.PDA_FLAG_TENSOR_CORES))

    assert need(2) < 4 << 20 and 4 << 20 < need(6) <= B.PDA_NO_ALLOC_WORKSPACE_BYTES
    # first call on the device: symbol lookup and kernel loading happen here
    B.paged_decode_attn_no_alloc(t["q"], t["k_pages"], t["v_pages"], t["page_table"],
                                 t["kv_lens"], num_splits=2, **kw)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    B.paged_decode_attn_no_alloc(t["q"], t["k_pages"], t["v_pages"], t["page_table"],
                                 t["kv_lens"], num_splits=6, **kw)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert B.last_device_error() == 0
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"
    got = (out.double().cpu().numpy(), lse.double().cpu().numpy())
    ref_out, ref_lse = U.run_oracle(inp)
    U.assert_parity(got[0], got[1], ref_out, ref_lse, W.KV_BF16, "no_alloc fresh process")
    print("fresh process: free memory unchanged", free0)


def test_no_alloc_allocates_nothing_in_a_fresh_process():
    r = subprocess.run(
        [sys.executable, "-c",
         "from tests.test_zz_no_alloc import _fresh_process_body as f; f()"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "free memory unchanged" in r.stdout
