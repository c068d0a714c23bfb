"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on
the same seeded inputs, element by element: small and mid sizes spanning
many tiles with ragged tails, and every row of the full workload sizes."""

import zlib

import numpy as np
import pytest
import torch

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

BF16, FP8, NV = W.KV_BF16, W.KV_FP8_E4M3, W.KV_NVFP4
BR = W.CAUSAL_BOTTOM_RIGHT


def wl(name, **kw):
    base = dict(route="pool", seed=zlib.crc32(name.encode()) % 100000)
    base.update(kw)
    return W.Workload(name=name, **base)


# Mid-size cases compared element by element.
CASES = [
    W.TINY,
    wl("varlen_mid", batch=4, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=64,
       kv_lens=("fixed", [1, 700, 64, 333]), extra_pages=5),
    wl("headline_shape_bf16", batch=3, num_q_heads=32, num_kv_heads=8, head_dim=128,
       page_size=16, kv_lens=("fixed", [1000, 517, 33]), extra_pages=3),
    wl("headline_shape_fp8", batch=3, num_q_heads=32, num_kv_heads=8, head_dim=128,
       page_size=16, kv_lens=("fixed", [1000, 517, 33]), extra_pages=3, kv_dtype=FP8),
    wl("longctx_mid_peaked", batch=2, num_q_heads=16, num_kv_heads=4, head_dim=256,
       page_size=128, scale=1 / 16, kv_lens=("fixed", [3000, 1111]), peaked_frac=0.01,
       route="dense"),
    wl("verify_fp8_window", batch=3, q_len=4, num_q_heads=64, num_kv_heads=8, head_dim=128,
       page_size=128, kv_dtype=FP8, causal_offset=BR, window=512,
       kv_lens=("fixed", [100, 700, 1500]), poison_invisible=True),
    wl("verify_bf16_window", batch=3, q_len=4, num_q_heads=64, num_kv_heads=8, head_dim=128,
       page_size=128, causal_offset=BR, window=512, kv_lens=("fixed", [100, 700, 1500]),
       poison_invisible=True),
    wl("d64_p8_mha", batch=3, num_q_heads=4, num_kv_heads=4, head_dim=64, page_size=8,
       kv_lens=("fixed", [77, 8, 300])),
    wl("d64_p256_gqa2_q3", batch=2, q_len=3, num_q_heads=4, num_kv_heads=2, head_dim=64,
       page_size=256, causal_offset=BR, kv_lens=("fixed", [600, 2])),
    wl("d128_p32_fixed_causal", batch=2, q_len=2, num_q_heads=8, num_kv_heads=1,
       head_dim=128, page_size=32, causal_offset=100, kv_lens=("fixed", [300, 50])),
    wl("d256_p16_window_noncausal", batch=2, num_q_heads=8, num_kv_heads=2, head_dim=256,
       page_size=16, window=40, kv_lens=("fixed", [200, 39]), poison_invisible=True),
    wl("empty_and_short_rows", batch=4, q_len=4, num_q_heads=8, num_kv_heads=2, head_dim=128,
       page_size=16, causal_offset=BR, kv_lens=("fixed", [0, 1, 3, 20]), extra_pages=2),
    wl("gqa8_q1_d128", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=128, page_size=64,
       kv_lens=("fixed", [900, 65])),
    wl("fp8_d64_gqa4", batch=2, num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=32,
       kv_dtype=FP8, kv_lens=("fixed", [500, 31])),
    wl("fp8_d256_q2", batch=2, q_len=2, num_q_heads=4, num_kv_heads=2, head_dim=256,
       page_size=128, kv_dtype=FP8, causal_offset=BR, kv_lens=("fixed", [700, 129])),
    # tensor-core path: FP8, head_dim 128, more than 8 packed rows per kv head
    wl("tc_fp8_p16_q2_g8", batch=4, q_len=2, num_q_heads=16, num_kv_heads=2, head_dim=128,
       page_size=16, kv_dtype=FP8, causal_offset=BR, kv_lens=("fixed", [1, 130, 1000, 2047]),
       extra_pages=4),
    wl("tc_fp8_p256_g16", batch=2, num_q_heads=32, num_kv_heads=2, head_dim=128,
       page_size=256, kv_dtype=FP8, kv_lens=("fixed", [300, 5000])),
    wl("tc_fp8_p64_q3_g16_window", batch=3, q_len=3, num_q_heads=32, num_kv_heads=2,
       head_dim=128, page_size=64, kv_dtype=FP8, causal_offset=BR, window=200,
       kv_lens=("fixed", [2, 333, 1500]), poison_invisible=True),
    wl("tc_fp8_fixed_offset_empty", batch=3, q_len=4, num_q_heads=64, num_kv_heads=8,
       head_dim=128, page_size=128, kv_dtype=FP8, causal_offset=40, window=30,
       kv_lens=("fixed", [0, 20, 700]), extra_pages=2),
    # FP8 tensor-core path with peaked scores: 1% of the keys scaled by 8 and a
    # large softmax scale, so the weights span many binades and most fall far
    # below the largest (the two-term e4m3 P and the lazy max rescale)
    wl("tc_fp8_peaked_g8_q4", batch=2, q_len=4, num_q_heads=32, num_kv_heads=4, head_dim=128,
       page_size=128, kv_dtype=FP8, scale=0.25, causal_offset=BR, peaked_frac=0.01,
       kv_lens=("fixed", [3000, 5000])),
    # the bf16 tensor-core path (4 packed rows) on the same kind of scores
    wl("tc_bf16_peaked_g4", batch=2, num_q_heads=16, num_kv_heads=4, head_dim=128,
       page_size=16, scale=0.25, peaked_frac=0.01, kv_lens=("fixed", [3000, 8000])),
    # NVFP4 K/V (e2m1 codes + an e4m3 scale per 16 elements), NaN scales in
    # the slots no row may read
    wl("nvfp4_headline_shape", batch=3, num_q_heads=32, num_kv_heads=8, head_dim=128,
       page_size=16, kv_dtype=NV, kv_lens=("fixed", [1000, 517, 33]), extra_pages=3),
    wl("nvfp4_verify_window", batch=3, q_len=4, num_q_heads=64, num_kv_heads=8,
       head_dim=128, page_size=128, kv_dtype=NV, causal_offset=BR, window=512,
       kv_lens=("fixed", [100, 700, 1500]), poison_invisible=True),
    wl("nvfp4_d64_p8_gqa4", batch=2, num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=8,
       kv_dtype=NV, kv_lens=("fixed", [77, 300]), extra_pages=2),
    wl("nvfp4_d256_p32_q2_window_peaked", batch=2, q_len=2, num_q_heads=4, num_kv_heads=2,
       head_dim=256, page_size=32, kv_dtype=NV, causal_offset=BR, window=100, scale=0.25,
       peaked_frac=0.02, kv_lens=("fixed", [700, 129]), poison_invisible=True, route="dense"),
    # NVFP4 on the tensor-core kernel: whole-tile pages, 8 packed rows,
    # peaked scores; then windowed verify rows with empty and 1-key sequences
    wl("nvfp4_tc_p256_g8_peaked", batch=3, num_q_heads=16, num_kv_heads=2, head_dim=128,
       page_size=256, kv_dtype=NV, scale=0.25, peaked_frac=0.01,
       kv_lens=("fixed", [3000, 257, 4096]), route="dense"),
    wl("nvfp4_tc_p64_q2_window_empty", batch=4, q_len=2, num_q_heads=8, num_kv_heads=4,
       head_dim=128, page_size=64, kv_dtype=NV, causal_offset=BR, window=300,
       kv_lens=("fixed", [0, 1, 900, 2000]), poison_invisible=True, extra_pages=2),
]


@pytest.fixture(scope="module")
def lib():
    return B.load()


@pytest.mark.parametrize("case", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [0, 1, 2, 3, 7, 64])
def test_parity_vs_oracle(lib, case, splits):
    inp = W.generate(case)
    ref_out, ref_lse = U.run_oracle(inp)
    out, lse, used = U.run_cuda(inp, num_splits=splits)
    if splits:
        assert 1 <= used <= splits
    U.assert_parity(out, lse, ref_out, ref_lse, case.kv_dtype, f"{case.name}/s={splits}")


# head_dim-128 cases: the planner picks the tensor-core kernel for some, the
# CUDA-core kernel for others; each is also run through the other kernel.
D128_CASES = [c for c in CASES if c.head_dim == 128]


@pytest.mark.parametrize("case", D128_CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [0, 1, 3, 64])
@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores", "tensor_cores_fused_merge"])
def test_parity_forced_kernel(lib, case, splits, kernel):
    """Both split kernels on every head_dim-128 case (flags force the choice),
    the tensor-core one also with the in-kernel merge of its splits."""
    flags = {"cuda_cores": B.PDA_FLAG_CUDA_CORES, "tensor_cores": B.PDA_FLAG_TENSOR_CORES,
             "tensor_cores_fused_merge": B.PDA_FLAG_TENSOR_CORES | B.PDA_FLAG_FUSED_MERGE}[kernel]
    inp = W.generate(case)
    ref_out, ref_lse = U.run_oracle(inp)
    out, lse, _ = U.run_cuda(inp, num_splits=splits, flags=flags)
    U.assert_parity(out, lse, ref_out, ref_lse, case.kv_dtype, f"{case.name}/{kernel}/s={splits}")


@pytest.mark.parametrize("case", [CASES[2], CASES[5], CASES[7]] +
                         [c for c in CASES if c.kv_dtype == NV][:2], ids=lambda w: w.name)
def test_page_permutation_invariance(lib, case):
    inp = W.generate(case)
    out0, lse0, _ = U.run_cuda(inp)
    n = inp["k_pages"].shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(7))
    moved = {}
    for key in ("k_pages", "v_pages", "k_scales", "v_scales"):
        if inp.get(key) is not None:
            moved[key] = torch.empty_like(inp[key])
            moved[key][perm] = inp[key]
    pt = inp["page_table"].to(torch.int64)
    pt2 = torch.where(pt >= 0, perm[pt.clamp(min=0)], pt).to(torch.int32)
    out1, lse1, _ = U.run_cuda(dict(inp, page_table=pt2, **moved))
    # the kernel's arithmetic depends only on logical token order
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


def test_split_counts_agree_with_each_other(lib):
    case = CASES[4]
    inp = W.generate(case)
    base_out, base_lse, _ = U.run_cuda(inp, num_splits=1)
    for s in (2, 5, 9, 31):
        out, lse, _ = U.run_cuda(inp, num_splits=s)
        assert U.max_err(out, base_out) <= 1e-5
        assert U.max_err(lse, base_lse) <= 1e-5


def test_lse_may_be_null(lib):
    inp = W.generate(CASES[2])
    t = U.to_device(inp)
    out, lse, _ = B.paged_decode_attn(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], num_kv_heads=8,
        scale=W.scale_of(CASES[2]), with_lse=False, num_splits=3)
    assert lse is None
    ref_out, _ = U.run_oracle(inp)
    assert U.max_err(out.double().cpu().numpy(), ref_out) <= 2e-3


def test_merge_kernel_vs_oracle_merge(lib):
    from oracle import oracle as orc
    g = torch.Generator().manual_seed(3)
    S, rows, D = 5, 300, 128
    o = torch.randn((S, rows, D), generator=g, dtype=torch.float32)
    ls = torch.randn((S, rows), generator=g, dtype=torch.float32) * 4
    ls[1, ::3] = -float("inf")
    o[1, ::3] = float("nan")          # never read when lse is -inf
    ls[:, 7] = -float("inf")           # an empty row
    o[:, 7] = float("nan")
    out, lse = B.merge_states(o.cuda(), ls.cuda())
    torch.cuda.synchronize()
    o_ref = torch.where(torch.isnan(o), torch.zeros_like(o), o).double().numpy()
    ref_out, ref_lse = orc.merge_states(o_ref, ls.double().numpy())
    assert U.max_err(out.double().cpu().numpy(), ref_out) <= 1e-5
    assert U.max_err(lse.double().cpu().numpy(), ref_lse) <= 1e-5


def test_bad_page_id_is_reported_not_dereferenced(lib):
    case = CASES[2]
    inp = W.generate(case)
    t = U.to_device(inp)
    pt = t["page_table"].clone()
    pt[1, 3] = inp["k_pages"].shape[0] + 1000   # outside the pool
    pt[2, 0] = -7
    B.last_device_error()
    out, lse, _ = B.paged_decode_attn(
        t["q"], t["k_pages"], t["v_pages"], pt, t["kv_lens"], num_kv_heads=8,
        scale=W.scale_of(case))
    assert B.last_device_error() == 6  # PDA_ERR_BAD_PAGE
    assert B.last_device_error() == 0  # reading clears it
    # sequence 0 never touched a bad page: still exact
    ref_out, ref_lse = U.run_oracle(inp, seqs=[0])
    U.assert_parity(out[:1].double().cpu().numpy(), lse[:1].double().cpu().numpy(),
                    ref_out, ref_lse, BF16, "untouched sequence")


def test_kv_len_beyond_page_table_is_reported(lib):
    case = CASES[2]
    inp = W.generate(case)
    t = U.to_device(inp)
    lens = t["kv_lens"].clone()
    lens[0] = t["page_table"].shape[1] * case.page_size + 1
    B.paged_decode_attn(t["q"], t["k_pages"], t["v_pages"], t["page_table"], lens,
                        num_kv_heads=8, scale=W.scale_of(case))
    assert B.last_device_error() == 6


# ---------------------------------------------------------------------------
# Full workload sizes, in the launch configuration the benchmark times.

def _full(name):
    return W.ALL[name]


def test_full_size_headline_every_row(lib):
    """The headline workload (B=128, kv_len 8192, bf16) in the benchmark's
    launch configuration, every row against the oracle (run on all host
    cores); then the same input through the CUDA-core kernel."""
    case = W.HEADLINE
    inp = W.generate(case, device="cuda")
    ref_out, ref_lse = U.run_oracle(inp)
    out, lse, _ = U.run_cuda(inp)
    U.assert_parity(out, lse, ref_out, ref_lse, BF16, f"{case.name}/full/auto")
    assert np.isfinite(out).all()
    out, lse, _ = U.run_cuda(inp, flags=B.PDA_FLAG_CUDA_CORES)
    U.assert_parity(out, lse, ref_out, ref_lse, BF16, f"{case.name}/full/cuda_cores")


def test_full_size_fp8_verify_every_row(lib):
    """The FP8 verify workload (B=64, q_len 4, lognormal lengths, window 4096)
    in the benchmark's launch configuration, every row against the oracle on
    the same e4m3 bytes: the exact two-term Q path, then native FP8 QK against
    the oracle run on the same quantised q."""
    case = W.FP8_VERIFY
    inp = W.generate(case, device="cuda")
    ref_out, ref_lse = U.run_oracle(inp)
    out, lse, _ = U.run_cuda(inp)
    U.assert_parity(out, lse, ref_out, ref_lse, FP8, f"{case.name}/full/auto")
    assert np.isfinite(out).all()
    ref_out, ref_lse = U.run_oracle(inp, native_qk=True)
    out, lse, _ = U.run_cuda(inp, flags=B.PDA_FLAG_NATIVE_FP8_QK)
    U.assert_parity(out, lse, ref_out, ref_lse, FP8, f"{case.name}/full/native_qk")


def test_full_size_nvfp4_headline_every_row(lib):
    """The headline shape with an NVFP4 KV cache, every row against the
    oracle on the same codes and block scales."""
    case = W.NVFP4_HEADLINE
    inp = W.generate(case, device="cuda")
    ref_out, ref_lse = U.run_oracle(inp)
    out, lse, _ = U.run_cuda(inp)
    U.assert_parity(out, lse, ref_out, ref_lse, NV, f"{case.name}/full")


@pytest.mark.parametrize("name", [W.VARLEN.name, W.LONGCTX.name])
def test_full_size_all_rows(lib, name):
    case = _full(name)
    inp = W.generate(case, device="cuda")
    out, lse, used = U.run_cuda(inp)
    ref_out, ref_lse = U.run_oracle(inp)
    U.assert_parity(out, lse, ref_out, ref_lse, case.kv_dtype, name)


@pytest.mark.parametrize("case", [c for c in CASES if c.name.startswith("tc_fp8")][:2] +
                         [c for c in CASES if c.kv_dtype == BF16 and c.head_dim == 128][:1],
                         ids=lambda w: w.name)
def test_workspace_contents_do_not_matter(lib, case):
    """The call zeroes the tensor-core kernel's counter header itself: a
    workspace full of random bytes, reused across calls, gives the same
    results as a fresh one."""
    inp = W.generate(case)
    ref_out, ref_lse = U.run_oracle(inp)
    params_kw = dict(num_splits=3, flags=B.PDA_FLAG_TENSOR_CORES | B.PDA_FLAG_FUSED_MERGE)
    t = U.to_device(inp)
    wl = inp["workload"]
    need = B.workspace_bytes(B.make_params(
        batch=wl.batch, q_len=wl.q_len, num_q_heads=wl.num_q_heads,
        num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, page_size=wl.page_size,
        max_pages_per_seq=t["page_table"].shape[1], num_pages=t["k_pages"].shape[0],
        scale=W.scale_of(wl), kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"], **params_kw))
    ws = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda",
                       generator=torch.Generator(device="cuda").manual_seed(11))
    for rep in range(3):
        out, lse, used = B.paged_decode_attn(
            t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"],
            num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl), causal_offset=wl.causal_offset,
            window=wl.window, kv_scale=inp["kv_scale"], workspace=ws, **params_kw)
        torch.cuda.synchronize()
        assert B.last_device_error() == 0
        U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse,
                        case.kv_dtype, f"{case.name}/garbage-ws/rep{rep}")


def test_cuda_graph_replays(lib):
    """A call captured in a CUDA graph replays correctly many times (the
    prologue kernel that zeroes the counters is part of the captured work)."""
    case = [c for c in CASES if c.name.startswith("tc_fp8")][0]
    inp = W.generate(case)
    ref_out, ref_lse = U.run_oracle(inp)
    t = U.to_device(inp)
    wl = inp["workload"]
    out = torch.empty((wl.batch, wl.q_len, wl.num_q_heads, wl.head_dim), dtype=torch.float32,
                      device="cuda")
    lse = torch.empty((wl.batch, wl.q_len, wl.num_q_heads), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    kw = dict(num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl), causal_offset=wl.causal_offset,
              window=wl.window, kv_scale=inp["kv_scale"], num_splits=2, out=out, lse=lse,
              workspace=ws, flags=B.PDA_FLAG_FUSED_MERGE)
    B.paged_decode_attn(t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], **kw)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        B.paged_decode_attn(t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"], **kw)
    for rep in range(4):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert B.last_device_error() == 0
        U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse,
                        case.kv_dtype, f"graph replay {rep}")


SINK_CASES = [c for c in CASES if c.head_dim == 128][:3] + \
    [c for c in CASES if c.name.startswith("tc_fp8")][:2] + [CASES[0]] + \
    [c for c in CASES if c.kv_dtype == NV][:1]


@pytest.mark.parametrize("case", SINK_CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [0, 1, 3])
@pytest.mark.parametrize("kernel", ["auto", "cuda_cores", "tensor_cores_fused_merge"])
def test_parity_attention_sink(lib, case, splits, kernel):
    """Per-head attention-sink logits (one dominating, one -inf): the sink
    joins the denominator in the single-split epilogue, the merge kernel or
    the in-kernel merge."""
    if kernel != "auto" and case.head_dim != 128:
        pytest.skip("forced kernels apply to head_dim 128")
    flags = {"auto": 0, "cuda_cores": B.PDA_FLAG_CUDA_CORES,
             "tensor_cores_fused_merge": B.PDA_FLAG_TENSOR_CORES | B.PDA_FLAG_FUSED_MERGE}[kernel]
    inp = W.generate(case)
    g = torch.Generator().manual_seed(77)
    sk = torch.randn(case.num_q_heads, generator=g) * 2.0
    sk[0] = 12.0
    sk[-1] = float("-inf")
    ref_out, ref_lse = U.run_oracle(inp, sinks=sk.numpy())
    out, lse, _ = U.run_cuda(inp, num_splits=splits, flags=flags, sinks=sk.cuda())
    U.assert_parity(out, lse, ref_out, ref_lse, case.kv_dtype, f"{case.name}/{kernel}/s={splits}/sink")


NATIVE_CASES = [c for c in CASES if c.kv_dtype == FP8 and c.head_dim == 128]


@pytest.mark.parametrize("case", NATIVE_CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_parity_native_fp8_qk(lib, case, splits):
    """Native FP8 QK (q as one e4m3 term per element) against the oracle run
    on the same per-row quantisation of q."""
    inp = W.generate(case)
    ref_out, ref_lse = U.run_oracle(inp, native_qk=True)
    flags = B.PDA_FLAG_TENSOR_CORES | B.PDA_FLAG_NATIVE_FP8_QK
    out, lse, _ = U.run_cuda(inp, num_splits=splits, flags=flags)
    U.assert_parity(out, lse, ref_out, ref_lse, FP8, f"{case.name}/native/s={splits}")


def _visible_tiles(wl, L, tile=128):
    """128-token tiles of the union of a sequence's rows' visible key ranges
    (readings R2, R3): the first query row's start to the last row's end."""
    W_ = wl.window

    def rng(i):
        if wl.causal_offset == B.PDA_CAUSAL_OFF:
            pos, hi = L - 1, L
        else:
            pos = (L - wl.q_len + i) if wl.causal_offset == B.PDA_CAUSAL_BOTTOM_RIGHT else wl.causal_offset + i
            hi = min(L, pos + 1)
        lo = max(0, pos - W_ + 1) if W_ > 0 else 0
        return lo, hi

    lo, _ = rng(0)
    _, hi = rng(wl.q_len - 1)
    return (hi + tile - 1) // tile - lo // tile if hi > lo else 0


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.VARLEN, W.FP8_VERIFY], ids=lambda w: w.name)
def test_work_queue_hands_out_longest_sequences_first(lib, wl):
    """The tensor-core kernel's prologue writes the queue order into the
    workspace after the counter header: a permutation of the sequences with
    their visible 128-token tiles non-increasing."""
    import torch
    inp = W.generate(wl, device="cuda")
    flags = B.PDA_FLAG_TENSOR_CORES
    params = B.make_params(
        batch=wl.batch, q_len=wl.q_len, num_q_heads=wl.num_q_heads,
        num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, page_size=wl.page_size,
        max_pages_per_seq=inp["page_table"].shape[1], num_pages=inp["k_pages"].shape[0],
        scale=W.scale_of(wl), causal_offset=wl.causal_offset, window=wl.window,
        kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"], num_splits=1, flags=flags)
    assert B.plan_kernel(params) == B.PDA_KERNEL_SPLIT_TMA
    ws = torch.full((B.workspace_bytes(params),), 0xAB, dtype=torch.uint8, device="cuda")
    B.paged_decode_attn(inp["q"], inp["k_pages"], inp["v_pages"], inp["page_table"],
                        inp["kv_lens"], num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl),
                        causal_offset=wl.causal_offset, window=wl.window,
                        kv_scale=inp["kv_scale"], num_splits=1, flags=flags, workspace=ws)
    torch.cuda.synchronize()
    M = wl.q_len * (wl.num_q_heads // wl.num_kv_heads)
    assert M <= 32  # one row tile per (sequence, kv head) at these shapes
    header = 64 + wl.batch * wl.num_kv_heads * 1 * 4 * 4
    off = (header + 255) // 256 * 256
    order = ws[off:off + 4 * wl.batch].cpu().view(torch.int32).tolist()
    assert sorted(order) == list(range(wl.batch))
    lens = inp["kv_lens"].cpu().tolist()
    tiles = [_visible_tiles(wl, lens[b]) for b in order]
    assert all(tiles[k] >= tiles[k + 1] for k in range(len(tiles) - 1)), tiles
    assert tiles[0] > tiles[-1]  # the workloads mix lengths: the order is not trivial


@pytest.mark.gpu
@pytest.mark.parametrize("flags", [B.PDA_FLAG_TENSOR_CORES, B.PDA_FLAG_CUDA_CORES],
                         ids=["tensor_cores", "cuda_cores"])
def test_fp8_value_decode_is_exact(lib, flags):
    """Every e4m3 code through the whole path, bit for bit: each sequence sees
    one key, so its weight is exactly 1 and out = fp32(decode(v) * kv_scale);
    the V row of sequence b holds codes 128 b .. 128 b + 127 (NaN codes give
    NaN)."""
    import torch
    Bn, Hq, Hkv, D, P = 2, 16, 1, 128, 16  # 16 packed rows: the FP8 tensor-core path
    g = torch.Generator().manual_seed(7)
    q = torch.randn(Bn, 1, Hq, D, generator=g).to(torch.bfloat16)
    k_pages = torch.randint(0, 0x7E, (Bn, Hkv, P, D), generator=g, dtype=torch.uint8)
    v_pages = torch.randint(0, 0x7E, (Bn, Hkv, P, D), generator=g, dtype=torch.uint8)
    for b in range(Bn):
        v_pages[b, 0, 0] = torch.arange(128 * b, 128 * b + 128, dtype=torch.int32).to(torch.uint8)
    page_table = torch.arange(Bn, dtype=torch.int32).reshape(Bn, 1)
    kv_lens = torch.ones(Bn, dtype=torch.int32)
    kv_scale = 0.0371
    out, lse, _ = B.paged_decode_attn(q.cuda(), k_pages.cuda(), v_pages.cuda(), page_table.cuda(),
                                      kv_lens.cuda(), num_kv_heads=Hkv, scale=D ** -0.5,
                                      kv_scale=kv_scale, num_splits=1, flags=flags)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    dec = v_pages[:, 0, 0].view(torch.float8_e4m3fn).float()          # [B, D], exact
    want = (dec * torch.tensor(kv_scale, dtype=torch.float32))[:, None, None, :].expand(Bn, 1, Hq, D)
    got = out.cpu()
    assert torch.equal(torch.isnan(got), torch.isnan(want))
    fin = ~torch.isnan(want)
    assert torch.equal(got[fin], want[fin]), (got[fin] - want[fin]).abs().max()
