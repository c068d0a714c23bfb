"""The C-ABI library: loads, exports what the header declares, validates on the
host (no GPU needed: every call here returns before any device work)."""

import ctypes
import glob
import os
import re

import pytest

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(
                r"^\s*(?:PDA_API\s+)?(?:const\s+)?(?:pda_status|size_t|int32_t|char|void)\s*\**\s*(\w+)\s*\(",
                text, flags=re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_binding_surface():
    assert declared_functions() == set(B.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_only_c_abi_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(B.EXPORTED) <= syms
    assert not any(s.startswith("_ZN3pda") for s in syms), "C++ internals leaked"


def test_abi_version_and_status_strings(lib):
    assert lib.pda_abi_version() == 3
    for code in range(8):
        assert B.status_string(code)
    assert B.status_string(99) == "unknown status"


def headline_params(**over):
    kw = dict(batch=128, q_len=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
              page_size=16, max_pages_per_seq=512, num_pages=65536,
              scale=0.08838834764831845)
    kw.update(over)
    return B.make_params(**kw)


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=96), 2),
    (dict(head_dim=0), 1),
    (dict(page_size=12), 2),
    (dict(page_size=4), 2),
    (dict(page_size=512), 2),
    (dict(q_len=0), 1),
    (dict(q_len=9), 2),
    (dict(num_q_heads=30), 1),
    (dict(scale=0.0), 1),
    (dict(scale=float("nan")), 1),
    (dict(causal_offset=-3), 1),
    (dict(kv_dtype=3), 1),
    (dict(kv_dtype=2, kv_scale=0.0), 1),
    (dict(kv_dtype=1, kv_scale=0.0), 1),
    (dict(num_pages=0), 1),
    (dict(max_pages_per_seq=0), 1),
    (dict(num_splits=-1), 1),
    (dict(batch=-1), 1),
    (dict(num_kv_heads=0), 1),
    (dict(scale=-1.0), 1),
    (dict(scale=float("inf")), 1),
    (dict(kv_dtype=1, kv_scale=float("nan")), 1),
    (dict(kv_dtype=1, kv_scale=float("inf")), 1),
    (dict(max_kv_len=-1), 1),
    (dict(max_pages_per_seq=1 << 27), 1),  # 2^27 pages x 16 tokens > INT_MAX
    (dict(batch=65536), 2),
])
def test_invalid_params_rejected_on_host(lib, over, status):
    p = headline_params(**over)
    dummy = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    st = lib.paged_decode_attn(dummy, dummy, dummy, dummy, dummy, ctypes.byref(p),
                               dummy, dummy, None)
    assert st == status, B.STATUS.get(st)


def test_null_params_and_pointers(lib):
    st = lib.paged_decode_attn(None, None, None, None, None, None, None, None, None)
    assert st == 1
    p = headline_params()
    st = lib.paged_decode_attn(None, None, None, None, None, ctypes.byref(p), None, None, None)
    assert st == 1


def test_misaligned_pointers(lib):
    p = headline_params()
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    st = lib.paged_decode_attn(bad, ok, ok, ok, ok, ctypes.byref(p), ok, ok, None)
    assert st == 3
    st = lib.paged_decode_attn(ok, ok, ok, ok, ok, ctypes.byref(p), bad, ok, None)
    assert st == 3
    # page table, kv_lens, lse and sinks need 4 bytes; the workspace 256
    odd = ctypes.c_void_p((1 << 20) + 2)
    for args in ((ok, ok, ok, odd, ok, ok, ok), (ok, ok, ok, ok, odd, ok, ok),
                 (ok, ok, ok, ok, ok, ok, odd)):
        q, k, v, pt, kl, out, lse = args
        assert lib.paged_decode_attn(q, k, v, pt, kl, ctypes.byref(p), out, lse, None) == 3
    p.sinks = (1 << 20) + 2
    assert lib.paged_decode_attn(ok, ok, ok, ok, ok, ctypes.byref(p), ok, ok, None) == 3
    p = headline_params()
    p.workspace = (1 << 20) + 16
    p.workspace_bytes = 1 << 20
    assert lib.paged_decode_attn(ok, ok, ok, ok, ok, ctypes.byref(p), ok, ok, None) == 3


def test_empty_batch_is_a_no_op(lib):
    p = headline_params(batch=0)
    n = ctypes.c_int32(-5)
    p.num_splits_out = ctypes.pointer(n)
    st = lib.paged_decode_attn(None, None, None, None, None, ctypes.byref(p), None, None, None)
    assert st == 0 and n.value == 1


def test_merge_states_validation(lib):
    st = lib.pda_merge_states(None, None, 0, 4, 128, None, None, None, 0, None)
    assert st == 1
    st = lib.pda_merge_states(None, None, 2, 4, 96, None, None, None, 0, None)
    assert st == 2
    st = lib.pda_merge_states(None, None, 2, 0, 128, None, None, None, 0, None)
    assert st == 0


def test_split_planner(lib):
    # headline: 1024 (b, kv head) units fill the 148 SMs ~7 times: no split
    assert B.choose_num_splits(headline_params(), 148) == 1
    # few long sequences: split to fill the machine
    longctx = B.make_params(batch=4, q_len=1, num_q_heads=16, num_kv_heads=4,
                            head_dim=256, page_size=128, max_pages_per_seq=256,
                            num_pages=1024, scale=1 / 16)
    s = B.choose_num_splits(longctx, 148)
    assert 8 <= s <= 40, s
    assert 16 * s <= 2 * 148
    # forced split count is honoured (clamped to the tile count)
    assert B.choose_num_splits(headline_params(num_splits=7), 148) == 7
    tiny = B.make_params(batch=2, q_len=1, num_q_heads=4, num_kv_heads=1, head_dim=64,
                         page_size=16, max_pages_per_seq=7, num_pages=16, scale=0.125)
    assert B.choose_num_splits(tiny, 148) >= 1
    assert B.choose_num_splits(B.make_params(
        batch=2, q_len=1, num_q_heads=4, num_kv_heads=1, head_dim=64, page_size=16,
        max_pages_per_seq=7, num_pages=16, scale=0.125, num_splits=1000), 148) <= 7
    # the window bounds the span a CTA walks
    win = headline_params(window=256, max_kv_len=8192, batch=4)
    assert B.choose_num_splits(win, 148) <= 256 // 16


def test_split_planner_persistent_kernel(lib):
    """The persistent tensor-core kernel takes no split once there are 1.5
    (sequence, kv head, row tile) units per SM (its queue hands out the longest
    sequences first); fewer units keep the wave model, as does the CUDA-core
    kernel."""
    def p(batch, **kw):
        return headline_params(batch=batch, num_q_heads=4, num_kv_heads=1, max_kv_len=65536,
                               max_pages_per_seq=4096, **kw)
    assert B.plan_kernel(p(222)) == B.PDA_KERNEL_SPLIT_TMA
    assert B.choose_num_splits(p(222), 148) == 1      # 2 * 222 = 3 * 148
    assert B.choose_num_splits(p(221), 148) > 1       # below: the wave model splits
    assert B.choose_num_splits(p(222, flags=B.PDA_FLAG_CUDA_CORES), 148) > 1
    fp8_verify = B.make_params(batch=64, q_len=4, num_q_heads=64, num_kv_heads=8, head_dim=128,
                               page_size=128, max_pages_per_seq=256, num_pages=16384,
                               scale=0.08838834764831845, kv_dtype=B.PDA_KV_FP8_E4M3,
                               kv_scale=0.01, causal_offset=B.PDA_CAUSAL_BOTTOM_RIGHT, window=4096)
    assert B.plan_kernel(fp8_verify) == B.PDA_KERNEL_SPLIT_TMA
    assert B.choose_num_splits(fp8_verify, 148) == 1


def test_workspace_bytes(lib):
    rows = 128 * 32
    expect_o = 4 * rows * 128 * 4
    # CUDA-core kernel: the split partials only
    got = B.workspace_bytes(headline_params(num_splits=4, flags=B.PDA_FLAG_CUDA_CORES))
    assert got >= expect_o + 4 * rows * 4 and got < expect_o + 4 * rows * 4 + 512
    assert B.workspace_bytes(headline_params(num_splits=1, flags=B.PDA_FLAG_CUDA_CORES)) == 0
    # tensor-core kernel: a counter header (the work-queue counter, then four
    # split-arrival counters per (sequence, kv head, row tile): one per softmax
    # row group) and the queue order (one int per sequence) before the partials
    header = (64 + 128 * 8 * 4 * 4 + 255) // 256 * 256 + (128 * 4 + 255) // 256 * 256
    assert B.workspace_bytes(headline_params(num_splits=1)) == header
    got = B.workspace_bytes(headline_params(num_splits=4))
    assert got >= header + expect_o + 4 * rows * 4 and got < header + expect_o + 4 * rows * 4 + 512
    assert B.workspace_bytes(headline_params(head_dim=96)) == ctypes.c_size_t(-1).value


def test_plan_kernel(lib):
    """Which split kernel the planner picks: tensor cores for FP8 K/V at
    head_dim 128 with more than 8 packed rows, bf16 only on request."""
    fp8 = dict(batch=64, q_len=4, num_q_heads=64, num_kv_heads=8, head_dim=128,
               page_size=128, max_pages_per_seq=256, num_pages=4096, scale=0.088,
               kv_dtype=B.PDA_KV_FP8_E4M3, kv_scale=0.01)
    assert B.plan_kernel(B.make_params(**fp8)) == B.PDA_KERNEL_SPLIT_TMA
    assert B.plan_kernel(B.make_params(**{**fp8, "q_len": 1})) == B.PDA_KERNEL_SPLIT_FMA
    assert B.plan_kernel(B.make_params(**{**fp8, "head_dim": 64})) == B.PDA_KERNEL_SPLIT_FMA
    assert B.plan_kernel(B.make_params(**fp8, flags=B.PDA_FLAG_CUDA_CORES)) == B.PDA_KERNEL_SPLIT_FMA
    assert B.plan_kernel(B.make_params(**{**fp8, "q_len": 1},
                                       flags=B.PDA_FLAG_TENSOR_CORES)) == B.PDA_KERNEL_SPLIT_TMA
    assert B.plan_kernel(headline_params()) == B.PDA_KERNEL_SPLIT_TMA
    assert B.plan_kernel(headline_params(flags=B.PDA_FLAG_CUDA_CORES)) == B.PDA_KERNEL_SPLIT_FMA
    assert B.plan_kernel(headline_params(num_q_heads=128)) == B.PDA_KERNEL_SPLIT_FMA  # 16 rows
    assert B.plan_kernel(headline_params(head_dim=64)) == B.PDA_KERNEL_SPLIT_FMA
    assert B.plan_kernel(headline_params(head_dim=96)) == -1


def test_append_validation(lib):
    """paged_kv_append rejects bad params and pointers on the host."""
    def call(**over):
        kw = dict(batch=2, num_new=1, num_kv_heads=2, head_dim=128, page_size=16,
                  max_pages_per_seq=4, num_pages=8, kv_dtype=B.PDA_KV_BF16, kv_scale=1.0)
        kw.update(over)
        p = B.PdaAppendParams(**kw)
        ptr = 1 << 20  # never dereferenced: every case returns before device work
        return lib.paged_kv_append(ptr, ptr, ptr, ptr, ctypes.byref(p), ptr, ptr, None)
    assert call(num_new=0) == 1 and call(num_new=65) == 1 and call(num_kv_heads=0) == 1
    assert call(kv_dtype=7) == 1 and call(kv_dtype=B.PDA_KV_FP8_E4M3, kv_scale=0.0) == 1
    assert call(head_dim=96) == 2 and call(page_size=12) == 2 and call(page_size=4) == 2
    assert call(batch=0) == 0
    assert lib.paged_kv_append(None, None, None, None, None, None, None, None) == 1
    p = B.PdaAppendParams(2, 1, 2, 128, 16, 4, 8, B.PDA_KV_BF16, 1.0)
    assert lib.paged_kv_append((1 << 20) + 8, 1 << 20, 1 << 20, 1 << 20, ctypes.byref(p),
                               1 << 20, 1 << 20, None) == 3


def test_binding_structs_match_the_header_layout(tmp_path):
    """The ctypes mirrors of pda_params and pda_append_params have the C
    header's size and field offsets (a C program compiled against the header
    prints them)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {"pda_params": B.PdaParams, "pda_append_params": B.PdaAppendParams}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "paged_decode_attn.h"',
             'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    got = {}
    for line in out.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_nvfp4_needs_aligned_scale_pools(lib):
    ok = ctypes.c_void_p(1 << 20)
    p = headline_params(kv_dtype=B.PDA_KV_NVFP4, kv_scale=0.01)
    st = lib.paged_decode_attn(ok, ok, ok, ok, ok, ctypes.byref(p), ok, ok, None)
    assert st == 1  # no block-scale pools
    p.k_scales = (1 << 20) + 4
    p.v_scales = 1 << 20
    st = lib.paged_decode_attn(ok, ok, ok, ok, ok, ctypes.byref(p), ok, ok, None)
    assert st == 3
    a = B.PdaAppendParams(4, 1, 8, 128, 16, 8, 64, B.PDA_KV_NVFP4, 0.01, None, None)
    st = lib.paged_kv_append(ok, ok, ok, ok, ctypes.byref(a), ok, ok, None)
    assert st == 1
    # head_dim 128 with at most 8 packed rows: the tensor-core kernel (NVFP4
    # decoded to f16 tiles); other head dims, or the flag: the CUDA-core one
    p = headline_params(kv_dtype=B.PDA_KV_NVFP4, kv_scale=0.01)
    assert B.plan_kernel(p) == B.PDA_KERNEL_SPLIT_TMA
    p = headline_params(kv_dtype=B.PDA_KV_NVFP4, kv_scale=0.01, flags=B.PDA_FLAG_CUDA_CORES)
    assert B.plan_kernel(p) == B.PDA_KERNEL_SPLIT_FMA
    p = headline_params(kv_dtype=B.PDA_KV_NVFP4, kv_scale=0.01, head_dim=64)
    assert B.plan_kernel(p) == B.PDA_KERNEL_SPLIT_FMA
