"""paged_kv_append through the C ABI against the oracle's append (bit-exact
pool bytes), plus append-then-decode parity."""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _case(seed, B_, T, Hkv, D, P, kv_dtype, max_pages=40, num_pages=None):
    g = torch.Generator().manual_seed(seed)
    num_pages = num_pages or B_ * max_pages + 7
    perm = torch.randperm(num_pages, generator=g)
    page_table = perm[:B_ * max_pages].reshape(B_, max_pages).to(torch.int32)
    cap = max_pages * P
    kv_lens = torch.randint(0, cap - T + 1, (B_,), generator=g).to(torch.int32)
    kv_lens[0] = 0                       # first slot of the first page
    if B_ > 1:
        kv_lens[1] = P - 1               # crosses a page boundary
    x = torch.randn((B_, T, Hkv, D), generator=g)
    # magnitudes across the e4m3 range: saturating, tiny, and ordinary values
    x = x * torch.where(torch.rand(x.shape, generator=g) < 0.02, 1e4, 1.0)
    x = x * torch.where(torch.rand(x.shape, generator=g) < 0.02, 1e-5, 1.0)
    k_new = x.to(torch.bfloat16)
    v_new = (-x * 0.5).to(torch.bfloat16)
    nv = kv_dtype == W.KV_NVFP4
    if not nv:  # NVFP4 leaves the codes of NaN inputs unspecified
        k_new.view(-1)[5] = float("nan")
    else:  # blocks of zeros (scale 0) and of one large value among tiny ones
        k_new.view(-1, 16)[3] = 0.0
        v_new.view(-1, 16)[5] = 1e-6
        v_new.view(-1, 16)[5, 7] = 3.0
    dt = torch.uint8 if kv_dtype != W.KV_BF16 else torch.int16
    shape = (num_pages, Hkv, P, D // 2 if nv else D)
    k_pages = torch.randint(-100, 100, shape, generator=g).to(dt)
    v_pages = torch.randint(-100, 100, shape, generator=g).to(dt)
    if dt == torch.int16:
        k_pages, v_pages = k_pages.view(torch.bfloat16), v_pages.view(torch.bfloat16)
    c = dict(k_new=k_new, v_new=v_new, page_table=page_table, kv_lens=kv_lens,
             k_pages=k_pages, v_pages=v_pages, P=P, kv_dtype=kv_dtype)
    if nv:
        sshape = (num_pages, Hkv, P, D // 16)
        c["k_scales"] = torch.randint(0, 255, sshape, generator=g).to(torch.uint8)
        c["v_scales"] = torch.randint(0, 255, sshape, generator=g).to(torch.uint8)
    return c


def _run_both(c, kv_scale=0.0123):
    """The library's append and the oracle's on the same pools: returns the
    library's pools, the oracle's, and the device error word (NVFP4 pools
    come with their block-scale pools: (codes, scales) pairs)."""
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in c.items()}
    kp, vp = d["k_pages"].clone(), d["v_pages"].clone()
    nv = c["kv_dtype"] == W.KV_NVFP4
    sc = {}
    if nv:
        sc = dict(k_scales=d["k_scales"].clone(), v_scales=d["v_scales"].clone())
    B.paged_kv_append(d["k_new"], d["v_new"], d["page_table"], d["kv_lens"], kp, vp,
                      kv_scale=kv_scale, **sc)
    torch.cuda.synchronize()
    err = B.last_device_error()
    res = orc.paged_kv_append(W.to_bits(c["k_new"]), W.to_bits(c["v_new"]),
                              c["page_table"].numpy(), c["kv_lens"].numpy(),
                              W.to_bits(c["k_pages"]), W.to_bits(c["v_pages"]),
                              page_size=c["P"], kv_dtype=c["kv_dtype"], kv_scale=kv_scale,
                              k_scales=c.get("k_scales"), v_scales=c.get("v_scales"))
    gk, gv = W.to_bits(kp.cpu()), W.to_bits(vp.cpu())
    if nv:
        return ((gk, W.to_bits(sc["k_scales"].cpu())), (gv, W.to_bits(sc["v_scales"].cpu())),
                (res[0], res[2]), (res[1], res[3]), err)
    return gk, gv, res[0], res[1], err


def _equal(a, b):
    if isinstance(a, tuple):
        return all(np.array_equal(x, y) for x, y in zip(a, b))
    return np.array_equal(a, b)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8_E4M3, W.KV_NVFP4],
                         ids=["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("D,P,T", [(64, 8, 1), (128, 16, 4), (128, 128, 13), (256, 32, 2)])
def test_append_bit_exact(kv_dtype, D, P, T):
    c = _case(100 + D + P + T, 5, T, 3, D, P, kv_dtype)
    gk, gv, ok, ov, err = _run_both(c)
    assert err == 0
    assert _equal(gk, ok) and _equal(gv, ov)


@pytest.mark.parametrize("kv_scale", [0.0123, 1.0, 2.0 ** -14, 37.5])
def test_append_nvfp4_bit_exact_across_scales(kv_scale):
    """Per-tensor scales that put the block scales in e4m3's subnormal,
    normal and saturating ranges."""
    c = _case(400, 6, 3, 2, 128, 16, W.KV_NVFP4)
    c["k_new"] = (c["k_new"].float() * torch.logspace(-6, 6, 128)).to(torch.bfloat16)
    gk, gv, ok, ov, err = _run_both(c, kv_scale=kv_scale)
    assert err == 0
    assert _equal(gk, ok) and _equal(gv, ov)


def test_append_large_batch_bit_exact():
    c = _case(7, 128, 1, 8, 128, 16, W.KV_FP8_E4M3, max_pages=8)
    gk, gv, ok, ov, err = _run_both(c, kv_scale=0.0071)
    assert err == 0
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)


def test_append_bad_page_is_reported_and_not_written():
    c = _case(9, 3, 2, 2, 64, 8, W.KV_BF16, max_pages=6)
    pt = c["page_table"].clone()
    b, pos = 2, int(c["kv_lens"][2])
    pt[b, pos // 8] = 10_000_000           # out of range for this call only
    c2 = dict(c, page_table=pt)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in c2.items()}
    kp, vp = d["k_pages"].clone(), d["v_pages"].clone()
    B.paged_kv_append(d["k_new"], d["v_new"], d["page_table"], d["kv_lens"], kp, vp)
    torch.cuda.synchronize()
    assert B.last_device_error() == 6       # PDA_ERR_BAD_PAGE
    # the sequences with valid pages were written as the oracle writes them
    c_ok = dict(c, k_new=c["k_new"][:2], v_new=c["v_new"][:2], page_table=c["page_table"][:2],
                kv_lens=c["kv_lens"][:2])
    ok, ov = orc.paged_kv_append(W.to_bits(c_ok["k_new"]), W.to_bits(c_ok["v_new"]),
                                 c_ok["page_table"].numpy(), c_ok["kv_lens"].numpy(),
                                 W.to_bits(c["k_pages"]), W.to_bits(c["v_pages"]), page_size=8)
    # except for the slot of sequence 2's second token when it shares no page
    # with the bad one; compare the pages the first two sequences own
    own = c["page_table"][:2].flatten().numpy()
    assert np.array_equal(W.to_bits(kp.cpu())[own], ok[own])
    assert np.array_equal(W.to_bits(vp.cpu())[own], ov[own])


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8_E4M3, W.KV_NVFP4],
                         ids=["bf16", "fp8", "nvfp4"])
def test_append_then_decode(kv_dtype):
    """Append a decode step's new token (the cache the oracle appends the same
    way), then decode over the longer cache: parity with the oracle."""
    wl = W.Workload(name="append_decode", batch=4, num_q_heads=16, num_kv_heads=2, head_dim=128,
                    page_size=16, kv_dtype=kv_dtype, kv_lens=("fixed", [5, 16, 100, 0]),
                    extra_pages=8, seed=31)
    inp = W.generate(wl)
    # give every sequence a page for its new token
    P = wl.page_size
    pt = inp["page_table"].clone()
    used = set(pt[pt >= 0].tolist())
    free = [p for p in range(inp["k_pages"].shape[0]) if p not in used]
    for b in range(wl.batch):
        L = int(inp["kv_lens"][b])
        if pt[b, L // P] < 0:
            pt[b, L // P] = free.pop()
    g = torch.Generator().manual_seed(4)
    k_new = torch.randn((wl.batch, 1, wl.num_kv_heads, wl.head_dim), generator=g).to(torch.bfloat16)
    v_new = torch.randn((wl.batch, 1, wl.num_kv_heads, wl.head_dim), generator=g).to(torch.bfloat16)
    nv = kv_dtype == W.KV_NVFP4
    res = orc.paged_kv_append(W.to_bits(k_new), W.to_bits(v_new), pt.numpy(),
                              inp["kv_lens"].numpy(), W.to_bits(inp["k_pages"]),
                              W.to_bits(inp["v_pages"]), page_size=P, kv_dtype=kv_dtype,
                              kv_scale=inp["kv_scale"],
                              k_scales=None if not nv else W.to_bits(inp["k_scales"]),
                              v_scales=None if not nv else W.to_bits(inp["v_scales"]))
    d = U.to_device(dict(inp, page_table=pt))
    kp, vp = d["k_pages"].clone(), d["v_pages"].clone()
    sc = {}
    if nv:
        sc = dict(k_scales=d["k_scales"].clone(), v_scales=d["v_scales"].clone())
    B.paged_kv_append(k_new.cuda(), v_new.cuda(), d["page_table"], d["kv_lens"], kp, vp,
                      kv_scale=inp["kv_scale"], **sc)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    assert np.array_equal(W.to_bits(kp.cpu()), res[0])
    assert np.array_equal(W.to_bits(vp.cpu()), res[1])
    new_lens = inp["kv_lens"] + 1
    after = dict(inp, page_table=pt, kv_lens=new_lens, k_pages=kp.cpu(), v_pages=vp.cpu())
    if nv:
        assert np.array_equal(W.to_bits(sc["k_scales"].cpu()), res[2])
        assert np.array_equal(W.to_bits(sc["v_scales"].cpu()), res[3])
        after.update(k_scales=sc["k_scales"].cpu(), v_scales=sc["v_scales"].cpu())
    ref_out, ref_lse = U.run_oracle(after)
    out, lse, _ = U.run_cuda(after)
    U.assert_parity(out, lse, ref_out, ref_lse, kv_dtype, "append then decode")
