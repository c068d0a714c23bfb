"""Checks that pin the fp64 oracle to things other than itself.

Each check takes the loaded oracle library as an argument, so the same checks
run against the real oracle (tests/test_oracle.py) and against copies of it
with a planted mistake (which must fail at least one check).

What pins what:
  * decode_bf16 / decode_e4m3: torch's own bfloat16 and float8_e4m3fn casts
    (an independent implementation) plus hand-worked E4M3 code values.
  * bruteforce: textbook dense attention (numpy matmul + scipy logsumexp)
    over the per-sequence K/V drawn BEFORE they were scattered into pages,
    so it never touches the page table; visibility is built as a dense
    boolean matrix rather than the oracle's per-key test.
  * page_permutation: relabelling physical pages changes nothing, bit for bit.
  * split_merge: partial states over disjoint key ranges, LSE-merged, equal
    the unsplit result.
  * closed forms: equal keys -> mean of visible V and lse = s + ln |V|;
    one-hot V -> softmax probabilities; single key -> v.
  * golden: hand-derived fixtures under tests/golden/.
  * e4m3 encode: inverts torch's decode on every finite code; equals torch's
    float8_e4m3fn cast (round to nearest even) on 200k log-uniform values and
    on every exact midpoint between adjacent codes.
  * quantize_q (native FP8 QK): equals torch's float8 cast of q * 2^e per
    row, with 2^e from torch.frexp of the row's max |q|.
  * sink: brute-force dense attention with the sink as one more key of zero
    value; a -inf sink is bit-identical to none.
  * append: new rows land where numpy indexing of the page table says
    (page_table[b][pos // P], slot pos % P), as torch-cast codes for FP8;
    every other slot is unchanged.
  * NVFP4: E2M1 decode of all 16 codes and E2M1 encoding (nearest even,
    saturating) against ml_dtypes' float4_e2m1fn (an independent
    implementation) and hand-worked codes; the block quantiser against
    hand-worked blocks and against a restatement built from numpy float32,
    torch's float8_e4m3fn cast and ml_dtypes; brute force decodes NVFP4 K/V
    through ml_dtypes and torch, never through the oracle.
"""

from __future__ import annotations

import json
import math
import os

import ml_dtypes
import numpy as np
import torch
from scipy.special import logsumexp, softmax

from oracle import oracle as orc
from paged_kv_decode_30_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Small cases: (name, Workload). All use the dense route so that the
# brute force has an unpaged copy of K/V.
SMALL_CASES = [
    W.TINY,
    W.Workload(name="gqa2_d32_p8", batch=3, num_q_heads=8, num_kv_heads=2,
               head_dim=32, page_size=8, kv_lens=("fixed", [1, 17, 64]),
               extra_pages=3, route="dense", seed=11),
    W.Workload(name="verify3_d16_p4", batch=2, q_len=3, num_q_heads=6,
               num_kv_heads=3, head_dim=16, page_size=4,
               causal_offset=W.CAUSAL_BOTTOM_RIGHT, kv_lens=("fixed", [9, 30]),
               route="dense", seed=12),
    W.Workload(name="verify4_window16", batch=2, q_len=4, num_q_heads=4,
               num_kv_heads=2, head_dim=16, page_size=8,
               causal_offset=W.CAUSAL_BOTTOM_RIGHT, window=16,
               kv_lens=("fixed", [50, 120]), route="dense",
               poison_invisible=True, seed=13),
    W.Workload(name="fixed_offset3", batch=2, q_len=2, num_q_heads=2,
               num_kv_heads=1, head_dim=8, page_size=16, causal_offset=3,
               kv_lens=("fixed", [40, 5]), route="dense", seed=14),
    W.Workload(name="window20_noncausal", batch=2, num_q_heads=4,
               num_kv_heads=2, head_dim=16, page_size=8, window=20,
               kv_lens=("fixed", [70, 33]), route="dense",
               poison_invisible=True, seed=15),
    W.Workload(name="fp8_verify4_window64", batch=2, q_len=4, num_q_heads=8,
               num_kv_heads=2, head_dim=32, page_size=16,
               kv_dtype=W.KV_FP8_E4M3, causal_offset=W.CAUSAL_BOTTOM_RIGHT,
               window=64, kv_lens=("fixed", [100, 300]), route="dense",
               poison_invisible=True, seed=16),
    W.Workload(name="empty_rows", batch=3, num_q_heads=4, num_kv_heads=4,
               head_dim=16, page_size=4, kv_lens=("fixed", [0, 10, 0]),
               extra_pages=2, route="dense", seed=17),
    W.Workload(name="peaked_d64_p32", batch=2, num_q_heads=4, num_kv_heads=1,
               head_dim=64, page_size=32, kv_lens=("fixed", [256, 130]),
               peaked_frac=0.05, route="dense", seed=18),
    W.Workload(name="nvfp4_verify4_window64", batch=2, q_len=4, num_q_heads=8,
               num_kv_heads=2, head_dim=32, page_size=16, kv_dtype=W.KV_NVFP4,
               causal_offset=W.CAUSAL_BOTTOM_RIGHT, window=64,
               kv_lens=("fixed", [100, 300]), route="dense", poison_invisible=True,
               extra_pages=2, seed=19),
    W.Workload(name="nvfp4_gqa4_d64_p8", batch=3, num_q_heads=8, num_kv_heads=2,
               head_dim=64, page_size=8, kv_dtype=W.KV_NVFP4,
               kv_lens=("fixed", [1, 37, 90]), route="dense", peaked_frac=0.05,
               extra_pages=1, seed=20),
]
NVFP4_CASES = [w for w in SMALL_CASES if w.kv_dtype == W.KV_NVFP4]


def run_oracle(inp, lib, tok_range=None, **over):
    wl = inp["workload"]
    kw = dict(num_kv_heads=wl.num_kv_heads, page_size=wl.page_size,
              scale=W.scale_of(wl), causal_offset=wl.causal_offset,
              window=wl.window, kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"],
              tok_range=tok_range)
    if inp.get("k_scales") is not None:
        kw.update(k_scales=W.to_bits(inp["k_scales"]), v_scales=W.to_bits(inp["v_scales"]))
    kw.update(over)
    return orc.paged_decode_attn(
        W.to_bits(inp["q"]), W.to_bits(inp["k_pages"]), W.to_bits(inp["v_pages"]),
        inp["page_table"].cpu().numpy(), inp["kv_lens"].cpu().numpy(), lib=lib, **kw)


def e2m1_values(codes: np.ndarray) -> np.ndarray:
    """float64 values of 4-bit E2M1 codes (one per byte), through ml_dtypes."""
    return np.asarray(codes, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def decode_dense(x, kv_dtype: int, kv_scale: float) -> np.ndarray:
    """Values of a bf16 / e4m3-code / NVFP4 (codes, scales) tensor as float64,
    through torch's and ml_dtypes' casts."""
    if kv_dtype == W.KV_BF16:
        return x.to(torch.float64).numpy()
    if kv_dtype == W.KV_FP8_E4M3:
        return x.view(torch.float8_e4m3fn).to(torch.float64).numpy() * kv_scale
    packed, scales = x
    packed = packed.numpy()
    codes = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(*packed.shape[:-1], -1)
    blk = scales.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return e2m1_values(codes) * np.repeat(blk, 16, axis=-1) * kv_scale


def visibility_matrix(L, q_len, causal_offset, window):
    """[q_len, L] boolean: may row i see key j. Dense restatement of the
    readings (bottom-right / fixed-offset causal, window including the query)."""
    j = np.arange(L)[None, :]
    i = np.arange(q_len)[:, None]
    if causal_offset >= 0:
        pos = causal_offset + i
    elif causal_offset == W.CAUSAL_BOTTOM_RIGHT:
        pos = L - q_len + i
    else:
        pos = np.full_like(i, L - 1)
    vis = np.ones((q_len, L), dtype=bool)
    if causal_offset != W.CAUSAL_OFF:
        vis &= j <= pos
    if window > 0:
        vis &= j >= pos - window + 1
    return vis


def bruteforce(inp, sinks=None):
    """Textbook dense softmax attention over the unpaged K/V copies. An
    attention sink enters as one more key with score sinks[h] and a zero
    value vector."""
    wl = inp["workload"]
    B, Lq, Hq, D = inp["q"].shape
    G = wl.group
    scale = W.scale_of(wl)
    q = inp["q"].to(torch.float64).numpy()
    out = np.zeros((B, Lq, Hq, D))
    lse = np.full((B, Lq, Hq), -np.inf)
    for b in range(B):
        K = decode_dense(inp["k_dense"][b], wl.kv_dtype, inp["kv_scale"])  # [Hkv, L, D]
        V = decode_dense(inp["v_dense"][b], wl.kv_dtype, inp["kv_scale"])
        L = K.shape[1]
        vis = visibility_matrix(L, Lq, wl.causal_offset, wl.window)
        for i in range(Lq):
            sel = vis[i]
            for h in range(Hq):
                g = h // G
                s = scale * (K[g][sel] @ q[b, i, h])
                Vs = V[g][sel]
                if sinks is not None:
                    s = np.append(s, float(sinks[h]))
                    Vs = np.vstack([Vs, np.zeros((1, D))])
                if s.size == 0 or np.all(np.isneginf(s)):
                    continue
                lse[b, i, h] = logsumexp(s)
                out[b, i, h] = np.exp(s - lse[b, i, h]) @ Vs
    return out, lse


def assert_close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):  # inf - inf where both are -inf
        err = np.where(both_inf, 0.0, np.abs(a - b))
    assert not np.isnan(err).any(), f"{what}: NaN mismatch"
    m = float(err.max()) if err.size else 0.0
    assert m <= tol, f"{what}: max abs err {m:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------
# individual checks


def check_decode_bf16(lib):
    bits = np.arange(65536, dtype=np.uint32)
    ref = torch.from_numpy(bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16)
    ref = ref.to(torch.float64).numpy()
    got = np.array([orc.bf16_to_double(int(b), lib=lib) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "bf16 NaN set differs"
    assert np.array_equal(got[~nan], ref[~nan]), "bf16 decode differs from torch"


def check_decode_e4m3(lib):
    codes = np.arange(256, dtype=np.int32)
    ref = torch.from_numpy(codes).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    got = np.array([orc.e4m3_to_double(int(c), lib=lib) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "e4m3 NaN set differs"
    assert np.array_equal(got[~nan], ref[~nan]), "e4m3 decode differs from torch"
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        g = json.load(f)
    for c, v in zip(g["codes"], g["values"]):
        x = orc.e4m3_to_double(c, lib=lib)
        if v == "nan":
            assert math.isnan(x), hex(c)
        else:
            assert x == v and math.copysign(1, x) == math.copysign(1, v), (hex(c), x, v)


def check_decode_e2m1(lib):
    codes = np.arange(16, dtype=np.uint8)
    ref = e2m1_values(codes)
    got = np.array([orc.e2m1_to_double(int(c), lib=lib) for c in codes])
    assert np.array_equal(got, ref), "e2m1 decode differs from ml_dtypes"
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    g = load_golden("e2m1_codes")
    for c, v in zip(g["codes"], g["values"]):
        x = orc.e2m1_to_double(c, lib=lib)
        assert x == v and math.copysign(1, x) == math.copysign(1, v), (hex(c), x, v)


def check_e2m1_encode_vs_ml_dtypes(lib, n=50_000, seed=6):
    """Against ml_dtypes' float4_e2m1fn cast (nearest even) of values clamped
    to +-6 as the quantiser saturates: log-uniform magnitudes, every exact
    midpoint between neighbouring codes, signed zeros and values past 6."""
    g = torch.Generator().manual_seed(seed)
    mag = torch.exp2(torch.rand(n, generator=g) * 8.0 - 4.0)          # 2^-4 .. 2^4
    sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0)
    x = (mag * sign).float().numpy()
    pos = e2m1_values(np.arange(8, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.array([0.0, -0.0, 6.0, -6.0, 7.5, -1e30, 1e30],
                                                 dtype=np.float32)]).astype(np.float32)
    ref = np.clip(x, -6.0, 6.0).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([orc.e2m1_encode(float(v), lib=lib) for v in x], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ref[i]), int(got[i])) for i in bad[:5]]


def nvfp4_block_restated(x_bits: np.ndarray, kv_scale: float):
    """The NVFP4 block rule restated with numpy float32 arithmetic, torch's
    e4m3 cast and ml_dtypes' e2m1 cast."""
    xf = torch.from_numpy(x_bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16)
    q = xf.float().numpy() / np.float32(kv_scale)
    amax = np.float32(np.abs(q).max())
    sc = torch.tensor([amax / np.float32(6.0)], dtype=torch.float32).clamp(max=448.0)
    sc = sc.to(torch.float8_e4m3fn)
    sd = np.float32(sc.float().item())
    code = int(sc.view(torch.uint8).item())
    if sd == 0:
        return np.zeros(16, dtype=np.uint8), code
    y = np.clip(q / sd, -6.0, 6.0).astype(np.float32)
    return y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF, code


def check_nvfp4_block_golden(lib):
    for blk in load_golden("nvfp4_blocks")["blocks"]:
        codes, sc = orc.nvfp4_encode_block(np.array(blk["x_bits"], dtype=np.uint16),
                                           blk["kv_scale"], lib=lib)
        assert sc == blk["scale_code"], (hex(sc), hex(blk["scale_code"]))
        assert codes.tolist() == blk["codes"], (codes.tolist(), blk["codes"])


def check_nvfp4_block_vs_restated(lib, n=400, seed=9):
    """Random blocks of mixed magnitude against the restated rule."""
    g = torch.Generator().manual_seed(seed)
    for k in range(n):
        x = torch.randn(16, generator=g) * torch.exp2(torch.randint(-20, 20, (1,), generator=g).float())
        if k % 7 == 0:
            x[torch.rand(16, generator=g) < 0.3] = 0.0
        bits = W.to_bits(x.to(torch.bfloat16))
        kv_scale = float(torch.exp2(torch.randint(-12, 6, (1,), generator=g).float()) *
                         (1 + torch.rand(1, generator=g)))
        kv_scale = float(np.float32(kv_scale))
        codes, sc = orc.nvfp4_encode_block(bits, kv_scale, lib=lib)
        rc, rsc = nvfp4_block_restated(bits, kv_scale)
        assert sc == rsc and np.array_equal(codes, rc), (k, kv_scale, sc, rsc, codes, rc)


def check_bruteforce(wl, lib, tol=1e-12):
    inp = W.generate(wl)
    out, lse = run_oracle(inp, lib)
    ref_out, ref_lse = bruteforce(inp)
    assert_close(out, ref_out, tol, f"{wl.name} out vs brute force")
    assert_close(lse, ref_lse, tol, f"{wl.name} lse vs brute force")


def check_page_permutation(wl, lib, seed=99):
    inp = W.generate(wl)
    out0, lse0 = run_oracle(inp, lib)
    n = inp["k_pages"].shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(seed))
    k2 = torch.empty_like(inp["k_pages"])
    v2 = torch.empty_like(inp["v_pages"])
    k2[perm] = inp["k_pages"]
    v2[perm] = inp["v_pages"]
    pt = inp["page_table"].clone().to(torch.int64)
    pt = torch.where(pt >= 0, perm[pt.clamp(min=0)], pt).to(torch.int32)
    inp2 = dict(inp, k_pages=k2, v_pages=v2, page_table=pt)
    out1, lse1 = run_oracle(inp2, lib)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1), \
        f"{wl.name}: page permutation changed the result"


def check_split_merge(wl, cuts, lib, tol=1e-12):
    inp = W.generate(wl)
    out, lse = run_oracle(inp, lib)
    bounds = [0, *cuts, 1 << 40]
    parts = [run_oracle(inp, lib, tok_range=(a, b)) for a, b in zip(bounds, bounds[1:])]
    B, Lq, Hq, D = out.shape
    o_parts = np.stack([p[0].reshape(-1, D) for p in parts])
    l_parts = np.stack([p[1].reshape(-1) for p in parts])
    mo, ml = orc.merge_states(o_parts, l_parts, lib=lib)
    assert_close(mo, out.reshape(-1, D), tol, f"{wl.name} split {cuts} out")
    assert_close(ml, lse.reshape(-1), tol, f"{wl.name} split {cuts} lse")


def check_equal_keys(lib, tol=1e-12):
    """All keys equal -> out = mean of the visible v, lse = s + ln |visible|."""
    wl = W.Workload(name="equal_keys", batch=2, q_len=3, num_q_heads=4,
                    num_kv_heads=2, head_dim=16, page_size=8,
                    causal_offset=W.CAUSAL_BOTTOM_RIGHT, window=20,
                    kv_lens=("fixed", [45, 7]), route="dense", seed=21)
    inp = W.generate(wl)
    kvec = torch.randn(wl.head_dim, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    valid = ~torch.isnan(inp["k_pages"].float())
    inp["k_pages"] = torch.where(valid, kvec.expand_as(inp["k_pages"]), inp["k_pages"])
    out, lse = run_oracle(inp, lib)
    q = inp["q"].to(torch.float64).numpy()
    k = kvec.to(torch.float64).numpy()
    scale = W.scale_of(wl)
    for b in range(wl.batch):
        V = inp["v_dense"][b].to(torch.float64).numpy()
        L = V.shape[1]
        vis = visibility_matrix(L, wl.q_len, wl.causal_offset, wl.window)
        for i in range(wl.q_len):
            n = int(vis[i].sum())
            for h in range(wl.num_q_heads):
                g = h // wl.group
                assert_close(out[b, i, h], V[g][vis[i]].mean(axis=0), tol, "equal keys mean")
                s = scale * float(q[b, i, h] @ k)
                assert_close(lse[b, i, h], s + math.log(n), tol, "equal keys lse")


def check_one_hot_values(lib, tol=1e-12):
    """V rows one-hot (v_j = e_j) -> out[:, j] is the softmax probability."""
    wl = W.Workload(name="one_hot", batch=1, num_q_heads=2, num_kv_heads=1,
                    head_dim=32, page_size=4, kv_lens=("fixed", [23]),
                    route="dense", seed=22)
    inp = W.generate(wl)
    L, D = 23, 32
    eye = torch.zeros((1, L, D), dtype=torch.bfloat16)
    eye[0, torch.arange(L), torch.arange(L)] = 1.0
    pt = inp["page_table"][0]
    vp = inp["v_pages"]
    for j in range(L):
        vp[int(pt[j // 4]), 0, j % 4] = eye[0, j]
    out, _ = run_oracle(inp, lib)
    K = inp["k_dense"][0].to(torch.float64).numpy()[0]
    q = inp["q"].to(torch.float64).numpy()
    for h in range(2):
        probs = softmax(W.scale_of(wl) * (K @ q[0, 0, h]))
        assert_close(out[0, 0, h, :L], probs, tol, "one-hot probabilities")
        assert_close(out[0, 0, h, L:], np.zeros(D - L), tol, "one-hot tail")


def check_poison_is_never_read(wl, lib):
    """NaN-filled unused pages, tails and invisible keys give the same result
    as the same slots holding zeros, and the result is finite."""
    inp = W.generate(wl)
    out0, lse0 = run_oracle(inp, lib)
    clean = dict(inp)
    keys = ("k_scales", "v_scales") if wl.kv_dtype == W.KV_NVFP4 else ("k_pages", "v_pages")
    for key in keys:
        x = inp[key].clone()
        if wl.kv_dtype == W.KV_BF16:
            x[torch.isnan(x.float())] = 0
        else:
            x[(x == W.E4M3_NAN_CODE) | (x == 0xFF)] = 0
        clean[key] = x
    out1, lse1 = run_oracle(clean, lib)
    assert np.isfinite(out0).all(), f"{wl.name}: poisoned slots reached out"
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


def load_golden(name):
    with open(os.path.join(GOLDEN, name + ".json")) as f:
        return json.load(f)


def check_golden(name, lib):
    g = load_golden(name)
    u16 = np.uint16
    q = np.array(g["q_bits"], dtype=u16)
    kp = np.array(g["k_pages_bits"], dtype=u16)
    vp = np.array(g["v_pages_bits"], dtype=u16)
    scale = g["scale"]
    if scale == "float32(ln 3)":
        scale = float(np.float32(math.log(3.0)))
    out, lse = orc.paged_decode_attn(
        q, kp, vp, np.array(g["page_table"], dtype=np.int32),
        np.array(g["kv_lens"], dtype=np.int32), num_kv_heads=g["num_kv_heads"],
        page_size=g["page_size"], scale=scale, causal_offset=g["causal_offset"],
        window=g["window"], kv_dtype=g["kv_dtype"], lib=lib)
    exp_lse = np.array([[[float(x) for x in r] for r in b] for b in g["expected_lse"]])
    assert_close(out, np.array(g["expected_out"], dtype=np.float64), g["tolerance"], name)
    assert_close(lse, exp_lse, g["tolerance"], name)


GOLDEN_NAMES = ["two_keys", "window_causal_equal_keys", "gqa_single_key", "empty_row"]


def run_all(lib):
    """Every check once; raises AssertionError at the first failure."""
    check_decode_bf16(lib)
    check_decode_e4m3(lib)
    for name in GOLDEN_NAMES:
        check_golden(name, lib)
    for wl in SMALL_CASES:
        check_bruteforce(wl, lib)
    check_page_permutation(SMALL_CASES[1], lib)
    check_split_merge(SMALL_CASES[3], [33, 70], lib)
    check_equal_keys(lib)
    check_one_hot_values(lib)
    check_poison_is_never_read(SMALL_CASES[3], lib)
    check_e4m3_encode_roundtrip(lib)
    check_e4m3_encode_vs_torch(lib, n=20_000)
    check_append(lib, W.KV_BF16)
    check_append(lib, W.KV_FP8_E4M3)
    check_decode_e2m1(lib)
    check_e2m1_encode_vs_ml_dtypes(lib, n=5_000)
    check_nvfp4_block_golden(lib)
    check_nvfp4_block_vs_restated(lib, n=100)
    check_append(lib, W.KV_NVFP4)
    for wl in NVFP4_CASES:
        check_bruteforce(wl, lib)
        check_poison_is_never_read(wl, lib)
    for wl in (SMALL_CASES[2], SMALL_CASES[6], SMALL_CASES[7]):
        check_sink_bruteforce(wl, lib)
    check_quantize_q_vs_torch(lib)


# ---------------------------------------------------------------------------
# KV append: e4m3 encoding and the page placement of new rows

def check_e4m3_encode_roundtrip(lib):
    """encode(decode(c)) == c for every finite code; values decoded by torch."""
    codes = torch.tensor([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).float().tolist()
    for c, v in zip(codes.tolist(), vals):
        got = orc.e4m3_encode(v, lib=lib)
        assert got == c, (hex(c), v, hex(got))


def check_e4m3_encode_vs_torch(lib, n=200_000, seed=5):
    """Against torch's float8_e4m3fn cast (round to nearest even) on
    log-uniform magnitudes across the whole range, clamped to +-448 as the
    quantiser saturates, and on every exact midpoint between adjacent codes."""
    g = torch.Generator().manual_seed(seed)
    mag = torch.exp2(torch.rand(n, generator=g) * 22.0 - 13.0)   # 2^-13 .. 2^9
    sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0)
    x = (mag * sign).float()
    pos = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    mids = ((pos[:-1] + pos[1:]) / 2).float()                     # exact in fp32
    x = torch.cat([x, mids, -mids, torch.tensor([0.0, -0.0, 448.0, -448.0, 1e30, -1e30])])
    ref = x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    enc = lib.oracle_e4m3_encode
    got = [enc(float(v)) for v in x.tolist()]
    bad = [(v, r, g_) for v, r, g_ in zip(x.tolist(), ref, got) if r != g_]
    assert not bad, bad[:5]


def check_append(lib, kv_dtype, seed=3):
    """New rows land at page_table[b][pos // P], slot pos % P for pos =
    kv_lens[b] + t (numpy indexing, independent of the oracle's loops), with
    bf16 bits copied / e4m3 codes from torch's cast of the fp32 quotient /
    NVFP4 codes and block scales from the restated block rule; every other
    slot is unchanged."""
    g = torch.Generator().manual_seed(seed)
    B, T, Hkv, D, P, max_pages, num_pages = 3, 5, 2, 32, 8, 6, 30
    kv_lens = np.array([0, 7, 22], dtype=np.int32)
    page_table = torch.randperm(num_pages, generator=g)[:B * max_pages].reshape(B, max_pages)
    page_table = page_table.to(torch.int32).numpy()
    k_new = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16)
    v_new = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16)
    fp8 = kv_dtype == W.KV_FP8_E4M3
    nv = kv_dtype == W.KV_NVFP4
    dt = np.uint16 if kv_dtype == W.KV_BF16 else np.uint8
    Dp = D // 2 if nv else D
    k_pages = np.random.default_rng(seed).integers(0, 255, (num_pages, Hkv, P, Dp)).astype(dt)
    v_pages = np.random.default_rng(seed + 1).integers(0, 255, (num_pages, Hkv, P, Dp)).astype(dt)
    scale = 0.0123
    extra = {}
    if nv:
        extra = dict(
            k_scales=np.random.default_rng(seed + 2).integers(0, 255, (num_pages, Hkv, P, D // 16)).astype(np.uint8),
            v_scales=np.random.default_rng(seed + 3).integers(0, 255, (num_pages, Hkv, P, D // 16)).astype(np.uint8))
    res = orc.paged_kv_append(W.to_bits(k_new), W.to_bits(v_new), page_table, kv_lens,
                              k_pages, v_pages, page_size=P, kv_dtype=kv_dtype,
                              kv_scale=scale, lib=lib, **extra)

    def coded(x):
        if nv:  # [T, Hkv, D] -> packed codes [T, Hkv, D/2], scales [T, Hkv, D/16]
            bits = W.to_bits(x).reshape(-1, 16)
            out = [nvfp4_block_restated(b_, scale) for b_ in bits]
            c = np.stack([o[0] for o in out]).reshape(*x.shape)
            sc = np.array([o[1] for o in out], dtype=np.uint8).reshape(*x.shape[:-1], D // 16)
            return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8), sc
        if not fp8:
            return W.to_bits(x)
        y = (x.float() / scale).clamp(-448.0, 448.0)
        return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    ek, ev = k_pages.copy(), v_pages.copy()
    if nv:
        eks, evs = extra["k_scales"].copy(), extra["v_scales"].copy()
    for b in range(B):
        pos = kv_lens[b] + np.arange(T)
        pages = page_table[b, pos // P]
        if nv:
            ek[pages, :, pos % P, :], eks[pages, :, pos % P, :] = coded(k_new[b])
            ev[pages, :, pos % P, :], evs[pages, :, pos % P, :] = coded(v_new[b])
        else:
            ek[pages, :, pos % P, :] = coded(k_new[b])
            ev[pages, :, pos % P, :] = coded(v_new[b])
    assert np.array_equal(res[0], ek) and np.array_equal(res[1], ev)
    if nv:
        assert np.array_equal(res[2], eks) and np.array_equal(res[3], evs)


# ---------------------------------------------------------------------------
# attention sink

def sink_logits(wl, seed=21):
    """Per-query-head sink logits on the scale of the scores, one of them far
    above every score (the sink takes almost all the weight) and one -inf."""
    g = torch.Generator().manual_seed(seed)
    sk = (torch.randn(wl.num_q_heads, generator=g) * 2.0).to(torch.float32)
    sk[0] = 30.0
    if wl.num_q_heads > 1:
        sk[-1] = float("-inf")
    return sk.numpy()


def check_sink_bruteforce(wl, lib, tol=1e-12):
    inp = W.generate(wl, device="cpu")
    sk = sink_logits(wl)
    ref_out, ref_lse = bruteforce(inp, sinks=sk)
    out, lse = run_oracle(inp, lib, sinks=sk)
    assert_close(out, ref_out, tol, f"{wl.name} sink out")
    assert_close(lse, ref_lse, tol, f"{wl.name} sink lse")


def check_sink_neg_inf_is_no_sink(wl, lib):
    inp = W.generate(wl, device="cpu")
    a_out, a_lse = run_oracle(inp, lib)
    b_out, b_lse = run_oracle(inp, lib, sinks=np.full(wl.num_q_heads, -np.inf, np.float32))
    assert np.array_equal(a_out, b_out) and np.array_equal(a_lse, b_lse)


# ---------------------------------------------------------------------------
# native FP8 QK: the per-row e4m3 quantisation of q

def check_quantize_q_vs_torch(lib, seed=8):
    """Against torch: per row, 2^e = 2^(8 - frexp exponent of max|q|) puts
    max|q| in [128, 256); q * 2^e through torch's float8_e4m3fn cast, back
    times 2^-e, as bf16 bits. Rows of mixed magnitude, and a zero row."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((37, 64), generator=g) * torch.exp2(torch.randint(-12, 12, (37, 1), generator=g).float())
    q[5] = 0.0
    qb = q.to(torch.bfloat16)
    mx = qb.float().abs().amax(dim=1, keepdim=True)
    _, ex = torch.frexp(torch.where(mx > 0, mx, torch.ones_like(mx)))
    e = torch.where(mx > 0, 8 - ex, torch.zeros_like(ex)).float()
    ref = (qb.float() * torch.exp2(e)).clamp(-448, 448).to(torch.float8_e4m3fn).float() * torch.exp2(-e)
    ref_bits = W.to_bits(ref.to(torch.bfloat16))
    got = orc.quantize_q_e4m3(W.to_bits(qb), lib=lib)
    assert np.array_equal(got, ref_bits)
