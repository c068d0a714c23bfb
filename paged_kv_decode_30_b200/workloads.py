"""Seeded synthetic inputs for paged-KV decode attention.

This module only draws inputs: query rows, paged K/V pools, page tables and
kv lengths. It holds none of the attention arithmetic, so both the CUDA path
and the fp64 oracle can consume what it produces.

Workload shapes follow the pages' paged-decode setting ("AstrAI commit log,
attn_paged_decode_split_kv_mma.cuh": split-KV paged decode with GQA packing;
"b12x 0.30.0, Kernel inventory, Attention table, Paged attention row": bf16
and FP8-E4M3 KV caches, page sizes 64/128, sliding window, verify rows).

Two ways of filling the K/V pool:
  * ``route="dense"``: each sequence's logical K/V ``[Hkv, L_b, D]`` is drawn
    first and then scattered into pages through the page table. The dense
    copies are returned, so a test can run textbook attention on them by a
    route that never touches the page table.
  * ``route="pool"``: the pool ``[num_pages, Hkv, P, D]`` is drawn directly
    (used for the large workloads, and on the GPU).

Pages that no sequence references, slots past ``kv_len`` in a sequence's last
page, and (optionally) keys that no query row can see are filled with NaN
(bf16 0x7FC0, e4m3 0x7F; NVFP4, whose codes have no NaN, gets NaN block
scales), so a kernel that reads or weights them shows it.

NVFP4 K/V (the cache builder's quantisation of the bf16 source, as the
"b12x 0.30.0, Kernel inventory" FP4 rows and the "sglang profiler skill,
fuse-overlap catalog" FP4 KV rows store it): packed E2M1 codes, two per
byte with the even element in the low nibble, ``[num_pages, Hkv, P, D/2]``,
plus one E4M3 scale per 16 consecutive elements of a row, ``[num_pages,
Hkv, P, D/16]``, and the per-tensor ``kv_scale``.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

KV_BF16 = 0
KV_FP8_E4M3 = 1
KV_NVFP4 = 2
CAUSAL_OFF = -1
CAUSAL_BOTTOM_RIGHT = -2

BF16_NAN_BITS = 0x7FC0
E4M3_NAN_CODE = 0x7F
E4M3_MAX = 448.0
E2M1_MAX = 6.0
NVFP4_BLOCK = 16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    q_len: int = 1
    kv_dtype: int = KV_BF16
    scale: Optional[float] = None        # None -> 1/sqrt(head_dim)
    causal_offset: int = CAUSAL_OFF
    window: int = 0
    # kv length recipe: ("fixed", [L0, L1, ...]) | ("const", L)
    # | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi)
    kv_lens: tuple = ("const", 1024)
    peaked_frac: float = 0.0             # fraction of K vectors scaled up
    peaked_factor: float = 8.0
    extra_pages: int = 0                 # unreferenced (poisoned) pool pages
    max_pages_per_seq: Optional[int] = None  # None -> max over sequences
    route: str = "pool"
    poison_invisible: bool = False       # NaN-fill keys no row can see
    seed: int = 20261202

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Names state what they are; sizes are in the fields.
TINY = Workload(
    name="tiny_b2_gqa4_d64_p16", batch=2, num_q_heads=4, num_kv_heads=1,
    head_dim=64, page_size=16, kv_lens=("fixed", [37, 100]), extra_pages=6,
    route="dense", seed=20261202 + 1)
VARLEN = Workload(
    name="varlen_b32_hq32_hkv8_d128_p64_l512to4096", batch=32, num_q_heads=32,
    num_kv_heads=8, head_dim=128, page_size=64, kv_lens=("uniform", 512, 4096),
    seed=20261202 + 2)
HEADLINE = Workload(
    name="b128_hq32_hkv8_d128_p16_l8192_bf16", batch=128, num_q_heads=32,
    num_kv_heads=8, head_dim=128, page_size=16, kv_lens=("const", 8192),
    seed=20261202 + 3)
LONGCTX = Workload(
    name="longctx_b4_hq16_hkv4_d256_p128_l32768_peaked", batch=4,
    num_q_heads=16, num_kv_heads=4, head_dim=256, page_size=128,
    scale=1.0 / 16.0, kv_lens=("const", 32768), peaked_frac=0.01,
    peaked_factor=8.0, seed=20261202 + 4)
FP8_VERIFY = Workload(
    name="fp8_verify_b64_q4_hq64_hkv8_d128_p128_w4096", batch=64, q_len=4,
    num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=128,
    kv_dtype=KV_FP8_E4M3, causal_offset=CAUSAL_BOTTOM_RIGHT, window=4096,
    kv_lens=("lognormal", 2048, 1.0, 128, 32768), poison_invisible=True,
    seed=20261202 + 5)

ALL = {w.name: w for w in (TINY, VARLEN, HEADLINE, LONGCTX, FP8_VERIFY)}

# The headline shape with an NVFP4 KV cache (a KV dtype beyond the five
# workloads: the same sequences, 72 bytes per token row of K or V instead of
# 256).
NVFP4_HEADLINE = HEADLINE.with_(name="nvfp4_b128_hq32_hkv8_d128_p16_l8192", kv_dtype=KV_NVFP4)
EXTRA = {NVFP4_HEADLINE.name: NVFP4_HEADLINE}


def _draw_kv_lens(wl: Workload, gen: torch.Generator) -> torch.Tensor:
    kind = wl.kv_lens[0]
    if kind == "fixed":
        lens = torch.tensor(list(wl.kv_lens[1]), dtype=torch.int64)
        assert lens.numel() == wl.batch
    elif kind == "const":
        lens = torch.full((wl.batch,), int(wl.kv_lens[1]), dtype=torch.int64)
    elif kind == "uniform":
        lo, hi = int(wl.kv_lens[1]), int(wl.kv_lens[2])
        lens = torch.randint(lo, hi + 1, (wl.batch,), generator=gen)
    elif kind == "lognormal":
        median, sigma, lo, hi = wl.kv_lens[1:]
        z = torch.randn((wl.batch,), generator=gen, dtype=torch.float64)
        lens = torch.exp(math.log(median) + sigma * z).round().clamp(lo, hi)
        lens = lens.to(torch.int64)
    else:
        raise ValueError(f"unknown kv_lens recipe {wl.kv_lens!r}")
    return lens


def _row_positions_span(wl: Workload, L: int):
    """[lo, hi) of keys that at least one query row of a sequence may see.

    Used only to decide which keys to NaN-poison; it restates the visibility
    rule of the readings (bottom-right causal, window including the query).
    """
    if wl.causal_offset >= 0:
        first, last = wl.causal_offset, wl.causal_offset + wl.q_len - 1
        hi = min(L, last + 1)
    elif wl.causal_offset == CAUSAL_BOTTOM_RIGHT:
        first, last = L - wl.q_len, L - 1
        hi = L
    else:
        first = last = L - 1
        hi = L
    lo = max(0, first - wl.window + 1) if wl.window > 0 else 0
    return lo, hi


def generate(wl: Workload, device: str | torch.device = "cpu",
             seed: Optional[int] = None, with_dense: Optional[bool] = None):
    """Draw one batch of inputs for ``wl``.

    Returns a dict with
      q           bf16 [B, q_len, Hq, D]
      k_pages     bf16 or uint8 (e4m3 codes) [num_pages, Hkv, P, D];
                  NVFP4: uint8 packed E2M1 codes [num_pages, Hkv, P, D/2]
      v_pages     same
      k_scales, v_scales  NVFP4: uint8 E4M3 block scales [num_pages, Hkv, P,
                  D/16]; None otherwise
      page_table  int32 [B, max_pages] (unused slots -1)
      kv_lens     int32 [B]
      kv_scale    float (1.0 for bf16)
      k_dense / v_dense  (route "dense" only) lists of [Hkv, L_b, D] tensors
                  holding the same values as the pages (bf16 or uint8);
                  NVFP4: lists of (codes [Hkv, L_b, D/2], scales [Hkv, L_b, D/16])
      workload    the Workload
    Generation happens on ``device`` with a generator seeded from the
    workload; the CPU and CUDA generators give different streams.
    """
    device = torch.device(device)
    seed = wl.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    cpu_gen = torch.Generator(device="cpu")
    cpu_gen.manual_seed(seed)

    B, Hkv, D, P = wl.batch, wl.num_kv_heads, wl.head_dim, wl.page_size
    lens = _draw_kv_lens(wl, cpu_gen)
    n_pages = [(int(L) + P - 1) // P for L in lens]
    used = sum(n_pages)
    num_pages = used + wl.extra_pages
    max_pages = wl.max_pages_per_seq or max(1, max(n_pages) if n_pages else 1)
    assert max_pages >= max(n_pages or [0])

    perm = torch.randperm(num_pages, generator=cpu_gen)
    page_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        page_table[b, : n_pages[b]] = perm[off: off + n_pages[b]].to(torch.int32)
        off += n_pages[b]

    fp8 = wl.kv_dtype == KV_FP8_E4M3
    nvfp4 = wl.kv_dtype == KV_NVFP4
    dense = (wl.route == "dense") if with_dense is None else with_dense
    shape = (num_pages, Hkv, P, D)

    k_dense = v_dense = None
    if wl.route == "dense":
        k_dense, v_dense = [], []
        for b in range(B):
            L = int(lens[b])
            k_dense.append(torch.randn((Hkv, L, D), generator=gen, device=device,
                                       dtype=torch.float32).to(torch.bfloat16))
            v_dense.append(torch.randn((Hkv, L, D), generator=gen, device=device,
                                       dtype=torch.float32).to(torch.bfloat16))
        if wl.peaked_frac > 0:
            for b in range(B):
                flat = k_dense[b].view(-1, D)
                nsel = int(round(wl.peaked_frac * flat.shape[0]))
                sel = torch.randperm(flat.shape[0], generator=cpu_gen)[:nsel].to(device)
                flat[sel] = (flat[sel].float() * wl.peaked_factor).to(torch.bfloat16)
        k_src = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        v_src = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        for b in range(B):
            L = int(lens[b])
            for t in range(n_pages[b]):
                pg = int(page_table[b, t])
                n = min(P, L - t * P)
                k_src[pg, :, :n, :] = k_dense[b][:, t * P: t * P + n, :]
                v_src[pg, :, :n, :] = v_dense[b][:, t * P: t * P + n, :]
    else:
        k_src = torch.randn(shape, generator=gen, device=device, dtype=torch.bfloat16)
        v_src = torch.randn(shape, generator=gen, device=device, dtype=torch.bfloat16)
        if wl.peaked_frac > 0:
            # Only referenced slots are candidates: pages are whole for the
            # workloads that use this (kv_len a multiple of page_size).
            flat = k_src.view(-1, D)
            nsel = int(round(wl.peaked_frac * B * Hkv * int(lens.max())))
            cand = torch.cat([
                (page_table[b, : n_pages[b]].to(torch.int64)[:, None, None] * Hkv * P
                 + torch.arange(Hkv)[None, :, None] * P
                 + torch.arange(P)[None, None, :]).reshape(-1)
                for b in range(B)]) if B else torch.zeros(0, dtype=torch.int64)
            sel = cand[torch.randperm(cand.numel(), generator=cpu_gen)[:nsel]].to(device)
            flat[sel] = (flat[sel].float() * wl.peaked_factor).to(torch.bfloat16)

    q = torch.randn((B, wl.q_len, wl.num_q_heads, D), generator=gen,
                    device=device, dtype=torch.float32).to(torch.bfloat16)

    kv_scale = 1.0
    k_scales = v_scales = None
    if nvfp4:
        # per-tensor scale that puts the largest block scale at the top of
        # the E4M3 range
        amax = max(float(k_src.float().abs().max()) if k_src.numel() else 0.0,
                   float(v_src.float().abs().max()) if v_src.numel() else 0.0)
        kv_scale = float(torch.tensor(amax / (E2M1_MAX * E4M3_MAX), dtype=torch.float32)) or 1.0
        k_pages, k_scales = encode_nvfp4(k_src, kv_scale)
        v_pages, v_scales = encode_nvfp4(v_src, kv_scale)
        if k_dense is not None:
            k_dense = [encode_nvfp4(x, kv_scale) for x in k_dense]
            v_dense = [encode_nvfp4(x, kv_scale) for x in v_dense]
        del k_src, v_src
    elif fp8:
        amax = max(float(k_src.float().abs().max()) if k_src.numel() else 0.0,
                   float(v_src.float().abs().max()) if v_src.numel() else 0.0)
        kv_scale = float(torch.tensor(amax / E4M3_MAX, dtype=torch.float32)) or 1.0
        k_pages = encode_e4m3(k_src, kv_scale)
        v_pages = encode_e4m3(v_src, kv_scale)
        if k_dense is not None:
            k_dense = [encode_e4m3(x, kv_scale) for x in k_dense]
            v_dense = [encode_e4m3(x, kv_scale) for x in v_dense]
        del k_src, v_src
    else:
        k_pages, v_pages = k_src, v_src

    if nvfp4:  # NaN lives in the block scales
        _poison(wl, k_scales, v_scales, page_table, lens, n_pages, True)
    else:
        _poison(wl, k_pages, v_pages, page_table, lens, n_pages, fp8)

    out = dict(q=q, k_pages=k_pages, v_pages=v_pages, k_scales=k_scales, v_scales=v_scales,
               page_table=page_table.to(device), kv_lens=lens.to(torch.int32).to(device),
               kv_scale=kv_scale, workload=wl, num_pages=num_pages,
               max_pages=max_pages)
    if dense and k_dense is not None:
        out["k_dense"], out["v_dense"] = k_dense, v_dense
    return out


def encode_e4m3(x: torch.Tensor, kv_scale: float) -> torch.Tensor:
    """Quantise a bf16 source to e4m3 codes: round-to-nearest-even of
    x / kv_scale, saturated to +-448, through torch's float8_e4m3fn cast."""
    y = (x.float() / kv_scale).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


# E2M1 magnitudes of codes 0..7 and the midpoints between neighbours.
_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def encode_nvfp4(x: torch.Tensor, kv_scale: float):
    """Quantise a bf16 source [..., D] to NVFP4: per block of 16 elements,
    q = x / kv_scale, block scale = e4m3(max |q| / 6) through torch's
    float8_e4m3fn cast, codes = the nearest E2M1 value of q / scale (ties to
    the even code, saturating at 6; +0 codes where the scale is zero).
    Returns (codes packed two per byte [..., D/2], scales [..., D/16])."""
    D = x.shape[-1]
    rows = x.reshape(-1, D)
    step = max(1, (1 << 24) // D)  # rows per chunk: bounded temporaries
    if rows.shape[0] > step:
        parts = [encode_nvfp4(rows[i:i + step], kv_scale) for i in range(0, rows.shape[0], step)]
        return (torch.cat([p_[0] for p_ in parts]).reshape(*x.shape[:-1], D // 2),
                torch.cat([p_[1] for p_ in parts]).reshape(*x.shape[:-1], D // NVFP4_BLOCK))
    q = x.float() / kv_scale
    blk = q.reshape(*q.shape[:-1], D // NVFP4_BLOCK, NVFP4_BLOCK)
    amax = blk.abs().amax(dim=-1)
    sc = (amax / E2M1_MAX).clamp(max=E4M3_MAX).to(torch.float8_e4m3fn)
    sd = sc.float()[..., None]
    y = torch.where(sd > 0, blk / torch.where(sd > 0, sd, torch.ones_like(sd)),
                    torch.zeros_like(blk))
    a = y.abs()
    mids = torch.tensor(_E2M1_MIDPOINTS, dtype=torch.float32, device=x.device)
    idx = torch.bucketize(a, mids)  # a <= mids[k] -> k
    at = mids[idx.clamp(max=len(_E2M1_MIDPOINTS) - 1)]
    idx = idx + ((a == at) & (idx % 2 == 1)).to(idx.dtype)  # ties to the even code
    codes = (idx | torch.where(torch.signbit(y), 8, 0)).to(torch.uint8)
    codes = codes.reshape(*q.shape[:-1], D)
    packed = codes[..., 0::2] | (codes[..., 1::2] << 4)
    return packed.contiguous(), sc.view(torch.uint8).contiguous()


def _nan_fill(pages: torch.Tensor, fp8: bool, index):
    if fp8:
        pages[index] = E4M3_NAN_CODE
    else:
        pages.view(torch.int16)[index] = BF16_NAN_BITS


def _poison(wl, k_pages, v_pages, page_table, lens, n_pages, fp8):
    num_pages = k_pages.shape[0]
    P = wl.page_size
    referenced = torch.zeros(num_pages, dtype=torch.bool)
    for b in range(wl.batch):
        referenced[page_table[b, : n_pages[b]].to(torch.int64)] = True
    unused = (~referenced).nonzero().flatten()
    if unused.numel():
        idx = unused.to(k_pages.device)
        for pool in (k_pages, v_pages):
            _nan_fill(pool, fp8, idx)
    for b in range(wl.batch):
        L = int(lens[b])
        if n_pages[b] and L % P:
            last = int(page_table[b, n_pages[b] - 1])
            for pool in (k_pages, v_pages):
                _nan_fill(pool, fp8, (last, slice(None), slice(L % P, P)))
        if wl.poison_invisible and L > 0:
            lo, hi = _row_positions_span(wl, L)
            for j0, j1 in ((0, lo), (hi, L)):
                for t in range(j0 // P, (j1 + P - 1) // P if j1 > j0 else j0 // P):
                    pg = int(page_table[b, t])
                    a, e = max(j0, t * P) - t * P, min(j1, (t + 1) * P) - t * P
                    for pool in (k_pages, v_pages):
                        _nan_fill(pool, fp8, (pg, slice(None), slice(a, e)))


def to_bits(x: torch.Tensor):
    """Host numpy view of a bf16 (as uint16 bit patterns) or uint8 tensor."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16")
    return x.numpy()


def scale_of(wl: Workload) -> float:
    """Softmax scale as the float32 the kernel receives."""
    return float(torch.tensor(wl.softmax_scale, dtype=torch.float32))


def visible_token_count(wl: Workload, kv_lens: Sequence[int]) -> int:
    """Number of (sequence, key) pairs that at least one query row may see;
    the algorithmic K/V bytes are this times Hkv * D * element size * 2."""
    total = 0
    for L in kv_lens:
        L = int(L)
        if L <= 0:
            continue
        lo, hi = _row_positions_span(wl, L)
        total += max(0, hi - lo)
    return total
