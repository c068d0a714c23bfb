"""Helpers for the GPU parity tests: run the CUDA library through the C ABI
and the oracle on the same seeded inputs, and compare."""

from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import oracle as orc
from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W

# Tolerances (max |err|) against the oracle on the same bytes.
TOL = {
    W.KV_BF16: dict(out=2e-3, lse=1e-3),
    W.KV_FP8_E4M3: dict(out=2e-2, lse=2e-2),
    W.KV_NVFP4: dict(out=2e-2, lse=2e-2),
}


# Max |err| of every parity comparison made in this process, in order:
# (what, kv dtype, out error, lse error). conftest prints them at the end of
# the run; PDA_PARITY_LOG=<path> also writes them there as JSON lines.
RECORDS = []


def _record(what, kv_dtype, eo, el):
    RECORDS.append((what, kv_dtype, eo, el))
    path = os.environ.get("PDA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, "kv_dtype": int(kv_dtype), "out": eo,
                                "lse": el}) + "\n")


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def to_device(inp):
    d = torch.device("cuda")
    out = {k: inp[k].to(d) for k in ("q", "k_pages", "v_pages", "page_table", "kv_lens")}
    for k in ("k_scales", "v_scales"):
        out[k] = inp[k].to(d) if inp.get(k) is not None else None
    return out


def run_cuda(inp, **kw):
    """The library on inp (moved to the GPU if needed). Returns host float64
    out, lse and the split count used; asserts the device error word is clear."""
    wl = inp["workload"]
    t = to_device(inp)
    if t["k_scales"] is not None:
        kw = dict(kw, k_scales=t["k_scales"], v_scales=t["v_scales"])
    out, lse, used = B.paged_decode_attn(
        t["q"], t["k_pages"], t["v_pages"], t["page_table"], t["kv_lens"],
        num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl),
        causal_offset=wl.causal_offset, window=wl.window, kv_scale=inp["kv_scale"], **kw)
    torch.cuda.synchronize()
    err = B.last_device_error()
    assert err == 0, f"device error word {B.STATUS.get(err, err)}"
    return out.double().cpu().numpy(), lse.double().cpu().numpy(), used


def run_oracle(inp, seqs=None, sinks=None, native_qk=False, threads=None):
    """The oracle on all sequences, or on the listed ones only (their pages
    are gathered into a small pool first). Returns out, lse for those rows.
    ``threads``: OpenMP threads of the oracle (None: one for small inputs,
    every host core for large ones; the rows are bit-identical either way)."""
    wl = inp["workload"]
    pt = inp["page_table"].cpu()
    lens = inp["kv_lens"].cpu()
    ks, vs = inp.get("k_scales"), inp.get("v_scales")
    if seqs is None:
        q, kp, vp, table, kv = inp["q"], inp["k_pages"], inp["v_pages"], pt, lens
    else:
        P = wl.page_size
        rows, pages = [], []
        for b in seqs:
            n = (int(lens[b]) + P - 1) // P
            rows.append(list(range(len(pages), len(pages) + n)))
            pages += [int(x) for x in pt[b, :n]]
        width = max(1, max(len(r) for r in rows))
        table = torch.full((len(seqs), width), -1, dtype=torch.int32)
        for i, r in enumerate(rows):
            table[i, : len(r)] = torch.tensor(r, dtype=torch.int32)
        idx = torch.tensor(pages or [0], dtype=torch.int64, device=inp["k_pages"].device)
        kp, vp = inp["k_pages"][idx], inp["v_pages"][idx]
        if ks is not None:
            ks, vs = ks[idx], vs[idx]
        q = inp["q"][torch.tensor(seqs, device=inp["q"].device)]
        kv = lens[seqs]
    qbits = W.to_bits(q)
    if native_qk:  # the oracle mirrors the Q quantisation of native FP8 QK
        qbits = orc.quantize_q_e4m3(qbits)
    if threads is None:
        threads = host_threads() if kp.numel() * kp.element_size() > (64 << 20) else 1
    return orc.paged_decode_attn(
        qbits, W.to_bits(kp), W.to_bits(vp), np.asarray(table, dtype=np.int32),
        np.asarray(kv, dtype=np.int32), num_kv_heads=wl.num_kv_heads,
        page_size=wl.page_size, scale=W.scale_of(wl), causal_offset=wl.causal_offset,
        window=wl.window, kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"], sinks=sinks,
        threads=threads, k_scales=None if ks is None else W.to_bits(ks),
        v_scales=None if vs is None else W.to_bits(vs))


def max_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    same_inf = np.isinf(got) & np.isinf(ref) & (np.sign(got) == np.sign(ref))
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), "empty-row pattern differs"
    d = np.where(same_inf, 0.0, np.abs(got - ref))
    assert not np.isnan(d).any(), "NaN in GPU output"
    return float(d.max()) if d.size else 0.0


def assert_parity(got_out, got_lse, ref_out, ref_lse, kv_dtype, what=""):
    tol = TOL[kv_dtype]
    eo = max_err(got_out, ref_out)
    el = max_err(got_lse, ref_lse)
    _record(what, kv_dtype, eo, el)
    assert eo <= tol["out"], f"{what}: out max|err| {eo:.3e} > {tol['out']}"
    assert el <= tol["lse"], f"{what}: lse max|err| {el:.3e} > {tol['lse']}"
    return eo, el
