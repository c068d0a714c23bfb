"""ctypes wrapper around ``oracle.c`` (test infrastructure only).

The C file is the oracle: plain single-threaded fp64 softmax attention that
walks the page table token by token. This module only builds it, loads it and
marshals numpy arrays in and out; it holds none of the method's arithmetic.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

ORACLE_KV_BF16 = 0
ORACLE_KV_FP8_E4M3 = 1
ORACLE_KV_NVFP4 = 2
CAUSAL_OFF = -1
CAUSAL_BOTTOM_RIGHT = -2

_lock = threading.Lock()
_lib = None


def build(out_path: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile oracle.c into a shared library with gcc and return its path.

    ``-ffp-contract=off`` keeps every multiply and add a separately rounded
    IEEE double operation.
    """
    cmd = [
        "gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-Wall",
        *extra_flags, _SRC, "-o", out_path, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return out_path


def _needs_build() -> bool:
    if not os.path.exists(_LIB_PATH):
        return True
    return os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)


def load(path: str | None = None):
    """Load (building first if stale) the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _needs_build():
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _declare(lib):
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_to_double.restype = ctypes.c_double
    lib.oracle_e2m1_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_encode.restype = ctypes.c_uint8
    lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
    lib.oracle_nvfp4_encode_block.restype = None
    lib.oracle_nvfp4_encode_block.argtypes = [ctypes.c_void_p, ctypes.c_float,
                                              ctypes.c_void_p, ctypes.c_void_p]
    p = ctypes.c_void_p
    i32 = ctypes.c_int
    lib.oracle_paged_decode_attn.restype = i32
    lib.oracle_paged_decode_attn.argtypes = [
        p, p, p, p, p,                      # q, k, v, k_scales, v_scales
        p, p,                               # page_table, kv_lens
        i32, i32, i32, i32, i32, i32, i32, i32,  # B Lq Hq Hkv D P max_pages num_pages
        ctypes.c_float, i32, i32, i32, ctypes.c_float,  # scale causal window dtype kv_scale
        p,                                  # sinks (float [Hq]) or NULL
        ctypes.c_int64, ctypes.c_int64,     # tok_lo, tok_hi
        p, p,                               # out, lse
    ]
    lib.oracle_paged_decode_attn_mt.restype = i32
    lib.oracle_paged_decode_attn_mt.argtypes = [
        p, p, p, p, p, p, p,
        i32, i32, i32, i32, i32, i32, i32, i32,
        ctypes.c_float, i32, i32, i32, ctypes.c_float,
        p,                                  # sinks or NULL
        p, p, i32,                          # out, lse, threads
    ]
    lib.oracle_max_threads.restype = i32
    lib.oracle_max_threads.argtypes = []
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_quantize_q_e4m3.restype = i32
    lib.oracle_quantize_q_e4m3.argtypes = [p, ctypes.c_int64, i32, p]
    lib.oracle_paged_kv_append.restype = i32
    lib.oracle_paged_kv_append.argtypes = [
        p, p, p, p,                          # k_new, v_new, page_table, kv_lens
        i32, i32, i32, i32, i32, i32, i32,   # B num_new Hkv D P max_pages num_pages
        i32, ctypes.c_float,                 # kv_dtype, kv_scale
        p, p,                                # k_pages, v_pages (in place)
        p, p,                                # k_scales, v_scales (NVFP4, in place)
    ]
    lib.oracle_merge_states.restype = i32
    lib.oracle_merge_states.argtypes = [p, p, i32, ctypes.c_int64, i32, p, p]
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _own_copy(a, dtype) -> np.ndarray:
    """A C-contiguous copy of `a` as `dtype` (array-likes that offer
    .numpy(), such as CPU tensors, are read through it)."""
    if not isinstance(a, np.ndarray) and hasattr(a, "numpy"):
        a = a.numpy()
    return np.array(a, dtype=dtype, copy=True, order="C")


def bf16_to_double(bits: int, lib=None) -> float:
    return (lib or load()).oracle_bf16_to_double(int(bits))


def e4m3_to_double(code: int, lib=None) -> float:
    return (lib or load()).oracle_e4m3_to_double(int(code))


def e2m1_to_double(code: int, lib=None) -> float:
    return (lib or load()).oracle_e2m1_to_double(int(code))


def e2m1_encode(x: float, lib=None) -> int:
    return int((lib or load()).oracle_e2m1_encode(float(x)))


def nvfp4_encode_block(x_bits, kv_scale: float, lib=None):
    """16 bf16 values (bits) -> (16 e2m1 codes, e4m3 scale code)."""
    lib = lib or load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    assert x.shape == (16,)
    codes = np.zeros(16, dtype=np.uint8)
    sc = np.zeros(1, dtype=np.uint8)
    lib.oracle_nvfp4_encode_block(_ptr(x), float(kv_scale), _ptr(codes), _ptr(sc))
    return codes, int(sc[0])


def paged_decode_attn(q_bits, k_pages, v_pages, page_table, kv_lens, *,
                      num_kv_heads, page_size, scale, causal_offset=CAUSAL_OFF,
                      window=0, kv_dtype=ORACLE_KV_BF16, kv_scale=1.0,
                      tok_range=None, threads=1, sinks=None, k_scales=None,
                      v_scales=None, lib=None):
    """Run the oracle on host arrays.

    q_bits      uint16 [B, q_len, Hq, D]   (bf16 bit patterns)
    k/v_pages   uint16 or uint8 [num_pages, Hkv, page_size, D], or (NVFP4)
                uint8 [num_pages, Hkv, page_size, D/2] packed codes
    k/v_scales  NVFP4 only: uint8 e4m3 block scales [num_pages, Hkv, page_size, D/16]
    page_table  int32 [B, max_pages];  kv_lens int32 [B]
    tok_range   optional (lo, hi): keep only keys with lo <= j < hi
    threads     > 1: the same rows on that many OpenMP threads (bit-identical
                results; no tok_range)
    sinks       optional float [Hq]: attention-sink logit per query head
    Returns (out float64 [B, q_len, Hq, D], lse float64 [B, q_len, Hq]).
    """
    lib = lib or load()
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kdt = np.uint16 if kv_dtype == ORACLE_KV_BF16 else np.uint8
    k_pages = np.ascontiguousarray(k_pages, dtype=kdt)
    v_pages = np.ascontiguousarray(v_pages, dtype=kdt)
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    kv_lens = np.ascontiguousarray(kv_lens, dtype=np.int32)
    B, q_len, Hq, D = q_bits.shape
    num_pages = k_pages.shape[0]
    assert k_pages.shape == v_pages.shape
    nv = kv_dtype == ORACLE_KV_NVFP4
    assert k_pages.shape[1:] == (num_kv_heads, page_size, D // 2 if nv else D), k_pages.shape
    ksp = vsp = None
    if nv:
        k_scales = np.ascontiguousarray(k_scales, dtype=np.uint8)
        v_scales = np.ascontiguousarray(v_scales, dtype=np.uint8)
        assert k_scales.shape == v_scales.shape == (num_pages, num_kv_heads, page_size, D // 16)
        ksp, vsp = _ptr(k_scales), _ptr(v_scales)
    max_pages = page_table.shape[1] if page_table.ndim == 2 else 0
    out = np.zeros((B, q_len, Hq, D), dtype=np.float64)
    lse = np.zeros((B, q_len, Hq), dtype=np.float64)
    lo, hi = (0, -1) if tok_range is None else tok_range
    sk = None if sinks is None else np.ascontiguousarray(sinks, dtype=np.float32)
    if sk is not None:
        assert sk.shape == (Hq,), sk.shape
    skp = None if sk is None else _ptr(sk)
    if threads > 1:
        if tok_range is not None:
            raise ValueError("tok_range is only supported single-threaded")
        rc = lib.oracle_paged_decode_attn_mt(
            _ptr(q_bits), _ptr(k_pages), _ptr(v_pages), ksp, vsp, _ptr(page_table),
            _ptr(kv_lens), B, q_len, Hq, num_kv_heads, D, page_size, max_pages,
            num_pages, float(scale), int(causal_offset), int(window),
            int(kv_dtype), float(kv_scale), skp, _ptr(out), _ptr(lse), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_paged_decode_attn_mt failed with status {rc}")
        return out, lse
    rc = lib.oracle_paged_decode_attn(
        _ptr(q_bits), _ptr(k_pages), _ptr(v_pages), ksp, vsp, _ptr(page_table),
        _ptr(kv_lens), B, q_len, Hq, num_kv_heads, D, page_size, max_pages,
        num_pages, float(scale), int(causal_offset), int(window),
        int(kv_dtype), float(kv_scale), skp, int(lo), int(hi), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_attn failed with status {rc}")
    return out, lse


def e4m3_encode(x: float, lib=None) -> int:
    return int((lib or load()).oracle_e4m3_encode(float(x)))


def paged_kv_append(k_new_bits, v_new_bits, page_table, kv_lens, k_pages, v_pages, *,
                    page_size, kv_dtype=ORACLE_KV_BF16, kv_scale=1.0, k_scales=None,
                    v_scales=None, lib=None):
    """Append new rows into copies of the pools; returns (k_pages, v_pages),
    or (k_pages, v_pages, k_scales, v_scales) for NVFP4.

    k/v_new_bits  uint16 [B, num_new, Hkv, D] (bf16 bit patterns)
    k/v_pages     uint16 or uint8 [num_pages, Hkv, page_size, D] (NVFP4: D/2)
    k/v_scales    NVFP4 only: uint8 [num_pages, Hkv, page_size, D/16]
    """
    lib = lib or load()
    k_new_bits = np.ascontiguousarray(k_new_bits, dtype=np.uint16)
    v_new_bits = np.ascontiguousarray(v_new_bits, dtype=np.uint16)
    kdt = np.uint16 if kv_dtype == ORACLE_KV_BF16 else np.uint8
    kp = _own_copy(k_pages, kdt)
    vp = _own_copy(v_pages, kdt)
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    kv_lens = np.ascontiguousarray(kv_lens, dtype=np.int32)
    B, num_new, Hkv, D = k_new_bits.shape
    nv = kv_dtype == ORACLE_KV_NVFP4
    ks = vs = None
    if nv:
        ks = _own_copy(k_scales, np.uint8)
        vs = _own_copy(v_scales, np.uint8)
    rc = lib.oracle_paged_kv_append(
        _ptr(k_new_bits), _ptr(v_new_bits), _ptr(page_table), _ptr(kv_lens), B, num_new,
        Hkv, D, page_size, page_table.shape[1], kp.shape[0], int(kv_dtype), float(kv_scale),
        _ptr(kp), _ptr(vp), None if ks is None else _ptr(ks), None if vs is None else _ptr(vs))
    if rc != 0:
        raise ValueError(f"oracle_paged_kv_append failed with status {rc}")
    return (kp, vp, ks, vs) if nv else (kp, vp)


def quantize_q_e4m3(q_bits, lib=None):
    """q (bf16 bits [..., D]) as native FP8 QK uses it, as bf16 bits."""
    lib = lib or load()
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    out = np.empty_like(q_bits)
    D = q_bits.shape[-1]
    rc = lib.oracle_quantize_q_e4m3(_ptr(q_bits), q_bits.size // D, D, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q_e4m3 failed with status {rc}")
    return out


def max_threads(lib=None) -> int:
    """OpenMP threads the multi-threaded entry point uses by default."""
    return int((lib or load()).oracle_max_threads())


def merge_states(o_parts, lse_parts, lib=None):
    """LSE merge of n states: o_parts [n, rows, D], lse_parts [n, rows]."""
    lib = lib or load()
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, rows, D = o_parts.shape
    out = np.zeros((rows, D), dtype=np.float64)
    lse = np.zeros((rows,), dtype=np.float64)
    rc = lib.oracle_merge_states(_ptr(o_parts), _ptr(lse_parts), n, rows, D,
                                 _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_merge_states failed with status {rc}")
    return out, lse
