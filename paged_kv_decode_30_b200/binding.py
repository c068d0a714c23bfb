"""ctypes binding of the C ABI in ``include/paged_decode_attn.h``.

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the CUDA stream, and the library does every step of the
computation. If the shared library is missing, loading raises; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpaged_decode_attn.so")

PDA_KV_BF16 = 0
PDA_KV_FP8_E4M3 = 1
PDA_KV_NVFP4 = 2
PDA_CAUSAL_OFF = -1
PDA_CAUSAL_BOTTOM_RIGHT = -2
PDA_FLAG_NO_PDL = 1
PDA_FLAG_TENSOR_CORES = 2
PDA_FLAG_CUDA_CORES = 4
PDA_FLAG_FUSED_MERGE = 8
PDA_FLAG_NATIVE_FP8_QK = 16
# Size of the library's fixed workspace array used by paged_decode_attn_no_alloc.
PDA_NO_ALLOC_WORKSPACE_BYTES = 16 * 1024 * 1024

STATUS = {
    0: "PDA_OK", 1: "PDA_ERR_INVALID_ARG", 2: "PDA_ERR_UNSUPPORTED",
    3: "PDA_ERR_MISALIGNED", 4: "PDA_ERR_WORKSPACE", 5: "PDA_ERR_CUDA",
    6: "PDA_ERR_BAD_PAGE", 7: "PDA_ERR_TIMEOUT",
}

# Every symbol the header declares (checked by the CPU test suite).
EXPORTED = (
    "paged_decode_attn", "paged_decode_attn_no_alloc", "paged_decode_attn_workspace_bytes",
    "pda_choose_num_splits", "pda_merge_states", "pda_status_string",
    "pda_last_device_error", "pda_abi_version", "pda_plan_kernel", "pda_hbm_read_probe",
    "paged_kv_append",
)
PDA_KERNEL_SPLIT_FMA = 0
PDA_KERNEL_SPLIT_TMA = 1
KERNEL_NAMES = {PDA_KERNEL_SPLIT_FMA: "split_fma_kernel", PDA_KERNEL_SPLIT_TMA: "split_tma_kernel"}


class PdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class PdaAppendParams(ctypes.Structure):
    """Mirror of ``pda_append_params``."""

    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_new", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
        ("kv_scale", ctypes.c_float),
        ("k_scales", ctypes.c_void_p),
        ("v_scales", ctypes.c_void_p),
    ]


class PdaParams(ctypes.Structure):
    """Mirror of ``pda_params``."""

    _fields_ = [
        ("batch", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("causal_offset", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
        ("kv_scale", ctypes.c_float),
        ("max_kv_len", ctypes.c_int32),
        ("num_splits", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("num_splits_out", ctypes.POINTER(ctypes.c_int32)),
        ("sinks", ctypes.c_void_p),
        ("k_scales", ctypes.c_void_p),
        ("v_scales", ctypes.c_void_p),
    ]


_lib = None


def load(path: Optional[str] = None):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m paged_kv_decode_30_b200.build`"
            " (there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    pp = ctypes.POINTER(PdaParams)
    lib.paged_decode_attn.restype = i32
    lib.paged_decode_attn.argtypes = [vp, vp, vp, vp, vp, pp, vp, vp, vp]
    lib.paged_decode_attn_no_alloc.restype = i32
    lib.paged_decode_attn_no_alloc.argtypes = [vp, vp, vp, vp, vp, pp, vp, vp, vp]
    lib.paged_decode_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.paged_decode_attn_workspace_bytes.argtypes = [pp]
    lib.pda_choose_num_splits.restype = i32
    lib.pda_choose_num_splits.argtypes = [pp, i32]
    lib.pda_merge_states.restype = i32
    lib.pda_merge_states.argtypes = [vp, vp, i32, i64, i32, vp, vp, vp, i32, vp]
    lib.pda_status_string.restype = ctypes.c_char_p
    lib.pda_status_string.argtypes = [i32]
    lib.pda_last_device_error.restype = i32
    lib.pda_last_device_error.argtypes = [vp]
    lib.pda_abi_version.restype = i32
    lib.pda_abi_version.argtypes = []
    lib.pda_plan_kernel.restype = i32
    lib.pda_plan_kernel.argtypes = [pp]
    lib.paged_kv_append.restype = i32
    lib.paged_kv_append.argtypes = [vp, vp, vp, vp, ctypes.POINTER(PdaAppendParams), vp, vp, vp]
    lib.pda_hbm_read_probe.restype = i32
    lib.pda_hbm_read_probe.argtypes = [vp, ctypes.c_size_t, vp, vp]
    if path is None:
        _lib = lib
    return lib


def make_params(*, batch, q_len, num_q_heads, num_kv_heads, head_dim, page_size,
                max_pages_per_seq, num_pages, scale, causal_offset=PDA_CAUSAL_OFF,
                window=0, kv_dtype=PDA_KV_BF16, kv_scale=1.0, max_kv_len=0,
                num_splits=0, flags=0) -> PdaParams:
    p = PdaParams()
    p.batch, p.q_len = batch, q_len
    p.num_q_heads, p.num_kv_heads = num_q_heads, num_kv_heads
    p.head_dim, p.page_size = head_dim, page_size
    p.max_pages_per_seq, p.num_pages = max_pages_per_seq, num_pages
    p.scale = scale
    p.causal_offset, p.window = causal_offset, window
    p.kv_dtype, p.kv_scale = kv_dtype, kv_scale
    p.max_kv_len, p.num_splits, p.flags = max_kv_len, num_splits, flags
    p.workspace = None
    p.workspace_bytes = 0
    return p


def status_string(status: int) -> str:
    return load().pda_status_string(status).decode()


def choose_num_splits(params: PdaParams, num_sms: int) -> int:
    return load().pda_choose_num_splits(ctypes.byref(params), num_sms)


def plan_kernel(params: PdaParams) -> int:
    """PDA_KERNEL_SPLIT_FMA or PDA_KERNEL_SPLIT_TMA (-1: invalid params)."""
    return load().pda_plan_kernel(ctypes.byref(params))


def hbm_read_probe(buf, sink, stream=None):
    """Read every byte of the CUDA tensor ``buf`` once (bandwidth probe);
    ``sink`` is an 8-byte CUDA tensor the kernel XORs into."""
    st = load().pda_hbm_read_probe(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink),
                                   _stream_handle(stream))
    if st != 0:
        raise PdaError(st, "pda_hbm_read_probe")


def workspace_bytes(params: PdaParams) -> int:
    return load().paged_decode_attn_workspace_bytes(ctypes.byref(params))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _params_for(q, k_pages, v_pages, page_table, kv_lens, k_scales, v_scales, **kw):
    """pda_params for CUDA tensors (checks they are contiguous CUDA tensors);
    the KV dtype follows the pools: bf16, uint8 e4m3 codes, or uint8 NVFP4
    codes when block-scale pools are given."""
    import torch
    B, q_len, Hq, D = q.shape
    for t in (q, k_pages, v_pages, page_table, kv_lens):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("all inputs must be contiguous CUDA tensors")
    if k_scales is not None or v_scales is not None:
        for t in (k_scales, v_scales):
            if t is None or not t.is_cuda or not t.is_contiguous() or t.dtype != torch.uint8:
                raise ValueError("k_scales and v_scales must be contiguous uint8 CUDA tensors")
        kv_dtype = PDA_KV_NVFP4
    else:
        kv_dtype = PDA_KV_FP8_E4M3 if k_pages.dtype == torch.uint8 else PDA_KV_BF16
    params = make_params(
        batch=B, q_len=q_len, num_q_heads=Hq, head_dim=D, page_size=k_pages.shape[2],
        max_pages_per_seq=page_table.shape[1], num_pages=k_pages.shape[0],
        kv_dtype=kv_dtype, **kw)
    if kv_dtype == PDA_KV_NVFP4:
        params.k_scales = k_scales.data_ptr()
        params.v_scales = v_scales.data_ptr()
    return params


def paged_decode_attn(q, k_pages, v_pages, page_table, kv_lens, *, num_kv_heads,
                      scale, causal_offset=PDA_CAUSAL_OFF, window=0, kv_scale=1.0,
                      max_kv_len=0, num_splits=0, flags=0, out=None, lse=None,
                      workspace=None, stream=None, with_lse=True, sinks=None,
                      library_workspace=False, k_scales=None, v_scales=None):
    """Run the library on CUDA tensors; returns (out, lse, num_splits_used).

    q [B, q_len, Hq, D] bf16; k/v_pages [num_pages, Hkv, P, D] bf16 or uint8
    (e4m3 codes), or with k_scales / v_scales (uint8 [num_pages, Hkv, P,
    D/16] e4m3 block scales) uint8 [num_pages, Hkv, P, D/2] NVFP4 codes;
    page_table int32 [B, max_pages]; kv_lens int32 [B];
    sinks: optional float32 CUDA tensor [Hq] of attention-sink logits.
    ``workspace``: a CUDA uint8 tensor (any contents; reusable across calls),
    or None to let the binding allocate exactly what the call needs.
    ``library_workspace``: pass no workspace, so the library uses (and grows
    in stream order) the buffer it owns on the device.
    """
    import torch
    lib = load()
    B, q_len, Hq, D = q.shape
    params = _params_for(q, k_pages, v_pages, page_table, kv_lens, k_scales, v_scales,
                         num_kv_heads=num_kv_heads, scale=scale, causal_offset=causal_offset,
                         window=window, kv_scale=kv_scale, max_kv_len=max_kv_len,
                         num_splits=num_splits, flags=flags)
    if out is None:
        out = torch.empty((B, q_len, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((B, q_len, Hq), dtype=torch.float32, device=q.device)
    if workspace is None and not library_workspace:
        need = lib.paged_decode_attn_workspace_bytes(ctypes.byref(params))
        if need == ctypes.c_size_t(-1).value:
            raise PdaError(1, "paged_decode_attn_workspace_bytes")
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        params.workspace = workspace.data_ptr()
        params.workspace_bytes = workspace.numel() * workspace.element_size()
    if sinks is not None:
        if not (sinks.is_cuda and sinks.dtype == torch.float32 and sinks.numel() == Hq):
            raise ValueError("sinks must be a float32 CUDA tensor of num_q_heads entries")
        params.sinks = sinks.data_ptr()
    used = ctypes.c_int32(0)
    params.num_splits_out = ctypes.pointer(used)
    st = lib.paged_decode_attn(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(kv_lens),
        ctypes.byref(params), _ptr(out), _ptr(lse), _stream_handle(stream))
    if st != 0:
        raise PdaError(st, "paged_decode_attn")
    return out, lse, used.value


def paged_decode_attn_no_alloc(q, k_pages, v_pages, page_table, kv_lens, *,
                               num_kv_heads, scale, causal_offset=PDA_CAUSAL_OFF,
                               window=0, kv_scale=1.0, max_kv_len=0, num_splits=0,
                               flags=0, out=None, lse=None, stream=None, sinks=None,
                               k_scales=None, v_scales=None):
    """The allocation-free entry point: the call's whole workspace goes to
    the library's fixed device array (see the C header). Same arguments as
    paged_decode_attn minus ``workspace``. ``out`` and ``lse`` are allocated
    here by torch only when the caller passes None."""
    import torch
    lib = load()
    B, q_len, Hq, D = q.shape
    params = _params_for(q, k_pages, v_pages, page_table, kv_lens, k_scales, v_scales,
                         num_kv_heads=num_kv_heads, scale=scale, causal_offset=causal_offset,
                         window=window, kv_scale=kv_scale, max_kv_len=max_kv_len,
                         num_splits=num_splits, flags=flags)
    if out is None:
        out = torch.empty((B, q_len, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, q_len, Hq), dtype=torch.float32, device=q.device)
    for t in (out, lse):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float32:
            raise ValueError("out and lse must be contiguous float32 CUDA tensors")
    if sinks is not None:
        if not (sinks.is_cuda and sinks.dtype == torch.float32 and sinks.numel() == Hq):
            raise ValueError("sinks must be a float32 CUDA tensor of num_q_heads entries")
        params.sinks = sinks.data_ptr()
    used = ctypes.c_int32(0)
    params.num_splits_out = ctypes.pointer(used)
    st = lib.paged_decode_attn_no_alloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(kv_lens),
        ctypes.byref(params), _ptr(out), _ptr(lse), _stream_handle(stream))
    if st != 0:
        raise PdaError(st, "paged_decode_attn_no_alloc")
    return out, lse, used.value


def paged_kv_append(k_new, v_new, page_table, kv_lens, k_pages, v_pages, *, kv_scale=1.0,
                    stream=None, k_scales=None, v_scales=None):
    """Write new K/V rows (bf16 [B, num_new, Hkv, D]) into the pools at
    positions kv_lens[b] + t (kv_lens is not advanced). Pools of uint8 are
    e4m3 codes quantised with kv_scale, or, with k_scales / v_scales (uint8
    block-scale pools), NVFP4 codes; bf16 pools get the bits."""
    import torch
    B, T, Hkv, D = k_new.shape
    kv_dtype = PDA_KV_FP8_E4M3 if k_pages.dtype == torch.uint8 else PDA_KV_BF16
    tensors = [k_new, v_new, page_table, kv_lens, k_pages, v_pages]
    if k_scales is not None or v_scales is not None:
        kv_dtype = PDA_KV_NVFP4
        tensors += [k_scales, v_scales]
    for t_ in tensors:
        if t_ is None or not t_.is_cuda or not t_.is_contiguous():
            raise ValueError("all inputs must be contiguous CUDA tensors")
    p = PdaAppendParams(B, T, Hkv, D, k_pages.shape[2], page_table.shape[1], k_pages.shape[0],
                        kv_dtype, kv_scale, _ptr(k_scales), _ptr(v_scales))
    st = load().paged_kv_append(_ptr(k_new), _ptr(v_new), _ptr(page_table), _ptr(kv_lens),
                                ctypes.byref(p), _ptr(k_pages), _ptr(v_pages),
                                _stream_handle(stream))
    if st != 0:
        raise PdaError(st, "paged_kv_append")


def merge_states(o_parts, lse_parts, *, out=None, lse=None, sinks=None, stream=None):
    """LSE merge: o_parts [S, rows, D] fp32, lse_parts [S, rows] fp32; sinks
    optional fp32 [Hq] (row r uses sinks[r % Hq])."""
    import torch
    S, rows, D = o_parts.shape
    if out is None:
        out = torch.empty((rows, D), dtype=torch.float32, device=o_parts.device)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=o_parts.device)
    st = load().pda_merge_states(_ptr(o_parts), _ptr(lse_parts), S, rows, D,
                                 _ptr(out), _ptr(lse), _ptr(sinks),
                                 0 if sinks is None else sinks.numel(), _stream_handle(stream))
    if st != 0:
        raise PdaError(st, "pda_merge_states")
    return out, lse


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (then clear) the device error word."""
    return load().pda_last_device_error(_stream_handle(stream))
