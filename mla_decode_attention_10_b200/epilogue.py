"""Python binding of ``libmla_epilogue.so``: argument marshalling only.

Every function here forwards to the C ABI declared in ``include/mla_epilogue.h``
and ``include/mla_harness.h`` under the same name; every step of the
epilogue runs in the library's CUDA kernels.  Torch is used for device memory
and streams only.  If the library has not been built, loading it raises:
there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_epilogue.so")

# constants of include/mla_epilogue.h (checked against the header by the tests)
MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_ALIGNMENT = 2
MLA_ERR_UNSUPPORTED = 3
MLA_ERR_CUDA = 4

MLA_FLAG_ROPE = 1
MLA_FLAG_Q_FP8 = 2
MLA_FLAG_KV_FP8 = 4
MLA_FLAG_PDL = 8
MLA_FLAG_FORCE_SPLIT = 16
MLA_FLAG_FORCE_ROWS = 32

MLA_STATUS_SLOT_RANGE = 1
MLA_STATUS_POS_RANGE = 2
MLA_STATUS_TIMEOUT = 4

MLA_MODE_SPLIT = 1
MLA_MODE_ROWS = 2

MLA_HARNESS_EMPTY_WAIT = 256

ROW = 576
NOPE = 512
PE = 64


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)}"
                         + (f" (cudaError {last_cuda_error()})" if code == MLA_ERR_CUDA else ""))
        self.code = code


class mla_plan(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("threads_per_block", ctypes.c_int32),
                ("blocks", ctypes.c_int64), ("rows_per_block", ctypes.c_int32),
                ("sm_count", ctypes.c_int32)]


class mla_tuning(ctypes.Structure):
    _fields_ = [("split_max_rows", ctypes.c_int64), ("split_rows_per_block", ctypes.c_int32),
                ("rows_warps_per_block", ctypes.c_int32), ("rows_blocks_per_sm", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m mla_decode_attention_10_b200.build` "
                               "(the epilogue has no CPU or PyTorch fallback)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, u32, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64
        L.mla_epilogue_launch.restype = ctypes.c_int
        L.mla_epilogue_launch.argtypes = [vp, i64, i64, vp, i64, i64, vp, i64, vp, i64,
                                          vp, vp, vp, i64, vp, vp,
                                          i64, i64, i64, i64, u32, vp, vp, vp, vp]
        L.mla_epilogue_plan.restype = ctypes.c_int
        L.mla_epilogue_plan.argtypes = [i64, i64, u32, i32, ctypes.POINTER(mla_plan)]
        L.mla_epilogue_set_tuning.restype = None
        L.mla_epilogue_set_tuning.argtypes = [ctypes.POINTER(mla_tuning)]
        L.mla_epilogue_get_tuning.restype = None
        L.mla_epilogue_get_tuning.argtypes = [ctypes.POINTER(mla_tuning)]
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_status_string.argtypes = [ctypes.c_int]
        L.mla_last_cuda_error.restype = ctypes.c_int32
        L.mla_last_cuda_error.argtypes = []
        L.mla_harness_produce.restype = ctypes.c_int
        L.mla_harness_produce.argtypes = [vp, vp, vp, i64, i64, vp, i64, i64, i64, i64, u32, vp]
        L.mla_harness_produce_after_weights.restype = ctypes.c_int
        L.mla_harness_produce_after_weights.argtypes = [vp, vp, vp, i64, i64, vp, i64, i64, vp, i64, vp, i64, i64,
                                                        u32, vp]
        L.mla_harness_empty.restype = ctypes.c_int
        L.mla_harness_empty.argtypes = [i64, i32, u32, vp]
        L.mla_harness_consume.restype = ctypes.c_int
        L.mla_harness_consume.argtypes = [vp, vp, vp, i64, i64, i64, u32, vp, vp]
        L.mla_absorb_launch.restype = ctypes.c_int
        L.mla_absorb_launch.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i64, vp, i64, i64, u32,
                                        vp, vp, vp]
        L.mla_harness_div_check.restype = ctypes.c_int
        L.mla_harness_div_check.argtypes = [ctypes.c_float, u64, u64, vp, vp]
        L.mla_harness_bf16_scale_check.restype = ctypes.c_int
        L.mla_harness_bf16_scale_check.argtypes = [u32, u32, vp, vp]
        _lib = L
    return _lib


# ---- the C ABI, one to one ------------------------------------------------------------

def mla_epilogue_launch(q_nope, q_nope_stride_t, q_nope_stride_h, q_pe, q_pe_stride_t, q_pe_stride_h,
                        kv_c, kv_c_stride_t, k_pe, k_pe_stride_t, slot_mapping, positions,
                        cos_sin, rope_rows, q_scale, kv_scale, T, H, block_size, num_blocks,
                        flags, q_out, cache, status, stream) -> int:
    """Pointers as ints (device addresses; 0/None for NULL); returns the mla_status code."""
    return lib().mla_epilogue_launch(q_nope, q_nope_stride_t, q_nope_stride_h, q_pe, q_pe_stride_t,
                                     q_pe_stride_h, kv_c, kv_c_stride_t, k_pe, k_pe_stride_t,
                                     slot_mapping, positions, cos_sin, rope_rows, q_scale, kv_scale,
                                     T, H, block_size, num_blocks, flags, q_out, cache, status, stream)


def mla_epilogue_plan(T: int, H: int, flags: int = 0, sm_count: int = 0) -> mla_plan:
    p = mla_plan()
    rc = lib().mla_epilogue_plan(T, H, flags, sm_count, ctypes.byref(p))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_epilogue_plan")
    return p


def mla_epilogue_set_tuning(split_max_rows: int = 0, split_rows_per_block: int = 0,
                            rows_warps_per_block: int = 0, rows_blocks_per_sm: int = 0) -> None:
    t = mla_tuning(split_max_rows, split_rows_per_block, rows_warps_per_block, rows_blocks_per_sm)
    lib().mla_epilogue_set_tuning(ctypes.byref(t))


def mla_epilogue_get_tuning() -> mla_tuning:
    t = mla_tuning()
    lib().mla_epilogue_get_tuning(ctypes.byref(t))
    return t


def status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def last_cuda_error() -> int:
    return lib().mla_last_cuda_error()


def mla_harness_produce(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h, q_pe,
                        q_pe_stride_t, q_pe_stride_h, T, H, flags, stream) -> int:
    return lib().mla_harness_produce(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h,
                                     q_pe, q_pe_stride_t, q_pe_stride_h, T, H, flags, stream)


def mla_harness_produce_after_weights(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h, q_pe,
                                     q_pe_stride_t, q_pe_stride_h, weights, weight_bytes, sink, T, H, flags,
                                     stream) -> int:
    return lib().mla_harness_produce_after_weights(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h, q_pe,
                                                   q_pe_stride_t, q_pe_stride_h, weights, weight_bytes, sink, T, H,
                                                   flags, stream)


def mla_harness_empty(blocks: int, threads: int, flags: int, stream) -> int:
    return lib().mla_harness_empty(blocks, threads, flags, stream)


def mla_harness_consume(q_out, cache, slot_mapping, T, H, cache_rows, flags, scores, stream) -> int:
    return lib().mla_harness_consume(q_out, cache, slot_mapping, T, H, cache_rows, flags, scores, stream)


def mla_harness_div_check(scale: float, first: int, count: int, result, stream) -> int:
    return lib().mla_harness_div_check(scale, first, count, result, stream)


def mla_harness_bf16_scale_check(first: int, count: int, result, stream) -> int:
    return lib().mla_harness_bf16_scale_check(first, count, result, stream)


def mla_absorb_launch(q_nope_c, q_nope_c_stride_t, q_nope_c_stride_h, w_uk, q_pe, q_pe_stride_t, q_pe_stride_h,
                      positions, cos_sin, rope_rows, q_scale, T, H, flags, q_out, status, stream) -> int:
    """The query rows from the absorption product (include/mla_absorb.h); returns the mla_status code."""
    return lib().mla_absorb_launch(q_nope_c, q_nope_c_stride_t, q_nope_c_stride_h, w_uk, q_pe, q_pe_stride_t,
                                   q_pe_stride_h, positions, cos_sin, rope_rows, q_scale, T, H, flags, q_out,
                                   status, stream)


# ---- torch convenience ------------------------------------------------------------------

def _dptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def fused_mla_decode_q_concat_kv_cache_insert(
        ql_nope: torch.Tensor, q_pe: torch.Tensor, kv_c: torch.Tensor, k_pe: torch.Tensor,
        cache: torch.Tensor, slot_mapping: torch.Tensor, *,
        positions: Optional[torch.Tensor] = None, cos_sin: Optional[torch.Tensor] = None,
        q_scale: Optional[torch.Tensor] = None, kv_scale: Optional[torch.Tensor] = None,
        q_out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
        pdl: bool = False, extra_flags: int = 0,
        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Torch-tensor form of ``mla_epilogue_launch`` (the Python op of the vLLM
    PR #54896 report's boundary test, extended with RoPE and FP8).

    RoPE is on when ``cos_sin`` is given, FP8 Q / KV when ``q_scale`` /
    ``kv_scale`` are given (one-element fp32 device tensors).  ``cache`` is
    updated in place; ``q_out`` ([T,H,576], bf16, or uint8 e4m3 bytes with FP8)
    is allocated when not given.  Raises ``MlaError`` when the library rejects
    the arguments.
    """
    T, H = ql_nope.shape[0], ql_nope.shape[1]
    flags = extra_flags
    if cos_sin is not None:
        flags |= MLA_FLAG_ROPE
    if q_scale is not None:
        flags |= MLA_FLAG_Q_FP8
    if kv_scale is not None:
        flags |= MLA_FLAG_KV_FP8
    if pdl:
        flags |= MLA_FLAG_PDL
    for name, t in (("ql_nope", ql_nope), ("q_pe", q_pe), ("kv_c", kv_c), ("k_pe", k_pe)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(-1) != 1:
            raise ValueError(f"{name}: a bf16 CUDA tensor with inner stride 1 is required")
    if tuple(ql_nope.shape) != (T, H, NOPE) or tuple(q_pe.shape) != (T, H, PE):
        raise ValueError("ql_nope must be [T,H,512] and q_pe [T,H,64]")
    if tuple(kv_c.shape) != (T, NOPE) or tuple(k_pe.shape) != (T, PE):
        raise ValueError("kv_c must be [T,512] and k_pe [T,64]")
    if slot_mapping.dtype != torch.int64 or not slot_mapping.is_contiguous() or slot_mapping.numel() != T:
        raise ValueError("slot_mapping must be a contiguous int64 [T] tensor")
    if cache.dim() != 3 or cache.shape[2] != ROW or not cache.is_contiguous():
        raise ValueError("cache must be a contiguous [num_blocks, block_size, 576] tensor")
    if cache.element_size() != (1 if kv_scale is not None else 2):
        raise ValueError("cache element size must be 1 (e4m3) with kv_scale, 2 (bf16) without")
    if cos_sin is not None:
        if positions is None or positions.dtype != torch.int32 or not positions.is_contiguous():
            raise ValueError("RoPE needs contiguous int32 positions [T]")
        if cos_sin.dtype != torch.float32 or not cos_sin.is_contiguous() or cos_sin.shape[-1] != PE:
            raise ValueError("cos_sin must be a contiguous fp32 [rows, 64] table")
    for name, sc in (("q_scale", q_scale), ("kv_scale", kv_scale)):
        if sc is not None and (sc.dtype != torch.float32 or not sc.is_cuda):
            raise ValueError(f"{name} must be a fp32 CUDA tensor")
    if q_out is None:
        q_out = torch.empty((T, H, ROW), device=ql_nope.device,
                            dtype=torch.uint8 if q_scale is not None else torch.bfloat16)
    rc = mla_epilogue_launch(
        _dptr(ql_nope), ql_nope.stride(0), ql_nope.stride(1),
        _dptr(q_pe), q_pe.stride(0), q_pe.stride(1),
        _dptr(kv_c), kv_c.stride(0), _dptr(k_pe), k_pe.stride(0),
        _dptr(slot_mapping), _dptr(positions) if cos_sin is not None else None,
        _dptr(cos_sin), cos_sin.shape[0] if cos_sin is not None else 0,
        _dptr(q_scale), _dptr(kv_scale),
        T, H, cache.shape[1], cache.shape[0], flags,
        _dptr(q_out), _dptr(cache), _dptr(status), _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_epilogue_launch")
    return q_out


def launch_absorb_workload(w, q_out: torch.Tensor, *, status: Optional[torch.Tensor] = None,
                           extra_flags: int = 0, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Launch mla_absorb_launch on a device-resident ``workloads.AbsorbWorkload``."""
    return mla_absorb_launch(
        _dptr(w.q_nope_c), w.q_nope_c.stride(0), w.q_nope_c.stride(1), _dptr(w.w_uk),
        _dptr(w.q_pe), w.q_pe.stride(0), w.q_pe.stride(1), _dptr(w.positions), _dptr(w.cos_sin),
        w.cos_sin.shape[0] if w.cos_sin is not None else 0, _dptr(w.q_scale), w.T, w.H,
        w.flags | extra_flags, _dptr(q_out), _dptr(status), _stream_handle(stream))


def launch_workload(w, q_out: torch.Tensor, *, status: Optional[torch.Tensor] = None,
                    extra_flags: int = 0, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Launch on a device-resident ``workloads.Workload`` (its own flags plus
    ``extra_flags``); returns the mla_status code."""
    return mla_epilogue_launch(
        _dptr(w.q_nope), w.q_nope.stride(0), w.q_nope.stride(1),
        _dptr(w.q_pe), w.q_pe.stride(0), w.q_pe.stride(1),
        _dptr(w.kv_c), w.kv_c.stride(0), _dptr(w.k_pe), w.k_pe.stride(0),
        _dptr(w.slot_mapping), _dptr(w.positions), _dptr(w.cos_sin),
        w.cos_sin.shape[0] if w.cos_sin is not None else 0,
        _dptr(w.q_scale), _dptr(w.kv_scale),
        w.T, w.H, w.block_size, w.num_blocks, w.flags | extra_flags,
        _dptr(q_out), _dptr(w.cache), _dptr(status), _stream_handle(stream))
