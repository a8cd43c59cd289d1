"""CPU oracle of the fused MLA decode epilogue -- TEST INFRASTRUCTURE ONLY.

A thin ctypes wrapper around ``libmla_oracle.so`` (plain single-threaded C++,
see ``mla_oracle.cpp`` for the definition it follows and its readings of the
pages).  Only ``tests/``, the smoke check and the benchmark's CPU-baseline /
reference arm may import this package; the product path never does, and this
package imports nothing from the product package.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import build as _build

FLAG_ROPE = 1
FLAG_Q_FP8 = 2
FLAG_KV_FP8 = 4

STATUS_SLOT_RANGE = 1
STATUS_POS_RANGE = 2

ROW = 576

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32
        L.mla_oracle_run.restype = ctypes.c_int
        L.mla_oracle_run.argtypes = [vp, i64, i64, vp, i64, i64, vp, i64, vp, i64,
                                     vp, vp, vp, i64, vp, vp,
                                     i64, i64, i64, i64, u32, vp, vp, vp]
        L.mla_oracle_run_threads.restype = ctypes.c_int
        L.mla_oracle_run_threads.argtypes = L.mla_oracle_run.argtypes + [ctypes.c_int]
        L.mla_oracle_absorb_run.restype = ctypes.c_int
        L.mla_oracle_absorb_run.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i64, vp,
                                            i64, i64, u32, vp, vp]
        L.mla_oracle_bf16_to_f32.restype = ctypes.c_float
        L.mla_oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.mla_oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.mla_oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.mla_oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.mla_oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    assert t.device.type == "cpu", "the oracle takes host tensors"
    return t.data_ptr()


def _check_inner(t: torch.Tensor, name: str) -> None:
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: inner stride must be 1")


def run(q_nope: torch.Tensor, q_pe: torch.Tensor, kv_c: torch.Tensor, k_pe: torch.Tensor,
        slot_mapping: torch.Tensor, cache: torch.Tensor, flags: int,
        positions: Optional[torch.Tensor] = None, cos_sin: Optional[torch.Tensor] = None,
        q_scale: Optional[torch.Tensor] = None, kv_scale: Optional[torch.Tensor] = None,
        threads: int = 1) -> Tuple[torch.Tensor, int]:
    """Run the oracle on host tensors.

    ``cache`` ([num_blocks, block_size, 576], bf16 or uint8 for e4m3 bytes) is
    updated in place.  Returns ``(q_out, status)`` where ``q_out`` is
    [T, H, 576] bf16, or uint8 e4m3 bytes when ``FLAG_Q_FP8`` is set.
    ``threads`` > 1 runs the same function on that many contiguous token
    slices at once (the benchmark's all-cores baseline; slots must be unique).
    """
    T, H = q_nope.shape[0], q_nope.shape[1]
    assert q_nope.dtype == torch.bfloat16 and q_pe.dtype == torch.bfloat16
    assert kv_c.dtype == torch.bfloat16 and k_pe.dtype == torch.bfloat16
    assert slot_mapping.dtype == torch.int64 and slot_mapping.is_contiguous()
    for t, n in ((q_nope, "q_nope"), (q_pe, "q_pe"), (kv_c, "kv_c"), (k_pe, "k_pe")):
        _check_inner(t, n)
    assert cache.is_contiguous() and cache.dim() == 3 and cache.shape[2] == ROW
    if flags & FLAG_ROPE:
        assert positions is not None and positions.dtype == torch.int32
        assert cos_sin is not None and cos_sin.dtype == torch.float32 and cos_sin.is_contiguous()
    q_fp8 = bool(flags & FLAG_Q_FP8)
    q_out = torch.empty((T, H, ROW), dtype=torch.uint8 if q_fp8 else torch.bfloat16)
    status = ctypes.c_int32(0)
    fn = lib().mla_oracle_run if threads <= 1 else lib().mla_oracle_run_threads
    extra = () if threads <= 1 else (int(threads),)
    rc = fn(
        _ptr(q_nope), q_nope.stride(0), q_nope.stride(1),
        _ptr(q_pe), q_pe.stride(0), q_pe.stride(1),
        _ptr(kv_c), kv_c.stride(0),
        _ptr(k_pe), k_pe.stride(0),
        _ptr(slot_mapping),
        _ptr(positions), _ptr(cos_sin), cos_sin.shape[0] if cos_sin is not None else 0,
        _ptr(q_scale), _ptr(kv_scale),
        T, H, cache.shape[1], cache.shape[0], flags,
        _ptr(q_out), _ptr(cache), ctypes.addressof(status), *extra)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return q_out, status.value


def absorb_run(q_nope_c: torch.Tensor, w_uk: torch.Tensor, q_pe: torch.Tensor, flags: int,
               positions: Optional[torch.Tensor] = None, cos_sin: Optional[torch.Tensor] = None,
               q_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, int]:
    """Latent query rows from the absorption product (see mla_oracle_absorb_run):
    q_nope_c [T,H,128] bf16, w_uk [H,512,128] bf16 contiguous, q_pe [T,H,64] bf16.
    Returns (q_out [T,H,576] bf16 or uint8 e4m3, status)."""
    T, H = q_nope_c.shape[0], q_nope_c.shape[1]
    assert q_nope_c.dtype == torch.bfloat16 and q_nope_c.stride(-1) == 1 and q_nope_c.shape[2] == 128
    assert w_uk.dtype == torch.bfloat16 and w_uk.is_contiguous() and tuple(w_uk.shape) == (H, 512, 128)
    assert q_pe.dtype == torch.bfloat16 and q_pe.stride(-1) == 1
    q_fp8 = bool(flags & FLAG_Q_FP8)
    q_out = torch.empty((T, H, ROW), dtype=torch.uint8 if q_fp8 else torch.bfloat16)
    status = ctypes.c_int32(0)
    rc = lib().mla_oracle_absorb_run(
        _ptr(q_nope_c), q_nope_c.stride(0), q_nope_c.stride(1), _ptr(w_uk),
        _ptr(q_pe), q_pe.stride(0), q_pe.stride(1),
        _ptr(positions), _ptr(cos_sin), cos_sin.shape[0] if cos_sin is not None else 0,
        _ptr(q_scale), T, H, flags, _ptr(q_out), ctypes.addressof(status))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return q_out, status.value


def bf16_to_f32(h: int) -> float:
    return lib().mla_oracle_bf16_to_f32(h)


def f32_to_bf16(f: float) -> int:
    return lib().mla_oracle_f32_to_bf16(f)


def f32_to_e4m3(f: float) -> int:
    return lib().mla_oracle_f32_to_e4m3(f)
