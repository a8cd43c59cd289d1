"""Seeded synthetic inputs for the fused MLA decode epilogue.

This module only draws random numbers and lays out buffers; it holds none of
the epilogue's arithmetic, so the CUDA path and the CPU oracle can both be fed
from it.  Every tensor is created on the host with a seeded
``torch.Generator`` so that both sides see identical bytes; ``Workload.to``
moves a workload to a device keeping every view's strides and offsets.

The named workloads follow the shapes the vLLM PR #54896 report describes for
the Kimi-K3 MLA decode epilogue (576 = 512 nope + 64 pe latent width, one
cache row per token, a 64/65-token row-split boundary test with seed 3), plus
a decode sweep, a full-head prefill chunk with strided inputs and a large
batch behind a synthetic producer.
"""

from __future__ import annotations

import dataclasses
import functools
from typing import Dict, List, Optional

import numpy as np
import torch

NOPE = 512
PE = 64
ROW = NOPE + PE

FLAG_ROPE = 1
FLAG_Q_FP8 = 2
FLAG_KV_FP8 = 4
FLAG_PDL = 8

ROPE_BASE = 10000.0


@dataclasses.dataclass
class Workload:
    """One call's worth of inputs (host or device tensors)."""

    name: str
    T: int
    H: int
    block_size: int
    num_blocks: int
    flags: int
    q_nope: torch.Tensor            # bf16 [T, H, 512], inner stride 1 (may be a view)
    q_pe: torch.Tensor              # bf16 [T, H, 64]
    kv_c: torch.Tensor              # bf16 [T, 512]
    k_pe: torch.Tensor              # bf16 [T, 64]
    slot_mapping: torch.Tensor      # int64 [T]
    cache: torch.Tensor             # [num_blocks, block_size, 576]; bf16, or uint8 holding e4m3 bytes
    positions: Optional[torch.Tensor] = None   # int32 [T]
    cos_sin: Optional[torch.Tensor] = None     # fp32 [rope_rows, 64] = [cos_0..31 | sin_0..31]
    q_scale: Optional[torch.Tensor] = None     # fp32 [1]
    kv_scale: Optional[torch.Tensor] = None    # fp32 [1]
    producer: bool = False          # q_nope / q_pe are written on the device by a producer kernel
    recipe: str = ""

    @property
    def rows(self) -> int:
        return self.T * (self.H + 1)

    @property
    def q_fp8(self) -> bool:
        return bool(self.flags & FLAG_Q_FP8)

    @property
    def kv_fp8(self) -> bool:
        return bool(self.flags & FLAG_KV_FP8)

    def q_out_dtype(self) -> torch.dtype:
        return torch.uint8 if self.q_fp8 else torch.bfloat16

    def to(self, device) -> "Workload":
        """Copy to ``device``; views keep their strides and storage offsets."""
        out = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            out[f.name] = _move(v, device) if isinstance(v, torch.Tensor) else v
        return Workload(**out)

    def algorithmic_bytes(self) -> int:
        """Bytes the operation must move once: every input row read once,
        every output row written once, plus per-token indices, positions and
        table rows, plus the scales."""
        T, H = self.T, self.H
        q_el = 1 if self.q_fp8 else 2
        kv_el = 1 if self.kv_fp8 else 2
        rd = T * H * ROW * 2 + T * ROW * 2 + T * 8
        if self.flags & FLAG_ROPE:
            rd += T * (4 + PE * 4)
        if self.q_fp8:
            rd += 4
        if self.kv_fp8:
            rd += 4
        wr = T * H * ROW * q_el + T * ROW * kv_el
        return rd + wr


def _move(v: torch.Tensor, device) -> torch.Tensor:
    base = v._base if v._base is not None else v
    assert base._base is None
    nb = base.to(device)
    return nb.as_strided(v.size(), v.stride(), v.storage_offset())


@functools.lru_cache(maxsize=4)
def _rope_table_np(rows: int, base: float) -> np.ndarray:
    p = np.arange(rows, dtype=np.float64)[:, None]
    w = base ** (-np.arange(PE // 2, dtype=np.float64) / (PE // 2))
    ang = p * w[None, :]
    tab = np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
    tab.setflags(write=False)
    return tab


def rope_table(rows: int, base: float = ROPE_BASE) -> torch.Tensor:
    """fp32 [rows, 64] table: row p = [cos(p*w_0..31) | sin(p*w_0..31)],
    w_j = base^(-j/32) (rotate-half frequencies for 64 rotary dims),
    evaluated in double precision and rounded once to fp32 (a fresh copy
    per call)."""
    return torch.from_numpy(np.array(_rope_table_np(rows, base), copy=True))


def _randn_bf16(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def make(name: str, T: int, H: int, flags: int, *, seed: int, num_blocks: int,
         block_size: int = 64, std: float = 1.0, rope_rows: int = 32768,
         scale: float = 0.05, cache_fill: str = "zero",
         q_nope_row: int = NOPE, q_pe_row: int = PE, kv_c_row: int = NOPE,
         kv_c_offset: int = 0, k_pe_row: int = PE, producer: bool = False,
         recipe: str = "") -> Workload:
    """General seeded workload.

    Draw order (one generator): slots = randperm(num_blocks*block_size)[:T],
    then q_nope, q_pe, kv_c, k_pe (normal, ``std``), then positions uniform in
    [0, rope_rows), then the cache pre-fill (``zero`` or ``random`` bytes).
    ``*_row`` > natural width makes the input a view into a wider row-major
    buffer (inner stride 1), ``kv_c_offset`` its column offset.
    """
    g = torch.Generator().manual_seed(seed)
    cap = num_blocks * block_size
    if T > cap:
        raise ValueError("more tokens than cache slots")
    slots = torch.randperm(cap, generator=g)[:T].to(torch.int64).contiguous()

    qn_buf = _randn_bf16(g, (T, H, q_nope_row), std)
    q_nope = qn_buf[:, :, :NOPE]
    qp_buf = _randn_bf16(g, (T, H, q_pe_row), std)
    q_pe = qp_buf[:, :, :PE]
    kv_buf = _randn_bf16(g, (T, kv_c_row), std)
    kv_c = kv_buf[:, kv_c_offset:kv_c_offset + NOPE]
    kp_buf = _randn_bf16(g, (T, k_pe_row), std)
    k_pe = kp_buf[:, :PE]

    positions = cos_sin = None
    if flags & FLAG_ROPE:
        positions = torch.randint(0, rope_rows, (T,), generator=g, dtype=torch.int64).to(torch.int32)
        cos_sin = rope_table(rope_rows)
    q_scale = torch.tensor([scale], dtype=torch.float32) if flags & FLAG_Q_FP8 else None
    kv_scale = torch.tensor([scale], dtype=torch.float32) if flags & FLAG_KV_FP8 else None

    cdt = torch.uint8 if flags & FLAG_KV_FP8 else torch.bfloat16
    if cache_fill == "zero":
        cache = torch.zeros((num_blocks, block_size, ROW), dtype=cdt)
    elif cache_fill == "random":
        nbytes = num_blocks * block_size * ROW * (1 if cdt == torch.uint8 else 2)
        raw = torch.randint(0, 256, (nbytes,), generator=g, dtype=torch.uint8)
        cache = raw.view(cdt).view(num_blocks, block_size, ROW)
    else:
        raise ValueError(cache_fill)
    return Workload(name=name, T=T, H=H, block_size=block_size, num_blocks=num_blocks,
                    flags=flags, q_nope=q_nope, q_pe=q_pe, kv_c=kv_c, k_pe=k_pe,
                    slot_mapping=slots, cache=cache, positions=positions, cos_sin=cos_sin,
                    q_scale=q_scale, kv_scale=kv_scale, producer=producer, recipe=recipe)


# --- the named workloads -------------------------------------------------------------

DECODE_SWEEP_T = (1, 2, 4, 8, 16, 32, 64, 128, 256)
_ALL_FP8 = FLAG_ROPE | FLAG_Q_FP8 | FLAG_KV_FP8


def _recipes() -> Dict[str, dict]:
    r = {
        "decode_t4_h16": dict(
            T=4, H=16, flags=0, seed=0, num_blocks=1,
            recipe="T=4 H=16 bf16 N(0,1), no RoPE/FP8, zero cache [1,64,576], slots randperm(64)[:4], seed 0"),
    }
    for T in (64, 65):
        r[f"split_boundary_t{T}_h16_rope"] = dict(
            T=T, H=16, flags=FLAG_ROPE, seed=3, num_blocks=2, rope_rows=32768,
            recipe=f"T={T} H=16 bf16 N(0,1), RoPE (32768-row table, positions U[0,32768)), "
                   "zero cache [2,64,576], slots randperm(128)[:T], seed 3")
    for T in DECODE_SWEEP_T:
        r[f"decode_sweep_t{T}_h16_rope_fp8"] = dict(
            T=T, H=16, flags=_ALL_FP8, seed=0, num_blocks=4096, std=2.0, rope_rows=32768, scale=0.05,
            cache_fill="random",
            recipe=f"T={T} H=16 bf16 N(0,2), RoPE, Q/KV e4m3 scale 0.05, random-byte e4m3 cache "
                   "[4096,64,576], slots randperm(262144)[:T], seed 0")
    r["prefill_t1024_h128_strided"] = dict(
        T=1024, H=128, flags=FLAG_ROPE, seed=0, num_blocks=1024, rope_rows=32768, q_nope_row=640,
        kv_c_row=1536, kv_c_offset=512,
        recipe="T=1024 H=128 bf16 N(0,1), RoPE; q_nope = [1024,128,640][:,:,:512], "
               "kv_c = [1024,1536][:,512:1024]; zero cache [1024,64,576]; slots randperm(65536)[:1024], seed 0")
    r["batch_t8192_h16_pdl_fp8"] = dict(
        T=8192, H=16, flags=_ALL_FP8, seed=0, num_blocks=16384, rope_rows=131072, scale=0.05,
        cache_fill="random", producer=True,
        recipe="T=8192 H=16 bf16 N(0,1), RoPE (131072-row table), Q/KV e4m3 scale 0.05, random-byte e4m3 "
               "cache [16384,64,576], slots randperm(1048576)[:8192], q_nope/q_pe written by a producer "
               "kernel, epilogue launched with PDL, seed 0")
    return r


RECIPES = _recipes()


def named(name: str, seed_offset: int = 0) -> Workload:
    """The named workload; ``seed_offset`` draws fresh values of the same recipe."""
    kw = dict(RECIPES[name])
    kw["seed"] += seed_offset
    return make(name, **kw)


def decode_t4_h16() -> Workload:
    return named("decode_t4_h16")


def split_boundary(T: int) -> Workload:
    return named(f"split_boundary_t{T}_h16_rope")


def decode_sweep(T: int) -> Workload:
    return named(f"decode_sweep_t{T}_h16_rope_fp8")


def prefill_t1024_h128_strided() -> Workload:
    return named("prefill_t1024_h128_strided")


def batch_t8192_h16_pdl_fp8() -> Workload:
    return named("batch_t8192_h16_pdl_fp8")


def all_named() -> Dict[str, "callable"]:
    return {n: (lambda nn: (lambda: named(nn)))(n) for n in RECIPES}


def names() -> List[str]:
    return list(RECIPES.keys())


# --- the query side with the absorption product folded in ----------------------------

ABSORB_IN = 128  # nope head dim before absorption


@dataclasses.dataclass
class AbsorbWorkload:
    """Inputs of the absorbed-query rows: q_out[t,h] = enc([q_nope_c[t,h] @ W_UK[h]^T | rope(q_pe[t,h])])."""

    name: str
    T: int
    H: int
    flags: int
    q_nope_c: torch.Tensor          # bf16 [T, H, 128], inner stride 1 (may be a view)
    w_uk: torch.Tensor              # bf16 [H, 512, 128] contiguous (per head: 512 latent rows of 128)
    q_pe: torch.Tensor              # bf16 [T, H, 64]
    positions: Optional[torch.Tensor] = None
    cos_sin: Optional[torch.Tensor] = None
    q_scale: Optional[torch.Tensor] = None
    recipe: str = ""

    @property
    def q_fp8(self) -> bool:
        return bool(self.flags & FLAG_Q_FP8)

    def q_out_dtype(self) -> torch.dtype:
        return torch.uint8 if self.q_fp8 else torch.bfloat16

    def to(self, device) -> "AbsorbWorkload":
        out = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            out[f.name] = _move(v, device) if isinstance(v, torch.Tensor) else v
        return AbsorbWorkload(**out)

    def flops(self) -> int:
        return 2 * self.T * self.H * ABSORB_IN * NOPE

    def algorithmic_bytes(self) -> int:
        """Every input read once (the weights once per call), every output row written once."""
        T, H = self.T, self.H
        rd = T * H * ABSORB_IN * 2 + H * NOPE * ABSORB_IN * 2 + T * H * PE * 2
        if self.flags & FLAG_ROPE:
            rd += T * (4 + PE * 4)
        if self.q_fp8:
            rd += 4
        return rd + T * H * ROW * (1 if self.q_fp8 else 2)


def make_absorb(name: str, T: int, H: int, flags: int, *, seed: int, std: float = 1.0,
                rope_rows: int = 32768, scale: float = 0.05, q_nope_row: int = ABSORB_IN,
                recipe: str = "") -> AbsorbWorkload:
    """Seeded absorbed-query inputs.  Draw order: q_nope_c ~ N(0, std), W_UK ~
    N(0, 1/128) (so the 128-term products are O(std)), q_pe ~ N(0, std), then
    positions uniform in [0, rope_rows).  ``q_nope_row`` > 128 makes q_nope_c
    a view into a wider row-major buffer."""
    g = torch.Generator().manual_seed(seed)
    qc = _randn_bf16(g, (T, H, q_nope_row), std)[:, :, :ABSORB_IN]
    w = _randn_bf16(g, (H, NOPE, ABSORB_IN), 1.0 / (ABSORB_IN ** 0.5))
    qp = _randn_bf16(g, (T, H, PE), std)
    positions = cos_sin = None
    if flags & FLAG_ROPE:
        positions = torch.randint(0, rope_rows, (T,), generator=g, dtype=torch.int64).to(torch.int32)
        cos_sin = rope_table(rope_rows)
    q_scale = torch.tensor([scale], dtype=torch.float32) if flags & FLAG_Q_FP8 else None
    return AbsorbWorkload(name=name, T=T, H=H, flags=flags, q_nope_c=qc, w_uk=w, q_pe=qp, positions=positions,
                          cos_sin=cos_sin, q_scale=q_scale, recipe=recipe)


def absorb_t8192_h16_fp8() -> AbsorbWorkload:
    return make_absorb("absorb_t8192_h16_rope_fp8", 8192, 16, FLAG_ROPE | FLAG_Q_FP8, seed=0, rope_rows=131072,
                       recipe="T=8192 H=16: q_nope_c [8192,16,128] and q_pe bf16 N(0,1), W_UK [16,512,128] "
                              "N(0,1/128), RoPE (131072-row table), e4m3 scale 0.05, seed 0")


def absorb_t64_h16() -> AbsorbWorkload:
    return make_absorb("absorb_t64_h16_rope", 64, 16, FLAG_ROPE, seed=3,
                       recipe="T=64 H=16: q_nope_c [64,16,128] and q_pe bf16 N(0,1), W_UK [16,512,128] N(0,1/128), "
                              "RoPE (32768-row table), bf16 out, seed 3")
