"""The C-ABI library without a GPU: it loads, exports every entry point the
headers declare, agrees with the binding's constants, and rejects bad host
arguments before it makes any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

from mla_decode_attention_10_b200 import build as B
from mla_decode_attention_10_b200 import epilogue as E

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("mla_epilogue.h", "mla_harness.h", "mla_absorb.h")]


@pytest.fixture(scope="module")
def lib():
    B.build()
    return E.lib()


def _declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing else leaks out of the library
    ours = {n for n in exported if n.startswith("mla_")}
    assert ours == set(names)


def test_header_constants_match_binding():
    text = "".join(open(h).read() for h in HEADERS)
    defines = dict(re.findall(r"#define\s+(MLA_\w+)\s+(\d+)u?", text))
    enums = dict(re.findall(r"(MLA_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    for name, val in list(defines.items()) + list(enums.items()):
        assert getattr(E, name) == int(val), name


def test_oracle_and_binding_flags_agree():
    import oracle
    from mla_decode_attention_10_b200 import workloads as W
    assert oracle.FLAG_ROPE == W.FLAG_ROPE == E.MLA_FLAG_ROPE
    assert oracle.FLAG_Q_FP8 == W.FLAG_Q_FP8 == E.MLA_FLAG_Q_FP8
    assert oracle.FLAG_KV_FP8 == W.FLAG_KV_FP8 == E.MLA_FLAG_KV_FP8
    assert W.FLAG_PDL == E.MLA_FLAG_PDL
    assert oracle.STATUS_SLOT_RANGE == E.MLA_STATUS_SLOT_RANGE
    assert oracle.STATUS_POS_RANGE == E.MLA_STATUS_POS_RANGE


# Fake, well-aligned addresses: every call below must return before touching them.
A = 1 << 20


def _call(**kw):
    args = dict(q_nope=A, q_nope_stride_t=16 * 512, q_nope_stride_h=512, q_pe=A, q_pe_stride_t=16 * 64,
                q_pe_stride_h=64, kv_c=A, kv_c_stride_t=512, k_pe=A, k_pe_stride_t=64, slot_mapping=A,
                positions=A, cos_sin=A, rope_rows=8, q_scale=A, kv_scale=A, T=4, H=16, block_size=64,
                num_blocks=1, flags=0, q_out=A, cache=A, status=None, stream=None)
    args.update(kw)
    return E.mla_epilogue_launch(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(flags=1 << 31), E.MLA_ERR_UNSUPPORTED),
    (dict(flags=128), E.MLA_ERR_UNSUPPORTED),
    (dict(flags=E.MLA_FLAG_FORCE_SPLIT | E.MLA_FLAG_FORCE_ROWS), E.MLA_ERR_INVALID_ARG),
    (dict(flags=64), E.MLA_ERR_UNSUPPORTED),
    (dict(T=-1), E.MLA_ERR_INVALID_ARG),
    (dict(H=0), E.MLA_ERR_INVALID_ARG),
    (dict(H=65537), E.MLA_ERR_INVALID_ARG),
    (dict(block_size=0), E.MLA_ERR_INVALID_ARG),
    (dict(num_blocks=-1), E.MLA_ERR_INVALID_ARG),
    (dict(T=2 ** 31 // 17 + 1), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_pe=None), E.MLA_ERR_INVALID_ARG),
    (dict(kv_c=None), E.MLA_ERR_INVALID_ARG),
    (dict(k_pe=None), E.MLA_ERR_INVALID_ARG),
    (dict(slot_mapping=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_out=None), E.MLA_ERR_INVALID_ARG),
    (dict(cache=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_ROPE, positions=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_ROPE, cos_sin=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_ROPE, rope_rows=0), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_Q_FP8, q_scale=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_KV_FP8, kv_scale=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope_stride_t=-8), E.MLA_ERR_INVALID_ARG),
    (dict(k_pe_stride_t=-1), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope=A + 8), E.MLA_ERR_ALIGNMENT),
    (dict(kv_c=A + 2), E.MLA_ERR_ALIGNMENT),
    (dict(q_out=A + 4), E.MLA_ERR_ALIGNMENT),
    (dict(cache=A + 8), E.MLA_ERR_ALIGNMENT),
    (dict(q_nope_stride_t=16 * 512 + 4), E.MLA_ERR_ALIGNMENT),
    (dict(q_nope_stride_h=516), E.MLA_ERR_ALIGNMENT),
    (dict(kv_c_stride_t=520 + 2), E.MLA_ERR_ALIGNMENT),
    (dict(q_pe=A + 1), E.MLA_ERR_ALIGNMENT),
    (dict(k_pe=A + 1), E.MLA_ERR_ALIGNMENT),
    (dict(slot_mapping=A + 4), E.MLA_ERR_ALIGNMENT),
    (dict(flags=E.MLA_FLAG_ROPE, positions=A + 2), E.MLA_ERR_ALIGNMENT),
    (dict(flags=E.MLA_FLAG_ROPE, cos_sin=A + 2), E.MLA_ERR_ALIGNMENT),
    (dict(flags=E.MLA_FLAG_Q_FP8, q_scale=A + 1), E.MLA_ERR_ALIGNMENT),
    (dict(status=A + 2), E.MLA_ERR_ALIGNMENT),
])
def test_host_validation_rejects_before_any_cuda_call(lib, kw, code):
    assert _call(**kw) == code


def test_zero_tokens_launches_nothing(lib):
    # T == 0 returns OK even with null buffers: nothing is read or written
    assert _call(T=0, q_nope=None, q_pe=None, kv_c=None, k_pe=None, slot_mapping=None,
                 q_out=None, cache=None) == E.MLA_OK


def test_size_one_dimensions_skip_stride_checks(lib):
    # a stride of a size-1 dimension is never used, so it is not checked; the
    # call then proceeds to the device query, which fails without a GPU
    import torch
    rc = _call(T=1, H=1, q_nope_stride_t=3, q_nope_stride_h=5, kv_c_stride_t=7)
    assert rc in ((E.MLA_OK,) if torch.cuda.is_available() else (E.MLA_ERR_CUDA,))


def test_plan_modes_and_grids(lib):
    t = E.mla_epilogue_get_tuning()
    assert t.split_rows_per_block == 0  # automatic
    p = E.mla_epilogue_plan(64, 16, 0, sm_count=148)
    # 64 * 17 = 1088 rows over 148 SMs: 8 rows a block would do, the automatic choice stops at 4
    assert p.mode == E.MLA_MODE_SPLIT and p.rows_per_block == 4 and p.threads_per_block == 96 * 4
    assert p.blocks == 64 * 17 // 4
    # the default split threshold counts rows: 4608 = 271 tokens x 17 rows, rounded up
    assert t.split_max_rows == 4608
    assert E.mla_epilogue_plan(65, 16, 0, sm_count=148).mode == E.MLA_MODE_SPLIT
    assert E.mla_epilogue_plan(271, 16, 0, sm_count=148).mode == E.MLA_MODE_SPLIT
    assert E.mla_epilogue_plan(272, 16, 0, sm_count=148).mode == E.MLA_MODE_ROWS
    assert E.mla_epilogue_plan(32, 128, 0, sm_count=148).mode == E.MLA_MODE_SPLIT
    assert E.mla_epilogue_plan(36, 128, 0, sm_count=148).mode == E.MLA_MODE_ROWS
    p = E.mla_epilogue_plan(300, 16, 0, sm_count=148)
    assert p.mode == E.MLA_MODE_ROWS and p.threads_per_block % 32 == 0 and p.rows_per_block == 1
    assert p.blocks <= 148 * t.rows_blocks_per_sm
    assert E.mla_epilogue_plan(1, 16, E.MLA_FLAG_FORCE_ROWS, sm_count=148).mode == E.MLA_MODE_ROWS
    big = E.mla_epilogue_plan(8192, 16, E.MLA_FLAG_FORCE_SPLIT, sm_count=148)
    assert big.mode == E.MLA_MODE_SPLIT and big.rows_per_block == 4 and big.blocks == 8192 * 17 // 4
    with pytest.raises(E.MlaError):
        E.mla_epilogue_plan(0, 16, 0, sm_count=148)
    with pytest.raises(E.MlaError):
        E.mla_epilogue_plan(4, 16, E.MLA_FLAG_FORCE_SPLIT | E.MLA_FLAG_FORCE_ROWS, sm_count=148)


@pytest.mark.parametrize("T,H,rpb,blocks", [(1, 16, 1, 17), (1, 1, 1, 2), (1, 128, 1, 129), (4, 16, 1, 68),
                                            (16, 16, 2, 136), (2, 16, 1, 34), (32, 16, 4, 136), (64, 16, 4, 272)])
def test_decode_sizes_spread_over_the_sms(lib, T, H, rpb, blocks):
    """At decode sizes every SM gets a block before a block gets a second row:
    a single token runs one row per SM (the num_tokens == 1 case)."""
    p = E.mla_epilogue_plan(T, H, E.MLA_FLAG_ROPE, sm_count=148)
    assert p.mode == E.MLA_MODE_SPLIT
    assert (p.rows_per_block, p.threads_per_block, p.blocks) == (rpb, 96 * rpb, blocks)


def test_tuning_moves_the_threshold_and_clamps(lib):
    old = E.mla_epilogue_get_tuning()
    try:
        E.mla_epilogue_set_tuning(split_max_rows=64 * 17)
        assert E.mla_epilogue_plan(64, 16, 0, sm_count=148).mode == E.MLA_MODE_SPLIT
        assert E.mla_epilogue_plan(65, 16, 0, sm_count=148).mode == E.MLA_MODE_ROWS
        E.mla_epilogue_set_tuning(split_rows_per_block=99, rows_warps_per_block=99, rows_blocks_per_sm=99)
        t = E.mla_epilogue_get_tuning()
        assert t.split_rows_per_block == 10
        assert t.rows_warps_per_block == 8 and t.rows_blocks_per_sm == 5
        E.mla_epilogue_set_tuning(split_rows_per_block=3)
        p = E.mla_epilogue_plan(5, 16, 0, sm_count=148)
        assert p.rows_per_block == 3 and p.threads_per_block == 288 and p.blocks == 29
        E.mla_epilogue_set_tuning()  # all zero: unchanged
        assert E.mla_epilogue_get_tuning().split_max_rows == 64 * 17
        assert E.mla_epilogue_get_tuning().split_rows_per_block == 3
        E.mla_epilogue_set_tuning(split_rows_per_block=-1)  # back to automatic
        assert E.mla_epilogue_get_tuning().split_rows_per_block == 0
    finally:
        E.mla_epilogue_set_tuning(old.split_max_rows, old.split_rows_per_block or -1,
                                  old.rows_warps_per_block, old.rows_blocks_per_sm)


def test_status_strings(lib):
    for c in range(5):
        assert E.status_string(c).startswith("MLA_")
    assert "unknown" in E.status_string(99)


@pytest.mark.parametrize("kw,code", [
    (dict(flags=1), E.MLA_ERR_UNSUPPORTED),
    (dict(T=-1), E.MLA_ERR_INVALID_ARG),
    (dict(src_nope=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope=A + 8), E.MLA_ERR_ALIGNMENT),
    (dict(q_pe_stride_h=65), E.MLA_ERR_ALIGNMENT),
])
def test_harness_validation(lib, kw, code):
    args = dict(src_nope=A, src_pe=A, q_nope=A, q_nope_stride_t=16 * 512, q_nope_stride_h=512, q_pe=A,
                q_pe_stride_t=16 * 64, q_pe_stride_h=64, T=4, H=16, flags=0, stream=None)
    args.update(kw)
    assert E.mla_harness_produce(**args) == code
    assert E.mla_harness_empty(0, 32, 0, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_empty(1, 2048, 0, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_div_check(1.0, 0, 2 ** 32 + 1, A, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_div_check(1.0, 0, 1, None, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_bf16_scale_check(2 ** 32 - 4, 5, A, None) == E.MLA_ERR_INVALID_ARG
    pw = dict(src_nope=A, src_pe=A, q_nope=A, q_nope_stride_t=16 * 512, q_nope_stride_h=512, q_pe=A,
              q_pe_stride_t=16 * 64, q_pe_stride_h=64, weights=A, weight_bytes=1 << 20, sink=A, T=4, H=16, flags=0,
              stream=None)
    for kw, want in ((dict(weights=None), E.MLA_ERR_INVALID_ARG), (dict(sink=None), E.MLA_ERR_INVALID_ARG),
                     (dict(weight_bytes=-16), E.MLA_ERR_INVALID_ARG), (dict(weight_bytes=24), E.MLA_ERR_ALIGNMENT),
                     (dict(weights=A + 8), E.MLA_ERR_ALIGNMENT), (dict(sink=A + 2), E.MLA_ERR_ALIGNMENT),
                     (dict(flags=4), E.MLA_ERR_UNSUPPORTED), (dict(T=0, weight_bytes=0), E.MLA_OK)):
        assert E.mla_harness_produce_after_weights(**{**pw, **kw}) == want, kw
    assert E.mla_harness_bf16_scale_check(0, 1, None, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_bf16_scale_check(0, 1, A + 4, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_consume(A, A, A, 4, 16, 64, 64, A, None) == E.MLA_ERR_UNSUPPORTED
    assert E.mla_harness_consume(A, A, A, -1, 16, 64, 0, A, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_consume(None, A, A, 4, 16, 64, 0, A, None) == E.MLA_ERR_INVALID_ARG
    assert E.mla_harness_consume(A + 8, A, A, 4, 16, 64, 0, A, None) == E.MLA_ERR_ALIGNMENT
    assert E.mla_harness_consume(A, A, A, 0, 16, 64, 0, None, None) == E.MLA_OK


@pytest.mark.parametrize("kw,code", [
    (dict(flags=E.MLA_FLAG_KV_FP8), E.MLA_ERR_UNSUPPORTED),
    (dict(T=-1), E.MLA_ERR_INVALID_ARG),
    (dict(H=0), E.MLA_ERR_INVALID_ARG),
    (dict(H=65536), E.MLA_ERR_INVALID_ARG),
    (dict(H=1, T=2 ** 31 - 100), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope_c=None), E.MLA_ERR_INVALID_ARG),
    (dict(w_uk=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_out=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_ROPE, positions=None), E.MLA_ERR_INVALID_ARG),
    (dict(flags=E.MLA_FLAG_Q_FP8, q_scale=None), E.MLA_ERR_INVALID_ARG),
    (dict(q_nope_c=A + 8), E.MLA_ERR_ALIGNMENT),
    (dict(w_uk=A + 2), E.MLA_ERR_ALIGNMENT),
    (dict(q_out=A + 4), E.MLA_ERR_ALIGNMENT),
    (dict(q_nope_c_stride_h=132), E.MLA_ERR_ALIGNMENT),
    (dict(q_pe=A + 1), E.MLA_ERR_ALIGNMENT),
])
def test_absorb_validation(lib, kw, code):
    args = dict(q_nope_c=A, q_nope_c_stride_t=16 * 128, q_nope_c_stride_h=128, w_uk=A, q_pe=A,
                q_pe_stride_t=16 * 64, q_pe_stride_h=64, positions=A, cos_sin=A, rope_rows=8, q_scale=A,
                T=4, H=16, flags=0, q_out=A, status=None, stream=None)
    args.update(kw)
    assert E.mla_absorb_launch(**args) == code
    args.update(T=0, q_nope_c=None, w_uk=None, q_out=None)
    if code != E.MLA_ERR_UNSUPPORTED and kw.get("H", 1) >= 1 and kw.get("H", 1) < 65536 and kw.get("T", 0) >= 0:
        assert E.mla_absorb_launch(**args) == E.MLA_OK


def test_cuda_failures_are_recorded_for_every_launcher(lib):
    """A launcher that gets past its host checks and is refused by the CUDA
    runtime returns MLA_ERR_CUDA and records the runtime's error code, which
    mla_last_cuda_error() then reports (checked where no GPU is visible, so
    the first runtime call fails)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a process without a visible GPU")
    calls = {
        "mla_absorb_launch": lambda: E.mla_absorb_launch(A, 16 * 128, 128, A, A, 16 * 64, 64, A, A, 8, A, 4, 16,
                                                         E.MLA_FLAG_ROPE, A, None, None),
        "mla_epilogue_launch": lambda: _call(),
        "mla_epilogue_plan": lambda: E.lib().mla_epilogue_plan(4, 16, 0, 0, ctypes.byref(E.mla_plan())),
        "mla_harness_produce": lambda: E.mla_harness_produce(A, A, A, 16 * 512, 512, A, 16 * 64, 64, 4, 16, 0, None),
        "mla_harness_empty": lambda: E.mla_harness_empty(1, 32, 0, None),
        "mla_harness_produce_after_weights": lambda: E.mla_harness_produce_after_weights(
            A, A, A, 16 * 512, 512, A, 16 * 64, 64, A, 1 << 20, A, 4, 16, 0, None),
        "mla_harness_consume": lambda: E.mla_harness_consume(A, A, A, 4, 16, 64, 0, A, None),
    }
    for name, call in calls.items():
        E.lib().mla_last_cuda_error.restype = ctypes.c_int32
        assert call() == E.MLA_ERR_CUDA, name
        assert E.last_cuda_error() != 0, name


C_USER = r"""
#include "mla_epilogue.h"
#include "mla_absorb.h"
#include "mla_harness.h"
#include <stdio.h>
#include <string.h>

int main(void) {
  mla_plan plan;
  if (mla_epilogue_plan(64, 16, MLA_FLAG_ROPE, 148, &plan) != MLA_OK) return 1;
  /* T == 0: nothing to read or write, no CUDA call */
  if (mla_epilogue_launch(NULL, 0, 0, NULL, 0, 0, NULL, 0, NULL, 0, NULL, NULL, NULL, 0, NULL, NULL,
                          0, 16, 64, 1, 0, NULL, NULL, NULL, NULL) != MLA_OK) return 2;
  if (mla_absorb_launch(NULL, 0, 0, NULL, NULL, 0, 0, NULL, NULL, 0, NULL, 0, 1, 0, NULL, NULL, NULL) != MLA_OK) return 3;
  /* a bad argument is refused on the host */
  if (mla_absorb_launch(NULL, 0, 0, NULL, NULL, 0, 0, NULL, NULL, 0, NULL, 4, 0, 0, NULL, NULL, NULL)
      != MLA_ERR_INVALID_ARG) return 4;
  if (strlen(mla_status_string(MLA_ERR_ALIGNMENT)) == 0) return 5;
  printf("%d %lld\n", (int)plan.mode, (long long)plan.blocks);
  return 0;
}
"""


def test_headers_are_plain_c_and_link(lib, tmp_path):
    """A C11 program (no C++, no CUDA headers) includes every header, links
    the library and calls its host-side paths."""
    src = tmp_path / "use.c"
    src.write_text(C_USER)
    exe = tmp_path / "use"
    libdir = os.path.dirname(B.LIB)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-l:" + os.path.basename(B.LIB), "-o", str(exe)], check=True)
    env = dict(os.environ, LD_LIBRARY_PATH=libdir + os.pathsep + os.environ.get("LD_LIBRARY_PATH", ""))
    out = subprocess.run([str(exe)], env=env, capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    mode, blocks = out.stdout.split()
    assert int(mode) == E.MLA_MODE_SPLIT and int(blocks) > 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No silent fallback: with the library absent, the binding raises before
    any work is done, and the torch-level call does too."""
    monkeypatch.setattr(E, "_lib", None)
    monkeypatch.setattr(E, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="no CPU or PyTorch fallback"):
        E.lib()
    with pytest.raises(RuntimeError):
        E.status_string(0)
    with pytest.raises(RuntimeError):
        E.mla_epilogue_launch(0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 1, 1, 64, 1, 0, 0, 0, 0, 0)
