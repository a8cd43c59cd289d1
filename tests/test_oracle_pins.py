"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin ties the oracle to what the pages, the number formats or plain
mathematics fix, chosen so that a plausible slip (a dropped term, a wrong sign,
a swapped cos/sin half, the wrong pairing or frequency index, a bf16 rounding
before quantisation, the wrong tie rule) fails at least one of them:

* neither RoPE nor FP8: q == cat(ql_nope, q_pe) and cache[slots] == cat(kv_c, k_pe),
  the assertions of the boundary test in the vLLM PR #54896 report (section
  关键源码片段, test_decode_epilogue_row_split_boundary), with torch.cat as the
  library routine;
* cache rows that no token maps to stay bit-identical;
* RoPE with exactly representable rotations (identity at position 0, quarter
  and half turns, and (1, 2^-k) rows whose result is exact in fp32) against
  values computed exactly in rational arithmetic;
* RoPE undone by the inverse rotation, with angles computed independently in
  double precision from the position, recovers the input (pins direction,
  pairing (i, i+32), frequency index and which token's position is used);
* pairwise norms are preserved;
* e4m3: all 65536 bf16 bit patterns through the full entry point against
  torch's own float8_e4m3fn cast of the fp32 quotient (clamped to +-448 for the
  satfinite form), special values from the OCP FP8 definition, and the
  round-trip bound of half an e4m3 spacing;
* bf16 rounding against torch's float -> bfloat16 cast;
* out-of-range slots and positions set the status bits and write as defined.
"""

import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_10_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(w, flags=None, table=None, positions=None):
    return oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, w.cache,
                      w.flags if flags is None else flags,
                      positions=w.positions if positions is None else positions,
                      cos_sin=w.cos_sin if table is None else table,
                      q_scale=w.q_scale, kv_scale=w.kv_scale)


def _bits16(t):
    return t.contiguous().view(torch.int16)


def _cat_q(w):
    return torch.cat((w.q_nope, w.q_pe), dim=-1)


def _cat_kv(w):
    return torch.cat((w.kv_c, w.k_pe), dim=-1)


# ---------------------------------------------------------------------------
# concat / scatter: the page's own assertions
# ---------------------------------------------------------------------------

def test_page_boundary_case_is_concat_and_scatter():
    g = json.load(open(os.path.join(GOLDEN, "row_split_boundary.json")))
    assert g["nope_width"] + g["pe_width"] == g["latent_width"] == oracle.ROW
    for T in g["num_tokens"]:
        nb = (T + 63) // 64
        w = W.make("boundary", T, 16, 0, seed=g["seed"], num_blocks=nb)
        prefill = w.cache.clone()
        q, st = _run(w)
        assert st == 0
        assert torch.equal(_bits16(q), _bits16(_cat_q(w)))
        rows = w.cache.view(-1, 576)[w.slot_mapping]
        assert torch.equal(_bits16(rows), _bits16(_cat_kv(w)))
        mask = torch.ones(w.cache.view(-1, 576).shape[0], dtype=torch.bool)
        mask[w.slot_mapping] = False
        assert torch.equal(_bits16(w.cache.view(-1, 576)[mask]), _bits16(prefill.view(-1, 576)[mask]))


@pytest.mark.parametrize("T,H", [(1, 1), (3, 7), (17, 16), (9, 128)])
def test_concat_scatter_strided_views_random_prefill(T, H):
    w = W.make("strided", T, H, 0, seed=T * 100 + H, num_blocks=4, block_size=16,
               cache_fill="random", q_nope_row=640, q_pe_row=72, kv_c_row=1536,
               kv_c_offset=512, k_pe_row=80)
    if T > 1:
        assert not w.q_nope.is_contiguous() and not w.kv_c.is_contiguous()
    prefill = w.cache.clone()
    q, st = _run(w)
    assert st == 0
    assert torch.equal(_bits16(q), _bits16(_cat_q(w)))
    flat, pre = w.cache.view(-1, 576), prefill.view(-1, 576)
    assert torch.equal(_bits16(flat[w.slot_mapping]), _bits16(_cat_kv(w)))
    mask = torch.ones(flat.shape[0], dtype=torch.bool)
    mask[w.slot_mapping] = False
    assert torch.equal(_bits16(flat[mask]), _bits16(pre[mask]))


def test_untouched_fp8_cache_bytes_identical():
    w = W.decode_sweep(32)
    prefill = w.cache.clone()
    _, st = _run(w)
    assert st == 0
    flat, pre = w.cache.view(-1, 576), prefill.view(-1, 576)
    mask = torch.ones(flat.shape[0], dtype=torch.bool)
    mask[w.slot_mapping] = False
    assert torch.equal(flat[mask], pre[mask])
    assert not torch.equal(flat[w.slot_mapping], pre[w.slot_mapping])


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def _nonzero_inputs(w):
    for t in (w.q_nope, w.q_pe, w.kv_c, w.k_pe):
        t[t == 0] = 1.0
    return w


def test_rope_position_zero_is_identity():
    w = W.make("pos0", 5, 16, W.FLAG_ROPE, seed=11, num_blocks=1, rope_rows=64)
    w.positions.zero_()
    # cos(0) = 1 and sin(0) = 0 exactly in the table.
    assert torch.all(w.cos_sin[0, :32] == 1.0) and torch.all(w.cos_sin[0, 32:] == 0.0)
    q, st = _run(w)
    assert st == 0
    assert torch.equal(q.float(), _cat_q(w).float())  # by value: +-0 may change sign
    rows = w.cache.view(-1, 576)[w.slot_mapping]
    assert torch.equal(rows.float(), _cat_kv(w).float())


def _one_row_table(c, s):
    tab = torch.empty((1, 64), dtype=torch.float32)
    tab[0, :32] = torch.as_tensor(c, dtype=torch.float32)
    tab[0, 32:] = torch.as_tensor(s, dtype=torch.float32)
    return tab


@pytest.mark.parametrize("c,s,name", [(0.0, 1.0, "quarter"), (-1.0, 0.0, "half"),
                                      (0.0, -1.0, "minus_quarter")])
def test_rope_exact_rotations(c, s, name):
    w = _nonzero_inputs(W.make(name, 3, 4, W.FLAG_ROPE, seed=5, num_blocks=1, rope_rows=1))
    w.positions.zero_()
    q, st = _run(w, table=_one_row_table(c, s))
    assert st == 0
    x = _cat_q(w).float()
    a, b = x[..., 512:544], x[..., 544:576]
    # rotate-half: (a, b) -> (a c - b s, b c + a s), exact for these (c, s)
    exp = x.clone()
    exp[..., 512:544] = a * c - b * s
    exp[..., 544:576] = b * c + a * s
    assert torch.equal(q.float(), exp)
    assert torch.equal(q[..., :512], w.q_nope)  # nope half untouched, bit for bit


@pytest.mark.parametrize("k", [1, 5, 9])
def test_rope_exact_fp32_results_round_like_torch(k):
    """Rows (cos, sin) = (1, -2^-k): y_i = x_i + x_{i+32} 2^-k and
    y_{i+32} = x_{i+32} - x_i 2^-k.  The exact rational result rounded once to
    fp32 (numpy) is what the fp32 formula must give, since each product is
    exact; the bf16 output must be torch's bf16 cast of that, and the e4m3
    output torch's e4m3 cast of its fp32 quotient (no bf16 step in between)."""
    s = -(2.0 ** -k)
    for flags in (W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8):
        w = W.make("exact", 4, 8, flags, seed=40 + k, num_blocks=1, rope_rows=1, std=3.0,
                   scale=0.37)
        w.positions.zero_()
        q, st = _run(w, table=_one_row_table(1.0, s))
        assert st == 0
        x = _cat_q(w).double().numpy()
        y = x.copy()
        fs = Fraction(s)
        for idx in np.ndindex(*x.shape[:-1]):
            for i in range(32):
                fa, fb = Fraction(float(x[idx + (512 + i,)])), Fraction(float(x[idx + (544 + i,)]))
                ra = fa * 1 - fb * fs
                rb = fb * 1 + fa * fs
                # exact in double, so numpy's float32() rounds the exact value once
                assert Fraction(float(ra)) == ra and Fraction(float(rb)) == rb
                y[idx + (512 + i,)] = float(np.float32(float(ra)))
                y[idx + (544 + i,)] = float(np.float32(float(rb)))
        y32 = torch.from_numpy(y.astype(np.float32))
        if flags & W.FLAG_Q_FP8:
            sc = torch.full_like(y32, 0.37)
            exp = (y32 / sc).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
            assert torch.equal(q, exp)
        else:
            exp = y32.to(torch.bfloat16)
            assert torch.equal(_bits16(q), _bits16(exp))


def test_rope_inverse_rotation_recovers_input():
    w = W.make("inv", 6, 16, W.FLAG_ROPE, seed=21, num_blocks=1, rope_rows=32768)
    q, st = _run(w)
    assert st == 0
    pos = w.positions.double().numpy()
    freq = 10000.0 ** (-np.arange(32, dtype=np.float64) / 32.0)
    th = pos[:, None] * freq[None, :]                    # [T, 32], independent of the table
    c, s = np.cos(th)[:, None, :], np.sin(th)[:, None, :]
    y = q.double().numpy()
    ya, yb = y[..., 512:544], y[..., 544:576]
    # inverse of (a, b) -> (a c - b s, b c + a s) is (u, v) -> (u c + v s, v c - u s)
    xa = ya * c + yb * s
    xb = yb * c - ya * s
    x = _cat_q(w).double().numpy()
    tol = 2.0 ** -7 * (np.abs(ya) + np.abs(yb)) + 1e-6
    assert np.all(np.abs(xa - x[..., 512:544]) <= tol)
    assert np.all(np.abs(xb - x[..., 544:576]) <= tol)
    # the cache row of each token rotates by that token's own angle
    kv = w.cache.view(-1, 576)[w.slot_mapping].double().numpy()
    ka, kb = kv[:, 512:544], kv[:, 544:576]
    c1, s1 = np.cos(th), np.sin(th)
    xk = _cat_kv(w).double().numpy()
    tolk = 2.0 ** -7 * (np.abs(ka) + np.abs(kb)) + 1e-6
    assert np.all(np.abs(ka * c1 + kb * s1 - xk[:, 512:544]) <= tolk)
    assert np.all(np.abs(kb * c1 - ka * s1 - xk[:, 544:576]) <= tolk)
    # and the rotation is not the identity for these positions
    assert not torch.equal(q[..., 512:].float(), _cat_q(w)[..., 512:].float())


def test_rope_preserves_pair_norms():
    w = W.make("norm", 8, 16, W.FLAG_ROPE, seed=22, num_blocks=1, rope_rows=32768)
    q, _ = _run(w)
    y = q.double().numpy()
    x = _cat_q(w).double().numpy()
    ny = np.hypot(y[..., 512:544], y[..., 544:576])
    nx = np.hypot(x[..., 512:544], x[..., 544:576])
    assert np.all(np.abs(ny - nx) <= 2.0 ** -7 * nx + 1e-6)


def _bf16_ulp(v):
    v = abs(v)
    if v == 0:
        return 2.0 ** -133
    e = math.floor(math.log2(v))
    return 2.0 ** (max(e, -126) - 7)


def test_rope_within_one_bf16_ulp_of_double():
    w = W.make("dbl", 4, 16, W.FLAG_ROPE, seed=23, num_blocks=1, rope_rows=32768)
    q, _ = _run(w)
    tab = w.cos_sin.double().numpy()[w.positions.long().numpy()]  # same fp32 table values
    c, s = tab[:, None, :32], tab[:, None, 32:]
    x = _cat_q(w).double().numpy()
    a, b = x[..., 512:544], x[..., 544:576]
    ref = np.concatenate([a * c - b * s, b * c + a * s], axis=-1)
    got = q[..., 512:].double().numpy()
    ulp = np.vectorize(_bf16_ulp)(ref)
    assert np.all(np.abs(got - ref) <= ulp)


# ---------------------------------------------------------------------------
# e4m3 and bf16 encoders
# ---------------------------------------------------------------------------

def _all_bf16_patterns_no_nan():
    u = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    b = u.view(torch.bfloat16)
    nan = torch.isnan(b.float())
    b = b.clone()
    b[nan] = 1.0  # NaN inputs are compared as "both NaN" elsewhere
    return b


# 7.0 and 0.9 are scales for which x * (1/scale) and x / scale give different
# e4m3 bytes for some bf16 x (60 and 30 of them), so a reciprocal-multiply fails here.
@pytest.mark.parametrize("scale", [0.05, 1.0, 0.37, 3.0, 7.0, 0.9])
def test_e4m3_exhaustive_bf16_through_entry_point(scale):
    """All bf16 patterns in q_nope (8 x 16 x 512 = 65536), flags Q_FP8|KV_FP8:
    each output byte equals torch's e4m3 cast of the fp32 quotient x / scale,
    clamped to +-448 (the satfinite form; torch alone would produce NaN)."""
    vals = _all_bf16_patterns_no_nan()
    w = W.make("e4m3x", 8, 16, W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=1, num_blocks=1,
               block_size=16, scale=scale)
    w.q_nope.copy_(vals.view(8, 16, 512))
    w.kv_c.copy_(vals[:8 * 512].view(8, 512))
    q, st = _run(w)
    assert st == 0
    x = _cat_q(w).float()
    exp = (x / torch.full_like(x, scale)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(q, exp)
    kx = _cat_kv(w).float()
    kexp = (kx / torch.full_like(kx, scale)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(w.cache.view(-1, 576)[w.slot_mapping], kexp)


def test_e4m3_special_values_from_format_definition():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_special_values.json")))
    for v, code in g["cases"]:
        assert oracle.f32_to_e4m3(float(v)) == int(code, 16), (v, code)
    assert oracle.f32_to_e4m3(float("nan")) & 0x7F == 0x7F


def test_e4m3_round_trip_within_half_spacing():
    w = W.make("rt", 16, 16, W.FLAG_Q_FP8, seed=31, num_blocks=1, std=2.0, scale=0.05)
    q, _ = _run(w)
    dec = q.view(torch.float8_e4m3fn).double()
    x = _cat_q(w).double() / float(np.float32(0.05))
    sat = x.abs() >= 448
    assert torch.all(dec[sat].abs() == 448)
    xs, ds = x[~sat], dec[~sat]
    # spacing of the e4m3 grid around |x|: 2^(e-3) for normals (e >= -6), 2^-9 below
    e = torch.floor(torch.log2(xs.abs().clamp_min(2.0 ** -6)))
    half = 2.0 ** (e - 3) / 2
    assert torch.all((ds - xs).abs() <= half * (1 + 1e-6))


def test_bf16_encoder_matches_torch_cast():
    g = torch.Generator().manual_seed(7)
    u = torch.randint(-2 ** 31, 2 ** 31 - 1, (40000,), generator=g, dtype=torch.int64).to(torch.int32)
    f = u.view(torch.float32)
    f = f[~torch.isnan(f)]
    # ties: low 16 bits exactly 0x8000, with both parities of the kept bit
    ties = (torch.arange(2000, dtype=torch.int32) * 65536 + 0x3f800000 + 0x8000).view(torch.float32)
    allf = torch.cat([f, ties, torch.tensor([0.0, -0.0, float("inf"), -float("inf"),
                                             3.4028234663852886e38, 1e-45, -1e-45])])
    exp = allf.to(torch.bfloat16).view(torch.int16).tolist()
    for v, e in zip(allf.tolist(), exp):
        got = oracle.f32_to_bf16(v)
        assert got == (e & 0xFFFF), (v, hex(got), hex(e & 0xFFFF))


def test_copy_path_preserves_every_bf16_pattern():
    """Without RoPE or FP8 the row is a copy: all 65536 bf16 bit patterns,
    NaN payloads (quiet and signalling) included, come out unchanged."""
    u = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    w = W.make("copy", 8, 16, 0, seed=2, num_blocks=1, block_size=16)
    w.q_nope.view(torch.int16).copy_(u.view(8, 16, 512))
    w.kv_c.view(torch.int16).copy_(u[-8 * 512:].view(8, 512))
    q, st = _run(w)
    assert st == 0
    assert torch.equal(_bits16(q), _bits16(_cat_q(w)))
    assert torch.equal(_bits16(w.cache.view(-1, 576)[w.slot_mapping]), _bits16(_cat_kv(w)))


# ---------------------------------------------------------------------------
# slot and position rules, status bits
# ---------------------------------------------------------------------------

def test_slot_and_position_rules():
    w = W.make("rules", 5, 3, W.FLAG_ROPE, seed=9, num_blocks=2, block_size=8,
               cache_fill="random", rope_rows=16)
    w.slot_mapping[1] = -1                   # skipped, no status
    w.slot_mapping[2] = 16                   # == capacity: skipped, status bit 1
    w.positions[3] = 16                      # == rope_rows: unrotated, status bit 2
    w.positions[4] = -5                      # negative: unrotated, status bit 2
    prefill = w.cache.clone()
    q, st = _run(w)
    assert st == oracle.STATUS_SLOT_RANGE | oracle.STATUS_POS_RANGE
    flat, pre = w.cache.view(-1, 576), prefill.view(-1, 576)
    written = {int(w.slot_mapping[t]) for t in (0, 3, 4)}
    for r in range(flat.shape[0]):
        if r not in written:
            assert torch.equal(_bits16(flat[r]), _bits16(pre[r]))
    for t in (3, 4):
        assert torch.equal(_bits16(q[t]), _bits16(_cat_q(w)[t]))
        assert torch.equal(_bits16(flat[int(w.slot_mapping[t])]), _bits16(_cat_kv(w)[t]))
    # in-range tokens are rotated
    assert not torch.equal(q[0, :, 512:].float(), _cat_q(w)[0, :, 512:].float())


def test_zero_tokens_is_a_no_op():
    w = W.make("empty", 0, 4, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=1,
               num_blocks=1, cache_fill="random", rope_rows=8)
    pre = w.cache.clone()
    q, st = _run(w)
    assert q.shape == (0, 4, 576) and st == 0
    assert torch.equal(w.cache, pre)


# ---------------------------------------------------------------------------
# brute force on tiny inputs, every flag combination
# ---------------------------------------------------------------------------

def _torch_restatement(w, flags):
    """Independent statement with torch CPU ops, one fp32 operation at a time."""
    def row(x, fp8, scale):
        x = x.float()
        y = x.clone()
        if flags & W.FLAG_ROPE:
            tab = w.cos_sin[w.positions.long()]
            c, s = tab[:, :32], tab[:, 32:]
            if x.dim() == 3:
                c, s = c[:, None, :], s[:, None, :]
            a, b = x[..., 512:544], x[..., 544:576]
            y[..., 512:544] = torch.sub(torch.mul(a, c), torch.mul(b, s))
            y[..., 544:576] = torch.add(torch.mul(b, c), torch.mul(a, s))
        if fp8:
            return (y / torch.full_like(y, float(scale))).clamp(-448, 448).to(
                torch.float8_e4m3fn).view(torch.uint8)
        return y.to(torch.bfloat16)
    q = row(_cat_q(w), flags & W.FLAG_Q_FP8, w.q_scale[0] if w.q_scale is not None else 1)
    kv = row(_cat_kv(w), flags & W.FLAG_KV_FP8, w.kv_scale[0] if w.kv_scale is not None else 1)
    return q, kv


@pytest.mark.parametrize("flags", list(range(8)))
@pytest.mark.parametrize("T", [1, 2, 4])
def test_brute_force_tiny_all_flags(flags, T):
    w = W.make("tiny", T, 3, flags, seed=1000 + 8 * T + flags, num_blocks=2, block_size=4,
               std=2.0, rope_rows=4096, scale=0.05, cache_fill="random")
    q, st = _run(w)
    assert st == 0
    eq, ekv = _torch_restatement(w, flags)
    if flags & W.FLAG_Q_FP8:
        assert torch.equal(q, eq)
    else:
        assert torch.equal(_bits16(q), _bits16(eq))
    rows = w.cache.view(-1, 576)[w.slot_mapping]
    if flags & W.FLAG_KV_FP8:
        assert torch.equal(rows, ekv)
    else:
        assert torch.equal(_bits16(rows), _bits16(ekv))


@pytest.mark.parametrize("flags", [0, W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8])
@pytest.mark.parametrize("threads", [2, 3, 64])
def test_threaded_driver_equals_single_thread(flags, threads):
    """The all-cores baseline runs the same per-token function on token
    slices: results and status bits equal the single-threaded run."""
    w = W.make("thr", 37, 5, flags, seed=41, num_blocks=4, block_size=16)
    cache1, cache2 = w.cache.clone(), w.cache.clone()
    if flags & W.FLAG_ROPE:
        w.positions[::9] = -3  # a status bit from some slices
    q1, s1 = oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, cache1, flags, positions=w.positions,
                        cos_sin=w.cos_sin, q_scale=w.q_scale, kv_scale=w.kv_scale)
    q2, s2 = oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, cache2, flags, positions=w.positions,
                        cos_sin=w.cos_sin, q_scale=w.q_scale, kv_scale=w.kv_scale, threads=threads)
    assert s1 == s2
    assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(cache1.view(torch.uint8), cache2.view(torch.uint8))


def test_query_and_cache_rows_use_their_own_scale():
    """q_scale 0.5, kv_scale 2.0, constant inputs: every query byte is the
    e4m3 code of 1 / 0.5 = 2 (0x40) and every cache byte that of 2 / 2 = 1
    (0x38), from the format's definition (bias 7, three mantissa bits).
    Swapping the two scales, or using one for both, changes one of them."""
    w = W.make("scales", 3, 2, W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=8, num_blocks=1, block_size=16)
    w.q_nope.fill_(1.0)
    w.q_pe.fill_(1.0)
    w.kv_c.fill_(2.0)
    w.k_pe.fill_(2.0)
    w.q_scale = torch.tensor([0.5], dtype=torch.float32)
    w.kv_scale = torch.tensor([2.0], dtype=torch.float32)
    cache = w.cache.clone()
    q, st = oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, cache, w.flags,
                       q_scale=w.q_scale, kv_scale=w.kv_scale)
    assert st == 0
    assert torch.all(q == 0x40)
    rows = cache.view(-1, 576)[w.slot_mapping]
    assert torch.all(rows == 0x38)
