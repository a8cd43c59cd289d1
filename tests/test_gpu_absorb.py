"""GPU parity of the absorbed query rows (tcgen05 tensor cores) against
independent references.

The 512 nope values accumulate in fp32 on the tensor cores in an order the
hardware chooses, so they are compared with the exact product (float64
numpy) within the bound the arithmetic gives: half an output step (bf16 ulp,
or e4m3 spacing of x / scale) plus the fp32 accumulation error over 128
terms, 128 * 2^-24 * sum |a_k b_k| (divided by the scale for e4m3).  The 64
rotary values do not touch the tensor cores and are compared with the
oracle bit for bit; so is everything where the oracle agrees (the vast
majority of the nope values).
"""

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_10_b200 import epilogue as E
from mla_decode_attention_10_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _gpu(w, extra=0, d=None):
    d = w.to("cuda") if d is None else d
    q = torch.full((w.T, w.H, 576), 0x7F if w.q_fp8 else 0, dtype=torch.uint8 if w.q_fp8 else torch.bfloat16,
                   device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = E.launch_absorb_workload(d, q, status=st, extra_flags=extra)
    assert rc == E.MLA_OK, E.status_string(rc)
    torch.cuda.synchronize()
    return q.cpu(), int(st.item())


def _spacing_e4m3(q):
    a = np.abs(q)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 2.0 ** (e - 3)


def _check(w, q_gpu, st_gpu):
    q_or, st_or = oracle.absorb_run(w.q_nope_c, w.w_uk, w.q_pe, w.flags, positions=w.positions,
                                    cos_sin=w.cos_sin, q_scale=w.q_scale)
    assert st_gpu == st_or
    # rotary half: bit for bit
    if w.q_fp8:
        assert torch.equal(q_gpu[..., 512:], q_or[..., 512:])
    else:
        assert torch.equal(q_gpu[..., 512:].view(torch.int16), q_or[..., 512:].view(torch.int16))
    # nope half: within the arithmetic's bound of the exact product
    a = w.q_nope_c.double().numpy()
    b = w.w_uk.double().numpy()
    exact = np.einsum("thk,hjk->thj", a, b)
    mag = np.einsum("thk,hjk->thj", np.abs(a), np.abs(b))
    acc = 128 * 2.0 ** -24 * mag
    if w.q_fp8:
        s = float(w.q_scale[0])
        got = q_gpu[..., :512].view(torch.float8_e4m3fn).double().numpy()
        qx = exact / s
        sat = np.abs(qx) >= 448 + acc / s
        assert np.all(np.abs(got[sat]) == 448)
        bound = _spacing_e4m3(qx) / 2 + acc / s + 1e-12
        assert np.all(np.abs(got - qx)[~sat] <= bound[~sat])
        same = (q_gpu[..., :512] == q_or[..., :512]).float().mean().item()
    else:
        got = q_gpu[..., :512].float().double().numpy()
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -126))) - 7)
        assert np.all(np.abs(got - exact) <= ulp / 2 + acc + 1e-30)
        same = (q_gpu[..., :512].view(torch.int16) == q_or[..., :512].view(torch.int16)).float().mean().item()
    assert same > 0.97, same


@pytest.mark.parametrize("flags", [0, W.FLAG_ROPE, W.FLAG_Q_FP8, W.FLAG_ROPE | W.FLAG_Q_FP8])
@pytest.mark.parametrize("T,H", [(1, 1), (5, 3), (128, 2), (130, 4), (300, 16)])
def test_absorbed_rows_match(flags, T, H):
    w = W.make_absorb("abs", T, H, flags, seed=T * 7 + H + flags, rope_rows=4096, scale=0.05, q_nope_row=136)
    q, st = _gpu(w)
    _check(w, q, st)


def test_absorbed_rows_named_workloads():
    for w in (W.absorb_t64_h16(), W.absorb_t8192_h16_fp8()):
        q, st = _gpu(w)
        _check(w, q, st)


@pytest.mark.parametrize("flags", [W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8])
@pytest.mark.parametrize("T,H", [(600, 40), (200, 80)])
def test_absorbed_rows_tile_assignments(flags, T, H):
    """(600, 40): one CTA per (head, half) takes the first token tiles, the
    other CTAs share out the last two of every pair, several pairs each (so
    their weights change between tiles).  (200, 80): more (head, half) pairs
    than SMs, so CTAs take contiguous runs of tiles."""
    w = W.make_absorb("assign", T, H, flags, seed=T + H + flags, rope_rows=4096, scale=0.05)
    q, st = _gpu(w)
    _check(w, q, st)


def test_identity_weights_copy_bit_for_bit():
    w = W.make_absorb("id", 200, 4, W.FLAG_ROPE, seed=5, rope_rows=512)
    w.w_uk.zero_()
    for h in range(4):
        w.w_uk[h, :128, :] = torch.eye(128, dtype=torch.bfloat16)
    q, _ = _gpu(w)
    assert torch.equal(q[..., :128].view(torch.int16), w.q_nope_c.contiguous().view(torch.int16))
    assert torch.all(q[..., 128:512].float() == 0)


def test_absorbed_rows_behind_producer_with_pdl():
    """q_nope_c written by a kernel just before (a device copy standing in for
    the projection), the absorbed rows launched as its programmatic dependent."""
    w = W.make_absorb("pdl", 777, 8, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=9, rope_rows=4096, scale=0.05)
    d = w.to("cuda")
    src = d.q_nope_c.clone()
    d.q_nope_c.fill_(float("nan"))
    q = torch.empty((w.T, w.H, 576), dtype=torch.uint8, device="cuda")
    d.q_nope_c.copy_(src)
    rc = E.launch_absorb_workload(d, q, extra_flags=E.MLA_FLAG_PDL)
    assert rc == E.MLA_OK
    torch.cuda.synchronize()
    _check(w, q.cpu(), 0)


@pytest.mark.parametrize("flags", [W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8])
def test_absorbed_rows_positions_out_of_range(flags):
    """Positions outside the table leave those tokens' pe values unrotated and
    set the status bit; 37 tokens leave a ragged last group of rows."""
    w = W.make_absorb("oor", 37, 3, flags, seed=11, rope_rows=64, scale=0.05)
    w.positions[::5] = -1
    w.positions[3::7] = 64
    q, st = _gpu(w)
    assert st == E.MLA_STATUS_POS_RANGE
    _check(w, q, st)


@pytest.mark.parametrize("layout", ["pe_offset", "table_offset", "pe_stride_68", "pe_stride_72"])
def test_absorbed_rows_unaligned_pe_and_table(layout):
    """q_pe or the cos/sin table off the 16-byte grid (2- or 4-byte aligned,
    or a row stride that is not a multiple of 8 elements) take the scalar
    load path; a stride of 72 keeps the vector path on a strided view."""
    w = W.make_absorb("ua", 70, 3, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=21, rope_rows=256, scale=0.05)
    d = w.to("cuda")
    if layout == "pe_offset":
        buf = torch.empty(w.T * w.H * 64 + 1, dtype=torch.bfloat16, device="cuda")
        buf[1:].copy_(d.q_pe.reshape(-1))
        d.q_pe = buf[1:].view(w.T, w.H, 64)
    elif layout == "table_offset":
        buf = torch.empty(d.cos_sin.numel() + 1, dtype=torch.float32, device="cuda")
        buf[1:].copy_(d.cos_sin.reshape(-1))
        d.cos_sin = buf[1:].view(d.cos_sin.shape)
    else:
        width = int(layout.rsplit("_", 1)[1])
        buf = torch.zeros(w.T, w.H, width, dtype=torch.bfloat16, device="cuda")
        buf[:, :, :64].copy_(d.q_pe)
        d.q_pe = buf[:, :, :64]
    q, st = _gpu(w, d=d)
    _check(w, q, st)
    w_bf16 = W.make_absorb("ua16", 70, 3, W.FLAG_ROPE, seed=22, rope_rows=256)
    d16 = w_bf16.to("cuda")
    buf = torch.empty(w_bf16.T * w_bf16.H * 64 + 1, dtype=torch.bfloat16, device="cuda")
    buf[1:].copy_(d16.q_pe.reshape(-1))
    d16.q_pe = buf[1:].view(w_bf16.T, w_bf16.H, 64)
    q, st = _gpu(w_bf16, d=d16)
    _check(w_bf16, q, st)


def test_absorbed_rows_many_heads_reload_weights():
    """T=100, H=200: 400 one-tile (head, column half) groups over at most 148
    persistent CTAs, so a CTA loads new weights for two or three successive
    groups (the weight buffer's empty/full phases alternate)."""
    w = W.make_absorb("heads", 100, 200, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=17, rope_rows=4096, scale=0.05)
    q, st = _gpu(w)
    _check(w, q, st)
