"""Pins for the oracle of the absorbed query rows (the query side of the
epilogue with the absorption product folded in)."""

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_10_b200 import workloads as W


def _bits(t):
    t = t.contiguous()
    return t.view(torch.int16) if t.element_size() == 2 else t


def _run(w):
    return oracle.absorb_run(w.q_nope_c, w.w_uk, w.q_pe, w.flags, positions=w.positions, cos_sin=w.cos_sin,
                             q_scale=w.q_scale)


def test_identity_weights_copy_the_input():
    """W_UK[h] = [I_128; 0]: the first 128 latent values are the input, bit
    for bit, the other 384 are zero."""
    w = W.make_absorb("id", 5, 3, 0, seed=1, q_nope_row=136)
    w.w_uk.zero_()
    for h in range(3):
        w.w_uk[h, :128, :] = torch.eye(128, dtype=torch.bfloat16)
    q, st = _run(w)
    assert st == 0
    assert torch.equal(_bits(q[..., :128]), _bits(w.q_nope_c))
    assert torch.all(q[..., 128:512].float() == 0)
    assert torch.equal(_bits(q[..., 512:]), _bits(w.q_pe))


def test_permutation_weights_select_one_input_each():
    """W_UK[h, j, k] = 1 exactly when k = (5 j + 3 h) mod 128: latent value j
    of head h is input element (5 j + 3 h) mod 128 of the same token and
    head, bit for bit.  The map differs per head and is not symmetric in
    (j, k), so a transposed weight index, a wrong head or a wrong token
    fails."""
    T, H = 4, 3
    w = W.make_absorb("perm", T, H, 0, seed=2, q_nope_row=136)
    w.w_uk.zero_()
    for h in range(H):
        for j in range(512):
            w.w_uk[h, j, (5 * j + 3 * h) % 128] = 1.0
    q, st = _run(w)
    assert st == 0
    src = w.q_nope_c.contiguous()
    for h in range(H):
        idx = torch.tensor([(5 * j + 3 * h) % 128 for j in range(512)])
        assert torch.equal(_bits(q[:, h, :512]), _bits(src[:, h, idx]))


def test_one_hot_queries_read_one_weight_column():
    """q_nope_c[t, h] = e_k with k = (7 t + h) mod 128: latent value j is
    W_UK[h, j, k], bit for bit (one exact product, one term)."""
    T, H = 3, 2
    w = W.make_absorb("onehot", T, H, 0, seed=4)
    w.q_nope_c.zero_()
    for t in range(T):
        for h in range(H):
            w.q_nope_c[t, h, (7 * t + h) % 128] = 1.0
    q, st = _run(w)
    assert st == 0
    for t in range(T):
        for h in range(H):
            assert torch.equal(_bits(q[t, h, :512]), _bits(w.w_uk[h, :, (7 * t + h) % 128]))


def test_exact_sums_cancellation_and_ties():
    """Sums whose exact value is known: 2^24 + 1 - 2^24 = 1 (lost by fp32
    accumulation in that order); 1 + 2^-9 + 2^-9 = 1 + 2^-8, a bf16 tie
    that rounds to even (1.0); 1 + 2^-9 + 2^-9 + 2^-20, just above the tie
    (1 + 2^-7).  The latent values are rounded once, from the exact sum."""
    w = W.make_absorb("sums", 1, 1, 0, seed=6)
    w.q_nope_c.zero_()
    w.w_uk.zero_()
    q_vals = {0: 2.0 ** 24, 1: 1.0, 2: -(2.0 ** 24), 3: 1.0, 4: 2.0 ** -9, 5: 2.0 ** -9, 6: 2.0 ** -20}
    for k, v in q_vals.items():
        w.q_nope_c[0, 0, k] = v
    for k in (0, 1, 2):
        w.w_uk[0, 0, k] = 1.0          # latent 0: cancellation
    for k in (3, 4, 5):
        w.w_uk[0, 1, k] = 1.0          # latent 1: exactly on the tie
    for k in (3, 4, 5, 6):
        w.w_uk[0, 2, k] = 1.0          # latent 2: just above it
    q, st = _run(w)
    assert st == 0
    got = q[0, 0, :3].float().tolist()
    assert got == [1.0, 1.0, 1.0 + 2.0 ** -7], got
    assert torch.all(q[0, 0, 3:512].float() == 0)


@pytest.mark.parametrize("flags", [0, W.FLAG_Q_FP8])
def test_small_integer_products_match_numpy(flags):
    """Inputs that are small integers times 2^-3 make every sum exact in
    double, so the oracle must equal numpy's float64 matmul rounded to fp32,
    then cast by torch to bf16 (or divided by the scale and cast to e4m3)."""
    g = torch.Generator().manual_seed(4)
    w = W.make_absorb("ints", 6, 4, flags, seed=2, scale=0.37)
    w.q_nope_c.copy_((torch.randint(-8, 9, w.q_nope_c.shape, generator=g).float() / 8).to(torch.bfloat16))
    w.w_uk.copy_((torch.randint(-8, 9, w.w_uk.shape, generator=g).float() / 8).to(torch.bfloat16))
    q, _ = _run(w)
    a = w.q_nope_c.double().numpy()
    b = w.w_uk.double().numpy()
    ql = np.einsum("thk,hjk->thj", a, b)
    ql32 = torch.from_numpy(ql.astype(np.float32))
    if flags & W.FLAG_Q_FP8:
        exp = (ql32 / torch.full_like(ql32, 0.37)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(q[..., :512], exp)
    else:
        assert torch.equal(_bits(q[..., :512]), _bits(ql32.to(torch.bfloat16)))


@pytest.mark.parametrize("flags", [W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8])
def test_pe_half_equals_the_epilogue_oracle(flags):
    """The rotated pe half of an absorbed row is the epilogue's pe half for
    the same q_pe, position and scale."""
    w = W.make_absorb("pe", 7, 5, flags, seed=6, rope_rows=512, scale=0.05)
    q, _ = _run(w)
    e = W.make("pe_e", 7, 5, flags, seed=6, num_blocks=1, rope_rows=512, scale=0.05)
    e.q_pe.copy_(w.q_pe)
    e.positions.copy_(w.positions)
    qe, _ = oracle.run(e.q_nope, e.q_pe, e.kv_c, e.k_pe, e.slot_mapping, e.cache, e.flags,
                       positions=e.positions, cos_sin=e.cos_sin, q_scale=e.q_scale, kv_scale=e.kv_scale)
    assert torch.equal(_bits(q[..., 512:]), _bits(qe[..., 512:]))


def test_general_inputs_within_fp32_rounding_of_numpy():
    w = W.make_absorb("gen", 9, 3, 0, seed=8)
    q, _ = _run(w)
    ql = np.einsum("thk,hjk->thj", w.q_nope_c.double().numpy(), w.w_uk.double().numpy())
    got = q[..., :512].double().numpy()
    ulp = np.abs(ql) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(got - ql) <= ulp)


def test_zero_tokens_and_bad_flags():
    w = W.make_absorb("z", 0, 2, 0, seed=1)
    q, st = _run(w)
    assert q.shape == (0, 2, 576) and st == 0
    w = W.make_absorb("f", 2, 2, 0, seed=1)
    with pytest.raises(ValueError):
        oracle.absorb_run(w.q_nope_c, w.w_uk, w.q_pe, W.FLAG_KV_FP8)


@pytest.mark.parametrize("flags", [W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8])
def test_positions_out_of_range_leave_pe_unrotated(flags):
    """The slot/position rule of the epilogue, on the absorbed rows: a
    position outside [0, rope_rows) sets status bit 2 and leaves that token's
    pe half unrotated (the bf16 input bits, or the e4m3 bytes of x / scale);
    tokens in range are rotated.  The table is a quarter turn everywhere
    (cos 0, sin 1), so a rotated pair (a, b) is exactly (-b, a) and the
    expected values need no rounding of a product."""
    T, H, rows = 6, 3, 8
    w = W.make_absorb("posrule", T, H, flags, seed=21, rope_rows=rows, scale=0.25)
    w.cos_sin = torch.cat((torch.zeros(rows, 32), torch.ones(rows, 32)), 1).contiguous()
    w.positions = torch.tensor([0, -1, rows, 3, 2 ** 31 - 1, rows - 1], dtype=torch.int32)
    q, st = _run(w)
    assert st == oracle.STATUS_POS_RANGE
    a, b = w.q_pe[..., :32], w.q_pe[..., 32:]
    rotated = torch.cat((-b, a), -1)
    for t in range(T):
        inside = 0 <= int(w.positions[t]) < rows
        want = rotated[t] if inside else w.q_pe[t]
        if flags & W.FLAG_Q_FP8:
            # x / 0.25 is exact (a power of two), so torch's cast of the
            # quotient is the e4m3 byte of the definition
            ref = (want.float() / 0.25).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
            assert torch.equal(q[t, :, 512:], ref), t
        else:
            assert torch.equal(_bits(q[t, :, 512:]), _bits(want)), t
