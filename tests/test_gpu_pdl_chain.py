"""Producer -> epilogue -> consumer, each a programmatic dependent of the one
before (the setting of the vLLM PR #54896 report, 实现拆解 item 2, and the
trigger-after-every-store rule of its 评论区精华).

q_out is filled with NaN bytes before every round, so a consumer that read a
row before the epilogue's store landed would produce a NaN or a wrong score.
The scores are checked against dot products of the oracle's q_out and cache
rows, computed in double precision on the host; q_out and the cache are
checked bit for bit as well.
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_10_b200 import epilogue as E
from mla_decode_attention_10_b200 import workloads as W
from parity_util import assert_same, run_oracle

pytestmark = pytest.mark.gpu


def _decode(t: torch.Tensor, fp8: bool) -> torch.Tensor:
    return (t.view(torch.float8_e4m3fn) if fp8 else t.view(torch.bfloat16)).double()


def _chain(w: W.Workload, extra: int, rounds_pdl: bool = True):
    d = w.to("cuda")
    s = torch.cuda.current_stream()
    src_n, src_p = d.q_nope.contiguous().clone(), d.q_pe.contiguous().clone()
    d.q_nope.fill_(float("nan"))
    d.q_pe.fill_(float("nan"))
    q_out = torch.full((w.T, w.H, W.ROW * (1 if w.q_fp8 else 2)), 0xFF, dtype=torch.uint8, device="cuda")
    q_out = q_out if w.q_fp8 else q_out.view(torch.bfloat16)
    scores = torch.full((w.T * w.H,), -1.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    pdl = E.MLA_FLAG_PDL if rounds_pdl else 0
    assert E.mla_harness_produce(src_n.data_ptr(), src_p.data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0),
                                 d.q_nope.stride(1), d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1),
                                 w.T, w.H, 0, s.cuda_stream) == E.MLA_OK
    assert E.launch_workload(d, q_out, extra_flags=extra | pdl) == E.MLA_OK
    cflags = pdl | (E.MLA_FLAG_Q_FP8 if w.q_fp8 else 0) | (E.MLA_FLAG_KV_FP8 if w.kv_fp8 else 0)
    assert E.mla_harness_consume(q_out.data_ptr(), d.cache.data_ptr(), d.slot_mapping.data_ptr(), w.T, w.H,
                                 w.num_blocks * w.block_size, cflags, scores.data_ptr(), s.cuda_stream) == E.MLA_OK
    torch.cuda.synchronize()
    return q_out.cpu(), d.cache.cpu(), scores.cpu()


def _expected_scores(w, q, cache):
    qd = _decode(q.contiguous().view(torch.uint8) if w.q_fp8 else q, w.q_fp8).reshape(w.T, w.H, W.ROW)
    rows = cache.view(-1, W.ROW)[w.slot_mapping]
    kd = _decode(rows, w.kv_fp8)
    prod = qd * kd[:, None, :]
    return prod.sum(-1).reshape(-1), prod.abs().sum(-1).reshape(-1)


@pytest.mark.parametrize("force", [0, E.MLA_FLAG_FORCE_SPLIT, E.MLA_FLAG_FORCE_ROWS])
@pytest.mark.parametrize("T,flags", [(7, W.FLAG_ROPE), (64, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8),
                                     (300, W.FLAG_ROPE | W.FLAG_KV_FP8), (1500, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8)])
def test_consumer_behind_epilogue_sees_every_store(force, T, flags):
    for rnd in range(3):
        w = W.make("chain", T, 16, flags, seed=900 + rnd + T, num_blocks=64, rope_rows=4096, scale=0.05,
                   cache_fill="random")
        q, cache, scores = _chain(w, force)
        qo, co, _ = run_oracle(w)
        assert_same(q, qo, "q_out")
        assert_same(cache, co, "cache")
        exp, mag = _expected_scores(w, qo, co)
        assert not torch.isnan(scores).any()
        err = (scores.double() - exp).abs()
        assert torch.all(err <= 1e-5 * mag + 1e-30), float((err / (mag + 1e-30)).max())


def test_consumer_marks_out_of_range_slots_nan():
    w = W.make("chain_bad", 5, 4, 0, seed=3, num_blocks=1, block_size=16)
    w.slot_mapping[2] = 16
    w.slot_mapping[4] = -1
    q, cache, scores = _chain(w, 0, rounds_pdl=False)
    s = scores.view(5, 4)
    assert torch.isnan(s[2]).all() and torch.isnan(s[4]).all()
    assert not torch.isnan(s[[0, 1, 3]]).any()


@pytest.mark.parametrize("T,flags", [(1, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8), (64, W.FLAG_ROPE)])
def test_epilogue_behind_a_producer_that_streams_weights_first(T, flags):
    """The producer reads 9 MiB of weights before it writes q (a projection
    GEMM's duration); the epilogue runs as its programmatic dependent.  The
    outputs are the oracle's bit for bit, and the producer's checksum of the
    weights is the XOR of all their 32-bit words."""
    w = W.make("gemm_like", T, 16, flags, seed=41 + T, num_blocks=8, rope_rows=4096, scale=0.05,
               cache_fill="random")
    d = w.to("cuda")
    s = torch.cuda.current_stream()
    g = torch.Generator().manual_seed(5)
    weights_host = torch.randint(-2 ** 31, 2 ** 31 - 1, ((9 << 20) // 4,), dtype=torch.int32, generator=g)
    weights = weights_host.to("cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    src_n, src_p = d.q_nope.contiguous().clone(), d.q_pe.contiguous().clone()
    d.q_nope.fill_(float("nan"))
    d.q_pe.fill_(float("nan"))
    q_out = torch.empty((w.T, w.H, W.ROW), dtype=w.q_out_dtype(), device="cuda")
    torch.cuda.synchronize()
    assert E.mla_harness_produce_after_weights(
        src_n.data_ptr(), src_p.data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0), d.q_nope.stride(1),
        d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1), weights.data_ptr(), weights.numel() * 4,
        sink.data_ptr(), w.T, w.H, 0, s.cuda_stream) == E.MLA_OK
    assert E.launch_workload(d, q_out, extra_flags=E.MLA_FLAG_PDL) == E.MLA_OK
    torch.cuda.synchronize()
    qo, co, _ = run_oracle(w)
    assert_same(q_out.cpu(), qo, "q_out")
    assert_same(d.cache.cpu(), co, "cache")
    x = weights_host.numpy().view("uint32")
    assert int(sink.cpu().numpy().view("uint32")[0]) == int(np.bitwise_xor.reduce(x))
