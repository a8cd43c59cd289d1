"""Shared helpers of the GPU parity tests: run a workload through the C ABI
and through the CPU oracle, compare bit for bit."""

from __future__ import annotations

import torch

import oracle
from mla_decode_attention_10_b200 import epilogue as E
from mla_decode_attention_10_b200 import workloads as W


def run_oracle(w: W.Workload, flags=None, table=None):
    """Oracle on a host workload; returns (q_out, cache_after, status)."""
    cache = w.cache.clone()
    q, st = oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, cache,
                       w.flags if flags is None else flags, positions=w.positions,
                       cos_sin=w.cos_sin if table is None else table,
                       q_scale=w.q_scale, kv_scale=w.kv_scale)
    return q, cache, st


def run_gpu(w: W.Workload, extra_flags: int = 0, producer: bool = False, stream=None):
    """The CUDA path on a copy of host workload ``w``; returns host
    (q_out, cache_after, status).  With ``producer`` the query inputs are
    written on the device by the synthetic producer kernel into zeroed buffers
    and the epilogue is launched behind it with programmatic dependent launch."""
    d = w.to("cuda")
    extra = extra_flags
    if producer:
        src_nope = d.q_nope.contiguous().clone()
        src_pe = d.q_pe.contiguous().clone()
        d.q_nope.zero_()
        d.q_pe.zero_()
        torch.cuda.synchronize()
        s = stream or torch.cuda.current_stream()
        rc = E.mla_harness_produce(src_nope.data_ptr(), src_pe.data_ptr(), d.q_nope.data_ptr(),
                                   d.q_nope.stride(0), d.q_nope.stride(1), d.q_pe.data_ptr(),
                                   d.q_pe.stride(0), d.q_pe.stride(1), d.T, d.H, 0, s.cuda_stream)
        assert rc == E.MLA_OK, E.status_string(rc)
        extra |= E.MLA_FLAG_PDL
    q_out = torch.empty((w.T, w.H, W.ROW), dtype=w.q_out_dtype(), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = E.launch_workload(d, q_out, status=status, extra_flags=extra, stream=stream)
    assert rc == E.MLA_OK, E.status_string(rc)
    torch.cuda.synchronize()
    return q_out.cpu(), d.cache.cpu(), int(status.item())


def bits(t: torch.Tensor) -> torch.Tensor:
    t = t.contiguous()
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.uint8)


def assert_same(gpu, ref, what: str):
    g, r = bits(gpu), bits(ref)
    if torch.equal(g, r):
        return
    diff = (g != r)
    idx = diff.nonzero()[:5].tolist()
    raise AssertionError(f"{what}: {int(diff.sum())} of {diff.numel()} elements differ; first at {idx}: "
                         f"gpu {[g[tuple(i)].item() for i in idx]} oracle {[r[tuple(i)].item() for i in idx]}")


def check_workload(w: W.Workload, extra_flags: int = 0, producer: bool = False):
    qg, cg, sg = run_gpu(w, extra_flags=extra_flags, producer=producer)
    qo, co, so = run_oracle(w)
    assert sg == so, (sg, so)
    assert_same(qg, qo, f"{w.name} q_out")
    assert_same(cg, co, f"{w.name} cache")
    return qg, cg
