"""GPU parity on boundary-dominant inputs: every query row carries one spike
(a key aligned with its query, about half of the row's softmax weight) at a
position where a kernel could lose, repeat or misplace a token: the first and
last token, block edges, partition and span edges, tile edges, the last tile
of a partition, and for several query tokens the key just past the causal
limit.  The CPU tests in test_boundary_sensitivity.py show, with the oracle
alone and on these same bytes, that each such slip moves the row's output by
more than ten times the tolerance; here the kernels must match the unchanged
oracle within the tolerance (max abs 2e-2 for fp16 / bf16 outputs, 1e-5 for
fp32).

Cases cover the CUDA-core kernel (G = 1, 2; f32 / D 64), the tcgen05 kernels
(G = 4, 8; 16-bit and E4M3 caches), block sizes 8 / 16 / 32, partitions of
128 / 256 / 512 / 4096 tokens, CTAs streaming several partitions with one
softmax, and pa_decode_multi for speculative verification and chunked prefill.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_443_b200 as pk
import workloads as W
from boundary_cases import DECODE, MULTI, mq_queries
from pa_harness import (TOL, as_f64, build, check_bookkeeping, check_caches, oracle_attention,
                        run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def clean_status():
    pk.pa_device_status(clear=True)
    yield


@pytest.mark.parametrize("case", DECODE, ids=[c.name for c in DECODE])
def test_boundary_decode(case):
    sc = case.scenario()
    spec = sc.spec
    assert sc.spikes.rows
    p, o = build(sc, draw_device="cpu")
    out = run_step(p, spec, partition_size=case.P)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    check_bookkeeping(p, o)
    check_caches(p, o)
    got = as_f64(out, spec)
    want = oracle_attention(o, spec)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[spec.dtype], (case.name, err)


@pytest.mark.parametrize("case", MULTI, ids=[c.name for c in MULTI])
def test_boundary_multi_query(case):
    sc = case.scenario()
    spec = sc.spec
    p, o = build(sc, draw_device="cpu")
    run_step(p, spec)                      # the step's tokens are appended
    torch.cuda.synchronize()
    q_cpu, qs = mq_queries(case, sc)
    q = q_cpu.cuda()
    T = q.shape[0]
    out = torch.full_like(q, float("nan"))
    maxq = int(np.diff(qs).max())
    n = pk.pa_decode_multi_workspace_bytes(T, spec.Hq, spec.D, p.max_ctx, case.P)
    ws = torch.empty(n // 4, dtype=torch.float32, device="cuda") if n else None
    pk.pa_decode_multi(out, q, p.cache.k_cache, p.cache.v_cache, p.tables, p.lens,
                       torch.from_numpy(qs).cuda(), spec.softmax_scale, p.max_ctx, maxq,
                       partition_size=case.P, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    got = as_f64(out, spec)
    want = oracle.paged_attention_mq(W.storage_view(q_cpu), o.k, o.v, spec.dtype_code, o.tables,
                                     o.lens, qs, spec.softmax_scale)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[spec.dtype], (case.name, err)
