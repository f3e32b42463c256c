"""GPU parity of pa_decode_grouped: families of sequences that share leading
physical blocks ("블록 공유" on the supersilo.blog vLLM summary: parallel
samples of one prompt, requests forked from one prefix) decoded with each
family's shared span read once for all its members.  The result is pa_decode's
attention; every query row carries a boundary spike (see boundary_cases.py),
including at the split between the shared span and the rest and at the rest's
partition edges, and the output must match the unchanged oracle within the
tolerance (max abs 2e-2).  The groups come from the library's own host helper
(pa_build_groups), whose rule is checked on the CPU in test_abi_host.py.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_443_b200 as pk
import workloads as W
from boundary_cases import GROUPED
from pa_harness import (TOL, as_f64, build, check_bookkeeping, check_caches, oracle_attention,
                        run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def clean_status():
    pk.pa_device_status(clear=True)
    yield


@pytest.mark.parametrize("case", GROUPED, ids=[c.name for c in GROUPED])
def test_grouped_decode_matches_oracle(case):
    sc = case.scenario()
    spec = sc.spec
    p, o = build(sc, draw_device="cpu")
    out = run_step(p, spec, partition_size=case.P, grouped=True)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    check_bookkeeping(p, o)
    check_caches(p, o)
    g = p.cache.groups(p.tables, p.lens)
    assert g.max_shared_len > 0 and g.num_groups < len(sc.batch)
    got = as_f64(out, spec)
    want = oracle_attention(o, spec)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[spec.dtype], (case.name, err)


def test_grouped_workspace_full_of_nan_is_all_written():
    """Every slot the reduce reads was written by the span or the rest kernel."""
    case = [c for c in GROUPED if c.name == "g_lp_g4_stream"][0]
    sc = case.scenario()
    spec = sc.spec
    p, o = build(sc, draw_device="cpu")
    g = p.cache.groups(p.tables, p.lens)
    ws = p.cache.grouped_workspace(p.q.shape[0], p.q.shape[1], p.max_ctx, g, case.P)
    ws.fill_(float("nan"))
    out = run_step(p, spec, partition_size=case.P, workspace=ws, grouped=True)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    got = as_f64(out, spec)
    assert np.isfinite(got).all()
    assert np.abs(got - oracle_attention(o, spec)).max() <= TOL[spec.dtype]


def test_grouped_equals_ungrouped_within_tolerance_and_no_groups_is_pa_decode():
    case = [c for c in GROUPED if c.name == "g_ps_g1_p128"][0]
    sc = case.scenario()
    spec = sc.spec
    p, _ = build(sc, with_oracle=False, draw_device="cpu")
    a = run_step(p, spec, partition_size=case.P, grouped=True).clone()
    b = run_step(p, spec, partition_size=case.P).clone()
    torch.cuda.synchronize()
    assert np.abs(as_f64(a, spec) - as_f64(b, spec)).max() <= TOL[spec.dtype]
    # groups that share nothing: the call is pa_decode, byte for byte
    B = p.q.shape[0]
    none = pk.Groups(torch.arange(B + 1, dtype=torch.int32, device="cuda"),
                     torch.zeros(B, dtype=torch.int32, device="cuda"), B, 1, 0)
    c = p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale,
                       partition_size=case.P, groups=none)
    torch.cuda.synchronize()
    assert torch.equal(c.view(torch.int16), b.view(torch.int16))


def test_inconsistent_groups_are_flagged_without_faulting():
    case = [c for c in GROUPED if c.name == "g_lp_g4_p128"][0]
    sc = case.scenario()
    spec = sc.spec
    p, _ = build(sc, with_oracle=False, draw_device="cpu")
    run_step(p, spec, partition_size=case.P)
    g = p.cache.groups(p.tables, p.lens)
    bad = pk.Groups(g.group_start.clone(), g.shared_lens.clone(), g.num_groups,
                    g.max_group_size, g.max_shared_len)
    bad.shared_lens[1] = g.max_shared_len - spec.block_size     # differs from its group's
    p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale, partition_size=case.P,
                   groups=bad)
    assert pk.pa_device_status() & pk.PA_DEVERR_CONTEXT
    bad = pk.Groups(g.group_start.clone(), g.shared_lens.clone(), g.num_groups,
                    g.max_group_size, g.max_shared_len)
    bad.group_start[-1] = len(sc.batch) + 3                      # past the batch
    p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale, partition_size=case.P,
                   groups=bad)
    assert pk.pa_device_status() & pk.PA_DEVERR_CONTEXT
    out = run_step(p, spec, partition_size=case.P, grouped=True)     # still healthy
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
