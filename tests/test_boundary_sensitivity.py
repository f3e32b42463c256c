"""The boundary-dominant parity cases are sensitive to one-token slips: for
every spiked query row, the oracle's output with the spike token dropped,
counted twice or replaced by its neighbour in the slot sequence (or, for a
spike just past a query's causal limit, with that key taken in) differs from
the unchanged output by more than ten times the output tolerance.  So a kernel
that makes any such slip at these positions fails its parity test
(test_gpu_boundary.py), which compares it with the unchanged oracle.

Oracle only, on the same CPU-drawn contents the GPU tests use; no kernel is
involved and no mistake is planted in one.
"""
import numpy as np
import pytest

import oracle
from boundary_cases import DECODE, GROUPED, MULTI, mq_offsets, mq_queries
from pa_harness import TOL, build_oracle, oracle_attention, oracle_row_perturbed

MARGIN = 10.0
MAX_ROWS = 160          # spiked rows checked per case (all when fewer)


def _rows(plan, seed):
    rows = sorted(plan.rows)
    if len(rows) > MAX_ROWS:
        rows = sorted(np.random.default_rng(seed).choice(rows, MAX_ROWS, replace=False).tolist())
    return rows


REPEAT_MIN_KEYS = 16


def _slips(kind, n, j):
    """The slips checked for a spike at position j of a row that sees n keys.
    A repeated spike moves the weight from about 1/2 to about 2/3; with fewer
    than REPEAT_MIN_KEYS keys the background's own spread can hide that, so
    there only the drop and the neighbour are required to show."""
    if kind == "past_limit":
        return ("include",)
    slips = ["drop"]
    if n > 1:
        slips.append("neighbour")
    if n >= REPEAT_MIN_KEYS:
        slips.append("repeat")
    return slips


@pytest.mark.parametrize("case", DECODE + GROUPED, ids=[c.name for c in DECODE + GROUPED])
def test_decode_case_is_sensitive(case):
    sc = case.scenario()
    spec = sc.spec
    o = build_oracle(sc)
    rows = _rows(sc.spikes, 7)
    assert rows, "the plan placed no spike"
    want = oracle_attention(o, spec, rows=np.array([divmod(r, spec.Hq) for r in rows]))
    tol = MARGIN * TOL[spec.dtype]
    for r, w in zip(rows, want):
        b, h, j, kind = sc.spikes.rows[r]
        n = int(o.lens[b])
        for how in _slips(kind, n, j):
            got = oracle_row_perturbed(o, spec, b, h, j, how)
            d = np.abs(got - w).max()
            assert d > tol, (case.name, b, h, j, kind, how, d)


@pytest.mark.parametrize("case", MULTI, ids=[c.name for c in MULTI])
def test_multi_query_case_is_sensitive(case):
    sc = case.scenario()
    spec = sc.spec
    o = build_oracle(sc)
    qt, qs = mq_queries(case, sc)
    from workloads import storage_view
    q = storage_view(qt)
    want_all = oracle.paged_attention_mq(q, o.k, o.v, spec.dtype_code, o.tables, o.lens, qs,
                                         spec.softmax_scale)
    rows = _rows(sc.spikes, 9)
    assert rows
    tol = MARGIN * TOL[spec.dtype]
    kinds = set()
    for r in rows:
        t, h, j, kind = sc.spikes.rows[r]
        b = int(np.searchsorted(qs, t, side="right") - 1)
        Qb = int(qs[b + 1] - qs[b])
        n = int(o.lens[b]) - Qb + (t - int(qs[b])) + 1       # keys query token t sees
        kinds.add(kind)
        for how in _slips(kind, n, j):
            got = oracle_row_perturbed(o, spec, b, h, j, how, n_keys=n, q_row=q[t, h])
            d = np.abs(got - want_all[t, h]).max()
            assert d > tol, (case.name, t, h, j, kind, how, d)
    assert "past_limit" in kinds


def test_cases_cover_every_kind_of_boundary():
    """Across the cases, the spikes sit at every kind of position a slip can
    hit: first and last token, block, partition and tile edges, the last tile
    of a partition, the split between a family's shared span and the rest, and
    the key just past a query's causal limit."""
    from collections import Counter
    kinds = Counter()
    for case in DECODE + GROUPED + MULTI:
        kinds.update(k for (_, _, _, k) in case.scenario().spikes.rows.values())
    for k in ("end", "start", "partition", "block", "tile", "last_tile", "shared", "past_limit"):
        assert kinds[k] >= 20, (k, kinds)
