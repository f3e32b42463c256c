"""The C-ABI library loads, exports every declared symbol and rejects bad
arguments on the host before any launch (CPU only: no device call is made)."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_443_b200 as pk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_443_b200 import build
    build.build()
    return pk.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    assert sorted(pk.EXPORTS) == names


def test_version_and_counters(L):
    assert "sm_100a" in pk.pa_version()
    assert pk.pa_launch_count() >= 0
    assert pk.pa_decode_default_partition_size() % 32 == 0


def test_partition_and_workspace_sizes(L):
    P = pk.pa_decode_default_partition_size()
    assert pk.pa_decode_num_partitions(0) == 1
    assert pk.pa_decode_num_partitions(P) == 1
    assert pk.pa_decode_num_partitions(P + 1) == 2
    assert pk.pa_decode_num_partitions(1000, 64) == 16
    assert pk.pa_decode_num_partitions(10, 48) == -1
    assert pk.pa_decode_workspace_bytes(64, 40, 128, P) == 0
    n = pk.pa_decode_workspace_bytes(3, 5, 64, 1000, 256)
    assert n >= 3 * 5 * 4 * 66 * 4 and n % 256 == 0


FAKE = 1 << 20   # a 16-byte aligned non-null address; never dereferenced on these paths


def decode_call(L, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, maxb=8, lens=FAKE, B=2, Hq=8, Hkv=2,
             D=128, bs=16, NB=100, scale=0.1, dtype=pk.PA_BF16, P=0, maxctx=100, ws=None,
             wsb=0, stream=None)
    a.update(kw)
    st = L.pa_decode(a["out"], a["q"], a["k"], a["v"], a["tables"], a["maxb"], a["lens"], a["B"],
                     a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"], a["scale"], a["dtype"], a["P"],
                     a["maxctx"], a["ws"], a["wsb"], a["stream"])
    return st


@pytest.mark.parametrize("kw,want", [
    (dict(dtype=7), pk.PA_ERR_INVALID),
    (dict(B=-1), pk.PA_ERR_INVALID),
    (dict(Hq=6, Hkv=4), pk.PA_ERR_INVALID),
    (dict(Hq=6, Hkv=2), pk.PA_ERR_UNSUPPORTED),
    (dict(Hq=32, Hkv=2), pk.PA_ERR_UNSUPPORTED),
    (dict(D=96), pk.PA_ERR_UNSUPPORTED),
    (dict(D=0), pk.PA_ERR_INVALID),
    (dict(bs=64), pk.PA_ERR_UNSUPPORTED),
    (dict(bs=0), pk.PA_ERR_INVALID),
    (dict(NB=0), pk.PA_ERR_INVALID),
    (dict(maxb=0), pk.PA_ERR_INVALID),
    (dict(P=100), pk.PA_ERR_INVALID),
    (dict(maxctx=-1), pk.PA_ERR_INVALID),
    (dict(maxctx=8 * 16 + 1), pk.PA_ERR_INVALID),
    (dict(scale=float("nan")), pk.PA_ERR_INVALID),
    (dict(q=None), pk.PA_ERR_INVALID),
    (dict(out=FAKE + 8), pk.PA_ERR_INVALID),
    (dict(tables=FAKE + 2), pk.PA_ERR_INVALID),
    (dict(maxctx=100, P=32), pk.PA_ERR_INVALID),            # workspace needed, none given
    (dict(maxctx=100, P=32, ws=FAKE, wsb=64), pk.PA_ERR_INVALID),
])
def test_decode_rejects_bad_arguments(L, kw, want):
    before = pk.pa_launch_count()
    assert decode_call(L, **kw) == want
    assert pk.pa_last_error()
    assert pk.pa_launch_count() == before


def test_decode_with_no_sequences_is_a_no_op(L):
    assert decode_call(L, B=0) == pk.PA_OK


def test_reshape_and_copy_reject_bad_arguments(L):
    r = lambda **kw: L.pa_reshape_and_cache(kw.get("key", FAKE), FAKE, FAKE, FAKE,
                                            kw.get("slots", FAKE), kw.get("N", 4), 2,
                                            kw.get("D", 128), kw.get("bs", 16), 10,
                                            kw.get("dtype", pk.PA_F16), None)
    assert r(dtype=5) == pk.PA_ERR_INVALID
    assert r(N=-1) == pk.PA_ERR_INVALID
    assert r(D=80) == pk.PA_ERR_UNSUPPORTED
    assert r(bs=12) == pk.PA_ERR_UNSUPPORTED
    assert r(key=None) == pk.PA_ERR_INVALID
    assert r(key=FAKE + 4) == pk.PA_ERR_INVALID
    assert r(slots=FAKE + 4) == pk.PA_ERR_INVALID
    assert r(N=0) == pk.PA_OK
    c = lambda **kw: L.pa_copy_blocks(FAKE, kw.get("v", FAKE), kw.get("pairs", FAKE),
                                      kw.get("P", 3), 2, 128, 16, 10, kw.get("dtype", pk.PA_BF16),
                                      None)
    assert c(P=-1) == pk.PA_ERR_INVALID
    assert c(v=None) == pk.PA_ERR_INVALID
    assert c(pairs=FAKE + 4) == pk.PA_ERR_INVALID
    assert c(dtype=9) == pk.PA_ERR_INVALID
    assert c(P=0) == pk.PA_OK


def test_auto_partition_size(L):
    bf = pk.PA_BF16
    # tensor-core shapes with plenty of work take long partitions
    assert pk.pa_decode_auto_partition_size(256, 64, 8, 128, bf, 4096) == 4096
    assert pk.pa_decode_auto_partition_size(128, 32, 8, 128, bf, 32768) == 4096
    assert pk.pa_decode_auto_partition_size(16, 64, 8, 128, bf, 32768) == 2048
    assert pk.pa_decode_auto_partition_size(8, 64, 8, 128, bf, 32768) == 1024
    # too few CTAs at long partitions: the default
    assert pk.pa_decode_auto_partition_size(1, 64, 8, 128, bf, 32768) == 512
    # the CUDA-core kernel: 1024 with enough CTAs, else the default
    assert pk.pa_decode_auto_partition_size(64, 40, 40, 128, pk.PA_F16, 2048) == 1024
    assert pk.pa_decode_auto_partition_size(64, 40, 40, 128, pk.PA_F16, 8192) == 1024
    assert pk.pa_decode_auto_partition_size(256, 64, 8, 64, bf, 4096) == 1024
    assert pk.pa_decode_auto_partition_size(256, 64, 8, 128, pk.PA_F32, 4096) == 1024
    assert pk.pa_decode_auto_partition_size(4, 40, 40, 128, pk.PA_F16, 2048) == 512
    assert pk.pa_decode_auto_partition_size(4, 6, 4, 128, bf, 100) == -1
    # the same rule over an E4M3 cache
    a8 = pk.pa_decode_fp8_auto_partition_size
    assert a8(256, 64, 8, 128, bf, 4096) == 4096
    assert a8(128, 32, 8, 128, bf, 32768) == 4096
    assert a8(16, 64, 8, 128, bf, 32768) == 2048
    assert a8(1, 64, 8, 128, bf, 32768) == 512
    assert a8(64, 40, 40, 128, pk.PA_F16, 2048) == 1024
    assert a8(4, 40, 40, 128, pk.PA_F16, 2048) == 512
    assert a8(256, 64, 8, 128, pk.PA_FP8_E4M3, 4096) == -1
    assert a8(4, 6, 4, 128, bf, 100) == -1
    # the default-sized workspace covers the automatic length
    for P in (1024, 2048, 4096):
        assert pk.pa_decode_workspace_bytes(256, 64, 128, 4096, P) <= \
            pk.pa_decode_workspace_bytes(256, 64, 128, 4096, 0)


def test_fp8_calls_reject_bad_arguments(L):
    assert decode_call(L, dtype=pk.PA_FP8_E4M3) == pk.PA_ERR_UNSUPPORTED

    def d8(k_scale=0.5, v_scale=2.0, dtype=pk.PA_BF16, **kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, maxb=8, lens=FAKE, B=2, Hq=8,
                 Hkv=2, D=128, bs=16, NB=100, scale=0.1, P=0, maxctx=100)
        a.update(kw)
        return L.pa_decode_fp8(a["out"], a["q"], a["k"], a["v"], a["tables"], a["maxb"],
                               a["lens"], a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"],
                               a["scale"], dtype, k_scale, v_scale, a["P"], a["maxctx"], None, 0,
                               None)

    before = pk.pa_launch_count()
    for bad in (dict(k_scale=0.0), dict(v_scale=-1.0), dict(k_scale=float("inf")),
                dict(v_scale=float("nan")), dict(dtype=pk.PA_FP8_E4M3), dict(dtype=9),
                dict(D=96), dict(maxctx=100, P=32)):
        want = pk.PA_ERR_UNSUPPORTED if ("D" in bad or bad.get("dtype") == pk.PA_FP8_E4M3) \
            else pk.PA_ERR_INVALID
        assert d8(**bad) == want, bad
    assert d8(B=0) == pk.PA_OK
    r = lambda dtype=pk.PA_F16, ks=1.0, vs=1.0, **kw: L.pa_reshape_and_cache_fp8(
        FAKE, FAKE, FAKE, FAKE, kw.get("slots", FAKE), kw.get("N", 4), 2, kw.get("D", 128), 16,
        10, dtype, ks, vs, None)
    assert r(dtype=pk.PA_FP8_E4M3) == pk.PA_ERR_INVALID
    assert r(ks=0.0) == pk.PA_ERR_INVALID
    assert r(vs=float("nan")) == pk.PA_ERR_INVALID
    assert r(D=80) == pk.PA_ERR_UNSUPPORTED
    assert r(slots=FAKE + 4) == pk.PA_ERR_INVALID
    assert r(N=0) == pk.PA_OK
    assert pk.pa_launch_count() == before


def test_multi_query_rejects_bad_arguments(L):
    def mq(**kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, maxb=8, lens=FAKE, qs=FAKE, B=2,
                 T=6, maxq=4, Hq=16, Hkv=2, D=128, bs=16, NB=100, scale=0.1, dtype=pk.PA_BF16,
                 P=0, maxctx=100, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.pa_decode_multi(a["out"], a["q"], a["k"], a["v"], a["tables"], a["maxb"],
                                 a["lens"], a["qs"], a["B"], a["T"], a["maxq"], a["Hq"], a["Hkv"],
                                 a["D"], a["bs"], a["NB"], a["scale"], a["dtype"], a["P"],
                                 a["maxctx"], a["ws"], a["wsb"], None)
    before = pk.pa_launch_count()
    cases = [
        (dict(dtype=pk.PA_F32), pk.PA_ERR_UNSUPPORTED),
        (dict(dtype=pk.PA_FP8_E4M3), pk.PA_ERR_UNSUPPORTED),
        (dict(dtype=9), pk.PA_ERR_INVALID),
        (dict(D=64), pk.PA_ERR_UNSUPPORTED),
        (dict(Hq=24), pk.PA_ERR_UNSUPPORTED),
        (dict(Hq=15), pk.PA_ERR_INVALID),
        (dict(bs=64), pk.PA_ERR_UNSUPPORTED),
        (dict(P=192), pk.PA_ERR_INVALID),          # not a multiple of 128
        (dict(maxq=0), pk.PA_ERR_INVALID),
        (dict(maxq=7), pk.PA_ERR_INVALID),         # above total_q
        (dict(maxctx=8 * 16 + 1), pk.PA_ERR_INVALID),
        (dict(qs=None), pk.PA_ERR_INVALID),
        (dict(qs=FAKE + 2), pk.PA_ERR_INVALID),
        (dict(q=FAKE + 8), pk.PA_ERR_INVALID),
        # 1000 tokens over 256-token partitions need split-K partials
        (dict(maxb=64, maxctx=1000, P=256, ws=None, wsb=0), pk.PA_ERR_INVALID),
        (dict(maxb=64, maxctx=1000, P=256, wsb=64), pk.PA_ERR_INVALID),
        (dict(scale=float("inf")), pk.PA_ERR_INVALID),
    ]
    for kw, want in cases:
        assert mq(**kw) == want, kw
        assert pk.pa_last_error()
    assert mq(B=0) == pk.PA_OK and mq(T=0) == pk.PA_OK
    assert pk.pa_launch_count() == before
    assert pk.pa_decode_multi_workspace_bytes(6, 16, 128, 100, 0) == 0
    assert pk.pa_decode_multi_workspace_bytes(6, 16, 128, 1000, 256) >= 6 * 16 * 4 * 130 * 4
    assert pk.pa_decode_multi_workspace_bytes(6, 16, 128, 1000, 96) == 0   # invalid length


# ---------------------------------------------------------------------------
# shared-prefix groups (host helper and argument checks)


def _groups_brute_force(tables, lens, bs):
    """Groups by the rule pa_build_groups documents, written out plainly."""
    B = len(lens)
    full = [int(x) // bs for x in lens]
    starts, shared = [], [0] * B
    b0 = 0
    while b0 < B:
        members = [b0]
        while (full[b0] > 0 and members[-1] + 1 < B and full[members[-1] + 1] > 0
               and tables[members[-1] + 1][0] == tables[b0][0]):
            members.append(members[-1] + 1)
        k = full[b0]
        for m in members[1:]:
            c = 0
            while c < min(k, full[m]) and tables[m][c] == tables[b0][c]:
                c += 1
            k = c
        for m in members:
            shared[m] = k * bs if len(members) > 1 else 0
        starts.append(b0)
        b0 = members[-1] + 1
    return starts + [B], shared


def test_build_groups_matches_its_rule():
    import numpy as np
    import torch
    rng = np.random.default_rng(11)
    for trial in range(200):
        bs = int(rng.choice([8, 16, 32]))
        B = int(rng.integers(1, 12))
        mb = 6
        tables = np.full((B, mb), -1, np.int32)
        lens = np.zeros(B, np.int32)
        pool = iter(range(1000))
        b = 0
        while b < B:
            # a family of forks sharing a random number of leading blocks
            size = int(rng.integers(1, 4))
            common = [next(pool) for _ in range(int(rng.integers(0, mb)))]
            for _ in range(min(size, B - b)):
                n_blk = int(rng.integers(len(common), mb + 1))
                row = common[:n_blk] + [next(pool) for _ in range(n_blk - len(common))]
                L = 0 if n_blk == 0 else int(rng.integers((n_blk - 1) * bs + 1, n_blk * bs + 1))
                tables[b, :n_blk] = row
                lens[b] = L
                b += 1
        g = pk.pa_build_groups(torch.from_numpy(tables), torch.from_numpy(lens), bs)
        starts, shared = _groups_brute_force(tables.tolist(), lens.tolist(), bs)
        assert g.group_start.tolist() == starts, trial
        assert g.shared_lens.tolist() == shared, trial
        assert g.num_groups == len(starts) - 1
        assert g.max_group_size == max(np.diff(starts))
        assert g.max_shared_len == max(shared)
        # what pa_decode_grouped requires of the groups
        for i in range(g.num_groups):
            mem = range(starts[i], starts[i + 1])
            S = shared[starts[i]]
            assert S % bs == 0 and all(shared[m] == S and lens[m] >= S for m in mem)
            assert all((tables[m, :S // bs] == tables[starts[i], :S // bs]).all() for m in mem)


def test_build_groups_of_the_workload_scripts():
    """Parallel samples: a group per prompt sharing its whole prompt blocks;
    shared prefix: one group of every request sharing the 4096-token prefix."""
    import torch
    import workloads as W
    for spec, want in ((W.small("llama13b_ps"), "per prompt"), (W.small("long_prefix"), "one")):
        sc = W.scenario(spec)
        alloc = pk.BlockAllocator(sc.num_blocks, spec.block_size, sc.free_order.tolist())
        for op in sc.setup_ops + sc.step_ops:
            if op.kind == "add":
                alloc.add(op.seq)
            elif op.kind == "fork":
                alloc.fork(op.seq, op.arg)
            elif op.kind == "release":
                alloc.release(op.seq)
            else:
                alloc.append(op.seq, op.arg)
        t, l = alloc.build_tables(sc.batch, sc.max_blocks)
        g = pk.pa_build_groups(torch.from_numpy(t), torch.from_numpy(l), spec.block_size)
        if want == "one":
            assert g.num_groups == 1 and g.max_shared_len == spec.prefix_len
        else:
            assert g.num_groups == spec.num_prompts
            assert g.max_group_size == spec.samples_per_prompt
            assert set(g.group_start.tolist()) == set(range(0, spec.num_seqs + 1,
                                                            spec.samples_per_prompt))


def test_grouped_decode_rejects_bad_arguments(L):
    import ctypes as C
    good = dict(num_groups=1, max_group_size=2, max_shared_len=16, B=2, Hq=8, Hkv=2, D=128,
                bs=16, max_ctx=64, P=0)

    def call(**kw):
        a = dict(good, **kw)
        fake = C.c_void_p(256)
        return L.pa_decode_grouped(fake, fake, fake, fake, fake, 8, fake, fake, fake,
                                   a["num_groups"], a["max_group_size"], a["max_shared_len"],
                                   a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], 100, 0.1,
                                   pk.PA_BF16, a["P"], a["max_ctx"], None, 0, None)

    n0 = pk.pa_launch_count()
    assert call(max_shared_len=8) == pk.PA_ERR_INVALID        # not a multiple of bs
    assert call(max_shared_len=80) == pk.PA_ERR_INVALID       # beyond max_context_len
    assert call(num_groups=3) == pk.PA_ERR_INVALID            # more groups than sequences
    assert call(max_group_size=0) == pk.PA_ERR_INVALID
    assert call() == pk.PA_ERR_INVALID                        # no workspace
    assert pk.pa_launch_count() == n0
    # the E4M3 variant checks the same, plus the cache scales and the query type
    def call8(q_dtype=pk.PA_BF16, k_scale=0.5, **kw):
        a = dict(good, **kw)
        fake = C.c_void_p(256)
        return L.pa_decode_grouped_fp8(fake, fake, fake, fake, fake, 8, fake, fake, fake,
                                       a["num_groups"], a["max_group_size"],
                                       a["max_shared_len"], a["B"], a["Hq"], a["Hkv"], a["D"],
                                       a["bs"], 100, 0.1, q_dtype, k_scale, 0.25, a["P"],
                                       a["max_ctx"], None, 0, None)

    assert call8(max_shared_len=8) == pk.PA_ERR_INVALID
    assert call8(num_groups=3) == pk.PA_ERR_INVALID
    assert call8(k_scale=0.0) == pk.PA_ERR_INVALID            # scales must be positive
    assert call8(q_dtype=pk.PA_FP8_E4M3) == pk.PA_ERR_UNSUPPORTED  # queries are not codes
    assert call8() == pk.PA_ERR_INVALID                       # no workspace
    assert pk.pa_launch_count() == n0
    need = L.pa_decode_grouped_workspace_bytes(2, 8, 128, 64, 16, 32)
    # slots: ceil(16/32) = 1 for the span + ceil(64/32) = 2 for the rest
    assert need == -(-2 * 8 * 3 * 130 * 4 // 256) * 256
    assert L.pa_decode_grouped_workspace_bytes(2, 8, 128, 64, 0, 32) == \
        L.pa_decode_workspace_bytes(2, 8, 128, 64, 32)
