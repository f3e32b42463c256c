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
    # other paths keep the default
    assert pk.pa_decode_auto_partition_size(64, 40, 40, 128, pk.PA_F16, 2048) == 512
    assert pk.pa_decode_auto_partition_size(256, 64, 8, 64, bf, 4096) == 512
    assert pk.pa_decode_auto_partition_size(256, 64, 8, 128, pk.PA_F32, 4096) == 512
    assert pk.pa_decode_auto_partition_size(4, 6, 4, 128, bf, 100) == -1
    # the same rule over an E4M3 cache
    a8 = pk.pa_decode_fp8_auto_partition_size
    assert a8(256, 64, 8, 128, bf, 4096) == 4096
    assert a8(128, 32, 8, 128, bf, 32768) == 4096
    assert a8(16, 64, 8, 128, bf, 32768) == 2048
    assert a8(1, 64, 8, 128, bf, 32768) == 512
    assert a8(64, 40, 40, 128, pk.PA_F16, 2048) == 512
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
