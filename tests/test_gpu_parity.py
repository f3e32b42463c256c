"""GPU parity: the CUDA library against the oracle, on the same seeded inputs.

Bit-exact: block tables, context lengths, slots, copy-on-write pairs (block
manager) and cache bytes after copy_blocks + reshape_and_cache.  Within the
stated tolerance (max abs error of the output, 2e-2 for fp16/bf16, 1e-5 for
fp32, fp32 accumulation): decode attention.  Every cache slot no token was
written to holds NaN, so reading an unused tail slot into a result shows up.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_443_b200 as pk
import workloads as W
from pa_harness import (TOL, as_f64, build, check_bookkeeping, check_caches, check_token_slots,
                        oracle_attention, poison_bits, run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def clean_status():
    pk.pa_device_status(clear=True)
    yield


def full_check(spec, partition_size=None):
    sc = W.scenario(spec)
    p, o = build(sc)
    out = run_step(p, spec, partition_size)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    check_bookkeeping(p, o)
    check_caches(p, o)
    got = as_f64(out, spec)
    want = oracle_attention(o, spec)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[spec.dtype], (spec.name, err)
    return got, want


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix"])
def test_small_workloads(name):
    full_check(W.small(name))


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_long_prefix_block_sizes(bs):
    full_check(replace(W.small("long_prefix"), block_size=bs, name=f"lp_small_bs{bs}"))


@pytest.mark.parametrize("P", [32, 64, 96, 256, 512, 4096])
def test_partition_sizes(P):
    full_check(W.small("opt13b"), partition_size=P)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_dtype_head_group_matrix(dtype, D, G):
    spec = W.Spec(f"m_{dtype}_{D}_{G}", dtype, 2 * G, 2, D, 16, "independent", 5, seed=77 + G + D,
                  ctx_dist="explicit", ctx_list=(1, 77, 300, 513, 1100), partition_size=256)
    full_check(spec)


def test_edge_context_lengths():
    lens = (0, 1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1024, 1025, 2047)
    spec = W.Spec("edges", "bf16", 8, 2, 128, 16, "independent", len(lens), seed=5,
                  ctx_dist="explicit", ctx_list=lens, partition_size=512)
    got, _ = full_check(spec)
    assert np.all(got[0] == 0.0)            # context 0 -> zero row
    spec32 = replace(spec, block_size=32, name="edges32", partition_size=64)
    full_check(spec32)


def test_physical_placement_gives_bit_identical_output():
    spec = W.small("gqa70b")
    sc1 = W.scenario(spec)
    sc2 = W.scenario(spec)
    sc2.free_order = np.random.default_rng(99).permutation(sc2.num_blocks).astype(np.int32)
    p1, _ = build(sc1, with_oracle=False)
    p2, _ = build(sc2, with_oracle=False)
    assert not torch.equal(p1.tables, p2.tables)
    o1 = run_step(p1, spec)
    o2 = run_step(p2, spec)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_two_phase_equals_one_call():
    spec = W.small("opt13b")
    p, _ = build(W.scenario(spec), with_oracle=False)
    run_step(p, spec)
    ws = p.cache.workspace(p.q.shape[0], p.q.shape[1], p.max_ctx, 64)
    a = torch.empty_like(p.q)
    b = torch.empty_like(p.q)
    pk.pa_decode(a, p.q, p.cache.k_cache, p.cache.v_cache, p.tables, p.lens, spec.softmax_scale,
                 p.max_ctx, partition_size=64, workspace=ws)
    pk.pa_decode_partitions(b, p.q, p.cache.k_cache, p.cache.v_cache, p.tables, p.lens,
                            spec.softmax_scale, p.max_ctx, partition_size=64, workspace=ws)
    pk.pa_decode_reduce(b, p.lens, p.max_ctx, partition_size=64, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_repeated_steps_are_idempotent():
    """The benchmark repeats one step; repeating it must give the same result.
    Re-running the copy-on-write after the in-place writer stored its tokens
    copies those into the copies' unused tail slots, so only slots holding
    tokens are compared byte for byte."""
    spec = W.small("llama13b_ps")
    p, o = build(W.scenario(spec))
    first = run_step(p, spec).clone()
    for _ in range(3):
        again = run_step(p, spec)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), again.view(torch.int16))
    check_token_slots(p, o)


def test_device_checks_flag_bad_values_without_faulting():
    spec = W.small("opt13b")
    p, _ = build(W.scenario(spec), with_oracle=False)
    cache = p.cache
    # block-table entry outside the pool
    bad = p.tables.clone()
    bad[0, 0] = cache.num_blocks + 5
    out = cache.decode(p.q, bad, p.lens, p.max_ctx, spec.softmax_scale)
    assert pk.pa_device_status() & pk.PA_DEVERR_TABLE
    # context longer than the table row / the declared maximum
    lens = p.lens.clone()
    lens[1] = p.tables.shape[1] * spec.block_size + 100
    cache.decode(p.q, p.tables, lens, p.max_ctx, spec.softmax_scale)
    assert pk.pa_device_status() & pk.PA_DEVERR_CONTEXT
    # slot beyond the cache
    slots = p.step_slots.clone()
    slots[0] = cache.num_blocks * spec.block_size
    cache.store(p.step_key, p.step_value, slots)
    assert pk.pa_device_status() & pk.PA_DEVERR_SLOT
    # copy pair outside the pool
    cache.copy_on_write(torch.tensor([[0, cache.num_blocks]], dtype=torch.int64, device="cuda"))
    assert pk.pa_device_status() & pk.PA_DEVERR_PAIR
    # swap pair outside the (smaller) destination pool
    hk = torch.zeros((4,) + tuple(cache.k_cache.shape[1:]), dtype=cache.dtype, device="cuda")
    hv = torch.zeros_like(hk)
    pk.pa_swap_blocks(hk, hv, cache.k_cache, cache.v_cache,
                      torch.tensor([[0, 4]], dtype=torch.int64, device="cuda"))
    assert pk.pa_device_status() & pk.PA_DEVERR_PAIR
    assert not hk.any()
    # the context is still healthy
    run_step(p, spec)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0


def test_bounded_wait_gives_up_and_context_survives():
    """A pipeline wait that nothing will satisfy returns after its limit with
    PA_DEVERR_TIMEOUT set; the device stays usable (no trap, no hang)."""
    flags = pk.pa_selftest_wait_timeout()
    assert flags & pk.PA_DEVERR_TIMEOUT
    assert pk.pa_device_status() == 0
    spec = W.small("opt13b")
    full_check(spec)


@pytest.mark.parametrize("name", ["tiny", "llama13b_ps"])
def test_swap_blocks_match_oracle(name):
    """Device -> pinned host -> second device pool, against the oracle's swap of
    the oracle's own caches: every byte of all three pools equal.  The pairs of
    the first copy live in pinned host memory, those of the second on the device."""
    spec = W.small(name)
    p, o = build(W.scenario(spec))
    run_step(p, spec)
    torch.cuda.synchronize()
    NB = p.cache.num_blocks
    rng = np.random.default_rng(3)
    nb_host, nb_dev2 = NB // 2 + 3, NB + 5
    src = rng.choice(NB, size=NB // 2, replace=False)
    out_pairs = np.stack([src, rng.permutation(nb_host)[:src.size]], 1).astype(np.int64)
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(nb_dev2)[:src.size]], 1).astype(np.int64)
    fill = W.poison_value(spec)
    shape = tuple(p.cache.k_cache.shape[1:])
    host = [torch.full((nb_host,) + shape, fill, dtype=p.cache.dtype).pin_memory() for _ in range(2)]
    dev2 = [torch.full((nb_dev2,) + shape, fill, dtype=p.cache.dtype, device="cuda")
            for _ in range(2)]
    pk.pa_swap_blocks(host[0], host[1], p.cache.k_cache, p.cache.v_cache,
                      torch.from_numpy(out_pairs).pin_memory())
    pk.pa_swap_blocks(dev2[0], dev2[1], host[0], host[1],
                      torch.from_numpy(in_pairs).cuda())
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    oh = [np.full((nb_host,) + shape, poison_bits(spec)) for _ in range(2)]
    od = [np.full((nb_dev2,) + shape, poison_bits(spec)) for _ in range(2)]
    oracle.swap_blocks(oh[0], oh[1], o.k, o.v, out_pairs, spec.dtype_code)
    oracle.swap_blocks(od[0], od[1], oh[0], oh[1], in_pairs, spec.dtype_code)
    for got, want in zip(host + dev2, oh + od):
        assert W.storage_view(got).tobytes() == want.tobytes()
    check_caches(p, o)       # the source pool is unchanged


def test_swap_out_and_in_keeps_attention():
    """Swap two whole sampling families and two samples of a third to the pinned
    host pool, poison every free device block, swap back into fresh blocks:
    decode output bit-identical to before and within tolerance of the oracle.
    Blocks shared among the moved samples stay shared; the two lone samples
    come back with private copies of their prompt."""
    spec = W.small("llama13b_ps")
    sc = W.scenario(spec)
    p, o = build(sc)
    before = run_step(p, spec).clone()
    cache = p.cache
    cache.enable_swap(cache.num_blocks)
    moved = [0, 1, 2, 3, 4, 5, 12, 13, 14, 15, 16, 17, 7, 9]
    out_pairs = cache.swap_out(moved)
    assert len({d for _, d in out_pairs}) == len(out_pairs)
    free_ids = torch.tensor(sorted(cache.alloc.free_stack()), dtype=torch.int64, device="cuda")
    cache.k_cache.index_fill_(0, free_ids, float("nan"))
    cache.v_cache.index_fill_(0, free_ids, float("nan"))
    in_pairs = cache.swap_in(moved)
    assert len(in_pairs) == len(out_pairs) and cache.host_alloc.num_free() == cache.num_blocks
    tables, lens, max_ctx = cache.tables(sc.batch, sc.max_blocks)
    assert torch.equal(lens, p.lens)
    assert not torch.equal(tables, p.tables)
    t, t0 = tables.cpu().numpy(), p.tables.cpu().numpy()

    def same_block(tab, rows):
        x = np.where(tab[rows] >= 0, tab[rows], -1 - np.arange(tab[rows].size).reshape(len(rows), -1))
        return x.reshape(-1)[:, None] == x.reshape(-1)[None, :]

    for fam in ([0, 1, 2, 3, 4, 5], [12, 13, 14, 15, 16, 17]):
        assert np.array_equal(same_block(t, fam), same_block(t0, fam))
    held = {int(b) for r in (6, 8, 10, 11) for b in t[r] if b >= 0}
    assert not held & {int(b) for r in (7, 9) for b in t[r] if b >= 0}
    after = cache.decode(p.q, tables, lens, max_ctx, spec.softmax_scale,
                         partition_size=spec.partition_size)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    err = np.abs(as_f64(after, spec) - oracle_attention(o, spec)).max()
    assert err <= TOL[spec.dtype]


def test_launch_counter_counts_kernels():
    spec = W.small("opt13b")
    p, _ = build(W.scenario(spec), with_oracle=False)
    n0 = pk.pa_launch_count()
    run_step(p, spec, partition_size=512)
    np_ = pk.pa_decode_num_partitions(p.max_ctx, 512)
    expect = (1 if p.step_pairs.numel() else 0) + 1 + 1 + (1 if np_ > 1 else 0)
    assert pk.pa_launch_count() - n0 == expect


# ---------------------------------------------------------------------------
# full sizes of the five workloads, in the launch configuration the benchmark
# times (default partition size), checked on sampled rows


def sampled_rows(o, spec, n=96, seed=0):
    rng = np.random.default_rng(seed)
    B = len(o.lens)
    rows = {(int(b), int(h)) for b, h in zip(rng.integers(0, B, n), rng.integers(0, spec.Hq, n))}
    for b in (int(np.argmax(o.lens)), int(np.argmin(o.lens))):
        rows |= {(b, 0), (b, spec.Hq - 1)}
    return np.array(sorted(rows), dtype=np.int64)


def compared_sequences(sc, n_random=32, seed=0):
    """Batch indices whose every head the full-size tests compare: the longest
    and the shortest sequence and n_random others."""
    lens = np.asarray(sc.context_lens)
    rng = np.random.default_rng(seed)
    pick = {int(np.argmax(lens)), int(np.argmin(lens))}
    rest = [b for b in range(len(lens)) if b not in pick]
    pick |= {int(b) for b in rng.choice(rest, size=min(n_random, len(rest)), replace=False)}
    return sorted(pick)


def full_size_check(spec, name):
    """One step of a full-size workload in the benchmark's launch configuration
    (its own partition length), with a spike (boundary-dominant key, see
    workloads.spike_plan) in every head of the compared sequences: bookkeeping
    and touched cache blocks bit-exact, every head of those sequences within
    tolerance of the oracle, and, for a few spiked rows, the oracle itself
    showing that losing the spike token would move the output far beyond it."""
    from pa_harness import oracle_row_perturbed
    sc = W.scenario(spec)
    seqs = compared_sequences(sc)
    # spikes at the edges of every partition length the automatic rule may take
    P = spec.partition_size
    sc = W.spike_plan(sc, tuple(sorted({P, 512, 1024, 2048, 4096} - {0})), seed=2, seqs=seqs)
    p, o = build(sc)
    out = run_step(p, spec)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    check_bookkeeping(p, o)
    touched = sorted({s // spec.block_size for s in o.slots} | {d for _, d in o.pairs})
    rng = np.random.default_rng(1)
    extra = rng.choice(sc.num_blocks, size=min(256, sc.num_blocks), replace=False).tolist()
    check_caches(p, o, blocks=sorted(set(touched) | set(extra)))
    rows = np.array([(b, h) for b in seqs for h in range(spec.Hq)], dtype=np.int64)
    want = oracle_attention(o, spec, rows=rows)
    got_all = as_f64(out, spec)
    got = got_all[rows[:, 0], rows[:, 1]]
    assert np.isfinite(got_all).all()
    err = np.abs(got - want).max()
    assert err <= TOL[spec.dtype], (name, err)
    # sensitivity on this very input: a few spiked rows, the spike token dropped
    spiked = sorted(sc.spikes.rows)
    for r in np.random.default_rng(3).choice(spiked, size=min(6, len(spiked)), replace=False):
        b, h, j, kind = sc.spikes.rows[int(r)]
        k = int(np.flatnonzero((rows[:, 0] == b) & (rows[:, 1] == h))[0])
        d = np.abs(oracle_row_perturbed(o, spec, b, h, j, "drop") - want[k]).max()
        assert d > 10 * TOL[spec.dtype], (name, b, h, j, kind, d)


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix_bs8",
                                  "long_prefix_bs16", "long_prefix_bs32"])
def test_full_size_workloads(name):
    spec = W.long_prefix(int(name[-2:].lstrip("s"))) if name.startswith("long_prefix") else W.FULL[name]
    full_size_check(spec, name)


# ---------------------------------------------------------------------------
# E4M3 caches: the quantising append bit-exact against the oracle's, attention
# within the output dtype's tolerance of the oracle's fp64 attention over the
# same codes (unused slots hold the E4M3 NaN code)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.0123, 0.0171)])
def test_fp8_append_is_bit_exact(dtype, scales):
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    code = W.DTYPE_CODES[dtype]
    g = torch.Generator().manual_seed(31)
    N, Hkv, D, bs, NB = 40, 2, 128, 16, 8
    k = torch.randn((N, Hkv, D), generator=g) * torch.exp(torch.randn((N, Hkv, D), generator=g) * 3)
    v = torch.randn((N, Hkv, D), generator=g)
    # saturation, signed zeros, subnormal codes, exact ties (for scale 1)
    special = torch.tensor([1e4, -1e4, 448.0, 464.0, 0.0, -0.0, 0.001953125, 0.0048828125,
                            1.0625, 17.0, -1.1875, 240.0 + 8.0])
    k[0, 0, :special.numel()] = special
    k, v = k.to(tdt), v.to(tdt)
    k_scale, v_scale = (float(np.float32(x)) for x in scales)
    kc = torch.full((NB, Hkv, bs, D), 0x7f, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
    vc = kc.clone()
    slots = torch.randperm(NB * bs, generator=g)[:N].to(torch.int64)
    slots[3] = -1
    pk.pa_reshape_and_cache_fp8(k.cuda(), v.cuda(), kc, vc, slots.cuda(), k_scale, v_scale)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    ok = np.full((NB, Hkv, bs, D), 0x7f, dtype=np.uint8)
    ov = ok.copy()
    oracle.reshape_and_cache_e4m3(W.storage_view(k), W.storage_view(v), ok, ov, slots.numpy(),
                                  code, k_scale, v_scale)
    assert np.array_equal(W.storage_view(kc), ok)
    assert np.array_equal(W.storage_view(vc), ov)


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix"])
def test_fp8_small_workloads(name):
    full_check(W.fp8(W.small(name)))


@pytest.mark.parametrize("P", [32, 64, 96, 256, 4096])
def test_fp8_partition_sizes(P):
    full_check(W.fp8(W.small("opt13b")), partition_size=P)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_fp8_dtype_head_group_matrix(dtype, D, G):
    spec = W.Spec(f"m8_{dtype}_{D}_{G}", dtype, 2 * G, 2, D, 16, "independent", 5,
                  seed=91 + G + D, ctx_dist="explicit", ctx_list=(1, 77, 300, 513, 1100),
                  partition_size=256)
    full_check(W.fp8(spec))


def test_fp8_edge_context_lengths():
    lens = (0, 1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 1024, 1025, 2047)
    spec = W.fp8(W.Spec("edges8", "f16", 8, 8, 128, 16, "independent", len(lens), seed=6,
                        ctx_dist="explicit", ctx_list=lens, partition_size=512))
    got, _ = full_check(spec)
    assert np.all(got[0] == 0.0)
    full_check(replace(spec, block_size=8, name="edges8_bs8", partition_size=96))
    full_check(replace(spec, block_size=32, name="edges8_bs32", partition_size=64))


@pytest.mark.parametrize("name", ["opt13b", "gqa70b", "long_prefix_bs16"])
def test_fp8_full_size_workloads(name):
    base = W.long_prefix(16) if name.startswith("long_prefix") else W.FULL[name]
    full_size_check(W.fp8(base), name + "_fp8")



# ---------------------------------------------------------------------------
# prefix caching: requests sharing a system prompt reuse its blocks


def _prefix_kv(tokens, Hkv, D, dtype):
    """K/V of every position of a prompt, a function of the prefix up to and
    including it (identical prefixes give identical K/V, as in a model)."""
    ks, vs = [], []
    h = 0
    for t in tokens:
        h = (h * 1_000_003 + int(t) + 1) % (1 << 61)
        g = torch.Generator().manual_seed(h)
        ks.append(torch.randn((Hkv, D), generator=g))
        vs.append(torch.randn((Hkv, D), generator=g))
    return torch.stack(ks).to(dtype), torch.stack(vs).to(dtype)


@pytest.mark.parametrize("fp8", [False, True])
def test_prefix_cached_requests_match_oracle_and_uncached_run(fp8):
    from oracle.allocator import BlockManager
    from pa_harness import oracle_append
    from paged_kv_cache_443_b200.cache import PagedKVCache
    base = W.Spec("prefix", "bf16", 8, 2, 128, 16, "independent", 6, seed=3, partition_size=128)
    spec = W.fp8(base) if fp8 else base
    rng = np.random.default_rng(5)
    system = rng.integers(0, 1000, 300).tolist()
    prompts = [system + rng.integers(0, 1000, int(rng.integers(1, 200))).tolist() for _ in range(6)]
    prompts.append(list(system))                       # the bare system prompt
    prompts.append(system[:150] + [7] + system[151:])  # diverges inside block 9
    NB = 200
    outs = []
    for cached in (True, False):
        cache = PagedKVCache(NB, 16, spec.Hkv, spec.D, W.torch_kv_dtype(spec), "cuda",
                             fill=float("nan"), k_scale=spec.k_scale, v_scale=spec.v_scale,
                             prefix_cache=cached)
        bm = BlockManager(NB, 16)
        if cached:
            bm.enable_prefix_cache()
        ok = np.full((NB, spec.Hkv, 16, spec.D), poison_bits(spec))
        ov = ok.copy()
        computed = []
        for r, toks in enumerate(prompts):
            n_c = cache.add_cached(r, toks)
            assert bm.add_cached(r, toks) == n_c
            k, v = _prefix_kv(toks, spec.Hkv, spec.D, W.torch_dtype(spec))
            slots, pairs = cache.append([r], [len(toks) - n_c], k[n_c:].cuda(), v[n_c:].cuda())
            want_slots, want_pairs = bm.append(r, len(toks) - n_c)
            assert slots == want_slots and pairs == want_pairs == []
            oracle_append(spec, k[n_c:], v[n_c:], ok, ov, want_slots)
            cache.commit(r, toks)
            bm.commit(r, toks)
            computed.append(len(toks) - n_c)
        B = len(prompts)
        tables, lens, max_ctx = cache.tables(list(range(B)))
        ot, ol = bm.build_tables(list(range(B)), tables.shape[1])
        assert np.array_equal(tables.cpu().numpy(), ot) and np.array_equal(lens.cpu().numpy(), ol)
        q = W.q_content(spec, B, "cuda")
        out = cache.decode(q, tables, lens, max_ctx, spec.softmax_scale, partition_size=128)
        torch.cuda.synchronize()
        assert pk.pa_device_status() == 0
        for dev, host in ((cache.k_cache, ok), (cache.v_cache, ov)):
            assert W.storage_view(dev).tobytes() == host.tobytes()
        o = Oracle_view(bm, ok, ov, ot, ol, W.storage_view(q))
        err = np.abs(as_f64(out, spec) - oracle_attention(o, spec)).max()
        assert err <= TOL[spec.dtype]
        if cached:
            # 18 full system blocks are reused by requests 1..5 and 6; the diverging
            # request shares the first 9
            assert computed[0] == len(prompts[0])
            assert all(c == len(p) - 288 for c, p in zip(computed[1:6], prompts[1:6]))
            assert computed[6] == 300 - 288 and computed[7] == 300 - 144
            t = tables.cpu().numpy()
            assert all((t[r, :18] == t[0, :18]).all() for r in range(1, 7))
            assert (t[7, :9] == t[0, :9]).all() and t[7, 9] != t[0, 9]
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


class Oracle_view:
    def __init__(self, bm, k, v, tables, lens, q):
        self.bm, self.k, self.v, self.tables, self.lens, self.q = bm, k, v, tables, lens, q


# ---------------------------------------------------------------------------
# E4M3 cache on the tensor-core kernel (G = 1, 2, 4, 8, D = 128, f16 / bf16 queries)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_tc_edges(dtype, G, bs):
    lens = (0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257, 700)
    spec = W.fp8(W.Spec(f"tc8_{dtype}_{G}_{bs}", dtype, 2 * G, 2, 128, bs, "independent",
                        len(lens), seed=300 + G + bs, ctx_dist="explicit", ctx_list=lens,
                        partition_size=256))
    got, _ = full_check(spec)
    assert np.all(got[0] == 0.0)
    full_check(spec, partition_size=128)
    full_check(spec, partition_size=4096)


@pytest.mark.parametrize("G", [1, 8])
@pytest.mark.parametrize("slope", [0.05, -0.05, 0.004])
@pytest.mark.parametrize("P", [0, 512])
def test_fp8_tc_score_ramps(G, slope, P):
    """Scores that rise along the sequence (the running max is raised in every
    tile, O rescaled each time), fall (every later P far below the first), or
    drift slowly: key j is a_j times a fixed sign pattern, the query that
    pattern, so s_j log2(e) = slope * j up to E4M3 rounding of a_j."""
    rng = np.random.default_rng(443 + G)
    B, Hkv, D, bs, L = 2, 2, 128, 16, (1500, 700)
    Hq = G * Hkv
    nb = [(n + bs - 1) // bs for n in L]
    NB = sum(nb) + 3
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((B, max(nb)), -1, np.int32)
    tables[0, :nb[0]] = perm[:nb[0]]
    tables[1, :nb[1]] = perm[nb[0]:nb[0] + nb[1]]
    sign = np.where(rng.random((Hkv, D)) < 0.5, -1.0, 1.0)
    scale = 1.0 / np.sqrt(D)
    k_scale, v_scale = 0.0123, 0.0171
    # s_j = scale * k_scale * a_j * D, so a_j = slope * j / (log2(e) * scale * k_scale * D)
    j = np.arange(max(L), dtype=np.float64)
    a = slope * (j - (max(L) if slope < 0 else 0)) / (np.log2(np.e) * scale * k_scale * D)
    a = np.clip(a, -440.0, 440.0)
    kf = np.zeros((NB, Hkv, bs, D))
    for b in range(B):
        for t in range(L[b]):
            kf[tables[b, t // bs], :, t % bs, :] = a[t] * sign
    kcodes = oracle.encode_e4m3(kf)
    vcodes = oracle.encode_e4m3(rng.standard_normal((NB, Hkv, bs, D)) / v_scale)
    q = np.repeat(sign[None, :, None, :], B, 0).repeat(G, 2).reshape(B, Hq, D)
    tdt = torch.bfloat16
    qt = torch.tensor(q, dtype=tdt)
    q_bits = W.storage_view(qt)
    lens = np.array(L, np.int32)
    want = oracle.paged_attention(q_bits, kcodes, vcodes, W.DTYPE_CODES["bf16"], tables, lens,
                                  scale, kv_dtype=oracle.E4M3, k_scale=k_scale, v_scale=v_scale)
    f8 = torch.float8_e4m3fn
    kc = torch.from_numpy(kcodes).view(f8).cuda()
    vc = torch.from_numpy(vcodes).view(f8).cuda()
    out = torch.empty((B, Hq, D), dtype=tdt, device="cuda")
    ws = torch.empty(pk.pa_decode_workspace_bytes(B, Hq, D, max(L), P), dtype=torch.uint8,
                     device="cuda")
    pk.pa_decode_fp8(out, qt.cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                     torch.from_numpy(lens).cuda(), scale, max(L), k_scale, v_scale,
                     partition_size=P, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    got = out.double().cpu().numpy()
    err = np.abs(got - want).max()
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("mag", [1e-6, 1e-2, 30.0, 2e3])
def test_fp8_tc_query_magnitudes(dtype, mag):
    """bf16 queries are staged as f16 times a per-head power of two; f16 ones as
    they are: tiny and large queries (near-uniform and near-one-hot softmax)."""
    if dtype == "f16" and mag > 1e3:
        mag = 1e3                                  # f16 q must stay finite
    spec = W.fp8(W.Spec(f"tc8q_{dtype}", dtype, 16, 2, 128, 16, "independent", 6, seed=77,
                        ctx_dist="explicit", ctx_list=(5, 130, 300, 513, 999, 1500),
                        partition_size=512))
    sc = W.scenario(spec)
    p, o = build(sc)
    scale = torch.tensor([mag] + [1.0] * 15, device="cuda").view(1, 16, 1)
    p.q.mul_(scale.to(p.q.dtype))
    o.q = W.storage_view(p.q)
    out = run_step(p, spec)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    got = as_f64(out, spec)
    want = oracle_attention(o, spec)
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[spec.dtype]


# ---------------------------------------------------------------------------
# several new query tokens per sequence (chunked prefill, speculative verify)


def mq_check(spec, qlens, partition_size=512, seed=0, bad_offsets=False):
    sc = W.scenario(spec)
    p, o = build(sc)
    run_step(p, spec)
    torch.cuda.synchronize()
    lens = o.lens.astype(np.int64)
    qlens = np.minimum(np.asarray(qlens, dtype=np.int64), lens)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((T, spec.Hq, spec.D), generator=g, device="cuda").to(W.torch_dtype(spec))
    out = torch.full_like(q, float("nan"))
    maxq = max(1, int(qlens.max()))
    n = pk.pa_decode_multi_workspace_bytes(T, spec.Hq, spec.D, p.max_ctx, partition_size)
    ws = torch.empty(n // 4, dtype=torch.float32, device="cuda") if n else None
    qs_dev = torch.from_numpy(qs).cuda()
    if bad_offsets:
        qs_dev[1] = qs_dev[2] + 1                  # not non-decreasing
    pk.pa_decode_multi(out, q, p.cache.k_cache, p.cache.v_cache, p.tables, p.lens, qs_dev,
                       spec.softmax_scale, p.max_ctx, maxq, partition_size=partition_size,
                       workspace=ws)
    torch.cuda.synchronize()
    if bad_offsets:
        return out, pk.pa_device_status()
    assert pk.pa_device_status() == 0
    got = as_f64(out, spec)
    want = oracle.paged_attention_mq(W.storage_view(q), o.k, o.v, spec.dtype_code, o.tables,
                                     o.lens, qs, spec.softmax_scale)
    assert np.isfinite(got).all()
    err = np.abs(got - want).max() if T else 0.0
    assert err <= TOL[spec.dtype], err
    return got, want


def mq_spec(dtype, G, bs, lens, seed, P=512):
    return W.Spec(f"mq_{dtype}_{G}_{bs}", dtype, 2 * G, 2, 128, bs, "independent", len(lens),
                  seed=seed, ctx_dist="explicit", ctx_list=tuple(lens), partition_size=P)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("P", [128, 512])
def test_mq_speculative_verify(dtype, G, P):
    spec = mq_spec(dtype, G, 16, (5, 40, 300, 513, 1100, 2000), seed=500 + G)
    mq_check(spec, (1, 4, 8, 3, 8, 5), partition_size=P)


@pytest.mark.parametrize("G", [1, 4, 8])
def test_mq_chunked_prefill(G):
    """Whole prompts and long chunks as queries: several query blocks per
    sequence (128/G tokens each) and several key partitions."""
    spec = mq_spec("bf16", G, 16, (200, 700, 1500, 90), seed=600 + G)
    mq_check(spec, (200, 300, 260, 90), partition_size=256)


@pytest.mark.parametrize("bs", [8, 32])
def test_mq_block_sizes(bs):
    spec = mq_spec("f16", 4, bs, (33, 257, 1000), seed=700 + bs)
    mq_check(spec, (33, 20, 129), partition_size=128)


def test_mq_edges():
    spec = mq_spec("bf16", 8, 16, (0, 1, 2, 127, 128, 129, 255), seed=801)
    mq_check(spec, (0, 1, 2, 127, 1, 129, 16), partition_size=128)


def test_mq_bad_offsets_are_flagged_without_faulting():
    spec = mq_spec("bf16", 4, 16, (50, 60, 70), seed=802)
    _, status = mq_check(spec, (3, 4, 5), bad_offsets=True)
    assert status & pk.PA_DEVERR_CONTEXT
    mq_check(spec, (3, 4, 5))                      # the context is still healthy


# ---------------------------------------------------------------------------
# the tcgen05 decode kernels streaming several partitions per CTA (chosen when the
# grid has at least 8 CTAs per SM) with one softmax: the merged partial and the
# empty partials of the span's other partitions must give the right result


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("P", [128, 256, 512])
def test_tc_several_partitions_per_cta(P, fp8):
    spec = W.Spec(f"ppc_{P}", "bf16", 32, 4, 128, 16, "independent", 320, seed=900 + P,
                  ctx_dist="uniform", ctx_lo=1, ctx_hi=2000, partition_size=P)
    spec = W.fp8(spec) if fp8 else spec
    sc = W.scenario(spec)
    p, o = build(sc)
    # a workspace full of NaN: every slot the reduce reads must have been written
    ws = p.cache.workspace(p.q.shape[0], p.q.shape[1], p.max_ctx, P)
    ws.fill_(float("nan"))
    out = run_step(p, spec, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    rows = sampled_rows(o, spec, n=160, seed=P)
    want = oracle_attention(o, spec, rows=rows)
    got_all = as_f64(out, spec)
    assert np.isfinite(got_all).all()
    assert np.abs(got_all[rows[:, 0], rows[:, 1]] - want).max() <= TOL[spec.dtype]
    # the same batch at one partition per CTA (long partitions) agrees
    out2 = run_step(p, spec, partition_size=4096)
    torch.cuda.synchronize()
    assert np.abs(as_f64(out2, spec) - got_all).max() <= TOL[spec.dtype]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [4, 8])
@pytest.mark.parametrize("P", [128, 512])
def test_mq_few_queries_token_major(dtype, G, P):
    """Q * G <= 16 takes the decode kernel with per-column causal limits."""
    spec = mq_spec(dtype, G, 16, (5, 40, 300, 513, 1100, 2000, 1, 2), seed=950 + G + P)
    qlens = (1, 4, 2, 3, 4, 1, 1, 2) if G == 4 else (1, 2, 2, 1, 2, 2, 1, 2)
    mq_check(spec, qlens, partition_size=P)


def test_mq_few_queries_several_partitions_per_cta():
    spec = W.Spec("mq_ppc", "bf16", 32, 4, 128, 16, "independent", 320, seed=977,
                  ctx_dist="uniform", ctx_lo=2, ctx_hi=2000, partition_size=128)
    mq_check(spec, [1 + (i % 4) for i in range(320)], partition_size=128)


# Repeated launches on the same inputs: every run finite and byte-identical to
# the first.  A missed wait between an asynchronous copy and the threads that
# patch its shared-memory tile shows up as an occasional run that differs (the
# cache's unused slots hold NaN, so a patch overtaken by a late copy turns the
# output non-finite); a single launch catches it only by chance.

REPEATS = 24


def _repeat_identical(launch):
    first = launch().clone()
    torch.cuda.synchronize()
    assert pk.pa_device_status() == 0
    assert torch.isfinite(first.float()).all()
    bad = 0
    for _ in range(REPEATS):
        again = launch()
        torch.cuda.synchronize()
        bad += int(not torch.equal(first.view(torch.int16), again.view(torch.int16)))
    assert pk.pa_device_status() == 0
    assert bad == 0, f"{bad} of {REPEATS} runs differ from the first"
    return first


@pytest.mark.parametrize("G,qmax", [(8, 4), (8, 2), (4, 4), (4, 8)])
def test_repeated_multi_query_launches_are_identical(G, qmax):
    """Token-major multi-query decode at N = 16 and N = 32 columns (two-slot
    ring), short last tiles after full ones."""
    n = 160
    spec = W.Spec(f"rep_mq_{G}_{qmax}", "bf16", 4 * G, 4, 128, 16, "independent", n,
                  seed=1200 + G + qmax, ctx_dist="uniform", ctx_lo=130, ctx_hi=1500,
                  partition_size=128)
    p, o = build(W.scenario(spec))
    run_step(p, spec)
    torch.cuda.synchronize()
    qlens = np.array([1 + (i % qmax) for i in range(n)], dtype=np.int64)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator(device="cuda").manual_seed(G)
    q = torch.randn((T, spec.Hq, spec.D), generator=g, device="cuda").to(W.torch_dtype(spec))
    qs_dev = torch.from_numpy(qs).cuda()
    ws_n = pk.pa_decode_multi_workspace_bytes(T, spec.Hq, spec.D, p.max_ctx, 128)
    ws = torch.empty(ws_n // 4, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)

    def launch():
        ws.fill_(float("nan"))
        pk.pa_decode_multi(out, q, p.cache.k_cache, p.cache.v_cache, p.tables, p.lens, qs_dev,
                           spec.softmax_scale, p.max_ctx, qmax, partition_size=128, workspace=ws)
        return out

    got = as_f64(_repeat_identical(launch), spec)
    want = oracle.paged_attention_mq(W.storage_view(q), o.k, o.v, spec.dtype_code, o.tables,
                                     o.lens, qs, spec.softmax_scale)
    assert np.abs(got - want).max() <= TOL[spec.dtype]


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_repeated_decode_launches_are_identical(dtype, fp8):
    """The tcgen05 decode kernels (E4M3: three-slot rings for f16 queries,
    two-slot rings for bf16 queries)."""
    spec = W.Spec(f"rep_dec_{dtype}", dtype, 32, 4, 128, 16, "independent", 256,
                  seed=1300 + fp8, ctx_dist="uniform", ctx_lo=130, ctx_hi=3000,
                  partition_size=512)
    spec = W.fp8(spec) if fp8 else spec
    p, o = build(W.scenario(spec))
    run_step(p, spec)
    torch.cuda.synchronize()
    ws = p.cache.workspace(p.q.shape[0], p.q.shape[1], p.max_ctx, 512)
    out = torch.empty_like(p.q)

    def launch():
        return p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale, out=out,
                              partition_size=512, workspace=ws)

    got = as_f64(_repeat_identical(launch), spec)
    rows = sampled_rows(o, spec, n=96, seed=5)
    want = oracle_attention(o, spec, rows=rows)
    assert np.abs(got[rows[:, 0], rows[:, 1]] - want).max() <= TOL[spec.dtype]


@pytest.mark.parametrize("dtype,G,samples", [("bf16", 1, 6), ("f16", 2, 4), ("bf16", 1, 20)])
def test_repeated_grouped_launches_are_identical(dtype, G, samples):
    """The grouped decode's span kernel at G = 1, 2 (rings of two tiles, three
    CTAs per SM; 8 / G or 16 / G members per CTA) and the rest kernel, with
    spans whose last tile is partial: every run finite and byte-identical."""
    spec = W.Spec(f"rep_grp_{G}_{samples}", dtype, 4 * G, 4, 128, 16, "parallel_sampling",
                  4 * samples, seed=1400 + G + samples, num_prompts=4,
                  samples_per_prompt=samples, prompt_lo=300, prompt_hi=900, div_lo=1,
                  div_hi=200, partition_size=0)
    p, o = build(W.scenario(spec))
    run_step(p, spec)
    torch.cuda.synchronize()
    groups = p.cache.groups(p.tables, p.lens)
    assert groups.max_shared_len > 0 and groups.max_group_size == samples
    ws = p.cache.grouped_workspace(p.q.shape[0], p.q.shape[1], p.max_ctx, groups, 0)
    out = torch.empty_like(p.q)

    def launch():
        ws.fill_(float("nan"))
        return p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale, out=out,
                              workspace=ws, groups=groups)

    got = as_f64(_repeat_identical(launch), spec)
    want = oracle_attention(o, spec)
    assert np.abs(got - want).max() <= TOL[spec.dtype]
