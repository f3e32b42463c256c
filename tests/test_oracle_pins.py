"""Pins of the oracle against what the pages and mathematics fix (CPU only).

Each pin comes from outside the oracle: a library routine (torch's fp64
scaled-dot-product attention, numpy's / torch's float decoders), a closed form,
the worked block-table example of the hjr-study-book Day 3 page, or an
invariant the pages state.  The last group plants plausible mistakes in a copy
of the oracle's steps and checks that the pins catch every one of them.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import kv_size

from pa_testlib import read_golden  # noqa: E402


# ---------------------------------------------------------------------------
# helpers: build a paged cache from contiguous per-sequence K/V (test side)


def paged_from_contiguous(Ks, Vs, bs, num_blocks, rng, fill=np.nan):
    """Scatter contiguous K/V ([L, Hkv, D] per sequence) into a [NB, Hkv, bs, D]
    cache at randomly chosen physical blocks; unused slots hold ``fill``."""
    B = len(Ks)
    Hkv, D = Ks[0].shape[1], Ks[0].shape[2]
    need = [-(-K.shape[0] // bs) for K in Ks]
    maxb = max(1, max(need))
    ids = rng.permutation(num_blocks)[: sum(need)]
    tables = np.full((B, maxb), -1, dtype=np.int32)
    kc = np.full((num_blocks, Hkv, bs, D), fill, dtype=np.float32)
    vc = np.full((num_blocks, Hkv, bs, D), fill, dtype=np.float32)
    pos = 0
    for b in range(B):
        for i in range(need[b]):
            tables[b, i] = ids[pos]
            pos += 1
        for j in range(Ks[b].shape[0]):
            kc[tables[b, j // bs], :, j % bs, :] = Ks[b][j]
            vc[tables[b, j // bs], :, j % bs, :] = Vs[b][j]
    lens = np.array([K.shape[0] for K in Ks], dtype=np.int32)
    return kc, vc, tables, lens


def sdpa_reference(q, Ks, Vs, scale):
    """torch's scaled_dot_product_attention in float64 on contiguous K/V; query
    head h uses kv head h // G (enable_gqa)."""
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        if Ks[b].shape[0] == 0:
            continue
        qq = torch.from_numpy(q[b].astype(np.float64))[None, :, None, :]
        kk = torch.from_numpy(Ks[b].astype(np.float64)).permute(1, 0, 2)[None]
        vv = torch.from_numpy(Vs[b].astype(np.float64)).permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(qq, kk, vv, scale=scale, enable_gqa=True)
        out[b] = o[0, :, 0, :].numpy()
    return out


def random_case(rng, B=5, Hq=4, Hkv=2, D=16, bs=8, lmax=70, lmin=1):
    lens = rng.integers(lmin, lmax + 1, size=B)
    Ks = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    nb = sum(-(-int(L) // bs) for L in lens) + 7
    return q, Ks, Vs, nb


# ---------------------------------------------------------------------------
# decoders


def test_f16_decoder_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, oracle.F16)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_bf16_decoder_exhaustive_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, oracle.BF16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


# ---------------------------------------------------------------------------
# attention against a library routine


@pytest.mark.parametrize("B,Hq,Hkv,D,bs,lmax", [
    (5, 4, 4, 16, 8, 70), (4, 8, 2, 32, 16, 100), (3, 8, 1, 8, 32, 90), (6, 6, 3, 64, 16, 40),
])
def test_attention_matches_torch_sdpa(B, Hq, Hkv, D, bs, lmax):
    rng = np.random.default_rng(100 + B * Hq + bs)
    q, Ks, Vs, nb = random_case(rng, B, Hq, Hkv, D, bs, lmax)
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, bs, nb, rng)
    scale = 1.0 / np.sqrt(D)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, scale)
    want = sdpa_reference(q, Ks, Vs, scale)
    assert np.abs(got - want).max() < 1e-12


def test_attention_bf16_storage_matches_sdpa_on_decoded_values():
    rng = np.random.default_rng(7)
    q, Ks, Vs, nb = random_case(rng, 4, 8, 2, 32, 16, 60)
    to_bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    back = lambda t: t.to(torch.float32).numpy()
    Kb = [to_bf(K) for K in Ks]
    Vb = [to_bf(V) for V in Vs]
    qb = to_bf(q)
    kc, vc, tables, lens = paged_from_contiguous([back(K) for K in Kb], [back(V) for V in Vb],
                                                 16, nb, rng, fill=0.0)
    kcb, vcb = bits(torch.from_numpy(kc).to(torch.bfloat16)), bits(torch.from_numpy(vc).to(torch.bfloat16))
    got = oracle.paged_attention(bits(qb), kcb, vcb, oracle.BF16, tables, lens, 0.25)
    want = sdpa_reference(back(qb), [back(K) for K in Kb], [back(V) for V in Vb], 0.25)
    assert np.abs(got - want).max() < 1e-12


# ---------------------------------------------------------------------------
# closed forms and special cases


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(1)
    q, Ks, Vs, nb = random_case(rng, 4, 4, 4, 16, 16, lmax=1, lmin=1)
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 16, nb, rng)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, 0.25)
    for b in range(4):
        assert np.array_equal(got[b], Vs[b][0].astype(np.float64))


def test_equal_keys_and_zero_query_give_mean_of_values():
    rng = np.random.default_rng(2)
    L, Hkv, D = 45, 2, 16
    k = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    Ks = [np.repeat(k, L, axis=0)]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(np.float32)]
    q = rng.standard_normal((1, 4, D)).astype(np.float32)
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 8, 20, rng)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, 0.3)
    mean = Vs[0].astype(np.float64).mean(axis=0)          # [Hkv, D]
    for h in range(4):
        assert np.abs(got[0, h] - mean[h // 2]).max() < 1e-13
    q0 = np.zeros_like(q)
    Ks2 = [rng.standard_normal((L, Hkv, D)).astype(np.float32)]
    kc, vc, tables, lens = paged_from_contiguous(Ks2, Vs, 8, 20, rng)
    got = oracle.paged_attention(q0, kc, vc, oracle.F32, tables, lens, 0.3)
    for h in range(4):
        assert np.abs(got[0, h] - mean[h // 2]).max() < 1e-13


def test_two_tokens_hand_computed():
    # q = (1, 2), k0 = (1, 0), k1 = (0, 1), scale 0.5: s0 = 0.5, s1 = 1.0,
    # w0 = 1 / (1 + e^{0.5}), w1 = 1 - w0; v0 = (2, 0), v1 = (0, 4).
    q = np.array([[[1.0, 2.0]]], dtype=np.float32)
    Ks = [np.array([[[1.0, 0.0]], [[0.0, 1.0]]], dtype=np.float32)]
    Vs = [np.array([[[2.0, 0.0]], [[0.0, 4.0]]], dtype=np.float32)]
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 8, 3, np.random.default_rng(0))
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, 0.5)[0, 0]
    w0 = 1.0 / (1.0 + np.exp(0.5))
    assert abs(got[0] - 2.0 * w0) < 1e-15 and abs(got[1] - 4.0 * (1 - w0)) < 1e-15


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    L, D = 33, 8
    Ks = [rng.standard_normal((L, 1, D)).astype(np.float32) * 0.01]
    Vs = [rng.standard_normal((L, 1, D)).astype(np.float32)]
    q = np.ones((1, 1, D), dtype=np.float32)
    Ks[0][17, 0, :] = 100.0
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 16, 5, rng)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, 1.0)
    assert np.abs(got[0, 0] - Vs[0][17, 0]).max() < 1e-12


def test_zero_context_gives_zero_row():
    rng = np.random.default_rng(4)
    q, Ks, Vs, nb = random_case(rng, 3, 2, 2, 8, 8, 20)
    Ks[1] = Ks[1][:0]
    Vs[1] = Vs[1][:0]
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 8, nb, rng)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, lens, 0.3)
    assert np.all(got[1] == 0.0)


# ---------------------------------------------------------------------------
# invariants the pages state


def test_physical_placement_does_not_matter():
    """"PagedAttention의 설계": logical order is kept whatever the physical
    blocks; permuting physical ids leaves the result bit-identical."""
    rng = np.random.default_rng(5)
    q, Ks, Vs, nb = random_case(rng, 5, 4, 2, 16, 8, 80)
    kc1, vc1, t1, l1 = paged_from_contiguous(Ks, Vs, 8, nb, np.random.default_rng(11))
    kc2, vc2, t2, l2 = paged_from_contiguous(Ks, Vs, 8, nb, np.random.default_rng(12))
    assert not np.array_equal(t1, t2)
    o1 = oracle.paged_attention(q, kc1, vc1, oracle.F32, t1, l1, 0.2)
    o2 = oracle.paged_attention(q, kc2, vc2, oracle.F32, t2, l2, 0.2)
    assert np.array_equal(o1, o2)


def test_block_size_does_not_matter():
    rng = np.random.default_rng(6)
    q, Ks, Vs, nb = random_case(rng, 4, 4, 4, 16, 8, 90)
    outs = []
    for bs in (8, 16, 32):
        kc, vc, t, l = paged_from_contiguous(Ks, Vs, bs, nb, np.random.default_rng(bs))
        outs.append(oracle.paged_attention(q, kc, vc, oracle.F32, t, l, 0.25))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_unused_tail_slots_are_never_read():
    """"PagedAttention의 설계": the last block may hold unused slots; poisoning
    them with NaN / inf must not change anything."""
    rng = np.random.default_rng(8)
    q, Ks, Vs, nb = random_case(rng, 5, 4, 2, 16, 16, 75)
    kc, vc, t, l = paged_from_contiguous(Ks, Vs, 16, nb, np.random.default_rng(1), fill=0.0)
    kn, vn, _, _ = paged_from_contiguous(Ks, Vs, 16, nb, np.random.default_rng(1), fill=np.nan)
    kn[np.isnan(kn)] = np.inf
    o1 = oracle.paged_attention(q, kc, vc, oracle.F32, t, l, 0.25)
    o2 = oracle.paged_attention(q, kn, vn, oracle.F32, t, l, 0.25)
    assert np.array_equal(o1, o2) and np.isfinite(o2).all()


def test_shared_prefix_blocks_equal_private_copies():
    """"블록 공유": sequences that point at the same prefix blocks get the same
    result as sequences holding private copies of the prefix."""
    rng = np.random.default_rng(9)
    bs, Hkv, D, P = 8, 2, 16, 24
    pre_k = rng.standard_normal((P, Hkv, D)).astype(np.float32)
    pre_v = rng.standard_normal((P, Hkv, D)).astype(np.float32)
    sfx = [rng.integers(1, 30) for _ in range(3)]
    Ks = [np.concatenate([pre_k, rng.standard_normal((s, Hkv, D)).astype(np.float32)]) for s in sfx]
    Vs = [np.concatenate([pre_v, rng.standard_normal((s, Hkv, D)).astype(np.float32)]) for s in sfx]
    q = rng.standard_normal((3, 4, D)).astype(np.float32)
    kc, vc, t, l = paged_from_contiguous(Ks, Vs, bs, 60, rng)
    private = oracle.paged_attention(q, kc, vc, oracle.F32, t, l, 0.25)
    # share: point every sequence's first P/bs table entries at sequence 0's blocks
    t2 = t.copy()
    t2[1:, : P // bs] = t[0, : P // bs]
    kc2, vc2 = kc.copy(), vc.copy()
    for b in (1, 2):
        for i in range(P // bs):
            kc2[t[b, i]] = np.nan
            vc2[t[b, i]] = np.nan
    shared = oracle.paged_attention(q, kc2, vc2, oracle.F32, t2, l, 0.25)
    assert np.array_equal(private, shared)


def test_out_of_range_table_is_rejected():
    rng = np.random.default_rng(10)
    q, Ks, Vs, nb = random_case(rng, 2, 2, 2, 8, 8, 20)
    kc, vc, t, l = paged_from_contiguous(Ks, Vs, 8, nb, rng)
    t = t.copy()
    t[0, 0] = nb
    with pytest.raises(ValueError):
        oracle.paged_attention(q, kc, vc, oracle.F32, t, l, 0.3)


# ---------------------------------------------------------------------------
# append and copy-on-write


def test_worked_block_table_example_slots():
    """The 37-token request of "4.2 PagedAttention의 접근": logical blocks 0, 1, 2
    in physical blocks 7, 2, 9, five tokens in the last one."""
    g = read_golden("block_table_example.txt")
    bs, L = g["block_size"][0], g["seq_len"][0]
    table = g["table"]
    NB, Hkv, D = 12, 2, 4
    # token t carries the value t in every element, so placement is visible
    key = np.repeat(np.arange(L, dtype=np.float32)[:, None, None], Hkv, 1).repeat(D, 2)
    kc = np.full((NB, Hkv, bs, D), -1.0, dtype=np.float32)
    vc = kc.copy()
    slots = np.array([table[t // bs] * bs + t % bs for t in range(L)], dtype=np.int64)
    assert slots[36] == 9 * 16 + 4 == 148
    oracle.reshape_and_cache(key, key + 0.5, kc, vc, slots, oracle.F32)
    for i, phys in enumerate(table):
        used = min(bs, L - i * bs)
        assert np.all(kc[phys, :, :used, 0] == np.arange(i * bs, i * bs + used)[None, :])
        assert np.all(vc[phys, :, :used, 0] == np.arange(i * bs, i * bs + used)[None, :] + 0.5)
        assert np.all(kc[phys, :, used:, :] == -1.0)
    assert L - (len(table) - 1) * bs == g["last_block_tokens"][0]
    untouched = [b for b in range(NB) if b not in table]
    assert np.all(kc[untouched] == -1.0)


def test_append_then_attend_matches_sdpa():
    """Tokens written one decode step at a time ("1. KV 캐시란": the new K, V
    pair is stored every step) and then attended over equal SDPA on the
    contiguous tokens."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, D, bs = 3, 4, 2, 16, 8
    lens = [13, 1, 30]
    NB = 12
    order = rng.permutation(NB)
    tables = np.full((B, 4), -1, dtype=np.int32)
    kc = np.full((NB, Hkv, bs, D), np.nan, dtype=np.float32)
    vc = kc.copy()
    Ks = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    nxt = 0
    for step in range(max(lens)):
        slots, keys, vals = [], [], []
        for b in range(B):
            if step >= lens[b]:
                slots.append(-1)   # finished sequence: nothing to store
            else:
                if step % bs == 0:
                    tables[b, step // bs] = order[nxt]
                    nxt += 1
                slots.append(int(tables[b, step // bs]) * bs + step % bs)
            keys.append(Ks[b][min(step, lens[b] - 1)])
            vals.append(Vs[b][min(step, lens[b] - 1)])
        oracle.reshape_and_cache(np.stack(keys), np.stack(vals), kc, vc, np.array(slots), oracle.F32)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    got = oracle.paged_attention(q, kc, vc, oracle.F32, tables, np.array(lens), 0.25)
    want = sdpa_reference(q, Ks, Vs, 0.25)
    assert np.abs(got - want).max() < 1e-12


def test_negative_slot_is_skipped_and_bad_slot_rejected():
    kc = np.zeros((2, 1, 4, 2), dtype=np.float32)
    vc = kc.copy()
    key = np.ones((2, 1, 2), dtype=np.float32)
    oracle.reshape_and_cache(key, key, kc, vc, np.array([-1, -5]), oracle.F32)
    assert np.all(kc == 0)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, key, kc, vc, np.array([0, 8]), oracle.F32)


def test_copy_on_write_leaves_source_and_sharers_unchanged():
    """"블록 공유" / copy-on-write: copying the shared partial block gives the
    writer a private block; the source block and the other sharer's result
    do not change, and the writer's result equals SDPA on its own tokens."""
    rng = np.random.default_rng(13)
    bs, Hkv, D, NB = 8, 2, 8, 10
    P = 11                                   # prompt ends inside block 1
    pk = rng.standard_normal((P, Hkv, D)).astype(np.float32)
    pv = rng.standard_normal((P, Hkv, D)).astype(np.float32)
    kc = np.full((NB, Hkv, bs, D), np.nan, dtype=np.float32)
    vc = kc.copy()
    oracle.reshape_and_cache(pk, pv, kc, vc, np.array([3 * bs + t if t < bs else 6 * bs + t - bs
                                                       for t in range(P)]), oracle.F32)
    table_parent = np.array([[3, 6]], dtype=np.int32)
    q = rng.standard_normal((1, 2, D)).astype(np.float32)
    before = oracle.paged_attention(q, kc, vc, oracle.F32, table_parent, np.array([P]), 0.3)
    src_bytes = kc[6].tobytes() + vc[6].tobytes()
    # child writes a new token into the shared block 6 -> copy it to block 8 first
    oracle.copy_blocks(kc, vc, np.array([[6, 8]]), oracle.F32)
    assert kc[8].tobytes() + vc[8].tobytes() == src_bytes
    nk = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    nv = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    oracle.reshape_and_cache(nk, nv, kc, vc, np.array([8 * bs + (P - bs)]), oracle.F32)
    assert kc[6].tobytes() + vc[6].tobytes() == src_bytes
    after = oracle.paged_attention(q, kc, vc, oracle.F32, table_parent, np.array([P]), 0.3)
    assert np.array_equal(before, after)
    child = oracle.paged_attention(q, kc, vc, oracle.F32, np.array([[3, 8]], dtype=np.int32),
                                   np.array([P + 1]), 0.3)
    want = sdpa_reference(q, [np.concatenate([pk, nk])], [np.concatenate([pv, nv])], 0.3)
    assert np.abs(child - want).max() < 1e-12


def test_copy_blocks_rejects_bad_ids():
    kc = np.zeros((2, 1, 4, 2), dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, kc.copy(), np.array([[0, 2]]), oracle.F32)


# ---------------------------------------------------------------------------
# KV size formula


def test_kv_size_formula_matches_opt13b_figure():
    g = read_golden("kv_size.txt")
    n = kv_size.kv_cache_bytes(g["num_layers"][0], g["num_heads"][0], g["head_dim"][0],
                               g["seq_len"][0], g["dtype_bytes"][0])
    assert n == 1_677_721_600
    about = g["about_gb"][0]
    # "about 1.6 GB": within 10% either way (1.68e9 B = 1.56 GiB)
    assert abs(n / 1e9 - about) / about < 0.1 and abs(n / 2**30 - about) / about < 0.1
    assert kv_size.kv_bytes_per_token(40, 128, 2) == 20480


# ---------------------------------------------------------------------------
# negative controls: plausible mistakes in a copy of the oracle's steps must
# each fail one of the pins above


def _mutant_attention(q, kc, vc, tables, lens, scale, mistake):
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = int(lens[b])
        n_attend = L - 1 if mistake == "drop_last" else L
        if mistake == "read_tail":
            n_attend = -(-L // bs) * bs
        for h in range(Hq):
            g = h % Hkv if mistake == "head_mod" else h // G
            K = np.zeros((n_attend, D))
            V = np.zeros((n_attend, D))
            for j in range(n_attend):
                blk, off = (j // bs, j % bs) if mistake != "swap_idx" else (j % bs, j // bs)
                blk = min(blk, tables.shape[1] - 1)
                off = min(off, bs - 1)
                K[j] = kc[tables[b, blk], g, off]
                V[j] = vc[tables[b, blk], g, off]
            s = (K @ q[b, h].astype(np.float64)) * (1.0 if mistake == "no_scale" else scale)
            if mistake == "per_block_softmax":
                o = np.zeros(D)
                for start in range(0, n_attend, bs):
                    ss = s[start:start + bs]
                    w = np.exp(ss - ss.max())
                    o += (w / w.sum()) @ V[start:start + bs]
                out[b, h] = o
                continue
            w = np.exp(s - s.max())
            if mistake == "unnormalised":
                out[b, h] = w @ V
            else:
                out[b, h] = (w / w.sum()) @ V
    return out


@pytest.mark.parametrize("mistake", ["per_block_softmax", "head_mod", "swap_idx", "no_scale",
                                     "drop_last", "read_tail", "unnormalised"])
def test_pins_catch_planted_mistakes(mistake):
    rng = np.random.default_rng(21)
    q, Ks, Vs, nb = random_case(rng, 5, 4, 2, 16, 8, 60, lmin=9)
    kc, vc, tables, lens = paged_from_contiguous(Ks, Vs, 8, nb, rng, fill=np.nan)
    want = sdpa_reference(q, Ks, Vs, 0.25)
    good = _mutant_attention(q, kc, vc, tables, lens, 0.25, mistake=None)
    assert np.abs(good - want).max() < 1e-12          # the unmutated copy passes
    bad = _mutant_attention(q, kc, vc, tables, lens, 0.25, mistake=mistake)
    caught = (not np.all(np.isfinite(bad))) or np.abs(bad - want).max() > 1e-6
    assert caught, mistake


def test_swap_out_and_back_in_restores_attention():
    """"적용 범위와 관련 연구": a sequence swapped out to host memory and back in
    (into other physical blocks) attends exactly as before; the host copy holds
    the blocks' bytes, and blocks not named are untouched."""
    rng = np.random.default_rng(31)
    q, Ks, Vs, nb = random_case(rng, 3, 4, 2, 16, 8, 60, lmin=20)
    kc, vc, t, l = paged_from_contiguous(Ks, Vs, 8, nb + 20, rng)
    before = oracle.paged_attention(q, kc, vc, oracle.F32, t, l, 0.25)
    b = 1
    blocks = [int(x) for x in t[b, : -(-int(l[b]) // 8)]]
    host_k = np.zeros((len(blocks) + 3,) + kc.shape[1:], dtype=np.float32)
    host_v = host_k.copy()
    out_pairs = np.array([[blk, i + 3] for i, blk in enumerate(blocks)])
    oracle.swap_blocks(host_k, host_v, kc, vc, out_pairs, oracle.F32)
    for i, blk in enumerate(blocks):
        assert host_k[i + 3].tobytes() == kc[blk].tobytes()
    assert np.all(host_k[:3] == 0)
    # the device blocks are recycled: poison them, then swap back into fresh ids
    used = set(int(x) for x in t[t >= 0])
    free = [x for x in range(kc.shape[0]) if x not in used]
    kc[blocks] = np.nan
    vc[blocks] = np.nan
    new_ids = free[: len(blocks)]
    oracle.swap_blocks(kc, vc, host_k, host_v,
                       np.array([[i + 3, nid] for i, nid in enumerate(new_ids)]), oracle.F32)
    t2 = t.copy()
    t2[b, : len(blocks)] = new_ids
    after = oracle.paged_attention(q, kc, vc, oracle.F32, t2, l, 0.25)
    assert np.array_equal(before[b], after[b])
    assert np.array_equal(np.delete(before, b, 0), np.delete(after, b, 0))
    with pytest.raises(ValueError):
        oracle.swap_blocks(host_k, host_v, kc, vc, np.array([[0, host_k.shape[0]]]), oracle.F32)


# ---------------------------------------------------------------------------
# E4M3 KV cache: the format's fixed points, torch's own float8_e4m3fn casts,
# brute-force nearest codes, and attention identities.


def _all_codes():
    return np.arange(256, dtype=np.uint8)


def test_e4m3_fixed_points_of_the_format():
    g = read_golden("e4m3_points.txt")
    for name, vals in g.items():
        code = vals[0]
        v = oracle.decode(np.array([code], dtype=np.uint8), oracle.E4M3)[0]
        if name == "nan":
            assert np.isnan(v)
            continue
        assert v == vals[1], name
        assert oracle.encode_e4m3(np.array([vals[1]]))[0] == code, name


def test_e4m3_decode_matches_torch_for_every_code():
    codes = _all_codes()
    ours = oracle.decode(codes, oracle.E4M3)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], theirs[~nan])
    # every finite code survives decode -> encode, -0 included
    back = oracle.encode_e4m3(ours[~nan])
    assert np.array_equal(back, codes[~nan])


def test_e4m3_encode_matches_torch_cast_and_rounds_ties_to_even():
    rng = np.random.default_rng(8)
    finite = oracle.decode(_all_codes(), oracle.E4M3)
    grid = np.unique(finite[np.isfinite(finite) & (finite >= 0)])       # 0 .. 448
    mids = (grid[:-1] + grid[1:]) / 2                                     # exact ties
    x = np.concatenate([
        rng.standard_normal(50000) * 10.0 ** rng.uniform(-3, 2.4, 50000),
        rng.uniform(-447.9, 447.9, 20000),
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1000), grid, -grid,
    ]).astype(np.float32)
    x = x[np.abs(x) < 448]
    ours = oracle.encode_e4m3(x.astype(np.float64))
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)
    # a tie goes to the neighbour whose fraction field is even
    t = oracle.encode_e4m3(mids)
    assert np.all((t & 1) == 0)


def test_e4m3_saturates_instead_of_overflowing():
    big = np.array([448.0, 449.0, 464.0, 479.9, 480.0, 1e6, np.inf])
    assert np.all(oracle.encode_e4m3(big) == 0x7e)
    assert np.all(oracle.encode_e4m3(-big) == 0xfe)


def _nearest_code_brute_force(q):
    """Nearest finite E4M3 value to each q by scanning all codes; ties to the
    even fraction field; |q| beyond 448 to +-448."""
    codes = _all_codes()
    vals = oracle.decode(codes, oracle.E4M3)
    ok = np.isfinite(vals)
    codes, vals = codes[ok], vals[ok]
    out = np.empty(q.shape, dtype=np.uint8)
    for i, v in enumerate(q.ravel()):
        v = min(max(float(v), -448.0), 448.0)
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        cand = codes[best]
        if len(cand) > 1:                       # +-0, or a tie between two codes
            same = [c for c in cand if (c & 0x80) == (0x80 if np.signbit(v) else 0)]
            cand = np.array(same or list(cand), dtype=np.uint8)
            even = [c for c in cand if (c & 1) == 0]
            cand = np.array(even or list(cand), dtype=np.uint8)
        out.ravel()[i] = cand[0]
    return out


@pytest.mark.parametrize("dtype", [oracle.F32, oracle.F16, oracle.BF16])
def test_e4m3_append_stores_nearest_code_of_the_fp32_quotient(dtype):
    rng = np.random.default_rng(40 + dtype)
    N, Hkv, D, bs, NB = 5, 2, 64, 8, 6
    tdt = {oracle.F32: torch.float32, oracle.F16: torch.float16, oracle.BF16: torch.bfloat16}[dtype]
    k = torch.from_numpy(rng.standard_normal((N, Hkv, D)) * 30).to(tdt)
    v = torch.from_numpy(rng.standard_normal((N, Hkv, D)) * 0.01).to(tdt)
    k[0, 0, :4] = torch.tensor([1e4, -1e4, 0.0, -0.0])             # saturate, signed zeros
    k_scale, v_scale = np.float32(0.37), np.float32(1.0 / 64)
    kc = np.zeros((NB, Hkv, bs, D), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.array([3, 17, -1, 40, 0], dtype=np.int64)
    st = lambda t: t.view(torch.int16).numpy().view(np.uint16) if t.dtype != torch.float32 else t.numpy()
    oracle.reshape_and_cache_e4m3(st(k), st(v), kc, vc, slots, dtype, k_scale, v_scale)
    kf = k.to(torch.float32).numpy()
    vf = v.to(torch.float32).numpy()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        blk, off = divmod(int(s), bs)
        want_k = _nearest_code_brute_force(kf[t] / k_scale)       # float32 / float32
        want_v = _nearest_code_brute_force(vf[t] / v_scale)
        assert np.array_equal(kc[blk, :, off], want_k)
        assert np.array_equal(vc[blk, :, off], want_v)
    assert kc[0, 0, 3, :4].tolist() == [0x7e, 0xfe, 0x00, 0x80]     # token 0 sits in slot 3
    # untouched slots stay as they were
    assert kc[1].sum() == 0
    with pytest.raises(ValueError):
        oracle.reshape_and_cache_e4m3(st(k), st(v), kc, vc, slots, dtype, 0.0, 1.0)


def test_e4m3_attention_identities():
    """With power-of-two scales the E4M3 cache equals an f32 cache of
    decode(code) * scale exactly, so the pinned f32 path must agree; with any
    scale, v_scale scales the output and k_scale multiplies the softmax scale."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, D, bs, NB = 3, 4, 2, 64, 16, 12
    codes_k = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    codes_v = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    for c in (codes_k, codes_v):                  # no NaN codes
        c[(c & 0x7f) == 0x7f] = 0x3c
    q = rng.standard_normal((B, Hq, D)).astype(np.float32) * 0.05
    tables = rng.permutation(NB)[: B * 4].reshape(B, 4).astype(np.int32)
    lens = np.array([1, 37, 64], dtype=np.int32)
    scale = 1 / 8
    dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = oracle.paged_attention(q, codes_k, codes_v, oracle.F32, tables, lens, scale,
                                 kv_dtype=oracle.E4M3, k_scale=0.25, v_scale=2.0)
    want = oracle.paged_attention(q, dec(codes_k) * np.float32(0.25), dec(codes_v) * np.float32(2.0),
                                  oracle.F32, tables, lens, scale)
    assert np.abs(got - want).max() <= 1e-12
    a = oracle.paged_attention(q, codes_k, codes_v, oracle.F32, tables, lens, scale,
                               kv_dtype=oracle.E4M3, k_scale=0.3, v_scale=0.7)
    b = oracle.paged_attention(q, codes_k, codes_v, oracle.F32, tables, lens, scale * 0.3,
                               kv_dtype=oracle.E4M3, k_scale=1.0, v_scale=1.0)
    assert np.abs(a - 0.7 * b).max() <= 1e-12 * max(1.0, np.abs(a).max())
    # a single token: the output is that token's dequantised V
    one = oracle.paged_attention(q, codes_k, codes_v, oracle.F32, tables, lens, scale,
                                 kv_dtype=oracle.E4M3, k_scale=0.3, v_scale=0.7)[0]
    v0 = oracle.decode(codes_v[tables[0, 0], :, 0], oracle.E4M3) * 0.7
    assert np.array_equal(one[:2], v0[0:1].repeat(2, 0)) and np.array_equal(one[2:], v0[1:2].repeat(2, 0))


# ---------------------------------------------------------------------------
# several new query tokens per sequence (chunked prefill, speculative verify)


def _mq_case(seed, dtype=oracle.F32, bs=16, G=2, D=64):
    rng = np.random.default_rng(seed)
    B, Hkv = 3, 2
    Hq = Hkv * G
    lens = np.array([7, 40, 130], dtype=np.int32)
    qlen = np.array([1, 5, 17], dtype=np.int32)
    qs = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    NB = 20
    order = rng.permutation(NB)
    maxb = -(-int(lens.max()) // bs)
    tables = np.full((B, maxb), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        nb = -(-int(lens[b]) // bs)
        tables[b, :nb] = order[k:k + nb]
        k += nb
    kc = rng.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
    vc = rng.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32)
    return q, kc, vc, tables, lens, qs, Hq, Hkv, D, bs


def test_multi_query_matches_causal_sdpa_on_contiguous_tokens():
    q, kc, vc, tables, lens, qs, Hq, Hkv, D, bs = _mq_case(21)
    scale = 1 / np.sqrt(D)
    got = oracle.paged_attention_mq(q, kc, vc, oracle.F32, tables, lens, qs, scale)
    for b in range(len(lens)):
        L, Qb = int(lens[b]), int(qs[b + 1] - qs[b])
        j = np.arange(L)
        K = kc[tables[b, j // bs], :, j % bs].transpose(1, 0, 2)      # [Hkv, L, D]
        V = vc[tables[b, j // bs], :, j % bs].transpose(1, 0, 2)
        Q = q[qs[b]:qs[b + 1]].transpose(1, 0, 2)                      # [Hq, Qb, D]
        mask = j[None, :] <= (L - Qb + np.arange(Qb))[:, None]         # bottom-right causal
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(Q).double()[None], torch.from_numpy(K).double()[None],
            torch.from_numpy(V).double()[None], attn_mask=torch.from_numpy(mask)[None, None],
            scale=scale, enable_gqa=True)[0].numpy().transpose(1, 0, 2)
        assert np.abs(got[qs[b]:qs[b + 1]] - ref).max() <= 1e-12


def test_multi_query_row_equals_decode_at_its_own_position():
    """A prompt processed as one chunk of queries: query i sees exactly what a
    single-query decode with context length L - Q + i + 1 sees."""
    q, kc, vc, tables, lens, qs, Hq, Hkv, D, bs = _mq_case(22, G=4)
    got = oracle.paged_attention_mq(q, kc, vc, oracle.F32, tables, lens, qs, 0.2)
    b = 2
    Qb = int(qs[b + 1] - qs[b])
    for i in (0, 7, Qb - 1):
        one = oracle.paged_attention(q[qs[b] + i][None], kc, vc, oracle.F32, tables[b:b + 1],
                                     np.array([lens[b] - Qb + i + 1], dtype=np.int32), 0.2)
        assert np.abs(got[qs[b] + i] - one[0]).max() == 0.0
    # one query per sequence is the plain decode
    q1 = q[qs[1:] - 1]
    dec = oracle.paged_attention(q1, kc, vc, oracle.F32, tables, lens, 0.2)
    one_each = oracle.paged_attention_mq(q1, kc, vc, oracle.F32, tables, lens,
                                         np.arange(len(lens) + 1, dtype=np.int32), 0.2)
    assert np.array_equal(dec, one_each)


def test_multi_query_rejects_bad_offsets():
    q, kc, vc, tables, lens, qs, Hq, Hkv, D, bs = _mq_case(23)
    with pytest.raises(ValueError):                 # more queries than context
        oracle.paged_attention_mq(q[:8], kc, vc, oracle.F32, tables, np.array([7, 0, 130], np.int32),
                                  np.array([0, 1, 3, 8], np.int32), 0.1)
    with pytest.raises(ValueError):                 # decreasing offsets
        oracle.paged_attention_mq(q[:8], kc, vc, oracle.F32, tables, lens,
                                  np.array([0, 5, 3, 8], np.int32), 0.1)
