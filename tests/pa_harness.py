"""Lockstep builder of a workload on the CUDA library and on the oracle.

Both sides replay the same block-manager script (from the workloads module)
on their own allocator, copy shared blocks and store the same seeded K/V with
their own routines, and build their own block tables.  The oracle receives
only generator output (host copies of the seeded draws) -- never a value
produced by the CUDA path.  Comparisons: tables / slots / pairs / cache bytes
bit-exact, attention within the stated tolerance.
"""
from dataclasses import dataclass
from typing import List, Optional, Tuple

import numpy as np
import torch

import oracle
import workloads as W
from oracle.allocator import BlockManager
from paged_kv_cache_443_b200.cache import PagedKVCache, _filled

# tolerances: fp32 accumulation; max abs error on outputs (fp16 / bf16 / fp32)
TOL = {"f32": 1e-5, "f16": 2e-2, "bf16": 2e-2}


def poison_bits(spec: W.Spec):
    """Bit pattern torch stores for NaN in the cache dtype (the fill of every
    slot no token was written to)."""
    return W.storage_view(_filled((1,), float("nan"), W.torch_kv_dtype(spec), "cpu"))[0]


def _zero_bits(spec: W.Spec):
    return W.storage_view(_filled((1,), 0.0, W.torch_kv_dtype(spec), "cpu"))[0]


def oracle_append(spec: W.Spec, key, value, k, v, slots):
    """The oracle's append of the same draws (E4M3 quantisation for E4M3 caches)."""
    if spec.fp8:
        oracle.reshape_and_cache_e4m3(W.storage_view(key), W.storage_view(value), k, v,
                                      np.asarray(slots, dtype=np.int64), spec.dtype_code,
                                      spec.k_scale, spec.v_scale)
    else:
        oracle.reshape_and_cache(W.storage_view(key), W.storage_view(value), k, v,
                                 np.asarray(slots, dtype=np.int64), spec.dtype_code)


@dataclass
class Product:
    cache: PagedKVCache
    step_slots: torch.Tensor
    step_pairs: torch.Tensor
    step_key: torch.Tensor
    step_value: torch.Tensor
    tables: torch.Tensor
    lens: torch.Tensor
    max_ctx: int
    q: torch.Tensor
    slots_host: List[int]
    pairs_host: List[Tuple[int, int]]


@dataclass
class Oracle:
    bm: BlockManager
    k: np.ndarray
    v: np.ndarray
    tables: np.ndarray
    lens: np.ndarray
    q: np.ndarray
    slots: List[int]
    pairs: List[Tuple[int, int]]


def build(sc: W.Scenario, device="cuda", with_oracle=True, poison=True, draw_device=None):
    """Builds the scenario on the library (on `device`) and, unless with_oracle
    is False, on the oracle.  K/V and q are drawn on draw_device (default:
    device) and copied; drawing on the CPU gives the same contents as an
    oracle-only build (build_oracle), whose sensitivity the CPU tests check."""
    spec = sc.spec
    draw = device if draw_device is None else draw_device
    shape = (sc.num_blocks, spec.Hkv, spec.block_size, spec.D)
    cache = PagedKVCache(sc.num_blocks, spec.block_size, spec.Hkv, spec.D, W.torch_kv_dtype(spec),
                         device, sc.free_order.tolist(),
                         fill=float("nan") if poison else 0.0, k_scale=spec.k_scale,
                         v_scale=spec.v_scale)
    orc = None
    if with_oracle:
        bm = BlockManager(sc.num_blocks, spec.block_size, sc.free_order.tolist())
        fill = poison_bits(spec) if poison else _zero_bits(spec)
        st = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16, "e4m3": np.uint8}[spec.kv]
        ok = np.full(shape, fill, dtype=st)
        ov = np.full(shape, fill, dtype=st)
    for op in sc.setup_ops:
        if op.kind == "add":
            cache.add(op.seq)
            with_oracle and bm.add(op.seq)
        elif op.kind == "fork":
            cache.fork(op.seq, op.arg)
            with_oracle and bm.fork(op.seq, op.arg)
        elif op.kind == "release":
            cache.release(op.seq)
            with_oracle and bm.release(op.seq)
        else:
            k, v = W.kv_content(spec, op.kv_id, op.arg, draw, sc.spikes)
            k, v = k.to(device), v.to(device)
            cache.append([op.seq], [op.arg], k, v)
            if with_oracle:
                slots, pairs = bm.append(op.seq, op.arg)
                if pairs:
                    oracle.copy_blocks(ok, ov, np.array(pairs), spec.kv_code)
                oracle_append(spec, k, v, ok, ov, slots)
            del k, v
    # the step's appends: reserved now, executed by run_step
    seqs = [op.seq for op in sc.step_ops]
    counts = [op.arg for op in sc.step_ops]
    draws = [tuple(x.to(device) for x in W.kv_content(spec, op.kv_id, op.arg, draw, sc.spikes))
             for op in sc.step_ops]
    key = torch.cat([d[0] for d in draws]) if draws else torch.empty((0, spec.Hkv, spec.D), dtype=W.torch_dtype(spec), device=device)
    value = torch.cat([d[1] for d in draws]) if draws else torch.empty_like(key)
    del draws
    slots, pairs = cache.reserve(seqs, counts)
    tables, lens, max_ctx = cache.tables(sc.batch, sc.max_blocks)
    q = W.q_content(spec, len(sc.batch), draw, sc.spikes).to(device)
    prod = Product(cache, torch.tensor(slots, dtype=torch.int64, device=device),
                   torch.tensor(pairs, dtype=torch.int64, device=device).reshape(-1, 2),
                   key.contiguous(), value.contiguous(), tables, lens, max_ctx, q, slots, pairs)
    if with_oracle:
        oslots, opairs = [], []
        for sid, n in zip(seqs, counts):
            s, p = bm.append(sid, n)
            oslots += s
            opairs += p
        if opairs:
            oracle.copy_blocks(ok, ov, np.array(opairs), spec.kv_code)
        oracle_append(spec, key, value, ok, ov, oslots)
        ot, ol = bm.build_tables(sc.batch, sc.max_blocks)
        orc = Oracle(bm, ok, ov, ot, ol, W.storage_view(q), oslots, opairs)
    return prod, orc


def run_step(p: Product, spec: W.Spec, partition_size: Optional[int] = None, out=None,
             workspace=None, stream=None, grouped=False):
    """One pass of the hot path: copy-on-write, append, decode (with `grouped`,
    the decode that reads each family's shared blocks once)."""
    P = spec.partition_size if partition_size is None else partition_size
    p.cache.copy_on_write(p.step_pairs, stream=stream)
    p.cache.store(p.step_key, p.step_value, p.step_slots, stream=stream)
    groups = p.cache.groups(p.tables, p.lens) if grouped else None
    return p.cache.decode(p.q, p.tables, p.lens, p.max_ctx, spec.softmax_scale, out=out,
                          partition_size=P, workspace=workspace, stream=stream, groups=groups)


def as_f64(t: torch.Tensor, spec: W.Spec) -> np.ndarray:
    return oracle.decode(W.storage_view(t), spec.dtype_code)


def oracle_attention(o: Oracle, spec: W.Spec, rows=None):
    return oracle.paged_attention(o.q, o.k, o.v, spec.dtype_code, o.tables, o.lens,
                                  spec.softmax_scale, rows=rows, kv_dtype=spec.kv_code,
                                  k_scale=spec.k_scale, v_scale=spec.v_scale)


def check_bookkeeping(p: Product, o: Oracle):
    assert p.slots_host == o.slots
    assert [tuple(x) for x in p.pairs_host] == [tuple(x) for x in o.pairs]
    assert np.array_equal(p.tables.cpu().numpy(), o.tables)
    assert np.array_equal(p.lens.cpu().numpy(), o.lens)


def check_caches(p: Product, o: Oracle, blocks=None):
    """Byte equality of the caches (all blocks, or the given block ids)."""
    for dev, host in ((p.cache.k_cache, o.k), (p.cache.v_cache, o.v)):
        if blocks is None:
            got = W.storage_view(dev)
            want = host
        else:
            idx = torch.as_tensor(np.asarray(blocks, dtype=np.int64), device=dev.device)
            got = W.storage_view(dev.index_select(0, idx))
            want = host[np.asarray(blocks)]
        assert got.tobytes() == want.tobytes()


def check_token_slots(p: Product, o: Oracle):
    """Byte equality of every cache slot that holds a token of the batch (unused
    tail slots excluded)."""
    bs = p.cache.block_size
    blk, off = [], []
    for b in range(len(o.lens)):
        j = np.arange(int(o.lens[b]))
        blk.append(o.tables[b, j // bs])
        off.append(j % bs)
    blk = np.concatenate(blk).astype(np.int64)
    off = np.concatenate(off).astype(np.int64)
    for dev, host in ((p.cache.k_cache, o.k), (p.cache.v_cache, o.v)):
        got = W.storage_view(dev)[blk, :, off, :]
        assert got.tobytes() == host[blk, :, off, :].tobytes()


def build_oracle(sc: W.Scenario, poison=True) -> Oracle:
    """The oracle side of build() alone (draws on the CPU): no GPU needed."""
    spec = sc.spec
    shape = (sc.num_blocks, spec.Hkv, spec.block_size, spec.D)
    bm = BlockManager(sc.num_blocks, spec.block_size, sc.free_order.tolist())
    fill = poison_bits(spec) if poison else _zero_bits(spec)
    st = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16, "e4m3": np.uint8}[spec.kv]
    ok = np.full(shape, fill, dtype=st)
    ov = np.full(shape, fill, dtype=st)
    for op in sc.setup_ops:
        if op.kind == "add":
            bm.add(op.seq)
        elif op.kind == "fork":
            bm.fork(op.seq, op.arg)
        elif op.kind == "release":
            bm.release(op.seq)
        else:
            k, v = W.kv_content(spec, op.kv_id, op.arg, "cpu", sc.spikes)
            slots, pairs = bm.append(op.seq, op.arg)
            if pairs:
                oracle.copy_blocks(ok, ov, np.array(pairs), spec.kv_code)
            oracle_append(spec, k, v, ok, ov, slots)
    oslots, opairs = [], []
    for op in sc.step_ops:
        k, v = W.kv_content(spec, op.kv_id, op.arg, "cpu", sc.spikes)
        s_, p_ = bm.append(op.seq, op.arg)
        if p_:
            oracle.copy_blocks(ok, ov, np.array(p_), spec.kv_code)
        oracle_append(spec, k, v, ok, ov, s_)
        oslots += s_
        opairs += p_
    ot, ol = bm.build_tables(sc.batch, sc.max_blocks)
    q = W.q_content(spec, len(sc.batch), "cpu", sc.spikes)
    return Oracle(bm, ok, ov, ot, ol, W.storage_view(q), oslots, opairs)


PERTURBATIONS = ("drop", "repeat", "neighbour")


def oracle_row_perturbed(o: Oracle, spec: W.Spec, b: int, h: int, j: int, how: str,
                         n_keys=None, q_row=None):
    """The oracle's output for query row (b, h) when its key/value sequence is
    changed at position j the way a slip in a kernel would change it:
      drop       token j left out;
      repeat     token j counted twice;
      neighbour  the slot next to j read in its place (j+1, or j-1 for the last);
      include    one key past the row's causal limit taken in as well.
    n_keys: keys the row attends to (default context_lens[b]); q_row: the
    query's storage row (default o.q[b, h]).  Rebuilds the row's keys
    contiguously through the block table, then calls the oracle on them."""
    bs = spec.block_size
    L = int(o.lens[b])
    n = L if n_keys is None else int(n_keys)
    g = h // spec.G
    pos = list(range(n))
    if how == "drop":
        pos.remove(j)
    elif how == "repeat":
        pos.insert(pos.index(j), j)
    elif how == "neighbour":
        pos[pos.index(j)] = j + 1 if j + 1 < n else j - 1
    elif how == "include":
        pos.append(n)
    else:
        raise ValueError(how)
    pos = np.asarray(pos, dtype=np.int64)
    blk = o.tables[b, pos // bs]
    kc = o.k[blk, g, pos % bs]                     # [m, D]
    vc = o.v[blk, g, pos % bs]
    m = len(pos)
    nb = -(-m // bs)
    fill = np.zeros(1, dtype=o.k.dtype)[0]
    k1 = np.full((nb * bs, spec.D), fill, dtype=o.k.dtype)
    v1 = np.full((nb * bs, spec.D), fill, dtype=o.v.dtype)
    k1[:m], v1[:m] = kc, vc
    q = (o.q[b, h] if q_row is None else q_row).reshape(1, 1, spec.D)
    return oracle.paged_attention(q, k1.reshape(nb, 1, bs, spec.D), v1.reshape(nb, 1, bs, spec.D),
                                  spec.dtype_code, np.arange(nb, dtype=np.int32).reshape(1, nb),
                                  np.array([m], np.int32), spec.softmax_scale,
                                  kv_dtype=spec.kv_code, k_scale=spec.k_scale,
                                  v_scale=spec.v_scale, nthreads=1)[0, 0]
