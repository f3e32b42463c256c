"""Oracle for the paged KV-cache decode path: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this; only
the tests, the smoke check of ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.

Parts:
  * ``pa_oracle.c`` (loaded here through ctypes): fp64 attention over the
    paged cache, the new-token append, the copy-on-write block copy and the
    block swap between two caches;
  * ``allocator.py``: the block manager (allocate on demand, share by
    reference count, copy on write, reclaim);
  * ``kv_size.py``: the KV-cache size formula of "1. KV 캐시란" (hjr-study-book
    Day 3).

Every function cites the passage of the three vLLM / PagedAttention pages it
follows; the module headers list the readings taken where the pages are silent.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, F16, BF16, E4M3 = 0, 1, 2, 3
_NP_STORAGE = {F32: np.float32, F16: np.uint16, BF16: np.uint16, E4M3: np.uint8}

_lib = None


def lib():
    """Load (building first if needed) the C oracle."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        p, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.or_decode.argtypes = [p, p, i32, i64]
        L.or_decode.restype = None
        L.or_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_f16_to_f64.restype = dbl
        L.or_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_f64.restype = dbl
        L.or_paged_attention.argtypes = [p, p, i64, p, p, p, i32, p, i32, p,
                                         i32, i32, i32, i32, i32, i32, dbl, i32]
        L.or_paged_attention.restype = i32
        L.or_paged_attention_kv.argtypes = [p, p, i64, p, p, p, i32, i32, dbl, dbl, p, i32, p,
                                            i32, i32, i32, i32, i32, i32, dbl, i32]
        L.or_paged_attention_kv.restype = i32
        L.or_paged_attention_mq.argtypes = [p, p, p, p, i32, p, i32, p, p, i32, i32, i32, i32,
                                            i32, i32, dbl, i32]
        L.or_paged_attention_mq.restype = i32
        L.or_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.or_e4m3_to_f64.restype = dbl
        L.or_encode_e4m3.argtypes = [p, p, i64]
        L.or_encode_e4m3.restype = None
        L.or_reshape_and_cache_e4m3.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i64, i32,
                                                ctypes.c_float, ctypes.c_float]
        L.or_reshape_and_cache_e4m3.restype = i32
        L.or_reshape_and_cache.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i64, i32]
        L.or_reshape_and_cache.restype = i32
        L.or_copy_blocks.argtypes = [p, p, p, i64, i32, i32, i32, i64, i32]
        L.or_copy_blocks.restype = i32
        L.or_swap_blocks.argtypes = [p, p, i64, p, p, i64, p, i64, i32, i32, i32, i32]
        L.or_swap_blocks.restype = i32
        L.or_max_threads.argtypes = []
        L.or_max_threads.restype = i32
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().or_max_threads())


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def decode(storage: np.ndarray, dtype: int) -> np.ndarray:
    """Exact fp64 values of stored fp32 / fp16 / bf16 bit patterns."""
    storage = np.ascontiguousarray(storage)
    out = np.empty(storage.size, dtype=np.float64)
    lib().or_decode(_ptr(out), _ptr(storage), dtype, storage.size)
    return out.reshape(storage.shape)


def encode_e4m3(values) -> np.ndarray:
    """Nearest OCP E4M3 codes (ties to even, saturating at +-448) of float64 values."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().or_encode_e4m3(_ptr(out), _ptr(v), v.size)
    return out


def paged_attention(q, k_cache, v_cache, dtype, block_tables, context_lens, scale,
                    rows=None, nthreads=None, kv_dtype=None, k_scale=1.0, v_scale=1.0):
    """Decode attention over the paged cache, fp64, for every (b, h) or for ``rows``.

    q: [B, Hq, D] storage array (float32, or uint16 bit patterns for fp16/bf16);
    k_cache, v_cache: [num_blocks, Hkv, block_size, D] storage arrays;
    block_tables: [B, max_blocks] int32; context_lens: [B] int32;
    rows: optional [n, 2] int64 array of (b, h).  Returns [B, Hq, D] or [n, D] float64.
    kv_dtype: storage type of the caches when it differs from q's (E4M3 codes,
    uint8), whose elements stand for decode(code) * k_scale / * v_scale.

    Follows "자기회귀 생성과 KV 캐시" (scores q.k/sqrt(d_k), softmax over valid
    past positions, weighted sum of V) and "PagedAttention의 설계" (gather
    through the block table in logical order, one normaliser over all tokens)
    of the supersilo.blog vLLM summary.
    """
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    block_tables, context_lens = _c(block_tables, np.int32), _c(context_lens, np.int32)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and block_tables.shape[0] == B
    if rows is not None:
        rows = _c(rows, np.int64).reshape(-1, 2)
        out = np.zeros((rows.shape[0], D), dtype=np.float64)
        n = rows.shape[0]
    else:
        out = np.zeros((B, Hq, D), dtype=np.float64)
        n = B * Hq
    nt = max_threads() if nthreads is None else int(nthreads)
    kvd = dtype if kv_dtype is None else kv_dtype
    rc = lib().or_paged_attention_kv(_ptr(out), _ptr(rows), n, _ptr(q), _ptr(k_cache),
                                     _ptr(v_cache), dtype, kvd, float(k_scale), float(v_scale),
                                     _ptr(block_tables), block_tables.shape[1],
                                     _ptr(context_lens), B, Hq, Hkv, D, bs, NB, float(scale), nt)
    if rc != 0:
        raise ValueError("oracle: input out of range")
    return out


def paged_attention_mq(q, k_cache, v_cache, dtype, block_tables, context_lens, query_start,
                       scale, nthreads=None):
    """Several new query tokens per sequence, causal among themselves.

    q: [total_q, Hq, D] storage array; query_start: [B+1] int32 offsets into q
    (sequence b's tokens are rows query_start[b] .. query_start[b+1]-1 and are
    its last context positions).  Returns [total_q, Hq, D] float64.  Reading
    of chunked prefill / speculative verification in "4. 이 밖의 기법들"
    (blog.aqudi.me): query token i of sequence b attends to positions
    0 .. context_lens[b] - Q_b + i.
    """
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    block_tables, context_lens = _c(block_tables, np.int32), _c(context_lens, np.int32)
    query_start = _c(query_start, np.int32)
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    B = context_lens.shape[0]
    assert query_start.shape[0] == B + 1 and int(query_start[-1]) == T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    nt = max_threads() if nthreads is None else int(nthreads)
    rc = lib().or_paged_attention_mq(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), dtype,
                                     _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                                     _ptr(query_start), B, Hq, Hkv, D, bs, NB, float(scale), nt)
    if rc != 0:
        raise ValueError("oracle: input out of range")
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, dtype):
    """Store the new tokens' K and V at their slots, in place (raw bytes).

    key, value: [N, Hkv, D] storage arrays; caches [num_blocks, Hkv, block_size, D]
    (modified in place, must be C-contiguous); slot_mapping: [N] int64, < 0 skips.
    Follows "1. KV 캐시란" (hjr-study-book Day 3) and its block-table example.
    """
    key, value = _c(key), _c(value)
    slot_mapping = _c(slot_mapping, np.int64)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    NB, Hkv, bs, D = k_cache.shape
    rc = lib().or_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(slot_mapping), slot_mapping.size, Hkv, D, bs, NB, dtype)
    if rc != 0:
        raise ValueError("oracle: slot out of range")


def reshape_and_cache_e4m3(key, value, k_cache, v_cache, slot_mapping, dtype, k_scale, v_scale):
    """Store the new tokens' K and V as E4M3 codes of x / scale (quotient in fp32).

    key, value: [N, Hkv, D] storage arrays of dtype (f32 / f16 / bf16); caches
    uint8 [num_blocks, Hkv, block_size, D], modified in place.  The precision
    reading for "quantization" of "4. 이 밖의 기법들" (blog.aqudi.me).
    """
    key, value = _c(key), _c(value)
    slot_mapping = _c(slot_mapping, np.int64)
    assert k_cache.dtype == np.uint8 and v_cache.dtype == np.uint8
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    NB, Hkv, bs, D = k_cache.shape
    rc = lib().or_reshape_and_cache_e4m3(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(slot_mapping), slot_mapping.size, Hkv, D, bs, NB,
                                         dtype, float(k_scale), float(v_scale))
    if rc != 0:
        raise ValueError("oracle: slot out of range or bad scale")


def copy_blocks(k_cache, v_cache, pairs, dtype):
    """Copy-on-write: block pairs[p,1] := block pairs[p,0] in both caches, in order.

    Follows "블록 공유" (supersilo.blog) and the copy-on-write bullet of
    "3. vLLM: KV cache를 블록 단위로 관리하기" (blog.aqudi.me).
    """
    pairs = _c(pairs, np.int64).reshape(-1, 2)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    NB, Hkv, bs, D = k_cache.shape
    rc = lib().or_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0],
                              Hkv, D, bs, NB, dtype)
    if rc != 0:
        raise ValueError("oracle: block id out of range")


def swap_blocks(dst_k, dst_v, src_k, src_v, pairs, dtype):
    """Block pairs[p,1] of the destination caches := block pairs[p,0] of the
    source caches, in order (swap out to host memory or back in).

    Follows "적용 범위와 관련 연구" of the supersilo.blog vLLM summary (sequences
    move to CPU memory when GPU memory is short).
    """
    pairs = _c(pairs, np.int64).reshape(-1, 2)
    for a in (dst_k, dst_v):
        assert a.flags.c_contiguous
    src_k, src_v = _c(src_k), _c(src_v)
    NBd, Hkv, bs, D = dst_k.shape
    NBs = src_k.shape[0]
    assert src_k.shape[1:] == dst_k.shape[1:]
    rc = lib().or_swap_blocks(_ptr(dst_k), _ptr(dst_v), NBd, _ptr(src_k), _ptr(src_v), NBs,
                              _ptr(pairs), pairs.shape[0], Hkv, D, bs, dtype)
    if rc != 0:
        raise ValueError("oracle: block id out of range")
