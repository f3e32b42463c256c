"""Python binding of libpagedkv.so (paged decode attention for B200 / sm_100a).

Argument marshalling only: every step of the decode path runs in the CUDA
library's kernels, and the block manager in its C++ host code.  The functions
carry the C names (pa_decode, pa_reshape_and_cache, pa_copy_blocks, pa_seq_*,
...); device arrays are torch CUDA tensors (torch provides device memory and
streams), shapes are read from them.  If the library was not built, importing
works but every call raises ``LibraryMissing``: there is no fallback path.

Layouts (see include/pagedkv.h): q / out [B, Hq, D]; k_cache / v_cache
[num_blocks, Hkv, block_size, D]; block_tables [B, max_blocks] int32;
context_lens [B] int32; key / value [N, Hkv, D]; slot_mapping [N] int64;
block_pairs [P, 2] int64.
"""
import ctypes
import os
from typing import List, Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PA_OK, PA_ERR_INVALID, PA_ERR_OOM, PA_ERR_CUDA, PA_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
PA_DEVERR_TABLE, PA_DEVERR_CONTEXT, PA_DEVERR_SLOT, PA_DEVERR_PAIR, PA_DEVERR_TIMEOUT = (
    0x1, 0x2, 0x4, 0x8, 0x10)

# every symbol include/pagedkv.h declares
EXPORTS = (
    "pa_last_error", "pa_version", "pa_launch_count", "pa_device_status",
    "pa_selftest_wait_timeout",
    "pa_decode_default_partition_size", "pa_decode_auto_partition_size",
    "pa_decode_fp8_auto_partition_size",
    "pa_decode_num_partitions", "pa_decode_workspace_bytes",
    "pa_decode", "pa_decode_partitions", "pa_decode_reduce", "pa_decode_noalloc",
    "pa_reshape_and_cache", "pa_reshape_and_cache_fp8", "pa_decode_fp8",
    "pa_decode_partitions_fp8", "pa_decode_multi", "pa_decode_multi_workspace_bytes",
    "pa_copy_blocks", "pa_swap_blocks", "pa_alloc_create", "pa_alloc_destroy", "pa_alloc_num_free",
    "pa_alloc_refcount", "pa_alloc_free_stack", "pa_seq_add", "pa_seq_fork", "pa_seq_append",
    "pa_seq_free", "pa_seq_move", "pa_seq_num_tokens", "pa_build_tables",
    "pa_alloc_enable_prefix_cache", "pa_alloc_evictable", "pa_seq_add_cached", "pa_seq_commit",
    "pa_decode_grouped", "pa_decode_grouped_fp8", "pa_decode_grouped_workspace_bytes",
    "pa_build_groups",
)


class LibraryMissing(RuntimeError):
    pass


class PagedKVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[status {status}] {message}")
        self.status = status


class OutOfBlocks(PagedKVError):
    pass


_lib = None


def lib():
    """The loaded ctypes library (raises LibraryMissing if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LibraryMissing(
            f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_443_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    pi32, pi64 = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    sig = {
        "pa_last_error": ([], ctypes.c_char_p),
        "pa_version": ([], ctypes.c_char_p),
        "pa_launch_count": ([], ctypes.c_uint64),
        "pa_device_status": ([ctypes.POINTER(ctypes.c_uint), i32], i32),
        "pa_selftest_wait_timeout": ([ctypes.POINTER(ctypes.c_uint)], i32),
        "pa_decode_default_partition_size": ([], i32),
        "pa_decode_auto_partition_size": ([i32, i32, i32, i32, i32, i32], i32),
        "pa_decode_fp8_auto_partition_size": ([i32, i32, i32, i32, i32, i32], i32),
        "pa_decode_num_partitions": ([i32, i32], i32),
        "pa_decode_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
        "pa_decode": ([vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                       i32, vp, sz, vp], i32),
        "pa_decode_partitions": ([vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, f32,
                                  i32, i32, i32, vp, sz, vp], i32),
        "pa_decode_reduce": ([vp, vp, i32, i32, i32, i32, i32, i32, vp, sz, vp], i32),
        "pa_decode_noalloc": ([vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, f32,
                               i32, i32, i32, vp], i32),
        "pa_reshape_and_cache": ([vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp], i32),
        "pa_reshape_and_cache_fp8": ([vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, f32,
                                      vp], i32),
        "pa_decode_multi": ([vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                             i32, f32, i32, i32, i32, vp, sz, vp], i32),
        "pa_decode_multi_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
        "pa_decode_fp8": ([vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, f32, i32,
                           f32, f32, i32, i32, vp, sz, vp], i32),
        "pa_decode_partitions_fp8": ([vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32,
                                      f32, i32, f32, f32, i32, i32, vp, sz, vp], i32),
        "pa_copy_blocks": ([vp, vp, vp, i32, i32, i32, i32, i32, i32, vp], i32),
        "pa_swap_blocks": ([vp, vp, i32, vp, vp, i32, vp, i32, i32, i32, i32, i32, vp], i32),
        "pa_alloc_create": ([i32, i32, pi32, ctypes.POINTER(vp)], i32),
        "pa_alloc_destroy": ([vp], None),
        "pa_alloc_num_free": ([vp], i32),
        "pa_alloc_refcount": ([vp, ctypes.c_int32], i32),
        "pa_alloc_free_stack": ([vp, pi32, i32, ctypes.POINTER(i32)], i32),
        "pa_seq_add": ([vp, i64], i32),
        "pa_seq_fork": ([vp, i64, i64], i32),
        "pa_seq_append": ([vp, i64, i32, pi64, pi64, ctypes.POINTER(i32)], i32),
        "pa_seq_free": ([vp, i64], i32),
        "pa_seq_move": ([vp, vp, pi64, i32, pi64, i32, ctypes.POINTER(i32)], i32),
        "pa_alloc_enable_prefix_cache": ([vp], i32),
        "pa_alloc_evictable": ([vp, pi32, i32, ctypes.POINTER(i32)], i32),
        "pa_seq_add_cached": ([vp, i64, pi32, i32, ctypes.POINTER(i32)], i32),
        "pa_seq_commit": ([vp, i64, pi32, i32], i32),
        "pa_seq_num_tokens": ([vp, i64, ctypes.POINTER(i32)], i32),
        "pa_build_tables": ([vp, pi64, i32, i32, pi32, pi32], i32),
        "pa_decode_grouped": ([vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                               i32, i32, i32, f32, i32, i32, i32, vp, sz, vp], i32),
        "pa_decode_grouped_fp8": ([vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32,
                                   i32, i32, i32, i32, f32, i32, f32, f32, i32, i32, vp, sz, vp],
                                  i32),
        "pa_decode_grouped_workspace_bytes": ([i32, i32, i32, i32, i32, i32], sz),
        "pa_build_groups": ([pi32, i32, i32, pi32, i32, pi32, pi32, ctypes.POINTER(i32),
                             ctypes.POINTER(i32), ctypes.POINTER(i32)], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(st: int) -> None:
    if st != PA_OK:
        msg = lib().pa_last_error().decode(errors="replace")
        raise (OutOfBlocks if st == PA_ERR_OOM else PagedKVError)(st, msg)


def _dtype_code(t) -> int:
    import torch
    codes = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
             torch.float8_e4m3fn: PA_FP8_E4M3}
    if t.dtype not in codes:
        raise PagedKVError(PA_ERR_INVALID, f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise PagedKVError(PA_ERR_INVALID, "tensors must be contiguous")


# ---------------------------------------------------------------------------
# library info


def pa_last_error() -> str:
    return lib().pa_last_error().decode(errors="replace")


def pa_version() -> str:
    return lib().pa_version().decode()


def pa_launch_count() -> int:
    return int(lib().pa_launch_count())


def pa_device_status(clear: bool = True) -> int:
    v = ctypes.c_uint(0)
    _check(lib().pa_device_status(ctypes.byref(v), int(clear)))
    return int(v.value)


def pa_selftest_wait_timeout() -> int:
    """Status bits of a launch whose internal wait is made to run out."""
    v = ctypes.c_uint(0)
    _check(lib().pa_selftest_wait_timeout(ctypes.byref(v)))
    return int(v.value)


def pa_decode_default_partition_size() -> int:
    return int(lib().pa_decode_default_partition_size())


def pa_decode_auto_partition_size(num_seqs: int, num_heads: int, num_kv_heads: int,
                                  head_size: int, dtype: int, max_context_len: int) -> int:
    """The partition length pa_decode picks for partition_size = 0 (dtype: PA_*)."""
    return int(lib().pa_decode_auto_partition_size(num_seqs, num_heads, num_kv_heads, head_size,
                                                   dtype, max_context_len))


def pa_decode_fp8_auto_partition_size(num_seqs: int, num_heads: int, num_kv_heads: int,
                                      head_size: int, dtype: int, max_context_len: int) -> int:
    """The partition length pa_decode_fp8 picks for partition_size = 0 (dtype:
    the queries' PA_* type)."""
    return int(lib().pa_decode_fp8_auto_partition_size(num_seqs, num_heads, num_kv_heads,
                                                       head_size, dtype, max_context_len))


def pa_decode_num_partitions(max_context_len: int, partition_size: int = 0) -> int:
    return int(lib().pa_decode_num_partitions(max_context_len, partition_size))


def pa_decode_workspace_bytes(num_seqs: int, num_heads: int, head_size: int,
                              max_context_len: int, partition_size: int = 0) -> int:
    return int(lib().pa_decode_workspace_bytes(num_seqs, num_heads, head_size, max_context_len,
                                               partition_size))


# ---------------------------------------------------------------------------
# device calls


def _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                 max_context_len, workspace, stream, kv_dtype=None):
    _contig(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (B, Hq, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise PagedKVError(PA_ERR_INVALID, "shape mismatch among q, out and the caches")
    for t, want in ((out, q.dtype), (k_cache, kv_dtype or q.dtype), (v_cache, kv_dtype or q.dtype)):
        if t.dtype != want:
            raise PagedKVError(PA_ERR_INVALID, f"dtype mismatch: {t.dtype} where {want} is expected")
    import torch
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PagedKVError(PA_ERR_INVALID, "block_tables and context_lens must be int32")
    if max_context_len is None:
        raise PagedKVError(PA_ERR_INVALID, "max_context_len is required (an upper bound)")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return (_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D, bs, NB, float(scale),
            _dtype_code(q), int(partition_size), int(max_context_len), _ptr(workspace), ws_bytes,
            _stream(stream))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
              partition_size=0, workspace=None, stream=None) -> None:
    """out[b,h] = softmax over j < context_lens[b] of scale*q[b,h].K_b[j], times V_b.
    ``workspace``: a CUDA tensor of at least pa_decode_workspace_bytes(...) bytes
    (or None when that is 0)."""
    _check(lib().pa_decode(*_decode_args(out, q, k_cache, v_cache, block_tables, context_lens,
                                         scale, partition_size, max_context_len, workspace,
                                         stream)))


class Groups:
    """Shared-prefix groups of a decode batch (pa_build_groups): group_start
    [num_groups + 1] and shared_lens [B] int32 tensors, and their bounds."""

    def __init__(self, group_start, shared_lens, num_groups, max_group_size, max_shared_len):
        self.group_start, self.shared_lens = group_start, shared_lens
        self.num_groups, self.max_group_size = int(num_groups), int(max_group_size)
        self.max_shared_len = int(max_shared_len)

    def to(self, device) -> "Groups":
        return Groups(self.group_start.to(device), self.shared_lens.to(device), self.num_groups,
                      self.max_group_size, self.max_shared_len)


def pa_build_groups(block_tables, context_lens, block_size: int) -> Groups:
    """Groups of consecutive sequences sharing leading physical blocks, from
    host (CPU) int32 block tables [B, max_blocks] and context lengths [B]."""
    import torch
    t = block_tables.to("cpu", torch.int32).contiguous()
    l = context_lens.to("cpu", torch.int32).contiguous()
    B, mb = t.shape
    gs = torch.empty(B + 1, dtype=torch.int32)
    sl = torch.empty(max(B, 1), dtype=torch.int32)
    ng, mg, ms = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    p32 = lambda x: ctypes.cast(x.data_ptr(), ctypes.POINTER(ctypes.c_int32))  # noqa: E731
    _check(lib().pa_build_groups(p32(t), B, mb, p32(l), int(block_size), p32(gs), p32(sl),
                                 ctypes.byref(ng), ctypes.byref(mg), ctypes.byref(ms)))
    return Groups(gs[:ng.value + 1].clone(), sl[:B].clone(), ng.value, mg.value, ms.value)


def pa_decode_grouped_workspace_bytes(num_seqs: int, num_heads: int, head_size: int,
                                      max_context_len: int, max_shared_len: int,
                                      partition_size: int = 0) -> int:
    return int(lib().pa_decode_grouped_workspace_bytes(num_seqs, num_heads, head_size,
                                                       max_context_len, max_shared_len,
                                                       partition_size))


def pa_decode_grouped(out, q, k_cache, v_cache, block_tables, context_lens, groups: Groups, scale,
                      max_context_len, partition_size=0, workspace=None, stream=None) -> None:
    """pa_decode's result, with each group's shared span read once for all its
    members (groups: device tensors, see pa_build_groups)."""
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                     max_context_len, workspace, stream)
    _contig(groups.group_start, groups.shared_lens)
    _check(lib().pa_decode_grouped(*a[:7], _ptr(groups.group_start), _ptr(groups.shared_lens),
                                   groups.num_groups, groups.max_group_size,
                                   groups.max_shared_len, *a[7:]))


def pa_decode_grouped_fp8(out, q, k_cache, v_cache, block_tables, context_lens, groups: Groups,
                          scale, max_context_len, k_scale, v_scale, partition_size=0,
                          workspace=None, stream=None) -> None:
    """pa_decode_fp8's result over E4M3 caches, with each group's shared span
    read once for all its members."""
    import torch
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                     max_context_len, workspace, stream, kv_dtype=torch.float8_e4m3fn)
    _contig(groups.group_start, groups.shared_lens)
    _check(lib().pa_decode_grouped_fp8(*a[:7], _ptr(groups.group_start), _ptr(groups.shared_lens),
                                       groups.num_groups, groups.max_group_size,
                                       groups.max_shared_len, *a[7:15], float(k_scale),
                                       float(v_scale), *a[15:]))


def pa_decode_partitions(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                         max_context_len, partition_size=0, workspace=None, stream=None) -> None:
    _check(lib().pa_decode_partitions(*_decode_args(out, q, k_cache, v_cache, block_tables,
                                                    context_lens, scale, partition_size,
                                                    max_context_len, workspace, stream)))


def pa_decode_reduce(out, context_lens, max_context_len, partition_size=0, workspace=None,
                     stream=None) -> None:
    _contig(out, context_lens, workspace)
    B, Hq, D = out.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_reduce(_ptr(out), _ptr(context_lens), B, Hq, D, _dtype_code(out),
                                  int(partition_size), int(max_context_len), _ptr(workspace),
                                  ws_bytes, _stream(stream)))


def pa_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                  k_scale, v_scale, partition_size=0, workspace=None, stream=None) -> None:
    """pa_decode over E4M3 caches (torch.float8_e4m3fn): keys stand for
    code * k_scale, values for code * v_scale; q and out f32 / f16 / bf16."""
    import torch
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                     max_context_len, workspace, stream, kv_dtype=torch.float8_e4m3fn)
    _check(lib().pa_decode_fp8(*a[:15], float(k_scale), float(v_scale), *a[15:]))


def pa_decode_partitions_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                             max_context_len, k_scale, v_scale, partition_size=0, workspace=None,
                             stream=None) -> None:
    import torch
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                     max_context_len, workspace, stream, kv_dtype=torch.float8_e4m3fn)
    _check(lib().pa_decode_partitions_fp8(*a[:15], float(k_scale), float(v_scale), *a[15:]))


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None) -> None:
    """Store key/value (f32 / f16 / bf16) as E4M3 codes of x / scale in the
    float8_e4m3fn caches at their slots."""
    _contig(key, value, k_cache, v_cache, slot_mapping)
    import torch
    N, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise PagedKVError(PA_ERR_INVALID, "shape mismatch")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != N:
        raise PagedKVError(PA_ERR_INVALID, "slot_mapping must be int64 [N]")
    if key.dtype != value.dtype or not (k_cache.dtype == v_cache.dtype == torch.float8_e4m3fn):
        raise PagedKVError(PA_ERR_INVALID, "key/value share a dtype; caches are float8_e4m3fn")
    _check(lib().pa_reshape_and_cache_fp8(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(slot_mapping), N, Hkv, D, bs, NB, _dtype_code(key),
                                          float(k_scale), float(v_scale), _stream(stream)))


def pa_decode_multi_workspace_bytes(total_q: int, num_heads: int, head_size: int,
                                    max_context_len: int, partition_size: int = 0) -> int:
    return int(lib().pa_decode_multi_workspace_bytes(total_q, num_heads, head_size,
                                                     max_context_len, partition_size))


def pa_decode_multi(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
                    max_context_len, max_query_len, partition_size=0, workspace=None,
                    stream=None) -> None:
    """Several new query tokens per sequence (chunked prefill / speculative
    verify): q, out [total_q, Hq, D]; query_start_loc int32 [B+1]; sequence b's
    queries are its last Q_b context tokens, each attending causally."""
    _contig(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc, workspace)
    import torch
    T, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (T, Hq, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise PagedKVError(PA_ERR_INVALID, "shape mismatch among q, out and the caches")
    for t_ in (out, k_cache, v_cache):
        if t_.dtype != q.dtype:
            raise PagedKVError(PA_ERR_INVALID, "q, out and the caches must share a dtype")
    if (block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32
            or query_start_loc.dtype != torch.int32):
        raise PagedKVError(PA_ERR_INVALID, "block_tables, context_lens, query_start_loc: int32")
    B = context_lens.shape[0]
    if query_start_loc.numel() != B + 1:
        raise PagedKVError(PA_ERR_INVALID, "query_start_loc must have num_seqs + 1 entries")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_multi(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                                 _ptr(query_start_loc), B, T, int(max_query_len), Hq, Hkv, D, bs,
                                 NB, float(scale), _dtype_code(q), int(partition_size),
                                 int(max_context_len), _ptr(workspace), ws_bytes,
                                 _stream(stream)))


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                      max_context_len, partition_size=0, stream=None) -> None:
    """pa_decode without a workspace argument, for callers that cannot allocate
    device memory: the split-K scratch is a fixed 32 MiB array inside the
    library (shared by all calls on a device; calls that overlap on the GPU
    race).  Batches needing more scratch raise PagedKVError (unsupported)."""
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, partition_size,
                     max_context_len, None, stream)
    _check(lib().pa_decode_noalloc(*a[:17], a[19]))


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """k_cache[s // bs, h, s % bs] = key[t, h] (same for value) for s = slot_mapping[t] >= 0."""
    _contig(key, value, k_cache, v_cache, slot_mapping)
    import torch
    N, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise PagedKVError(PA_ERR_INVALID, "shape mismatch")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != N:
        raise PagedKVError(PA_ERR_INVALID, "slot_mapping must be int64 [N]")
    if not (key.dtype == value.dtype == k_cache.dtype == v_cache.dtype):
        raise PagedKVError(PA_ERR_INVALID, "dtype mismatch")
    _check(lib().pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(slot_mapping), N, Hkv, D, bs, NB, _dtype_code(key),
                                      _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, block_pairs, stream=None) -> None:
    """Block block_pairs[p,1] := block block_pairs[p,0] in both caches."""
    _contig(k_cache, v_cache, block_pairs)
    import torch
    NB, Hkv, bs, D = k_cache.shape
    if block_pairs.dtype != torch.int64 or (block_pairs.numel() and block_pairs.shape[-1] != 2):
        raise PagedKVError(PA_ERR_INVALID, "block_pairs must be int64 [P, 2]")
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise PagedKVError(PA_ERR_INVALID, "cache mismatch")
    P = block_pairs.numel() // 2
    _check(lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_pairs) if P else None,
                                P, Hkv, D, bs, NB, _dtype_code(k_cache), _stream(stream)))


def pa_swap_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, block_pairs,
                   stream=None) -> None:
    """Block block_pairs[p,1] of the destination caches := block block_pairs[p,0]
    of the source caches.  A cache pair may be pinned host memory (torch
    pin_memory()); block_pairs is an int64 [P, 2] tensor on the device or pinned."""
    _contig(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, block_pairs)
    import torch
    NBd, Hkv, bs, D = dst_k_cache.shape
    NBs = src_k_cache.shape[0]
    if (tuple(src_k_cache.shape[1:]) != (Hkv, bs, D) or src_v_cache.shape != src_k_cache.shape
            or dst_v_cache.shape != dst_k_cache.shape):
        raise PagedKVError(PA_ERR_INVALID, "cache shape mismatch")
    if not (dst_k_cache.dtype == dst_v_cache.dtype == src_k_cache.dtype == src_v_cache.dtype):
        raise PagedKVError(PA_ERR_INVALID, "dtype mismatch")
    if block_pairs.dtype != torch.int64 or (block_pairs.numel() and block_pairs.shape[-1] != 2):
        raise PagedKVError(PA_ERR_INVALID, "block_pairs must be int64 [P, 2]")
    P = block_pairs.numel() // 2
    _check(lib().pa_swap_blocks(_ptr(dst_k_cache), _ptr(dst_v_cache), NBd, _ptr(src_k_cache),
                                _ptr(src_v_cache), NBs, _ptr(block_pairs) if P else None, P, Hkv,
                                D, bs, _dtype_code(dst_k_cache), _stream(stream)))


# ---------------------------------------------------------------------------
# block manager (host)


def pa_alloc_create(num_blocks: int, block_size: int,
                    initial_free_order: Optional[Sequence[int]] = None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    arr = None
    if initial_free_order is not None:
        arr = (ctypes.c_int32 * len(initial_free_order))(*[int(x) for x in initial_free_order])
        if len(initial_free_order) != num_blocks:
            raise PagedKVError(PA_ERR_INVALID, "initial_free_order must have num_blocks entries")
    _check(lib().pa_alloc_create(num_blocks, block_size, arr, ctypes.byref(h)))
    return h


def pa_alloc_destroy(h) -> None:
    lib().pa_alloc_destroy(h)


def pa_alloc_num_free(h) -> int:
    return int(lib().pa_alloc_num_free(h))


def pa_alloc_refcount(h, block: int) -> int:
    return int(lib().pa_alloc_refcount(h, block))


def pa_alloc_free_stack(h) -> List[int]:
    n = ctypes.c_int(0)
    _check(lib().pa_alloc_free_stack(h, None, 0, ctypes.byref(n)))
    buf = (ctypes.c_int32 * max(1, n.value))()
    _check(lib().pa_alloc_free_stack(h, buf, n.value, ctypes.byref(n)))
    return list(buf[: n.value])


def pa_seq_add(h, seq_id: int) -> None:
    _check(lib().pa_seq_add(h, seq_id))


def pa_seq_fork(h, parent: int, child: int) -> None:
    _check(lib().pa_seq_fork(h, parent, child))


def pa_seq_append(h, seq_id: int, n_tokens: int) -> Tuple[List[int], List[Tuple[int, int]]]:
    """Returns (slots, cow_pairs); cow_pairs holds at most one (src, dst) pair."""
    slots = (ctypes.c_int64 * max(1, n_tokens))()
    pair = (ctypes.c_int64 * 2)()
    n_cow = ctypes.c_int(0)
    _check(lib().pa_seq_append(h, seq_id, n_tokens, slots, pair, ctypes.byref(n_cow)))
    return list(slots[:n_tokens]), ([(pair[0], pair[1])] if n_cow.value else [])


def pa_seq_free(h, seq_id: int) -> None:
    _check(lib().pa_seq_free(h, seq_id))


def pa_seq_move(src, dst, seq_ids: Sequence[int], capacity: int) -> List[Tuple[int, int]]:
    """Move sequences from manager src to dst keeping their sharing; returns the
    (src block, dst block) pairs to copy.  capacity >= the sequences' block count."""
    ids = (ctypes.c_int64 * max(1, len(seq_ids)))(*[int(x) for x in seq_ids])
    buf = (ctypes.c_int64 * max(2, 2 * capacity))()
    n = ctypes.c_int(0)
    _check(lib().pa_seq_move(src, dst, ids, len(seq_ids), buf, capacity, ctypes.byref(n)))
    return [(buf[2 * i], buf[2 * i + 1]) for i in range(n.value)]


def pa_alloc_enable_prefix_cache(h) -> None:
    _check(lib().pa_alloc_enable_prefix_cache(h))


def pa_alloc_evictable(h) -> List[int]:
    n = ctypes.c_int(0)
    _check(lib().pa_alloc_evictable(h, None, 0, ctypes.byref(n)))
    buf = (ctypes.c_int32 * max(1, n.value))()
    _check(lib().pa_alloc_evictable(h, buf, n.value, ctypes.byref(n)))
    return list(buf[:n.value])


def _tokens(token_ids):
    t = [int(x) for x in token_ids]
    return (ctypes.c_int32 * max(1, len(t)))(*t), len(t)


def pa_seq_add_cached(h, seq_id: int, token_ids) -> int:
    """New sequence holding the cached blocks of its prompt's leading full
    blocks; returns the number of tokens they cover."""
    buf, n = _tokens(token_ids)
    got = ctypes.c_int(0)
    _check(lib().pa_seq_add_cached(h, seq_id, buf, n, ctypes.byref(got)))
    return got.value


def pa_seq_commit(h, seq_id: int, token_ids) -> None:
    buf, n = _tokens(token_ids)
    _check(lib().pa_seq_commit(h, seq_id, buf, n))


def pa_seq_num_tokens(h, seq_id: int) -> int:
    n = ctypes.c_int(0)
    _check(lib().pa_seq_num_tokens(h, seq_id, ctypes.byref(n)))
    return n.value


def pa_build_tables(h, seq_ids: Sequence[int], max_blocks_per_seq: int):
    """(block_tables int32 [B, max_blocks], context_lens int32 [B]) as numpy arrays."""
    import numpy as np
    B = len(seq_ids)
    ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
    tables = np.empty((B, max_blocks_per_seq), dtype=np.int32)
    lens = np.empty(B, dtype=np.int32)
    as_p = lambda a, t: a.ctypes.data_as(ctypes.POINTER(t))
    _check(lib().pa_build_tables(h, as_p(ids, ctypes.c_int64), B, max_blocks_per_seq,
                                 as_p(tables, ctypes.c_int32), as_p(lens, ctypes.c_int32)))
    return tables, lens


class BlockAllocator:
    """Owning wrapper of a pa_allocator handle (same operations, Python names)."""

    def __init__(self, num_blocks: int, block_size: int,
                 initial_free_order: Optional[Sequence[int]] = None):
        self.num_blocks, self.block_size = num_blocks, block_size
        self.h = pa_alloc_create(num_blocks, block_size, initial_free_order)

    def close(self):
        if self.h:
            pa_alloc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq_id):
        pa_seq_add(self.h, seq_id)

    def fork(self, parent, child):
        pa_seq_fork(self.h, parent, child)

    def append(self, seq_id, n_tokens):
        return pa_seq_append(self.h, seq_id, n_tokens)

    def release(self, seq_id):
        pa_seq_free(self.h, seq_id)

    def num_free(self):
        return pa_alloc_num_free(self.h)

    def refcount(self, block):
        return pa_alloc_refcount(self.h, block)

    def free_stack(self):
        return pa_alloc_free_stack(self.h)

    def num_tokens(self, seq_id):
        return pa_seq_num_tokens(self.h, seq_id)

    def enable_prefix_cache(self):
        pa_alloc_enable_prefix_cache(self.h)

    def evictable(self):
        return pa_alloc_evictable(self.h)

    def add_cached(self, seq_id, token_ids) -> int:
        return pa_seq_add_cached(self.h, seq_id, token_ids)

    def commit(self, seq_id, token_ids):
        pa_seq_commit(self.h, seq_id, token_ids)

    def move_to(self, dst: "BlockAllocator", seq_ids):
        """Move sequences to another manager (sharing kept); returns copy pairs."""
        cap = sum(-(-self.num_tokens(s) // self.block_size) for s in seq_ids)
        return pa_seq_move(self.h, dst.h, list(seq_ids), cap)

    def build_tables(self, seq_ids, max_blocks_per_seq):
        return pa_build_tables(self.h, seq_ids, max_blocks_per_seq)
