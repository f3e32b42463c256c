"""PagedKVCache: one layer's paged K/V cache with its block manager.

Orchestration of the C-ABI calls a decode step makes, in the order the
vLLM / PagedAttention pages describe: the block manager reserves slots for new
tokens, taking a fresh block only when the current one is full and copying a
shared block before it is modified ("PagedAttention의 설계", "블록 공유" on the
supersilo.blog summary; section 3 of the blog.aqudi.me write-up); the new
tokens' K/V are stored at their slots ("1. KV 캐시란", hjr-study-book Day 3);
attention then reads every sequence's K/V through its block table.  When GPU
memory runs short a sequence can be swapped out to a pinned host pool and back
("적용 범위와 관련 연구", supersilo.blog): the host pool has its own C++ block
manager, and both directions are one pa_swap_blocks launch.  No arithmetic
happens here: slots and copy pairs come from the C++ block managers, every
device operation is a libpagedkv.so kernel.
"""
from typing import List, Optional, Sequence, Tuple

import torch

from . import (BlockAllocator, Groups, pa_build_groups, pa_copy_blocks, pa_decode,
               pa_decode_fp8, pa_decode_grouped, pa_decode_grouped_fp8,
               pa_decode_grouped_workspace_bytes,
               pa_decode_workspace_bytes, pa_reshape_and_cache, pa_reshape_and_cache_fp8,
               pa_swap_blocks)


def _filled(shape, fill: float, dtype: torch.dtype, device) -> torch.Tensor:
    if dtype == torch.float8_e4m3fn:   # fill the byte code (NaN -> the E4M3 NaN code)
        code = int(torch.tensor([float(fill)]).to(dtype).view(torch.uint8)[0])
        return torch.full(shape, code, dtype=torch.uint8, device=device).view(dtype)
    return torch.full(shape, fill, dtype=dtype, device=device)


class PagedKVCache:
    """dtype: the cache's element type, or torch.float8_e4m3fn for a cache of
    E4M3 codes standing for code * k_scale (keys) and code * v_scale (values);
    new K/V and queries are then f32 / f16 / bf16 and quantised on append."""

    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int, head_size: int,
                 dtype: torch.dtype, device="cuda", initial_free_order: Optional[Sequence[int]] = None,
                 fill: Optional[float] = None, k_scale: float = 1.0, v_scale: float = 1.0,
                 prefix_cache: bool = False):
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_kv_heads, self.head_size = num_kv_heads, head_size
        self.dtype, self.device = dtype, torch.device(device)
        self.fp8 = dtype == torch.float8_e4m3fn
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        shape = (num_blocks, num_kv_heads, block_size, head_size)
        if fill is None:
            self.k_cache = torch.empty(shape, dtype=dtype, device=self.device)
            self.v_cache = torch.empty(shape, dtype=dtype, device=self.device)
        else:
            self.k_cache = _filled(shape, fill, dtype, self.device)
            self.v_cache = _filled(shape, fill, dtype, self.device)
        self.alloc = BlockAllocator(num_blocks, block_size, initial_free_order)
        if prefix_cache:
            self.alloc.enable_prefix_cache()
        self.host_alloc = None
        self.host_k = self.host_v = None

    # ---- block manager ----
    def add(self, seq_id: int) -> None:
        self.alloc.add(seq_id)

    def fork(self, parent: int, child: int) -> None:
        self.alloc.fork(parent, child)

    def release(self, seq_id: int) -> None:
        self.alloc.release(seq_id)

    # ---- prefix caching ("5. Prefix Caching", hjr-study-book Day 3) ----
    def add_cached(self, seq_id: int, token_ids: Sequence[int]) -> int:
        """New request: takes the cached blocks of its prompt's leading full
        blocks and returns how many tokens they cover; the caller appends the
        K/V of the rest (append) and then commits the prompt."""
        return self.alloc.add_cached(seq_id, token_ids)

    def commit(self, seq_id: int, token_ids: Sequence[int]) -> None:
        """Make the sequence's full blocks of token_ids reusable by later requests."""
        self.alloc.commit(seq_id, token_ids)

    def reserve(self, seq_ids: Sequence[int], counts: Sequence[int]
                ) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Host only: slots for counts[i] new tokens of seq_ids[i] (concatenated in
        that order) and the copy-on-write pairs to run before writing them."""
        slots: List[int] = []
        pairs: List[Tuple[int, int]] = []
        for sid, n in zip(seq_ids, counts):
            s, p = self.alloc.append(sid, int(n))
            slots += s
            pairs += p
        return slots, pairs

    # ---- device steps ----
    def copy_on_write(self, pairs, stream=None) -> None:
        if isinstance(pairs, torch.Tensor):
            t = pairs
        else:
            if not pairs:
                return
            t = torch.tensor(pairs, dtype=torch.int64, device=self.device)
        if t.numel():
            pa_copy_blocks(self.k_cache, self.v_cache, t, stream=stream)

    def store(self, key: torch.Tensor, value: torch.Tensor, slot_mapping, stream=None) -> None:
        if not isinstance(slot_mapping, torch.Tensor):
            slot_mapping = torch.tensor(slot_mapping, dtype=torch.int64, device=self.device)
        if not slot_mapping.numel():
            return
        if self.fp8:
            pa_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slot_mapping,
                                     self.k_scale, self.v_scale, stream=stream)
        else:
            pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slot_mapping, stream=stream)

    def append(self, seq_ids: Sequence[int], counts: Sequence[int], key: torch.Tensor,
               value: torch.Tensor, stream=None) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Reserve, copy shared blocks, then store key/value ([sum(counts), Hkv, D])."""
        slots, pairs = self.reserve(seq_ids, counts)
        self.copy_on_write(pairs, stream=stream)
        self.store(key, value, slots, stream=stream)
        return slots, pairs

    def tables(self, seq_ids: Sequence[int], max_blocks: Optional[int] = None):
        """Device block tables [B, max_blocks] int32 and context lengths [B] int32,
        plus the longest context (host int)."""
        if max_blocks is None:
            n = [self.alloc.num_tokens(s) for s in seq_ids]
            max_blocks = max(1, -(-max(n, default=1) // self.block_size))
        t, l = self.alloc.build_tables(list(seq_ids), max_blocks)
        return (torch.from_numpy(t).to(self.device), torch.from_numpy(l).to(self.device),
                int(l.max()) if l.size else 0)

    def workspace(self, num_seqs: int, num_heads: int, max_context_len: int,
                  partition_size: int = 0) -> Optional[torch.Tensor]:
        n = pa_decode_workspace_bytes(num_seqs, num_heads, self.head_size, max_context_len,
                                      partition_size)
        if n == 0:
            return None
        return torch.empty(n // 4, dtype=torch.float32, device=self.device)

    def groups(self, block_tables: torch.Tensor, context_lens: torch.Tensor) -> Groups:
        """Shared-prefix groups of a batch (on this cache's device), from its tables."""
        return pa_build_groups(block_tables.cpu(), context_lens.cpu(),
                               self.block_size).to(self.device)

    def grouped_workspace(self, num_seqs: int, num_heads: int, max_context_len: int,
                          groups: Groups, partition_size: int = 0) -> Optional[torch.Tensor]:
        n = pa_decode_grouped_workspace_bytes(num_seqs, num_heads, self.head_size,
                                              max_context_len, groups.max_shared_len,
                                              partition_size)
        return torch.empty(n // 4, dtype=torch.float32, device=self.device) if n else None

    def decode(self, q: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
               max_context_len: int, scale: float, out: Optional[torch.Tensor] = None,
               partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
               stream=None, groups: Optional[Groups] = None) -> torch.Tensor:
        """Decode attention of the batch; with `groups` (self.groups(...)) each
        group's shared leading blocks are read once for all its members (the
        result is the same)."""
        if out is None:
            out = torch.empty_like(q)
        if groups is not None:
            if workspace is None:
                workspace = self.grouped_workspace(q.shape[0], q.shape[1], max_context_len,
                                                   groups, partition_size)
            if self.fp8:
                pa_decode_grouped_fp8(out, q, self.k_cache, self.v_cache, block_tables,
                                      context_lens, groups, scale, max_context_len, self.k_scale,
                                      self.v_scale, partition_size=partition_size,
                                      workspace=workspace, stream=stream)
            else:
                pa_decode_grouped(out, q, self.k_cache, self.v_cache, block_tables, context_lens,
                                  groups, scale, max_context_len, partition_size=partition_size,
                                  workspace=workspace, stream=stream)
            return out
        if workspace is None:
            workspace = self.workspace(q.shape[0], q.shape[1], max_context_len, partition_size)
        if self.fp8:
            pa_decode_fp8(out, q, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                          max_context_len, self.k_scale, self.v_scale,
                          partition_size=partition_size, workspace=workspace, stream=stream)
        else:
            pa_decode(out, q, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                      max_context_len, partition_size=partition_size, workspace=workspace,
                      stream=stream)
        return out

    # ---- swap to / from pinned host memory ----
    def enable_swap(self, num_host_blocks: int) -> None:
        """Pinned host caches of num_host_blocks blocks, with their own block manager."""
        shape = (num_host_blocks, self.num_kv_heads, self.block_size, self.head_size)
        self.host_k = torch.empty(shape, dtype=self.dtype, pin_memory=True)
        self.host_v = torch.empty(shape, dtype=self.dtype, pin_memory=True)
        self.host_alloc = BlockAllocator(num_host_blocks, self.block_size)

    def _move(self, src_alloc, dst_alloc, src_caches, dst_caches, seq_ids, stream):
        pairs = src_alloc.move_to(dst_alloc, seq_ids)    # host: sharing kept, all or nothing
        if pairs:
            t = torch.tensor(pairs, dtype=torch.int64, device=self.device)
            pa_swap_blocks(dst_caches[0], dst_caches[1], src_caches[0], src_caches[1], t,
                           stream=stream)
        return pairs

    def swap_out(self, seq_ids: Sequence[int], stream=None) -> List[Tuple[int, int]]:
        """Move the sequences' blocks to the host pool and release them here
        (blocks shared among them stay shared).  Returns the (device block,
        host block) pairs copied; stream order keeps any later write to a
        released block after the copy."""
        if self.host_alloc is None:
            raise RuntimeError("enable_swap() first")
        return self._move(self.alloc, self.host_alloc, (self.k_cache, self.v_cache),
                          (self.host_k, self.host_v), seq_ids, stream)

    def swap_in(self, seq_ids: Sequence[int], stream=None) -> List[Tuple[int, int]]:
        """Bring swapped-out sequences back into fresh device blocks.  Returns the
        (host block, device block) pairs copied; block tables change accordingly."""
        if self.host_alloc is None:
            raise RuntimeError("enable_swap() first")
        return self._move(self.host_alloc, self.alloc, (self.host_k, self.host_v),
                          (self.k_cache, self.v_cache), seq_ids, stream)
