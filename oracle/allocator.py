"""Oracle block manager: the bookkeeping behind the block tables, in plain Python.

TEST INFRASTRUCTURE ONLY (see the package docstring).  An independent model of
the host allocator exported by the CUDA library; the tests require the two to
agree bit for bit on block tables, context lengths, slots, copy-on-write pairs,
reference counts and the free list.

What the pages fix:
  * "PagedAttention의 설계" (supersilo.blog vLLM summary): the cache is cut into
    fixed-size blocks; a block table links each request's logical blocks to
    physical blocks; the block manager allocates the blocks a request needs as
    it grows and reclaims them.
  * "3. vLLM: KV cache를 블록 단위로 관리하기" (blog.aqudi.me): physical blocks
    need not be contiguous; a new block is taken only when the tokens fill the
    current one; requests with a common prompt point at the same physical
    blocks, copied only when one side has to modify one (copy-on-write).
  * "블록 공유" (supersilo.blog): parallel samples / beams start from one prompt
    and share its blocks.
  * "4.2 PagedAttention의 접근" (hjr-study-book Day 3): worked example, 16-token
    blocks, a 37-token request mapped to physical blocks 7, 2, 9 with 5 tokens
    in the last one.

Readings where the pages are silent (a chosen convention, stated so two
implementations can agree exactly):
  * free blocks form a LIFO stack; the caller may give its initial order (the
    last entry is handed out first), else it is [num_blocks-1, ..., 1, 0] so
    block 0 comes first;
  * freeing a sequence drops one reference from each of its blocks in logical
    order; a block whose count reaches zero is pushed onto the stack;
  * an append that writes into a partially filled last block whose reference
    count is above one first takes a fresh block dst, records the pair
    (old, dst), drops one reference from old and puts dst in the table (the
    copy-on-write); the copy is taken before any new blocks, which follow in
    logical order;
  * an append or fork that cannot get all its blocks changes nothing and fails
    with OOM;
  * moving sequences to another manager (swap to CPU memory and back, "적용
    범위와 관련 연구" of the supersilo.blog summary, which gives no mechanism)
    keeps the sharing among the sequences moved together: going through them in
    the caller's order and through each one's blocks in logical order, a block
    seen for the first time takes the destination's next free block, and later
    holders share it; the sequences are then released in the source in the
    caller's order;
  * prefix caching ("5. Prefix Caching", hjr-study-book Day 3, and "prefix
    caching" in "4. 이 밖의 기법들", blog.aqudi.me: the KV blocks of a prompt
    prefix repeated across requests are reused; no mechanism is given): a full
    block's key is its content chain (previous block's key, its token ids); a
    new request takes the cached blocks of its leading full blocks up to the
    first key with no block, leaving at least one token to compute; committing
    a sequence registers its full blocks (a key keeps its first block, a block
    its first key); a cached block whose count drops to zero waits on an
    evictable list (least recently released evicted first), and an allocation
    takes the free stack before evicting.
"""
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple


class OOM(Exception):
    pass


class Invalid(Exception):
    pass


@dataclass
class _Seq:
    blocks: List[int] = field(default_factory=list)
    num_tokens: int = 0


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int,
                 initial_free_order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise Invalid("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if initial_free_order is None:
            self.free = list(range(num_blocks - 1, -1, -1))
        else:
            order = [int(x) for x in initial_free_order]
            if sorted(order) != list(range(num_blocks)):
                raise Invalid("initial_free_order must be a permutation of 0..num_blocks-1")
            self.free = order
        self.refcount = [0] * num_blocks
        self.seqs: Dict[int, _Seq] = {}
        self.prefix = False
        self.block_of_key: Dict[tuple, int] = {}
        self.key_of_block: Dict[int, tuple] = {}
        self.evictable: List[int] = []

    # -- block hand-out and release (shared by every operation) --
    def _take(self) -> int:
        if self.free:
            blk = self.free.pop()
        else:                                   # evict the least recently released
            blk = self.evictable.pop(0)
            del self.block_of_key[self.key_of_block.pop(blk)]
        self.refcount[blk] = 1
        return blk

    def _drop(self, blk: int) -> None:
        self.refcount[blk] -= 1
        if self.refcount[blk] == 0:
            if self.prefix and blk in self.key_of_block:
                self.evictable.append(blk)
            else:
                self.free.append(blk)

    # -- queries --
    def num_free(self) -> int:
        """Blocks an allocation can take (free stack + evictable)."""
        return len(self.free) + len(self.evictable)

    def free_stack(self) -> List[int]:
        """The free stack bottom to top (the last entry is handed out next)."""
        return list(self.free)

    def blocks_of(self, seq_id: int) -> List[int]:
        return list(self.seqs[seq_id].blocks)

    def num_tokens(self, seq_id: int) -> int:
        return self.seqs[seq_id].num_tokens

    # -- operations --
    def add(self, seq_id: int) -> None:
        if seq_id in self.seqs:
            raise Invalid("sequence exists")
        self.seqs[seq_id] = _Seq()

    def fork(self, parent: int, child: int) -> None:
        """The child shares every block of the parent ("블록 공유")."""
        if parent not in self.seqs or child in self.seqs:
            raise Invalid("missing parent or existing child")
        p = self.seqs[parent]
        for blk in p.blocks:
            self.refcount[blk] += 1
        self.seqs[child] = _Seq(list(p.blocks), p.num_tokens)

    def append(self, seq_id: int, n_tokens: int) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Reserve slots for n_tokens new tokens; returns (slots, cow_pairs).

        slot = physical_block * block_size + offset_in_block, as in the
        37-token example of "4.2 PagedAttention의 접근".
        """
        if seq_id not in self.seqs:
            raise Invalid("unknown sequence")
        if n_tokens < 0:
            raise Invalid("negative token count")
        s = self.seqs[seq_id]
        bs = self.block_size
        T = s.num_tokens
        if n_tokens == 0:
            return [], []
        # Copy-on-write is needed when the first new token lands inside an
        # existing, shared last block.
        cow = (T % bs != 0) and self.refcount[s.blocks[-1]] > 1
        blocks_after = -(-(T + n_tokens) // bs)
        new_blocks = blocks_after - len(s.blocks)
        need = new_blocks + (1 if cow else 0)
        if need > self.num_free():
            raise OOM("not enough free blocks")
        pairs: List[Tuple[int, int]] = []
        if cow:
            old = s.blocks[-1]
            dst = self._take()
            self._drop(old)                     # still held by its other sharers
            s.blocks[-1] = dst
            pairs.append((old, dst))
        for _ in range(new_blocks):
            s.blocks.append(self._take())
        slots = [s.blocks[t // bs] * bs + t % bs for t in range(T, T + n_tokens)]
        s.num_tokens = T + n_tokens
        return slots, pairs

    def release(self, seq_id: int) -> None:
        """Drop the sequence; blocks nobody references go back to the stack."""
        if seq_id not in self.seqs:
            raise Invalid("unknown sequence")
        for blk in self.seqs.pop(seq_id).blocks:
            self._drop(blk)

    def move_to(self, dst: "BlockManager", seq_ids: Sequence[int]) -> List[Tuple[int, int]]:
        """Move the sequences into dst; returns the (source block, dst block)
        pairs whose contents must be copied."""
        seq_ids = [int(x) for x in seq_ids]
        if dst is self or dst.block_size != self.block_size:
            raise Invalid("bad destination")
        if len(set(seq_ids)) != len(seq_ids):
            raise Invalid("repeated sequence")
        for sid in seq_ids:
            if sid not in self.seqs or sid in dst.seqs:
                raise Invalid("unknown sequence or already in the destination")
        distinct = {blk for sid in seq_ids for blk in self.seqs[sid].blocks}
        if len(distinct) > dst.num_free():
            raise OOM("not enough free blocks in the destination")
        where: Dict[int, int] = {}
        pairs: List[Tuple[int, int]] = []
        for sid in seq_ids:
            s = self.seqs[sid]
            mapped = []
            for blk in s.blocks:
                if blk in where:
                    dst.refcount[where[blk]] += 1
                else:
                    new = dst._take()
                    where[blk] = new
                    pairs.append((blk, new))
                mapped.append(where[blk])
            dst.seqs[sid] = _Seq(mapped, s.num_tokens)
        for sid in seq_ids:
            self.release(sid)
        return pairs

    # -- prefix caching --
    def enable_prefix_cache(self) -> None:
        self.prefix = True

    def add_cached(self, seq_id: int, token_ids: Sequence[int]) -> int:
        """New sequence holding the cached blocks of its leading full blocks;
        returns the number of tokens they cover."""
        if seq_id in self.seqs:
            raise Invalid("sequence exists")
        toks = [int(t) for t in token_ids]
        bs = self.block_size
        blocks: List[int] = []
        if self.prefix and toks:
            key = None
            for k in range((len(toks) - 1) // bs):
                key = (key, tuple(toks[k * bs:(k + 1) * bs]))
                blk = self.block_of_key.get(key)
                if blk is None:
                    break
                if self.refcount[blk] == 0:
                    self.evictable.remove(blk)
                self.refcount[blk] += 1
                blocks.append(blk)
        self.seqs[seq_id] = _Seq(blocks, len(blocks) * bs)
        return len(blocks) * bs

    def commit(self, seq_id: int, token_ids: Sequence[int]) -> None:
        """Register the sequence's full blocks under their content keys."""
        if seq_id not in self.seqs:
            raise Invalid("unknown sequence")
        toks = [int(t) for t in token_ids]
        s = self.seqs[seq_id]
        if len(toks) > s.num_tokens:
            raise Invalid("more tokens than the sequence holds")
        if not self.prefix:
            return
        bs = self.block_size
        key = None
        for k in range(len(toks) // bs):
            key = (key, tuple(toks[k * bs:(k + 1) * bs]))
            blk = s.blocks[k]
            if key not in self.block_of_key and blk not in self.key_of_block:
                self.block_of_key[key] = blk
                self.key_of_block[blk] = key

    def build_tables(self, seq_ids: Sequence[int], max_blocks: int):
        """Block tables [B][max_blocks] (padding -1) and context lengths [B]."""
        import numpy as np
        B = len(seq_ids)
        tables = np.full((B, max_blocks), -1, dtype=np.int32)
        lens = np.zeros(B, dtype=np.int32)
        for i, sid in enumerate(seq_ids):
            if sid not in self.seqs:
                raise Invalid("unknown sequence")
            s = self.seqs[sid]
            if len(s.blocks) > max_blocks:
                raise Invalid("table row too short")
            tables[i, :len(s.blocks)] = s.blocks
            lens[i] = s.num_tokens
        return tables, lens
