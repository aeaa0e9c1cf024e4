"""Host-side block manager used to build block tables for the synthetic workloads.

This is input construction, not attention arithmetic: it decides which physical
block of the pool each logical block of a sequence lives in, and which blocks are
shared between sequences.

Rules followed (nano vllm KV-cache practice page):
  * a block holds a fixed number of token positions and has an id, a reference
    count, a content hash (-1 when unset) and the token ids it holds
    (section 3.2.1, "Block设计");
  * allocation walks a request's blocks; the hash of each block is looked up in a
    hash -> block id map: a hit reuses the block and increments its reference
    count, a miss takes a fresh block with reference count 1 and records its hash
    (section 3.2.2, "BlockManager核心逻辑");
  * finishing a request decrements the reference count of each of its blocks and a
    block whose count reaches zero is returned to the free list (section 3.2.1);
  * the hash of a block is a rolling hash h = (h * 31 + token) mod 2**32 seeded
    with the hash of the previous block, so a hit implies the whole prefix matched
    (section 4.2, "前缀共享实现").

Readings where the page is silent:
  * a hash hit is confirmed by comparing token ids (the Block keeps them), which
    guards against 32-bit collisions;
  * a trailing partial chunk (fewer tokens than a block) whose whole prefix chain
    matched and whose tokens are a prefix of an already cached full block's tokens
    reuses that block; it is read, never written, by a decode-only workload.
  * the free list is consumed in a caller-given order (a seeded permutation), so
    physical ids are scattered over the pool.
"""
from __future__ import annotations

from dataclasses import dataclass, field

MASK32 = 0xFFFFFFFF


def compute_hash(token_ids, prefix_hash: int) -> int:
    """Rolling hash of one block's tokens chained on the previous block's hash.

    nano vllm KV-cache practice page, section 4.2: multiply by 31, add the token,
    keep the low 32 bits.
    """
    h = int(prefix_hash)
    for t in token_ids:
        h = (h * 31 + int(t)) & MASK32
    return h


@dataclass
class Block:
    """One physical KV-cache block (nano vllm page, section 3.2.1)."""

    block_id: int
    ref_count: int = 0
    hash: int = -1
    token_ids: list = field(default_factory=list)
    parent_hash: int = -1


class BlockManager:
    """Reference-counted, hash-shared allocator of physical KV blocks."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.block_size = int(block_size)
        self.blocks = [Block(i) for i in range(num_blocks)]
        order = list(range(num_blocks)) if free_order is None else [int(i) for i in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        # consumed from the front
        self.free = list(order)
        self._free_pos = 0
        self.hash_to_block_id: dict[int, int] = {}
        # parent hash -> ids of cached full blocks chained on it (partial-tail reuse)
        self._children: dict[int, list[int]] = {}

    # -- allocation -------------------------------------------------------
    def _take_free(self) -> Block:
        while self._free_pos < len(self.free):
            bid = self.free[self._free_pos]
            self._free_pos += 1
            blk = self.blocks[bid]
            if blk.ref_count == 0:
                if blk.hash != -1:
                    self._forget(blk)
                return blk
        raise MemoryError("KV block pool exhausted")

    def _forget(self, blk: Block) -> None:
        if self.hash_to_block_id.get(blk.hash) == blk.block_id:
            del self.hash_to_block_id[blk.hash]
        kids = self._children.get(blk.parent_hash)
        if kids and blk.block_id in kids:
            kids.remove(blk.block_id)
        blk.hash = -1
        blk.token_ids = []
        blk.parent_hash = -1

    def allocate(self, token_ids) -> list[int]:
        """Return the block table (physical ids) for a request's tokens."""
        bs = self.block_size
        table: list[int] = []
        h = 0
        chain_ok = True
        n = len(token_ids)
        for start in range(0, n, bs):
            chunk = [int(t) for t in token_ids[start:start + bs]]
            if len(chunk) == bs:
                parent = h
                h = compute_hash(chunk, h)
                bid = self.hash_to_block_id.get(h) if chain_ok else None
                if bid is not None and self.blocks[bid].token_ids == chunk:
                    blk = self.blocks[bid]
                    blk.ref_count += 1
                else:
                    chain_ok = False
                    blk = self._take_free()
                    blk.ref_count = 1
                    blk.hash = h
                    blk.token_ids = chunk
                    blk.parent_hash = parent
                    self.hash_to_block_id[h] = blk.block_id
                    self._children.setdefault(parent, []).append(blk.block_id)
                table.append(blk.block_id)
            else:
                blk = None
                if chain_ok:
                    for bid in self._children.get(h, []):
                        cand = self.blocks[bid]
                        if cand.token_ids[:len(chunk)] == chunk:
                            blk = cand
                            break
                if blk is not None:
                    blk.ref_count += 1
                else:
                    blk = self._take_free()
                    blk.ref_count = 1
                    blk.hash = -1
                    blk.token_ids = chunk
                table.append(blk.block_id)
        return table

    def free_table(self, table) -> None:
        """Finish a request: drop one reference on each of its blocks."""
        for bid in table:
            blk = self.blocks[int(bid)]
            if blk.ref_count <= 0:
                raise RuntimeError(f"double free of block {bid}")
            blk.ref_count -= 1
            if blk.ref_count == 0:
                self._forget(blk)
                self.free.append(blk.block_id)

    def append(self, table: list, pos: int, token_id: int):
        """Decode append: the slot of position `pos` (the sequence's current length)
        of a sequence whose blocks are `table` (updated in place), and the
        (src, dst) block copy the step needs first, or None.

        Readings (the pages share blocks by reference count and never write into a
        shared one): a position that starts a block takes a fresh block; a block
        other sequences also hold (ref_count > 1) is replaced by a private copy
        (copy-on-write); a private block that is still registered under a hash is
        dropped from the hash map before it is written (a later request must not
        find it by a hash its contents no longer match). Blocks filled by appends
        are not hashed.
        """
        bs = self.block_size
        bi, off = divmod(int(pos), bs)
        if bi == len(table):
            if off:
                raise ValueError("pos skips a block")
            blk = self._take_free()
            blk.ref_count = 1
            blk.hash = -1
            blk.token_ids = [int(token_id)]
            table.append(blk.block_id)
            return blk.block_id * bs, None
        if bi > len(table) or bi < 0:
            raise ValueError("pos outside the table")
        blk = self.blocks[int(table[bi])]
        copy = None
        if blk.ref_count > 1:
            new = self._take_free()
            new.ref_count = 1
            new.hash = -1
            new.token_ids = list(blk.token_ids[:off])
            blk.ref_count -= 1
            copy = (blk.block_id, new.block_id)
            table[bi] = new.block_id
            blk = new
        elif blk.hash != -1:
            keep = list(blk.token_ids[:off])
            self._forget(blk)
            blk.token_ids = keep
        del blk.token_ids[off:]
        blk.token_ids.append(int(token_id))
        return blk.block_id * bs + off, copy

    # -- introspection ----------------------------------------------------
    def num_used(self) -> int:
        return sum(1 for b in self.blocks if b.ref_count > 0)

    def ref_counts(self) -> list[int]:
        return [b.ref_count for b in self.blocks]
