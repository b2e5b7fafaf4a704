"""Block pool with reference counts, on-demand growth, fork and copy-on-write
(oracle; test infrastructure only).

* The pool is pre-cut into fixed-size frames handed out slab-style from a
  free pool in O(1) ([csdn-QA] §三 item 7; [tech] §2.1, §4.2 item 3).
* Each physical block carries a reference count; ``is_allocated`` is
  ref_count > 0 ([tech] §2.1, struct ``Block``).
* A block whose count drops to zero is reclaimed at once ([tech] §4.2
  item 1; [csdn-QA] §四, pages are released as soon as a request ends).
* A sequence only holds the blocks its tokens need: a new block is taken
  when the current last block is full ([course] ch.2 §2.4.2).
* Fork: a child shares its parent's blocks; the shared blocks' counts go up
  ([tech] §2.1, fork-like sharing; [course] §2.4.3).
* Copy-on-write: a write into a block whose count exceeds one first copies it
  into a fresh block ([course] §2.4.3 pitfall note).

* Compaction: periodic defragmentation ([tech] §2.1 "defragmentation only
  moves block pointers", §4.2 item 2 "defragment every 1000 iterations").
  With fixed-size blocks a free block always serves any request, so the
  useful form is packing live blocks below a target so the pool's tail can
  be released: the data of each moved block is copied (the caller runs the
  copies) and every pointer to it -- table entries -- is rewritten.

Readings where the pages are silent:
* Free pool order: a stack.  It starts as ``initial_free_order`` (element 0
  handed out first); a reclaimed block is pushed on top (LIFO).
* Out of blocks: the call raises ``OutOfBlocks`` and changes nothing.
* Compaction moves the live blocks at or above the target, in ascending id,
  into the free blocks below it, in ascending id; the pool then holds
  exactly the target number of blocks and its free stack lists the remaining
  free blocks in their previous stack order.  It raises ``OutOfBlocks`` (and
  changes nothing) when more blocks are live than the target holds.
* Batched appends process sequences in ascending index; when many sequences
  share one partial block, each but the last one to write copies it, and the
  last one (which then holds the only reference) writes in place.
"""

from __future__ import annotations


class OutOfBlocks(Exception):
    pass


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if initial_free_order is None \
            else [int(b) for b in initial_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial_free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = order                 # free[0] is the top of the stack
        self.ref = [0] * num_blocks

    def allocate(self) -> int:
        if not self.free:
            raise OutOfBlocks()
        block = self.free.pop(0)
        self.ref[block] = 1
        return block

    def incref(self, block: int) -> None:
        if not (0 <= block < self.num_blocks) or self.ref[block] <= 0:
            raise ValueError("incref of a block that is not allocated")
        self.ref[block] += 1

    def decref(self, block: int) -> None:
        if not (0 <= block < self.num_blocks) or self.ref[block] <= 0:
            raise ValueError("decref of a block that is not allocated")
        self.ref[block] -= 1
        if self.ref[block] == 0:
            self.free.insert(0, block)

    def num_free(self) -> int:
        return len(self.free)

    def ref_count(self, block: int) -> int:
        return self.ref[block]

    def free_order(self) -> list:
        return list(self.free)


def append_slot(alloc: BlockAllocator, table: list, length: int):
    """Append one token to a sequence whose blocks are ``table`` (mutated).

    Returns (slot, cow, new_length); ``cow`` is (src, dst) when the last
    block was shared and had to be copied first, else None."""
    bs = alloc.block_size
    if len(table) != -(-length // bs):
        raise ValueError("table length does not match the sequence length")
    cow = None
    if length % bs == 0:
        table.append(alloc.allocate())
    else:
        last = table[length // bs]
        if alloc.ref_count(last) > 1:
            fresh = alloc.allocate()
            alloc.decref(last)
            table[length // bs] = fresh
            cow = (last, fresh)
    slot = table[length // bs] * bs + length % bs
    return slot, cow, length + 1


def _blocks_needed_for_batch(alloc: BlockAllocator, tables, lengths) -> int:
    bs = alloc.block_size
    pending = {}
    need = 0
    for table, length in zip(tables, lengths):
        if length % bs == 0:
            need += 1
        else:
            last = table[length // bs]
            count = pending.get(last, alloc.ref_count(last))
            if count > 1:
                need += 1
                pending[last] = count - 1
    return need


def append_slots(alloc: BlockAllocator, tables: list, lengths: list):
    """One token for each sequence, in ascending index.  Atomic: on
    ``OutOfBlocks`` nothing changes.  Returns (slots, cow_pairs) and updates
    ``tables`` and ``lengths`` in place."""
    if _blocks_needed_for_batch(alloc, tables, lengths) > alloc.num_free():
        raise OutOfBlocks()
    slots, cows = [], []
    for i in range(len(tables)):
        slot, cow, lengths[i] = append_slot(alloc, tables[i], lengths[i])
        slots.append(slot)
        if cow is not None:
            cows.append(cow)
    return slots, cows


def extend(alloc: BlockAllocator, table: list, length: int, num_tokens: int):
    """``num_tokens`` successive appends to one sequence.  Atomic.
    Returns (slots, cow or None, new_length)."""
    bs = alloc.block_size
    if num_tokens <= 0:
        return [], None, length
    cow_needed = length % bs != 0 and alloc.ref_count(table[length // bs]) > 1
    new_blocks = -(-(length + num_tokens) // bs) - (-(-length // bs))
    if new_blocks + int(cow_needed) > alloc.num_free():
        raise OutOfBlocks()
    slots, first_cow = [], None
    for k in range(num_tokens):
        slot, cow, length = append_slot(alloc, table, length)
        slots.append(slot)
        if k == 0:
            first_cow = cow
    return slots, first_cow, length


def fork(alloc: BlockAllocator, parent_table: list) -> list:
    """The child shares every block of the parent."""
    for block in parent_table:
        alloc.incref(block)
    return list(parent_table)


def free_sequence(alloc: BlockAllocator, table: list) -> None:
    for block in table:
        alloc.decref(block)


def compact(alloc: BlockAllocator, target: int) -> list:
    """Shrink the pool to ``target`` blocks; returns the (src, dst) moves."""
    if target < 0 or target > alloc.num_blocks:
        raise ValueError("target outside [0, num_blocks]")
    live_high = [b for b in range(target, alloc.num_blocks) if alloc.ref[b] > 0]
    free_low = sorted(b for b in alloc.free if b < target)
    if len(live_high) > len(free_low):
        raise OutOfBlocks()
    moves = list(zip(live_high, free_low[:len(live_high)]))
    taken = {dst for _, dst in moves}
    for src, dst in moves:
        alloc.ref[dst] = alloc.ref[src]
        alloc.ref[src] = 0
    alloc.free = [b for b in alloc.free if b < target and b not in taken]
    alloc.ref = alloc.ref[:target]
    alloc.num_blocks = target
    return moves


def remap(table: list, moves) -> list:
    """The table with every moved block replaced by its destination."""
    where = {src: dst for src, dst in moves}
    return [where.get(b, b) for b in table]
