"""Pins for the oracle's block allocator: invariants that the pages fix
(reference counts, immediate reclamation, on-demand growth, sharing,
copy-on-write), checked on scripted and seeded random operation sequences."""

import random

import pytest

import oracle
from conftest import read_golden


def check_invariants(alloc, tables):
    """tables: the block lists of every live sequence."""
    nb = alloc.num_blocks
    held = [0] * nb
    for t in tables:
        for b in t:
            held[b] += 1
    # every reference is a table entry, and every table entry a reference
    assert held == alloc.ref
    free = alloc.free_order()
    assert len(set(free)) == len(free)
    assert all(alloc.ref_count(b) == 0 for b in free)
    # a block is either free or referenced
    assert alloc.num_free() + sum(1 for r in alloc.ref if r > 0) == nb


def test_waste_example_on_demand_allocation():
    """An average 128-token request holds 8 blocks of 16 (no waste), where
    reserving the 2048-token maximum would waste 93.75 %."""
    vals = {k: v for k, v in read_golden("waste_example.txt")}
    avg, mx = int(vals["avg_tokens"]), int(vals["max_tokens"])
    bs = int(vals["block_size"])
    assert 100.0 * (mx - avg) / mx == float(vals["waste_percent"])
    alloc = oracle.BlockAllocator(mx // bs, bs)
    table, length = [], 0
    for _ in range(avg):
        _, _, length = oracle.append_slot(alloc, table, length)
    assert len(table) == avg // bs
    assert len(table) * bs - length == 0
    assert alloc.num_free() == mx // bs - avg // bs


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_internal_fragmentation_below_one_block(bs):
    alloc = oracle.BlockAllocator(400, bs)
    for length_target in [1, bs - 1, bs, bs + 1, 5 * bs + 3]:
        table, length = [], 0
        for _ in range(length_target):
            _, _, length = oracle.append_slot(alloc, table, length)
        assert len(table) == -(-length_target // bs)
        assert 0 <= len(table) * bs - length_target < bs
        oracle.free_sequence(alloc, table)
    assert alloc.num_free() == 400


def test_initial_order_and_lifo_reuse():
    alloc = oracle.BlockAllocator(5, 16, [3, 1, 4, 0, 2])
    assert [alloc.allocate() for _ in range(3)] == [3, 1, 4]
    alloc.decref(1)
    alloc.decref(3)
    assert alloc.free_order() == [3, 1, 0, 2]
    assert alloc.allocate() == 3


def test_out_of_blocks_changes_nothing():
    alloc = oracle.BlockAllocator(2, 4)
    tables = [[], []]
    lengths = [0, 0]
    oracle.append_slots(alloc, tables, lengths)
    before = (alloc.free_order(), list(alloc.ref), [list(t) for t in tables], list(lengths))
    lengths = [4, 4]
    with pytest.raises(oracle.OutOfBlocks):
        oracle.append_slots(alloc, tables, lengths)
    assert (alloc.free_order(), list(alloc.ref), [list(t) for t in tables], list(lengths)) == \
        (before[0], before[1], before[2], [4, 4])
    with pytest.raises(oracle.OutOfBlocks):
        oracle.extend(alloc, tables[0], 4, 1)
    assert alloc.free_order() == before[0] and alloc.ref == before[1]


def test_fork_shares_and_counts():
    alloc = oracle.BlockAllocator(20, 4)
    parent, length = [], 0
    _, _, length = oracle.extend(alloc, parent, length, 10)
    children = [oracle.fork(alloc, parent) for _ in range(3)]
    assert all(c == parent for c in children)
    assert all(alloc.ref_count(b) == 4 for b in parent)
    check_invariants(alloc, [parent] + children)


def test_copy_on_write_of_a_shared_partial_block():
    """The shared last block is copied before a write; the sharers keep the
    old block; the last sharer to write holds the only reference and writes
    in place."""
    bs = 4
    alloc = oracle.BlockAllocator(30, bs)
    parent, plen = [], 0
    _, _, plen = oracle.extend(alloc, parent, plen, 10)      # last block half full
    shared_last = parent[-1]
    seqs = [parent] + [oracle.fork(alloc, parent) for _ in range(3)]
    lengths = [plen] * 4
    slots, cows = oracle.append_slots(alloc, seqs, lengths)
    # three copies (the first three writers), the fourth writes in place
    assert [c[0] for c in cows] == [shared_last] * 3
    assert seqs[3][-1] == shared_last
    assert alloc.ref_count(shared_last) == 1
    for i in range(3):
        assert seqs[i][-1] == cows[i][1]
        assert slots[i] == cows[i][1] * bs + plen % bs
    assert slots[3] == shared_last * bs + plen % bs
    # untouched shared full blocks keep their counts
    assert all(alloc.ref_count(b) == 4 for b in parent[:-1])
    check_invariants(alloc, seqs)


def test_extend_equals_repeated_append_slot():
    a1 = oracle.BlockAllocator(50, 8, list(reversed(range(50))))
    a2 = oracle.BlockAllocator(50, 8, list(reversed(range(50))))
    t1, t2 = [], []
    s1, _, l1 = oracle.extend(a1, t1, 0, 37)
    l2, s2 = 0, []
    for _ in range(37):
        s, _, l2 = oracle.append_slot(a2, t2, l2)
        s2.append(s)
    assert (s1, t1, l1) == (s2, t2, l2)
    assert a1.free_order() == a2.free_order() and a1.ref == a2.ref


def test_free_all_returns_every_block():
    alloc = oracle.BlockAllocator(64, 8)
    seqs, lens = [], []
    for n in [3, 17, 8, 0, 40]:
        t, length = [], 0
        _, _, length = oracle.extend(alloc, t, length, n)
        seqs.append(t)
        lens.append(length)
    seqs.append(oracle.fork(alloc, seqs[1]))
    for t in seqs:
        oracle.free_sequence(alloc, t)
    assert alloc.num_free() == 64
    assert all(r == 0 for r in alloc.ref)


@pytest.mark.parametrize("seed", range(6))
def test_random_operation_sequences_keep_invariants(seed):
    rng = random.Random(seed)
    bs = rng.choice([4, 8, 16])
    nb = rng.randint(8, 60)
    order = list(range(nb))
    rng.shuffle(order)
    alloc = oracle.BlockAllocator(nb, bs, order)
    seqs, lens = [], []
    for _ in range(300):
        op = rng.random()
        try:
            if op < 0.45 and seqs:
                i = rng.randrange(len(seqs))
                _, _, lens[i] = oracle.append_slot(alloc, seqs[i], lens[i])
            elif op < 0.6:
                t, length = [], 0
                _, _, length = oracle.extend(alloc, t, 0, rng.randint(0, 3 * bs))
                seqs.append(t)
                lens.append(length)
            elif op < 0.75 and seqs:
                i = rng.randrange(len(seqs))
                seqs.append(oracle.fork(alloc, seqs[i]))
                lens.append(lens[i])
            elif op < 0.85 and seqs:
                i = rng.randrange(len(seqs))
                oracle.free_sequence(alloc, seqs.pop(i))
                lens.pop(i)
            elif seqs:
                oracle.append_slots(alloc, seqs, lens)
        except oracle.OutOfBlocks:
            pass
        check_invariants(alloc, seqs)
        for t, length in zip(seqs, lens):
            assert len(t) == -(-length // bs)


@pytest.mark.parametrize("seed", range(5))
def test_compaction_packs_live_blocks_below_the_target(seed):
    """After compaction every table points below the target, every moved
    block's count travelled with it, the pool invariants hold at the new
    size, and the moves are distinct high sources onto distinct free low
    destinations."""
    rng = random.Random(500 + seed)
    bs = rng.choice([4, 8])
    nb = 96
    order = list(range(nb))
    rng.shuffle(order)
    alloc = oracle.BlockAllocator(nb, bs, order)
    seqs, lens = [], []
    for _ in range(8):
        t, length = [], 0
        _, _, length = oracle.extend(alloc, t, 0, rng.randint(1, 5 * bs))
        seqs.append(t)
        lens.append(length)
    for i in range(3):
        seqs.append(oracle.fork(alloc, seqs[i]))
        lens.append(lens[i])
    for i in (1, 4):
        oracle.free_sequence(alloc, seqs[i])
    seqs = [t for i, t in enumerate(seqs) if i not in (1, 4)]
    live = sum(1 for r in alloc.ref if r > 0)
    counts = {b: alloc.ref[b] for b in range(nb) if alloc.ref[b] > 0}
    target = live + rng.randint(0, 5)
    moves = oracle.compact(alloc, target)
    assert len({s for s, _ in moves}) == len(moves) == len({d for _, d in moves})
    assert all(s >= target > d for s, d in moves)
    seqs = [oracle.remap(t, moves) for t in seqs]
    assert all(b < target for t in seqs for b in t)
    where = dict(moves)
    for b, c in counts.items():
        assert alloc.ref[where.get(b, b)] == c
    assert alloc.num_blocks == target
    check_invariants(alloc, seqs)


def test_compaction_beyond_the_live_blocks_changes_nothing():
    alloc = oracle.BlockAllocator(10, 4)
    t = []
    oracle.extend(alloc, t, 0, 24)                     # 6 live blocks
    before = (alloc.free_order(), list(alloc.ref))
    with pytest.raises(oracle.OutOfBlocks):
        oracle.compact(alloc, 5)
    assert (alloc.free_order(), list(alloc.ref)) == before
