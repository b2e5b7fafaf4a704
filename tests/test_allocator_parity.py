"""The C++ host allocator (through the C ABI) against the oracle allocator:
identical slots, tables, copy-on-write pairs, reference counts and free
stack, bit for bit, on scripted and seeded random operation sequences."""

import random

import numpy as np
import pytest

import oracle
from paged_kv_cache_359_b200 import BlockAllocator, OutOfBlocks, PagedAttnError


def same_state(c, o):
    assert c.free_order() == o.free_order()
    assert c.ref_counts() == o.ref
    assert c.num_free() == o.num_free()


def test_create_and_lifo():
    order = [3, 1, 4, 0, 2]
    c, o = BlockAllocator(5, 16, order), oracle.BlockAllocator(5, 16, order)
    same_state(c, o)
    for _ in range(3):
        assert c.allocate() == o.allocate()
    c.decref(1); o.decref(1)
    c.decref(3); o.decref(3)
    same_state(c, o)
    with pytest.raises(Exception):
        c.decref(1)


def test_out_of_blocks_is_atomic():
    c = BlockAllocator(3, 4)
    tables = np.full((2, 4), -1, dtype=np.int32)
    lengths = np.array([4, 4], dtype=np.int32)
    for i in range(2):
        _, _, lengths[i] = c.extend(tables[i], 0, 4)
    before = (c.free_order(), c.ref_counts(), tables.copy(), lengths.copy())
    with pytest.raises(OutOfBlocks):
        c.append_slots(tables, lengths)
    assert (c.free_order(), c.ref_counts()) == before[:2]
    assert (tables == before[2]).all() and (lengths == before[3]).all()


@pytest.mark.parametrize("bs", [4, 16])
def test_prefix_fork_and_copy_on_write(bs):
    nb, cap = 64, 16
    order = list(np.random.default_rng(bs).permutation(nb))
    c, o = BlockAllocator(nb, bs, order), oracle.BlockAllocator(nb, bs, order)
    plen = 3 * bs + bs // 2
    ct = np.full((8, cap), -1, dtype=np.int32)
    slots_c, cow_c, lc = c.extend(ct[0], 0, plen)
    ot0 = []
    slots_o, cow_o, lo = oracle.extend(o, ot0, 0, plen)
    assert list(slots_c) == slots_o and cow_c is None and cow_o is None and lc == lo
    n = -(-plen // bs)
    ots = [ot0]
    for i in range(1, 8):
        c.fork(ct[0], n, ct[i])
        ots.append(oracle.fork(o, ot0))
    same_state(c, o)
    lens_c = np.full(8, plen, dtype=np.int32)
    lens_o = [plen] * 8
    for step in range(bs):
        sc, pc = c.append_slots(ct, lens_c)
        so, po = oracle.append_slots(o, ots, lens_o)
        assert list(sc) == so
        assert [tuple(p) for p in pc.tolist()] == po
        assert list(lens_c) == lens_o
        for i in range(8):
            assert list(ct[i, : -(-lens_c[i] // bs)]) == ots[i]
        same_state(c, o)
    for i in range(8):
        c.free(ct[i], -(-int(lens_c[i]) // bs))
        oracle.free_sequence(o, ots[i])
    same_state(c, o)
    assert c.num_free() == nb


@pytest.mark.parametrize("seed", range(8))
def test_random_operation_sequences(seed):
    rng = random.Random(100 + seed)
    bs = rng.choice([4, 8, 16])
    nb = rng.randint(8, 80)
    cap = 40
    order = list(range(nb))
    rng.shuffle(order)
    c, o = BlockAllocator(nb, bs, order), oracle.BlockAllocator(nb, bs, order)
    ctabs, otabs, lens = [], [], []
    for _ in range(400):
        op = rng.random()
        if op < 0.4 and ctabs:
            i = rng.randrange(len(ctabs))
            try:
                so, cow_o, lo = oracle.append_slot(o, otabs[i], lens[i])
            except oracle.OutOfBlocks:
                with pytest.raises(OutOfBlocks):
                    c.append_slot(ctabs[i], lens[i])
            else:
                sc, cow_c, lc = c.append_slot(ctabs[i], lens[i])
                assert (sc, cow_c, lc) == (so, cow_o, lo)
                lens[i] = lo
        elif op < 0.55:
            k = rng.randint(0, 3 * bs)
            t = np.full(cap, -1, dtype=np.int32)
            ot = []
            try:
                so, _, lo = oracle.extend(o, ot, 0, k)
            except oracle.OutOfBlocks:
                with pytest.raises(OutOfBlocks):
                    c.extend(t, 0, k)
                continue
            sc, _, lc = c.extend(t, 0, k)
            assert list(sc) == so and lc == lo
            ctabs.append(t); otabs.append(ot); lens.append(lo)
        elif op < 0.7 and ctabs:
            i = rng.randrange(len(ctabs))
            t = np.full(cap, -1, dtype=np.int32)
            c.fork(ctabs[i], -(-lens[i] // bs), t)
            ctabs.append(t); otabs.append(oracle.fork(o, otabs[i])); lens.append(lens[i])
        elif op < 0.8 and ctabs:
            i = rng.randrange(len(ctabs))
            c.free(ctabs.pop(i), -(-lens[i] // bs))
            oracle.free_sequence(o, otabs.pop(i))
            lens.pop(i)
        elif ctabs:
            tabs = np.stack(ctabs)
            ln = np.array(lens, dtype=np.int32)
            olens = list(lens)
            try:
                so, po = oracle.append_slots(o, otabs, olens)
            except oracle.OutOfBlocks:
                with pytest.raises(OutOfBlocks):
                    c.append_slots(tabs, ln)
            else:
                sc, pc = c.append_slots(tabs, ln)
                assert list(sc) == so and [tuple(p) for p in pc.tolist()] == po
                for i in range(len(ctabs)):
                    ctabs[i][:] = tabs[i]
                lens = list(ln)
                assert lens == olens
        same_state(c, o)
        for t, ot, ln in zip(ctabs, otabs, lens):
            assert list(t[: -(-ln // bs)]) == ot


@pytest.mark.parametrize("seed", range(4))
def test_compaction_matches_the_oracle(seed):
    rng = random.Random(900 + seed)
    bs, nb, cap = 8, 120, 20
    order = list(range(nb))
    rng.shuffle(order)
    c, o = BlockAllocator(nb, bs, order), oracle.BlockAllocator(nb, bs, order)
    ctabs, otabs, lens = [], [], []
    for _ in range(10):
        k = rng.randint(1, 6 * bs)
        t = np.full(cap, -1, dtype=np.int32)
        ot = []
        c.extend(t, 0, k)
        oracle.extend(o, ot, 0, k)
        ctabs.append(t); otabs.append(ot); lens.append(k)
    for i in (0, 3):
        t = np.full(cap, -1, dtype=np.int32)
        c.fork(ctabs[i], -(-lens[i] // bs), t)
        ctabs.append(t); otabs.append(oracle.fork(o, otabs[i])); lens.append(lens[i])
    for i in (2, 5, 7):
        c.free(ctabs[i], -(-lens[i] // bs))
        oracle.free_sequence(o, otabs[i])
    keep = [i for i in range(len(ctabs)) if i not in (2, 5, 7)]
    live = sum(1 for r in o.ref if r > 0)
    target = live + rng.randint(0, 3)
    cm = c.compact(target)
    om = oracle.compact(o, target)
    assert [tuple(m) for m in cm.tolist()] == om
    # the batch call on a copy of the kept tables (entries past each row's
    # length stay untouched), then the per-table call
    batch = np.stack([ctabs[i] for i in keep])
    nblk = np.array([-(-lens[i] // bs) for i in keep], dtype=np.int32)
    tail = [batch[r, n:].copy() for r, n in enumerate(nblk)]
    BlockAllocator.remap_batch(batch, nblk, cm)
    for r, i in enumerate(keep):
        n = int(nblk[r])
        assert list(batch[r, :n]) == oracle.remap(otabs[i], om)
        assert (batch[r, n:] == tail[r]).all()
    for i in keep:
        n = -(-lens[i] // bs)
        BlockAllocator.remap(ctabs[i], n, cm)
        assert list(ctabs[i][:n]) == oracle.remap(otabs[i], om)
    assert c.free_order() == o.free_order()
    assert c.ref_counts() == o.ref
    # below the live count: refused, nothing changes
    before = (c.free_order(), c.ref_counts())
    with pytest.raises(OutOfBlocks):
        c.compact(live - 1)
    assert (c.free_order(), c.ref_counts()) == before and c.num_blocks == target
    # remap leaves entries that are not a source alone
    t = np.array([0, 5, 7], dtype=np.int32)
    BlockAllocator.remap(t, 3, np.array([[7, 2], [9, 1]], dtype=np.int32))
    assert list(t) == [0, 5, 2]
    tb = np.array([[0, 5, 7], [9, 7, 9]], dtype=np.int32)
    BlockAllocator.remap_batch(tb, np.array([3, 2]), np.array([[7, 2], [9, 1]], dtype=np.int32))
    assert tb.tolist() == [[0, 5, 2], [1, 2, 9]]
    with pytest.raises(PagedAttnError):        # a row longer than the stride changes nothing
        BlockAllocator.remap_batch(tb, np.array([3, 4]), np.array([[0, 1]], dtype=np.int32))
    assert tb.tolist() == [[0, 5, 2], [1, 2, 9]]
