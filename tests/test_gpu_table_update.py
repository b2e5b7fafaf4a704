"""pa_update_block_tables, the "update the mapping" step of a decode step:
after the oracle allocator appends one token per sequence (new blocks,
copy-on-write replacements of a shared half-full block, in-place writes),
the device tables updated from the step's lengths and slots must equal the
oracle's host tables bit for bit, step after step, and entries past each
sequence's length must keep their old values."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_359_b200 as pa
from gpu_common import device_clean

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_device_tables_follow_the_host_allocator(bs):
    rng = np.random.default_rng(300 + bs)
    nb, s, cap = 400, 12, 40
    alloc = oracle.BlockAllocator(nb, bs, rng.permutation(nb).astype(np.int32))
    tables, lens = [], []
    # sequences 0..5 fork one prompt whose last block is half full (their
    # first appends copy it), 6..11 are independent with ragged lengths
    root = []
    _, _, plen = oracle.extend(alloc, root, 0, 3 * bs + bs // 2)
    for _ in range(6):
        tables.append(oracle.fork(alloc, root))
        lens.append(plen)
    oracle.free_sequence(alloc, root)
    for _ in range(6):
        t = []
        _, _, ln = oracle.extend(alloc, t, 0, int(rng.integers(1, 4 * bs)))
        tables.append(t)
        lens.append(ln)

    def host_array():
        a = np.full((s, cap), -7, dtype=np.int32)        # a sentinel past every length
        for i, t in enumerate(tables):
            a[i, :len(t)] = t
        return a

    dev = torch.from_numpy(host_array()).cuda()
    cows_seen = 0
    for step in range(2 * bs + 3):
        slots, cows = oracle.append_slots(alloc, tables, lens)
        cows_seen += len(cows)
        slots = np.array(slots, dtype=np.int64)
        if step % 5 == 4:
            slots[step % s] = -1        # a sequence that gains no token keeps its entry
            want = host_array()
            want[step % s] = dev[step % s].cpu().numpy()
        else:
            want = host_array()
        pa.pa_update_block_tables(dev, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                  torch.from_numpy(slots).cuda(), bs, nb)
        torch.cuda.synchronize()
        got = dev.cpu().numpy()
        assert (got == want).all(), step
        if step % 5 == 4:                # bring the skipped entry in line for the next step
            dev[step % s] = torch.from_numpy(host_array()[step % s]).cuda()
    assert cows_seen == 5               # every sharer but the last copied the shared block
    device_clean()


def test_out_of_pool_slot_is_flagged_and_skipped():
    dev = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    lens = torch.tensor([3, 5], dtype=torch.int32, device="cuda")
    slots = torch.tensor([16 * 100 + 2, 16 + 4], dtype=torch.int64, device="cuda")
    pa.pa_update_block_tables(dev, lens, slots, 16, 50)
    flags = pa.pa_device_error(clear=True)
    assert flags == 8
    assert dev.cpu().tolist() == [[0, 0, 0, 0], [1, 0, 0, 0]]
