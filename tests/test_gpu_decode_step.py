"""pa_decode_step (the mapping update, the cache write of one new token per
sequence and the decode, in one launch) against the oracle, step after step:

* the batch forks one prompt whose last block is half full (the sharers'
  first appends copy it) beside independent sequences of ragged lengths, and
  some sequences skip a step;
* the device tables never receive the step's new block before the call: an
  entry past a sequence's length holds a value outside the pool, so a kernel
  that read it would raise the block-id error and decode zeros;
* after each call the device tables equal the oracle allocator's host tables,
  the caches equal the oracle's copy-on-write copies and row writes bit for
  bit, the attention is within tolerance of the oracle's decode, and the
  output bits equal pa_update_block_tables followed by pa_decode_append on a
  second copy of the same state."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, same_bits

pytestmark = pytest.mark.gpu

OUTSIDE = -7          # table entries past every length


def _host_array(tables, cap):
    a = np.full((len(tables), cap), OUTSIDE, dtype=np.int32)
    for i, t in enumerate(tables):
        a[i, :len(t)] = t
    return a


def _run(bs, d, hq, hk, steps, seed, ctas=0):
    rng = np.random.default_rng(seed)
    nb, cap, n_fork, n_ind = 320, 48, 6, 7
    dt = torch.bfloat16
    alloc = oracle.BlockAllocator(nb, bs, rng.permutation(nb).astype(np.int32))
    tables, lens = [], []
    root = []
    _, _, plen = oracle.extend(alloc, root, 0, 3 * bs + bs // 2)
    for _ in range(n_fork):
        tables.append(oracle.fork(alloc, root))
        lens.append(plen)
    oracle.free_sequence(alloc, root)
    for _ in range(n_ind):
        t = []
        _, _, ln = oracle.extend(alloc, t, 0, int(rng.integers(0, 4 * bs)))
        tables.append(t)
        lens.append(ln)
    s = len(tables)
    gen = pa_inputs.generator("cpu", seed)
    kc_h = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cpu")
    vc_h = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cpu")
    kc, vc = kc_h.cuda(), vc_h.cuda()              # pa_decode_step's state
    kc2, vc2 = kc_h.cuda(), vc_h.cuda()            # update + append's state
    tab = torch.from_numpy(_host_array(tables, cap)).cuda()
    tab2 = tab.clone()
    scale = d ** -0.5
    cows_seen = 0
    if ctas:
        pa.pa_set_option("decode_split_ctas", ctas)
    try:
        for step in range(steps):
            skip = {(step * 5 + 3) % s} if step % 4 == 3 else set()
            slots, cows = [], []
            for i in range(s):
                if i in skip:
                    slots.append(-1)
                    continue
                slot, cow, lens[i] = oracle.append_slot(alloc, tables[i], lens[i])
                slots.append(slot)
                if cow is not None:
                    cows.append(cow)
            cows_seen += len(cows)
            new = pa_inputs.step_tokens(s, hq, hk, d, "bf16", seed, step, "cpu")
            if cows:
                kc_h, vc_h = oracle.copy_blocks(kc_h, vc_h, cows)
                pairs = torch.tensor(cows, dtype=torch.int64, device="cuda")
                pa.pa_copy_blocks(kc, vc, pairs)
                pa.pa_copy_blocks(kc2, vc2, pairs)
            kc_h, vc_h = oracle.reshape_and_cache(new["key"], new["value"], kc_h, vc_h, slots)
            want_tab = _host_array(tables, cap)
            ref = oracle.paged_decode(new["q"], kc_h, vc_h, want_tab, np.array(lens, np.int32),
                                      scale)
            q, key, value = new["q"].cuda(), new["key"].cuda(), new["value"].cuda()
            slots_d = torch.tensor(slots, dtype=torch.int64, device="cuda")
            lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
            out = torch.empty_like(q)
            pa.pa_decode_step(out, q, key, value, kc, vc, slots_d, tab, lens_d, scale)
            out2 = torch.empty_like(q)
            pa.pa_update_block_tables(tab2, lens_d, slots_d, bs, nb)
            pa.pa_decode_append(out2, q, key, value, kc2, vc2, slots_d, tab2, lens_d, scale)
            torch.cuda.synchronize()
            device_clean()
            assert (tab.cpu().numpy() == want_tab).all(), step
            assert same_bits(kc, kc_h) and same_bits(vc, vc_h), step
            assert same_bits(out, out2), step
            assert_close(out, ref)
    finally:
        if ctas:
            pa.pa_set_option("decode_split_ctas", 0)
    assert cows_seen == n_fork - 1          # every sharer but the last copied the shared block


@pytest.mark.parametrize("bs,d,hq,hk", [(16, 128, 32, 8), (8, 64, 8, 8), (32, 256, 16, 2),
                                        (8, 128, 32, 8), (128, 64, 8, 2)])
def test_decode_step_follows_the_allocator(bs, d, hq, hk):
    _run(bs, d, hq, hk, steps=min(bs, 32) + 3, seed=700 + bs + d)


@pytest.mark.parametrize("ctas", [2, 4])
def test_decode_step_in_cluster_mode(ctas):
    _run(16, 128, 32, 8, steps=19, seed=790 + ctas, ctas=ctas)


def test_validate_mode_rejects_a_slot_off_the_new_row():
    bs, d, hk, hq, nb = 16, 128, 2, 8, 64
    gen = pa_inputs.generator("cuda", 5)
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cuda")
    vc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cuda")
    tab = torch.tensor([[3, 9, OUTSIDE], [4, OUTSIDE, OUTSIDE]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([33, 7], dtype=torch.int32, device="cuda")
    new = pa_inputs.step_tokens(2, hq, hk, d, "bf16", 6, 0, "cuda")
    out = torch.empty_like(new["q"])
    pa.pa_set_option("validate", 1)
    try:
        # sequence 0's new token is row 0 of its third block; row 1 is wrong
        bad = torch.tensor([11 * bs + 1, 4 * bs + 6], dtype=torch.int64, device="cuda")
        with pytest.raises(pa.PagedAttnError) as e:
            pa.pa_decode_step(out, new["q"], new["key"], new["value"], kc, vc, bad, tab, lens,
                              d ** -0.5)
        assert e.value.status == 4
        assert tab.cpu().tolist()[0] == [3, 9, OUTSIDE]          # nothing ran
        good = torch.tensor([11 * bs, 4 * bs + 6], dtype=torch.int64, device="cuda")
        pa.pa_decode_step(out, new["q"], new["key"], new["value"], kc, vc, good, tab, lens,
                          d ** -0.5)
        torch.cuda.synchronize()
        assert tab.cpu().tolist() == [[3, 9, 11], [4, OUTSIDE, OUTSIDE]]
    finally:
        pa.pa_set_option("validate", 0)
    device_clean()
