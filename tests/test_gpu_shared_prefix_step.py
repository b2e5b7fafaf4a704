"""pa_decode_shared_prefix_step (the cascade decode as a whole step: the
own-token pass also stores each sequence's new token and sets its last table
entry from the new slot) against the oracle, step after step:

* groups of forks share whole-block prefixes beside singletons and groups
  without a prefix, G in {1, 4, 8}; and the prefix workload (64 forks of a
  prompt whose half-full last block is copied on the first append of each
  sharer that has not written yet);
* the device tables never receive a step's new block before the call
  (entries past every length hold an id outside the pool);
* after each call the tables equal the oracle allocator's, the caches equal
  the oracle's copy-on-write copies and row writes bit for bit, the output is
  within tolerance of the oracle's decode and bit-identical to
  pa_update_block_tables, pa_reshape_and_cache and pa_decode_shared_prefix
  run on a second copy of the state."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, same_bits

pytestmark = pytest.mark.gpu

OUTSIDE = -7


def _host_array(tables, cap):
    a = np.full((len(tables), cap), OUTSIDE, dtype=np.int32)
    for i, t in enumerate(tables):
        a[i, :len(t)] = t
    return a


def _steps(alloc, tables, lens, starts, prefixes, hq, hk, d, steps, seed, skip_every=3):
    """Run ``steps`` decode steps through the fused call and the three-call
    reference path on two copies of one state; check each against the oracle."""
    bs, nb = alloc.block_size, alloc.num_blocks
    s = len(tables)
    cap = max(len(t) for t in tables) + steps // bs + 3
    lens_np = np.array(lens, dtype=np.int32)
    owned = pa_inputs.owned_rows(_host_array(tables, cap), lens_np, bs, nb)
    gen = pa_inputs.generator("cpu", seed)
    kc_h = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cpu", owned)
    vc_h = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cpu", owned)
    kc, vc = kc_h.cuda(), vc_h.cuda()
    kc2, vc2 = kc_h.cuda(), vc_h.cuda()
    tab = torch.from_numpy(_host_array(tables, cap)).cuda()
    tab2 = tab.clone()
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    pl = torch.tensor(prefixes, dtype=torch.int32, device="cuda")
    max_group = int(np.max(np.diff(starts)))
    max_prefix = int(max(prefixes))
    member_prefix = np.repeat(np.array(prefixes), np.diff(starts))
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(s, hq, d, max_prefix),
                     dtype=torch.uint8, device="cuda")
    ws2 = torch.empty_like(ws)
    scale = d ** -0.5
    cows_seen = 0
    for step in range(steps):
        skip = {(7 * step + 1) % s} if step % skip_every == skip_every - 1 else set()
        slots, cows = [], []
        for i in range(s):
            if i in skip:
                slots.append(-1)
                continue
            slot, cow, lens[i] = oracle.append_slot(alloc, tables[i], lens[i])
            assert lens[i] - 1 >= member_prefix[i]       # the new token is past the prefix
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
        lens_now = np.array(lens, dtype=np.int32)
        ref = oracle.paged_decode(new["q"], kc_h, vc_h, want_tab, lens_now, scale)
        q, key, value = new["q"].cuda(), new["key"].cuda(), new["value"].cuda()
        slots_d = torch.tensor(slots, dtype=torch.int64, device="cuda")
        lens_d = torch.from_numpy(lens_now).cuda()
        out = torch.empty_like(q)
        pa.pa_set_option("validate", 1 if step == 0 else 0)
        try:
            pa.pa_decode_shared_prefix_step(out, q, key, value, kc, vc, slots_d, tab, lens_d,
                                            scale, gs, pl, max_group, max_prefix, ws)
        finally:
            pa.pa_set_option("validate", 0)
        out2 = torch.empty_like(q)
        pa.pa_update_block_tables(tab2, lens_d, slots_d, bs, nb)
        pa.pa_reshape_and_cache(key, value, kc2, vc2, slots_d)
        pa.pa_decode_shared_prefix(out2, q, kc2, vc2, tab2, lens_d, scale, gs, pl, max_group,
                                   max_prefix, ws2)
        torch.cuda.synchronize()
        device_clean()
        assert (tab.cpu().numpy() == want_tab).all(), step
        assert same_bits(kc, kc_h) and same_bits(vc, vc_h), step
        assert same_bits(out, out2), step
        assert_close(out, ref)
    return cows_seen


@pytest.mark.parametrize("g", [1, 4, 8])
def test_step_over_mixed_groups(g):
    rng = np.random.default_rng(900 + g)
    bs, d, hk = 16, 128, 4
    sizes = [40, 1, 7, 3, 1, 12]
    prefixes = [48 * 16, 0, 5 * 16, 16, 0, 33 * 16]
    nb = 4000
    alloc = oracle.BlockAllocator(nb, bs, rng.permutation(nb).astype(np.int32))
    tables, lens = [], []
    for size, plen in zip(sizes, prefixes):
        parent = []
        _, _, p_len = oracle.extend(alloc, parent, 0, plen)
        members = [parent] + [oracle.fork(alloc, parent) for _ in range(size - 1)]
        for t in members:
            _, _, ln = oracle.extend(alloc, t, p_len, int(rng.integers(0, 90)))
            tables.append(t)
            lens.append(ln)
    starts = np.cumsum([0] + sizes).astype(np.int32)
    _steps(alloc, tables, lens, starts, prefixes, hk * g, hk, d, steps=2 * bs + 3,
           seed=910 + g)


@pytest.mark.parametrize("bs,d", [(16, 128), (8, 64), (32, 256)])
def test_step_over_the_prefix_workload(bs, d):
    problem = pa_inputs.prefix(bs, d)
    alloc = oracle.BlockAllocator(problem.num_blocks, bs, problem.free_order)
    parent = []
    _, _, plen = oracle.extend(alloc, parent, 0, problem.prefix_len)
    tables = [parent] + [oracle.fork(alloc, parent) for _ in range(problem.num_seqs - 1)]
    lens = [plen] * problem.num_seqs
    for i, t in enumerate(tables):
        _, _, lens[i] = oracle.extend(alloc, t, plen, int(problem.tail_lens[i]))
    shared = (problem.prefix_len // bs) * bs
    shared -= shared % 16
    sharers = sum(1 for t in tables if alloc.ref_count(t[plen // bs]) > 1)
    cows = _steps(alloc, tables, lens, [0, problem.num_seqs], [shared], problem.num_heads,
                  problem.num_kv_heads, d, steps=3, seed=920 + bs + d, skip_every=10)
    # the sequences that had not written past the prompt copy its shared
    # half-full block on their first append, all but the last of them
    assert cows == max(sharers - 1, 0)
