"""GPU parity for prefix sharing and copy-on-write: 64 sequences forked from
one prefix (the last shared block half full, so the first write of each
sharer but the last copies it), divergent tails, one copy_blocks, one
reshape_and_cache, then decode -- for block_size {8,16,32,64,128} x head_dim
{64,128,256}, 32 q / 8 kv heads, bf16."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, same_bits

pytestmark = pytest.mark.gpu


def build(problem):
    """Run the allocator script on both allocators; they must agree exactly."""
    bs, nb, s = problem.block_size, problem.num_blocks, problem.num_seqs
    cap = problem.max_blocks_per_seq
    o = oracle.BlockAllocator(nb, bs, problem.free_order)
    c = pa.BlockAllocator(nb, bs, problem.free_order)
    ot = [[] for _ in range(s)]
    ct = np.full((s, cap), -1, dtype=np.int32)
    _, _, plen = oracle.extend(o, ot[0], 0, problem.prefix_len)
    _, _, plen_c = c.extend(ct[0], 0, problem.prefix_len)
    assert plen == plen_c
    prefix_table = np.array(ot[0], dtype=np.int32)[None]   # before any copy-on-write
    n = -(-plen // bs)
    for i in range(1, s):
        ot[i] = oracle.fork(o, ot[0])
        c.fork(ct[0], n, ct[i])
    lens = [plen] * s
    slots, cows = [], []
    for i in range(s):
        sl, cow, lens[i] = oracle.extend(o, ot[i], plen, int(problem.tail_lens[i]))
        slc, cowc, ln = c.extend(ct[i], plen, int(problem.tail_lens[i]))
        assert list(slc) == sl and cowc == cow and ln == lens[i]
        slots += sl
        if cow is not None:
            cows.append(cow)
    assert c.free_order() == o.free_order() and c.ref_counts() == o.ref
    tables = np.full((s, cap), -1, dtype=np.int32)
    for i in range(s):
        tables[i, :len(ot[i])] = ot[i]
        assert list(ct[i, :len(ot[i])]) == ot[i]
    return tables, np.array(lens, dtype=np.int32), slots, cows, prefix_table


@pytest.mark.parametrize("aligned", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_prefix_sharing_copy_on_write(bs, d, aligned):
    problem = pa_inputs.prefix(bs, d, aligned=aligned)
    tables, lens, slots, cows, prefix_table = build(problem)
    writers = int((problem.tail_lens > 0).sum())
    if aligned:
        assert not cows
    else:
        # every writer but the last sharer standing copies the shared block
        assert len(cows) == writers - 1 if writers == problem.num_seqs else len(cows) == writers
        assert len({c[0] for c in cows}) <= 1

    hk, dt = problem.num_kv_heads, pa_inputs.torch_dtype(problem.dtype)
    # pool: the prefix rows filled, everything else NaN
    prefix_owned = pa_inputs.owned_rows(prefix_table, np.array([problem.prefix_len]), bs,
                                        problem.num_blocks)
    gen = pa_inputs.generator("cuda", problem.seed)
    kc = pa_inputs.poisoned_pool(problem.num_blocks, bs, hk, d, dt, gen, "cuda", prefix_owned)
    vc = pa_inputs.poisoned_pool(problem.num_blocks, bs, hk, d, dt, gen, "cuda", prefix_owned)
    key, value = pa_inputs.token_rows(len(slots), hk, d, problem.dtype, problem.seed + 1, "cuda")
    q = pa_inputs.randn((problem.num_seqs, problem.num_heads, d), dt, gen, "cuda")

    k_ref, v_ref = oracle.copy_blocks(kc.cpu(), vc.cpu(), cows)
    k_ref, v_ref = oracle.reshape_and_cache(key.cpu(), value.cpu(), k_ref, v_ref, slots)
    old_shared = [c[0] for c in cows]
    shared_before = kc[old_shared].clone() if old_shared else None

    if cows:
        pa.pa_copy_blocks(kc, vc, torch.tensor(cows, dtype=torch.int64, device="cuda"))
    pa.pa_reshape_and_cache(key, value, kc, vc, torch.tensor(slots, dtype=torch.int64,
                                                             device="cuda"))
    torch.cuda.synchronize()
    assert same_bits(kc, k_ref) and same_bits(vc, v_ref)
    if old_shared:
        # the shared block itself is only written by the last sharer's tail,
        # at rows past the prefix; its prefix rows never change
        r = problem.prefix_len % bs
        assert same_bits(kc[old_shared][:, :r], shared_before[:, :r])

    out = torch.empty_like(q)
    pa.pa_decode(out, q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                 problem.scale)
    torch.cuda.synchronize()
    seqs = [0, 1, 31, problem.num_seqs - 1, int(np.argmax(lens)), int(np.argmin(lens))]
    ref = oracle.paged_decode(q.cpu(), k_ref, v_ref, tables, lens, problem.scale, seqs=seqs)
    assert_close(out[seqs], ref[seqs])
    device_clean()
