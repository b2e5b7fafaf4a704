"""GPU parity for pa_decode_shared_prefix (cascade decode over groups that
share a prefix) against the oracle's plain decode of the same batch."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, same_bits
from test_gpu_prefix import build

pytestmark = pytest.mark.gpu


def _prefix_batch(bs, d, aligned):
    """The prefix/copy-on-write workload (64 forks, tails U[0, 512]) built
    through the oracle allocator, cache filled on the GPU and checked."""
    problem = pa_inputs.prefix(bs, d, aligned=aligned)
    tables, lens, slots, cows, prefix_table = build(problem)
    hk, dt = problem.num_kv_heads, pa_inputs.torch_dtype(problem.dtype)
    owned = pa_inputs.owned_rows(prefix_table, np.array([problem.prefix_len]), bs,
                                 problem.num_blocks)
    gen = pa_inputs.generator("cuda", problem.seed)
    kc = pa_inputs.poisoned_pool(problem.num_blocks, bs, hk, d, dt, gen, "cuda", owned)
    vc = pa_inputs.poisoned_pool(problem.num_blocks, bs, hk, d, dt, gen, "cuda", owned)
    key, value = pa_inputs.token_rows(len(slots), hk, d, problem.dtype, problem.seed + 1, "cuda")
    q = pa_inputs.randn((problem.num_seqs, problem.num_heads, d), dt, gen, "cuda")
    k_ref, v_ref = oracle.copy_blocks(kc.cpu(), vc.cpu(), cows)
    k_ref, v_ref = oracle.reshape_and_cache(key.cpu(), value.cpu(), k_ref, v_ref, slots)
    if cows:
        pa.pa_copy_blocks(kc, vc, torch.tensor(cows, dtype=torch.int64, device="cuda"))
    pa.pa_reshape_and_cache(key, value, kc, vc, torch.tensor(slots, dtype=torch.int64,
                                                             device="cuda"))
    torch.cuda.synchronize()
    assert same_bits(kc, k_ref) and same_bits(vc, v_ref)
    return problem, tables, lens, kc, vc, q, k_ref, v_ref


@pytest.mark.parametrize("aligned", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_shared_prefix_workload(bs, d, aligned):
    problem, tables, lens, kc, vc, q, k_ref, v_ref = _prefix_batch(bs, d, aligned)
    # the shared part is the prefix's whole blocks before any copy-on-write
    shared = (problem.prefix_len // bs) * bs
    shared -= shared % 16
    gs = torch.tensor([0, problem.num_seqs], dtype=torch.int32, device="cuda")
    pl = torch.tensor([shared], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.pa_set_option("validate", 1)
    try:
        pa.pa_decode_shared_prefix(out, q, kc, vc, torch.from_numpy(tables).cuda(),
                                   torch.from_numpy(lens).cuda(), problem.scale, gs, pl,
                                   max_group_size=problem.num_seqs, max_prefix_len=shared)
    finally:
        pa.pa_set_option("validate", 0)
    torch.cuda.synchronize()
    seqs = [0, 1, 31, problem.num_seqs - 1, int(np.argmax(lens)), int(np.argmin(lens))]
    ref = oracle.paged_decode(q.cpu(), k_ref, v_ref, tables, lens, problem.scale, seqs=seqs)
    assert_close(out[seqs], ref[seqs])
    # and the whole batch agrees with plain decode of the same cache
    plain = torch.empty_like(q)
    pa.pa_decode(plain, q, kc, vc, torch.from_numpy(tables).cuda(),
                 torch.from_numpy(lens).cuda(), problem.scale)
    full_ref = oracle.paged_decode(q.cpu(), k_ref, v_ref, tables, lens, problem.scale)
    assert_close(out, full_ref)
    assert_close(plain, full_ref)
    device_clean()


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_mixed_groups_and_singletons(g):
    """Groups of different sizes (1 .. 40 members, some with no shared
    prefix), random tails, one pool; every output against the oracle."""
    rng = np.random.default_rng(700 + g)
    bs, d, hk = 16, 128, 4
    hq = hk * g
    sizes = [40, 1, 7, 3, 1, 12]
    prefixes = [48 * 16, 0, 5 * 16, 16, 0, 33 * 16]
    nb = 4000
    alloc = oracle.BlockAllocator(nb, bs, rng.permutation(nb))
    tables, lens = [], []
    for size, plen in zip(sizes, prefixes):
        parent = []
        _, _, pl = oracle.extend(alloc, parent, 0, plen)
        members = [parent] + [oracle.fork(alloc, parent) for _ in range(size - 1)]
        for t in members:
            _, _, ln = oracle.extend(alloc, t, pl, int(rng.integers(0 if plen else 1, 300)))
            tables.append(t)
            lens.append(ln)
    s = len(tables)
    cap = max(len(t) for t in tables) + 1
    tab = np.full((s, cap), -1, dtype=np.int32)
    for i, t in enumerate(tables):
        tab[i, :len(t)] = t
    lens = np.array(lens, dtype=np.int32)
    owned = pa_inputs.owned_rows(tab, lens, bs, nb)
    gen = pa_inputs.generator("cuda", 9 + g)
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cuda", owned)
    vc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cuda", owned)
    q = pa_inputs.randn((s, hq, d), torch.bfloat16, gen, "cuda")
    starts = np.cumsum([0] + sizes).astype(np.int32)
    out = torch.empty_like(q)
    pa.pa_set_option("validate", 1)
    try:
        pa.pa_decode_shared_prefix(out, q, kc, vc, torch.from_numpy(tab).cuda(),
                                   torch.from_numpy(lens).cuda(), d ** -0.5,
                                   torch.from_numpy(starts).cuda(),
                                   torch.tensor(prefixes, dtype=torch.int32, device="cuda"),
                                   max_group_size=max(sizes), max_prefix_len=max(prefixes))
    finally:
        pa.pa_set_option("validate", 0)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(q.cpu(), kc.cpu(), vc.cpu(), tab, lens, d ** -0.5)
    assert_close(out, ref)
    device_clean()


def test_validate_mode_rejects_a_member_that_does_not_share_the_prefix():
    problem, tables, lens, kc, vc, q, _, _ = _prefix_batch(16, 128, True)
    tables = tables.copy()
    tables[5, 3] = tables[5, 3] + 1 if tables[5, 3] + 1 < problem.num_blocks else 0
    gs = torch.tensor([0, problem.num_seqs], dtype=torch.int32, device="cuda")
    pl = torch.tensor([problem.prefix_len], dtype=torch.int32, device="cuda")
    pa.pa_set_option("validate", 1)
    try:
        with pytest.raises(pa.PagedAttnError) as e:
            pa.pa_decode_shared_prefix(torch.empty_like(q), q, kc, vc,
                                       torch.from_numpy(tables).cuda(),
                                       torch.from_numpy(lens).cuda(), problem.scale, gs, pl,
                                       max_group_size=64, max_prefix_len=problem.prefix_len)
        assert e.value.status == 4
    finally:
        pa.pa_set_option("validate", 0)
