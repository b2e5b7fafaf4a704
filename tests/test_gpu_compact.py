"""GPU check of compaction end to end: a fragmented pool built through the
C++ allocator (tokens written with pa_reshape_and_cache, sequences forked
and freed), then pa_alloc_compact -> pa_copy_blocks of the moves ->
pa_seq_remap of every table.  The compacted pool's first ``target`` blocks
equal the oracle's copy bit for bit, and decoding over just those blocks
gives the same output bits as before."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import BlockAllocator
from gpu_common import device_clean, same_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs,hq,hk,d,dt", [(16, 32, 8, 128, "bf16"), (8, 8, 8, 64, "f32"),
                                           (32, 16, 2, 256, "bf16"), (8, 32, 8, 128, "bf16"),
                                           (64, 32, 8, 128, "bf16")])
def test_compaction_preserves_decode_bits(bs, hq, hk, d, dt):
    rng = np.random.default_rng(bs * 7 + d)
    nb, cap = 900, 64
    order = rng.permutation(nb).astype(np.int32)
    alloc = BlockAllocator(nb, bs, order)
    torch_dt = pa_inputs.torch_dtype(dt)
    gen = pa_inputs.generator("cuda", 77 + bs)
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch_dt, gen, "cuda",
                                 np.zeros((nb, bs), dtype=bool))
    vc = kc.clone()
    tables, lens = [], []
    for _ in range(24):
        n = int(rng.integers(1, cap * bs // 2))
        t = np.full(cap, -1, dtype=np.int32)
        slots, _, ln = alloc.extend(t, 0, n)
        key, value = pa_inputs.token_rows(n, hk, d, dt, int(rng.integers(1 << 30)))
        pa.pa_reshape_and_cache(key.cuda(), value.cuda(), kc, vc,
                                torch.from_numpy(slots).cuda())
        tables.append(t)
        lens.append(ln)
    for i in (1, 6):                                  # forks share their parent's blocks
        t = np.full(cap, -1, dtype=np.int32)
        alloc.fork(tables[i], -(-lens[i] // bs), t)
        tables.append(t)
        lens.append(lens[i])
    for i in sorted((0, 3, 4, 9, 12, 17, 20), reverse=True):   # holes all over the pool
        alloc.free(tables[i], -(-lens[i] // bs))
        del tables[i], lens[i]
    torch.cuda.synchronize()

    s = len(tables)
    q = pa_inputs.randn((s, hq, d), torch_dt, pa_inputs.generator("cuda", 5), "cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    out0 = torch.empty_like(q)
    pa.pa_decode(out0, q, kc, vc, torch.from_numpy(np.stack(tables)).cuda(), ctx, scale)

    live = sum(1 for r in alloc.ref_counts() if r > 0)
    target = live + 3
    before_k, before_v = kc.cpu(), vc.cpu()
    moves = alloc.compact(target)
    assert len(moves) > 0 and alloc.num_blocks == target
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(moves.astype(np.int64)).cuda())
    ref_k, ref_v = oracle.copy_blocks(before_k, before_v, moves.tolist())
    torch.cuda.synchronize()
    assert same_bits(kc[:target], ref_k[:target]) and same_bits(vc[:target], ref_v[:target])

    # every table in one call; the per-table call must agree with it
    batch = np.stack(tables)
    nblk = np.array([-(-ln // bs) for ln in lens], dtype=np.int32)
    BlockAllocator.remap_batch(batch, nblk, moves)
    for r, (t, ln) in enumerate(zip(tables, lens)):
        BlockAllocator.remap(t, -(-ln // bs), moves)
        assert t[: -(-ln // bs)].max() < target
        assert (t[: nblk[r]] == batch[r, : nblk[r]]).all()
    kc[target:] = float("nan")                        # the released tail
    vc[target:] = float("nan")
    out1 = torch.empty_like(q)
    pa.pa_decode(out1, q, kc[:target], vc[:target], torch.from_numpy(np.stack(tables)).cuda(),
                 ctx, scale)
    torch.cuda.synchronize()
    assert same_bits(out0, out1)
    device_clean()
