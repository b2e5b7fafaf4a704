"""GPU parity for pa_decode_append (cache write of one new token per
sequence fused with decode) against the oracle's reshape_and_cache followed
by its decode: cache bits exact, attention within tolerance."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, same_bits, tables_via_oracle_allocator

pytestmark = pytest.mark.gpu


def _step(problem, data, seed, skip=()):
    """One decode step through the oracle allocator: slots for a new token of
    every sequence (-1 for sequences listed in ``skip``), updated tables."""
    alloc, tables, lengths = tables_via_oracle_allocator(problem)
    slots = []
    for i in range(problem.num_seqs):
        if i in skip:
            slots.append(-1)
            continue
        slot, cow, lengths[i] = oracle.append_slot(alloc, tables[i], lengths[i])
        assert cow is None
        slots.append(slot)
    tab = np.full((problem.num_seqs, problem.max_blocks_per_seq), -1, dtype=np.int32)
    for i, t in enumerate(tables):
        tab[i, :len(t)] = t
    new = pa_inputs.step_tokens(problem.num_seqs, problem.num_heads, problem.num_kv_heads,
                                problem.head_dim, problem.dtype, seed, 0, "cuda")
    return tab, np.array(lengths, dtype=np.int32), slots, new


def _check(problem, data, tab, lens, slots, new):
    k0, v0 = data["k_cache"].cpu(), data["v_cache"].cpu()
    out = torch.empty_like(new["q"])
    pa.pa_decode_append(out, new["q"], new["key"], new["value"], data["k_cache"],
                        data["v_cache"], torch.tensor(slots, dtype=torch.int64, device="cuda"),
                        torch.from_numpy(tab).cuda(), torch.from_numpy(lens).cuda(),
                        problem.scale)
    torch.cuda.synchronize()
    k1, v1 = oracle.reshape_and_cache(new["key"].cpu(), new["value"].cpu(), k0, v0, slots)
    assert same_bits(data["k_cache"], k1) and same_bits(data["v_cache"], v1)
    ref = oracle.paged_decode(new["q"].cpu(), k1, v1, tab, lens, problem.scale)
    assert_close(out, ref)
    device_clean()


def test_tiny_fp32_append():
    problem = pa_inputs.tiny()                    # lengths 5, 16, 37 -> 16 opens a block
    data = pa_inputs.materialize(problem, "cuda")
    _check(problem, data, *_step(problem, data, 11))


@pytest.mark.parametrize("d,bs,hq,hk", [(128, 16, 32, 8), (64, 8, 8, 8), (256, 32, 16, 2),
                                        (128, 16, 32, 32), (128, 8, 32, 8), (128, 64, 32, 8),
                                        (64, 128, 8, 2)])
def test_append_block_boundaries_and_skips(d, bs, hq, hk):
    # lengths ending on, just past and inside a block; two sequences skip
    fixed = {0: bs, 1: bs - 1, 2: 1, 3: 3 * bs + 5, 4: 0}
    problem = pa_inputs.random_small(60 + d + bs, num_seqs=9, max_len=300, num_heads=hq,
                                     num_kv_heads=hk, head_dim=d, block_size=bs, dtype="bf16",
                                     zero_len=True, fixed=fixed)
    data = pa_inputs.materialize(problem, "cuda")
    _check(problem, data, *_step(problem, data, 12, skip=(5, 7)))


def test_gqa_workload_step():
    problem = pa_inputs.gqa(extra_tokens=4)
    data = pa_inputs.materialize(problem, "cuda")
    _check(problem, data, *_step(problem, data, 13))


@pytest.mark.parametrize("ctas", [2, 4])
def test_append_in_cluster_mode(ctas):
    problem = pa_inputs.random_small(88, num_seqs=4, max_len=1500, num_heads=32, num_kv_heads=8,
                                     head_dim=128, block_size=16, dtype="bf16")
    data = pa_inputs.materialize(problem, "cuda")
    pa.pa_set_option("decode_split_ctas", ctas)
    try:
        _check(problem, data, *_step(problem, data, 14))
    finally:
        pa.pa_set_option("decode_split_ctas", 0)


def test_validate_mode_rejects_a_slot_that_is_not_the_last_position():
    problem = pa_inputs.random_small(89, num_seqs=3, max_len=100, num_heads=8, num_kv_heads=2,
                                     head_dim=128, block_size=16, dtype="bf16")
    data = pa_inputs.materialize(problem, "cuda")
    tab, lens, slots, new = _step(problem, data, 15)
    slots[1] += 1 if (lens[1] - 1) % 16 != 15 else -1
    out = torch.empty_like(new["q"])
    pa.pa_set_option("validate", 1)
    try:
        with pytest.raises(pa.PagedAttnError) as e:
            pa.pa_decode_append(out, new["q"], new["key"], new["value"], data["k_cache"],
                                data["v_cache"], torch.tensor(slots, dtype=torch.int64,
                                                              device="cuda"),
                                torch.from_numpy(tab).cuda(), torch.from_numpy(lens).cuda(),
                                problem.scale)
        assert e.value.status == 4
    finally:
        pa.pa_set_option("validate", 0)
