"""GPU parity: cache writes and block copies through the C ABI are bit-exact
against the oracle, and leave every other row (NaN poison included) alone."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import device_clean, same_bits, tables_via_oracle_allocator

pytestmark = pytest.mark.gpu


def _step_slots(problem):
    alloc, tables, lengths = tables_via_oracle_allocator(problem)
    slots, cows = oracle.append_slots(alloc, tables, lengths)
    return slots, cows


@pytest.mark.parametrize("make", [pa_inputs.tiny, lambda: pa_inputs.gqa(num_seqs=256)])
def test_reshape_and_cache_one_token_per_sequence(make):
    problem = make()
    data = pa_inputs.materialize(problem, "cuda")
    slots, cows = _step_slots(problem)
    assert not cows
    new = pa_inputs.step_tokens(problem.num_seqs, problem.num_heads, problem.num_kv_heads,
                                problem.head_dim, problem.dtype, problem.seed, 0, "cuda")
    k_ref, v_ref = oracle.reshape_and_cache(new["key"].cpu(), new["value"].cpu(),
                                            data["k_cache"].cpu(), data["v_cache"].cpu(), slots)
    slot_t = torch.tensor(slots, dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache(new["key"], new["value"], data["k_cache"], data["v_cache"], slot_t)
    torch.cuda.synchronize()
    assert same_bits(data["k_cache"], k_ref)
    assert same_bits(data["v_cache"], v_ref)
    device_clean()


@pytest.mark.parametrize("dtype,hk,d,bs", [("bf16", 8, 64, 8), ("bf16", 8, 256, 32),
                                           ("f32", 4, 128, 16), ("f32", 2, 256, 8)])
def test_reshape_and_cache_skips_negative_slots(dtype, hk, d, bs):
    nb = 40
    gen = pa_inputs.generator("cuda", 5)
    dt = pa_inputs.torch_dtype(dtype)
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cuda", np.zeros((nb, bs), bool))
    vc = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cuda", np.zeros((nb, bs), bool))
    key, value = pa_inputs.token_rows(300, hk, d, dtype, 6, "cuda")
    rng = np.random.default_rng(7)
    slots = rng.choice(nb * bs, size=300, replace=False).astype(np.int64)
    slots[::7] = -1
    k_ref, v_ref = oracle.reshape_and_cache(key.cpu(), value.cpu(), kc.cpu(), vc.cpu(), slots)
    pa.pa_reshape_and_cache(key, value, kc, vc, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    assert same_bits(kc, k_ref) and same_bits(vc, v_ref)
    device_clean()


def test_reshape_and_cache_out_of_pool_slot_is_reported_and_skipped():
    nb, bs, hk, d = 4, 16, 2, 64
    gen = pa_inputs.generator("cuda", 8)
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, torch.bfloat16, gen, "cuda")
    vc = kc.clone()
    before_k, before_v = kc.clone(), vc.clone()
    key, value = pa_inputs.token_rows(2, hk, d, "bf16", 9, "cuda")
    slots = torch.tensor([nb * bs, nb * bs + 5], dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache(key, value, kc, vc, slots)
    flags = pa.pa_device_error(clear=True)
    assert flags == 8
    assert same_bits(kc, before_k) and same_bits(vc, before_v)


@pytest.mark.parametrize("dtype,hk,d,bs", [("bf16", 8, 128, 16), ("bf16", 8, 64, 8),
                                           ("bf16", 8, 256, 32), ("f32", 4, 64, 16)])
def test_copy_blocks_bitwise(dtype, hk, d, bs):
    nb = 64
    gen = pa_inputs.generator("cuda", 11)
    dt = pa_inputs.torch_dtype(dtype)
    owned = np.random.default_rng(12).random((nb, bs)) < 0.7
    kc = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cuda", owned)
    vc = pa_inputs.poisoned_pool(nb, bs, hk, d, dt, gen, "cuda", owned)
    rng = np.random.default_rng(13)
    ids = rng.permutation(nb)
    pairs = np.stack([ids[:20], ids[20:40]], axis=1).astype(np.int64)
    k_ref, v_ref = oracle.copy_blocks(kc.cpu(), vc.cpu(), pairs.tolist())
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert same_bits(kc, k_ref) and same_bits(vc, v_ref)
    device_clean()
