"""GPU parity for pa_swap_blocks: blocks move between the device cache and a
pinned host cache bit-exactly (against the oracle), and a sequence swapped
out and back in to other blocks decodes to the same bits."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import _native
from gpu_common import device_clean, same_bits

pytestmark = pytest.mark.gpu


def _pools(nb_dev, nb_host, bs=16, hk=8, d=128, dtype=torch.bfloat16, seed=0):
    gen = pa_inputs.generator("cuda", seed)
    kc = pa_inputs.poisoned_pool(nb_dev, bs, hk, d, dtype, gen, "cuda")
    vc = pa_inputs.poisoned_pool(nb_dev, bs, hk, d, dtype, gen, "cuda")
    hk_pool = pa_inputs.poisoned_pool(nb_host, bs, hk, d, dtype, gen, "cuda").cpu().pin_memory()
    hv_pool = pa_inputs.poisoned_pool(nb_host, bs, hk, d, dtype, gen, "cuda").cpu().pin_memory()
    return kc, vc, hk_pool, hv_pool


@pytest.mark.parametrize("bs,d,dt", [(16, 128, torch.bfloat16), (8, 64, torch.float32),
                                     (32, 256, torch.bfloat16), (64, 128, torch.bfloat16),
                                     (128, 64, torch.bfloat16)])
@pytest.mark.parametrize("mapping_on_device", [True, False])
def test_swap_out_and_in_bitwise(bs, d, dt, mapping_on_device):
    rng = np.random.default_rng(bs + d)
    kc, vc, hkp, hvp = _pools(300, 200, bs=bs, d=d, dtype=dt, seed=bs)
    out = np.stack([rng.choice(300, 150, replace=False), rng.choice(200, 150, replace=False)],
                   axis=1).astype(np.int64)
    m = torch.from_numpy(out)
    m = m.cuda() if mapping_on_device else m.pin_memory()
    ref_k, ref_v = oracle.swap_blocks(kc.cpu(), vc.cpu(), hkp.clone(), hvp.clone(), out.tolist())
    pa.pa_swap_blocks(hkp, hvp, kc, vc, m)
    torch.cuda.synchronize()
    assert same_bits(hkp, ref_k) and same_bits(hvp, ref_v)
    back = np.stack([out[:, 1], rng.permutation(300)[:150]], axis=1).astype(np.int64)
    ref2_k, ref2_v = oracle.swap_blocks(hkp.clone(), hvp.clone(), kc.cpu(), vc.cpu(), back.tolist())
    m2 = torch.from_numpy(back)
    pa.pa_swap_blocks(kc, vc, hkp, hvp, m2.cuda() if mapping_on_device else m2.pin_memory())
    torch.cuda.synchronize()
    assert same_bits(kc, ref2_k) and same_bits(vc, ref2_v)
    device_clean()


def test_swapped_sequence_decodes_to_the_same_bits():
    """Decode a GQA batch, swap every block of one sequence out to the host,
    free and reuse nothing else, swap it back into fresh blocks, rewrite its
    table, decode again: identical output bits for every sequence."""
    problem = pa_inputs.random_small(31, num_seqs=6, max_len=900, num_heads=32, num_kv_heads=8,
                                     head_dim=128, block_size=16, dtype="bf16", slack_blocks=80)
    data = pa_inputs.materialize(problem, "cuda")
    out0 = torch.empty_like(data["q"])
    pa.pa_decode(out0, data["q"], data["k_cache"], data["v_cache"], data["block_tables"],
                 data["context_lens"], problem.scale)
    s = 2
    n = -(-int(problem.context_lens[s]) // 16)
    used = set(problem.block_tables[problem.block_tables >= 0].tolist())
    fresh = [b for b in range(problem.num_blocks) if b not in used][:n]
    assert len(fresh) == n
    host_k = torch.empty((n, 16, 8, 128), dtype=torch.bfloat16).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    own = problem.block_tables[s, :n].astype(np.int64)
    pa.pa_swap_blocks(host_k, host_v, data["k_cache"], data["v_cache"],
                      torch.from_numpy(np.stack([own, np.arange(n)], 1)).cuda())
    data["k_cache"][torch.from_numpy(own).cuda()] = float("nan")      # the old blocks are gone
    data["v_cache"][torch.from_numpy(own).cuda()] = float("nan")
    pa.pa_swap_blocks(data["k_cache"], data["v_cache"], host_k, host_v,
                      torch.from_numpy(np.stack([np.arange(n), np.array(fresh)], 1)).cuda())
    tables = problem.block_tables.copy()
    tables[s, :n] = fresh
    out1 = torch.empty_like(out0)
    pa.pa_decode(out1, data["q"], data["k_cache"], data["v_cache"],
                 torch.from_numpy(tables).cuda(), data["context_lens"], problem.scale)
    torch.cuda.synchronize()
    assert same_bits(out0, out1)
    device_clean()


def test_pageable_host_pool_is_rejected():
    kc, vc, _, _ = _pools(8, 4, seed=3)
    pageable_k = torch.empty((4, 16, 8, 128), dtype=torch.bfloat16)
    pageable_v = torch.empty_like(pageable_k)
    m = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    vp = ctypes.c_void_p
    status = _native.lib().pa_swap_blocks(vp(pageable_k.data_ptr()), vp(pageable_v.data_ptr()),
                                          vp(kc.data_ptr()), vp(vc.data_ptr()), vp(m.data_ptr()),
                                          1, 8, 128, 16, 8, 4, _native.PA_DTYPE_BF16, None)
    assert status == 2 and b"pinned" in _native.lib().pa_last_error()


def test_validate_mode_rejects_out_of_pool_ids():
    kc, vc, hkp, hvp = _pools(8, 4, seed=4)
    pa.pa_set_option("validate", 1)
    try:
        with pytest.raises(pa.PagedAttnError):
            pa.pa_swap_blocks(hkp, hvp, kc, vc,
                              torch.tensor([[0, 4]], dtype=torch.int64, device="cuda"))
    finally:
        pa.pa_set_option("validate", 0)
