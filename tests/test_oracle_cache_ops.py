"""Pins for the oracle's cache write and block copy (CPU only)."""

import numpy as np
import torch

import oracle
import pa_inputs
from conftest import read_golden


def _pool(nb, bs, hk, d, dtype=torch.bfloat16, seed=0):
    gen = pa_inputs.generator("cpu", seed)
    owned = np.zeros((nb, bs), dtype=bool)
    owned[: nb // 2] = True
    return pa_inputs.poisoned_pool(nb, bs, hk, d, dtype, gen, "cpu", owned)


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_reshape_and_cache_matches_library_index_copy():
    """Row ``slot`` of the flattened [NB*bs, Hk, D] cache receives key[t]; the
    library's index_copy on the flattened view is the same definition."""
    nb, bs, hk, d = 12, 16, 2, 8
    kc, vc = _pool(nb, bs, hk, d, seed=1), _pool(nb, bs, hk, d, seed=2)
    key, value = pa_inputs.token_rows(5, hk, d, "bf16", 3)
    slots = torch.tensor([112, 5, -1, 191, 48], dtype=torch.int64)
    k_out, v_out = oracle.reshape_and_cache(key, value, kc, vc, slots)
    keep = slots >= 0
    ref_k = kc.clone().reshape(nb * bs, hk, d).index_copy_(0, slots[keep], key[keep])
    ref_v = vc.clone().reshape(nb * bs, hk, d).index_copy_(0, slots[keep], value[keep])
    assert _same_bits(k_out.reshape(nb * bs, hk, d), ref_k)
    assert _same_bits(v_out.reshape(nb * bs, hk, d), ref_v)
    # inputs untouched
    assert _same_bits(kc, _pool(nb, bs, hk, d, seed=1))


def test_reshape_and_cache_worked_mapping_rows():
    """Appending token 0, 16 and 32 of the worked example's request lands in
    physical pages 7, 3 and 12 at row 0; every other row keeps its bits,
    including NaN poison."""
    rows = read_golden("worked_mapping.txt")
    bs = int(rows[0][1])
    table = [int(b) for _, b in rows[1:]]
    nb, hk, d = 16, 2, 4
    kc, vc = _pool(nb, bs, hk, d, dtype=torch.float32, seed=4), _pool(nb, bs, hk, d,
                                                                      dtype=torch.float32, seed=5)
    key, value = pa_inputs.token_rows(3, hk, d, "f32", 6)
    slots = [oracle.physical_slot(table, t, bs) for t in (0, 16, 32)]
    k_out, v_out = oracle.reshape_and_cache(key, value, kc, vc, slots)
    changed = torch.zeros((nb, bs), dtype=torch.bool)
    for i, page in enumerate(table):
        assert _same_bits(k_out[page, 0], key[i])
        assert _same_bits(v_out[page, 0], value[i])
        changed[page, 0] = True
    assert _same_bits(k_out[~changed], kc[~changed])
    assert _same_bits(v_out[~changed], vc[~changed])


def test_copy_blocks_copies_whole_blocks_bitwise():
    nb, bs, hk, d = 10, 8, 2, 4
    kc, vc = _pool(nb, bs, hk, d, seed=7), _pool(nb, bs, hk, d, seed=8)
    pairs = [(0, 7), (3, 9), (4, 6)]
    k_out, v_out = oracle.copy_blocks(kc, vc, pairs)
    for src, dst in pairs:
        assert _same_bits(k_out[dst], kc[src])
        assert _same_bits(v_out[dst], vc[src])
    untouched = [b for b in range(nb) if b not in (7, 9, 6)]
    assert _same_bits(k_out[untouched], kc[untouched])
    assert _same_bits(v_out[untouched], vc[untouched])


def test_swap_blocks_round_trip_restores_every_bit():
    """Swap a set of device blocks out to a host pool and back into other
    device blocks: the moved blocks carry the same bits, nothing else in
    either pool changes, and the library's index_copy gives the same pool."""
    nb, hb, bs, hk, d = 20, 12, 16, 2, 8
    kc, vc = _pool(nb, bs, hk, d, seed=21), _pool(nb, bs, hk, d, seed=22)
    hk_pool, hv_pool = _pool(hb, bs, hk, d, seed=23), _pool(hb, bs, hk, d, seed=24)
    out = [(3, 0), (7, 5), (11, 2)]
    h_k, h_v = oracle.swap_blocks(kc, vc, hk_pool, hv_pool, out)
    src = torch.tensor([s for s, _ in out])
    dst = torch.tensor([t for _, t in out])
    assert _same_bits(h_k, hk_pool.clone().index_copy_(0, dst, kc[src]))
    assert _same_bits(h_v, hv_pool.clone().index_copy_(0, dst, vc[src]))
    back = [(0, 15), (5, 16), (2, 17)]
    k2, v2 = oracle.swap_blocks(h_k, h_v, kc, vc, back)
    for (s0, _), (_, t1) in zip(out, back):
        assert _same_bits(k2[t1], kc[s0]) and _same_bits(v2[t1], vc[s0])
    keep = [b for b in range(nb) if b not in (15, 16, 17)]
    assert _same_bits(k2[keep], kc[keep]) and _same_bits(v2[keep], vc[keep])
