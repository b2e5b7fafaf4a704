"""Pins for the oracle's address translation and page gather (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
from conftest import read_golden


def test_worked_mapping_example():
    """Logical page -> physical page as printed in the worked example; every
    token of logical page p sits in physical page table[p] at row t % 16."""
    rows = read_golden("worked_mapping.txt")
    bs = int(rows[0][1])
    mapping = {int(a): int(b) for a, b in rows[1:]}
    table = [mapping[p] for p in range(len(mapping))]
    for t in range(bs * len(table)):
        slot = oracle.physical_slot(table, t, bs)
        assert slot // bs == mapping[t // bs]
        assert slot % bs == t % bs


def _scatter_contiguous(contig, perm, bs, num_blocks, fill=float("nan")):
    """Build a pool from contiguous tokens by whole-block copies: logical block
    j goes to physical block perm[j].  No per-token slot arithmetic."""
    length, hk, d = contig.shape
    pool = torch.full((num_blocks, bs, hk, d), fill, dtype=contig.dtype)
    n = -(-length // bs)
    padded = torch.full((n * bs, hk, d), fill, dtype=contig.dtype)
    padded[:length] = contig
    for j in range(n):
        pool[perm[j]] = padded[j * bs:(j + 1) * bs]
    return pool


@pytest.mark.parametrize("length,bs", [(1, 16), (16, 16), (37, 16), (50, 8), (97, 32)])
def test_gather_inverts_blockwise_scatter(length, bs):
    rng = np.random.default_rng(length * 31 + bs)
    hk, d = 3, 8
    contig = torch.from_numpy(rng.standard_normal((length, hk, d))).to(torch.float32)
    num_blocks = -(-length // bs) + 5
    perm = rng.permutation(num_blocks)
    pool = _scatter_contiguous(contig, perm, bs, num_blocks)
    got = oracle.gather_sequence(pool, perm, length, bs)
    assert torch.equal(got, contig.to(torch.float64))
    assert not torch.isnan(got).any()


def test_gather_empty():
    pool = torch.zeros((4, 16, 2, 8))
    assert oracle.gather_sequence(pool, [0], 0, 16).shape == (0, 2, 8)


def test_block_bytes_formula_matches_pool_tensors():
    """Bytes per block = tokens x heads x head_dim x 2 x element size."""
    for bs, hk, d, dt in [(16, 8, 128, "bf16"), (8, 4, 64, "f32"), (32, 8, 256, "bf16")]:
        gen = pa_inputs.generator("cpu", 0)
        k = pa_inputs.poisoned_pool(2, bs, hk, d, pa_inputs.torch_dtype(dt), gen, "cpu")
        v = pa_inputs.poisoned_pool(2, bs, hk, d, pa_inputs.torch_dtype(dt), gen, "cpu")
        per_block = (k[0].numel() * k.element_size()) + (v[0].numel() * v.element_size())
        assert oracle.block_bytes(bs, hk, d, k.element_size()) == per_block
    # the configuration the decode benchmark uses: 16 tokens, 8 kv heads,
    # head_dim 128, bf16 -> 64 KiB of keys and values per block
    assert oracle.block_bytes(16, 8, 128, 2) == 65536
