"""Address translation and page gather (oracle; test infrastructure only).

A sequence's KV cache is logically contiguous and physically scattered over
fixed-size blocks; a per-sequence block table maps logical block i to a
physical block id ([course] ch.2 §2.2, worked example: logical 0 -> 7,
1 -> 3, 2 -> 12).  The attention kernel computes the logical block from the
token position, looks up the physical block, and reads the row inside it
([csdn-QA] §三 items 1-4; [course] §2.5 step 1).  One logical block maps to
exactly one physical block ([course] §2.2 table; [csdn-QA] §三 item 2 says
"one or more", read here as one-to-one).

Cache layout: ``[num_blocks, block_size, num_kv_heads, head_dim]`` -- a
block holds block_size tokens, each token's key (or value) for every head
and every dimension ([course] §2.3), with keys and values in two separate
tensors ([csdn-QA] §三, ``KVCachePage`` holds separate k_data / v_data).
"""

from __future__ import annotations

import torch


def physical_slot(block_table_row, token: int, block_size: int) -> int:
    """Flat slot (physical_block * block_size + row) of logical token ``token``.

    logical block = token // block_size, row = token % block_size, physical
    block = table[logical block]  ([csdn-QA] §三 item 4; [course] §2.2).
    """
    logical_block = token // block_size
    row = token % block_size
    physical = int(block_table_row[logical_block])
    return physical * block_size + row


def gather_sequence(cache: torch.Tensor, block_table_row, length: int,
                    block_size: int) -> torch.Tensor:
    """The sequence's ``length`` tokens in logical order, fp64 [L, Hk, D].

    Token t is read from slot ``physical_slot(table, t, block_size)`` of the
    flattened cache ([course] §2.5: find the physical block via the table,
    load it, repeat for every block)."""
    assert cache.device.type == "cpu"
    nb, bs, hk, d = cache.shape
    assert bs == block_size
    flat = cache.reshape(nb * bs, hk, d)
    slots = [physical_slot(block_table_row, t, block_size) for t in range(int(length))]
    if not slots:
        return torch.zeros((0, hk, d), dtype=torch.float64)
    idx = torch.tensor(slots, dtype=torch.int64)
    return flat.index_select(0, idx).to(torch.float64)


def block_bytes(block_size: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """Bytes of one physical block, key plus value: tokens x heads x head_dim
    x 2 (K and V) x element size ([course] §2.3)."""
    return block_size * num_kv_heads * head_dim * 2 * elem_bytes
