"""Cache writes and block copies (oracle; test infrastructure only).

* ``reshape_and_cache``: a generated token's key and value go into the row
  named by its slot (physical block * block_size + row); a new block is only
  needed once the current one is full ([course] ch.2 §2.4.2; [csdn-QA] §四
  flow: allocate a free page, update the mapping).  Slot -1 means "skip".
  The copy is exact: the cache has the dtype of the incoming rows.
* ``copy_blocks``: copy-on-write of a shared block -- a write to a block whose
  reference count exceeds one first copies the whole block (keys and values)
  into a fresh block ([course] §2.4.3 pitfall note).

* ``swap_blocks``: a page moves between two pools -- the device cache and a
  pinned host cache -- whole blocks of keys and values ([csdn-QA] §三
  item 10: page migration through pinned memory and asynchronous copies).

All return new tensors and leave their inputs untouched.  Duplicate slots,
duplicate destinations or a destination that is also a source are outside
the definition (read as invalid input).
"""

from __future__ import annotations

import torch


def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping) -> tuple:
    """key/value [T, Hk, D]; caches [NB, bs, Hk, D]; slot_mapping [T] int."""
    k_out = k_cache.clone()
    v_out = v_cache.clone()
    bs = k_cache.shape[1]
    for t in range(key.shape[0]):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        block, row = slot // bs, slot % bs
        k_out[block, row] = key[t]
        v_out[block, row] = value[t]
    return k_out, v_out


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping) -> tuple:
    """block_mapping: sequence of (src, dst) physical block ids."""
    k_out = k_cache.clone()
    v_out = v_cache.clone()
    for src, dst in block_mapping:
        k_out[int(dst)] = k_cache[int(src)]
        v_out[int(dst)] = v_cache[int(src)]
    return k_out, v_out


def swap_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor,
                dst_v: torch.Tensor, block_mapping) -> tuple:
    """block_mapping: (src, dst) pairs; block dst of the destination pool
    receives block src of the source pool.  Returns the new destination."""
    k_out = dst_k.clone()
    v_out = dst_v.clone()
    for src, dst in block_mapping:
        k_out[int(dst)] = src_k[int(src)]
        v_out[int(dst)] = src_v[int(src)]
    return k_out, v_out
