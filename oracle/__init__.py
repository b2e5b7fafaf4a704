"""CPU oracle for paged KV-cache decode -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct restatement of what the
paged decode path computes, written from the pages' description of
PagedAttention.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product (``paged_kv_cache_359_b200``) never imports it, and it imports
nothing from the product: the two share no code, headers, tables or helpers.

Sources, cited by page title and section throughout:

* [csdn-QA]  "VLLM中PagedAttention如何降低显存碎片？" (How does PagedAttention
  in vLLM reduce GPU-memory fragmentation?), ask.csdn.net answer, sections
  一..四 and the page-table pseudo-structs under 三.
* [tech]     "PagedAttention技术解析：优化Transformer显存管理" (PagedAttention
  technical analysis), sections 2.1, 2.2, 3.1, 3.2, 4.2.
* [course]   "vLLM内存管理与PagedAttention精讲", chapter 2 "PagedAttention核心
  思想", sections 2.2 (worked mapping), 2.3 (block contents and size),
  2.4 (on-demand allocation, sharing, copy-on-write), 2.5 (block-wise
  attention loop).

Arithmetic is fp64 (inputs in fp32 or bf16 are upcast exactly).  Every
function is pinned by ``tests/test_oracle_*.py`` against something other
than itself: the worked mapping example, brute-force pure-Python loops,
closed forms, ``torch.nn.functional.scaled_dot_product_attention`` in fp64,
permutation invariance, and allocator invariants.  No oracle function is
"parity unpinned".
"""

from .paging import physical_slot, gather_sequence, block_bytes
from .attention import (attention, paged_decode, split_partials, lse_merge,
                        paged_decode_split)
from .cache_ops import reshape_and_cache, copy_blocks, swap_blocks
from .allocator import (BlockAllocator, OutOfBlocks, append_slot, append_slots,
                        extend, fork, free_sequence, compact, remap)

__all__ = [
    "physical_slot", "gather_sequence", "block_bytes",
    "attention", "paged_decode", "split_partials", "lse_merge", "paged_decode_split",
    "reshape_and_cache", "copy_blocks", "swap_blocks",
    "BlockAllocator", "OutOfBlocks", "append_slot", "append_slots", "extend", "fork",
    "free_sequence", "compact", "remap",
]
