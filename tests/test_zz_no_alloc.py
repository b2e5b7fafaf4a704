"""pa_decode_split_noalloc: the split decode for callers that cannot allocate
device memory (a plugin whose host framework owns all device memory, a
serving process with a fixed budget and no allocation after start-up).  It
must give what pa_decode_split gives with a caller workspace, call after
call, although every call reuses the library's one built-in scratch array.

Each call is checked against the oracle at the attention tolerance and
against pa_decode_split with a caller workspace bit for bit: both run the
same kernels, and the merge adds partitions in a fixed order, so a stale or
misplaced partial left in the shared scratch by an earlier call would show
as a bit difference even where it stays inside the tolerance.  The calls
change shape from one to the next, and two of them split the merge of each
(sequence, head) into several chunks, whose arrival counts and per-chunk
sums live in the scratch across calls.

This file is collected last, so a stop-at-first-failure run has already run
every other test; it also passes on its own in a fresh process."""

import ctypes

import numpy as np
import pytest
import torch

import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import _native
from gpu_common import assert_close, device_clean, oracle_decode, same_bits

pytestmark = pytest.mark.gpu

SCRATCH = 16 * 1024 * 1024


def _noalloc(out, data, problem, max_len, partition):
    """Straight through the C ABI."""
    q, kc = data["q"], data["k_cache"]
    s, hq, d = q.shape
    nb, bs, hk, _ = kc.shape
    vp = ctypes.c_void_p
    status = _native.lib().pa_decode_split_noalloc(
        vp(out.data_ptr()), vp(q.data_ptr()), vp(kc.data_ptr()), vp(data["v_cache"].data_ptr()),
        vp(data["block_tables"].data_ptr()), data["block_tables"].shape[1],
        vp(data["context_lens"].data_ptr()), s, hq, hk, d, bs, nb, problem.scale,
        _native.PA_DTYPE_BF16, max_len, partition, vp(torch.cuda.current_stream().cuda_stream))
    _native.check(status)


def _merge_chunks(num_seqs, num_heads, parts):
    """Chunks per (sequence, head) of the split merge: the library's rule
    (about 600 merge CTAs, at least 16 partitions per chunk), restated so
    the test can say which calls take the chunked path."""
    heads = num_seqs * num_heads
    return max(1, min(-(-600 // heads), -(-parts // 16)))


# (seed, sequences, longest length, partition): the first call merges in one
# chunk per head, the second in four (64 partitions of 256 tokens), the
# third in one again at another shape, the fourth in several again with
# other lengths, so each call inherits the scratch in another layout.
CALLS = [(41, 5, 2500, 256), (43, 2, 16384, 256), (42, 5, 3200, 512), (44, 3, 12000, 256)]


def test_noalloc_matches_oracle_and_caller_workspace_call_after_call():
    chunked = 0
    for seed, num_seqs, max_len, partition in CALLS:
        problem = pa_inputs.random_small(seed, num_seqs=num_seqs, max_len=max_len,
                                         num_heads=32, num_kv_heads=8, head_dim=128,
                                         block_size=16, dtype="bf16",
                                         fixed={0: 1, 1: max_len})
        data = pa_inputs.materialize(problem, "cuda")
        longest = int(problem.context_lens.max())
        need = pa.pa_decode_split_workspace_bytes(num_seqs, 32, 128, longest, partition)
        assert need <= SCRATCH                     # fits the built-in scratch
        chunked += _merge_chunks(num_seqs, 32, -(-longest // partition)) > 1
        expect = torch.empty_like(data["q"])
        pa.pa_decode_split(expect, data["q"], data["k_cache"], data["v_cache"],
                           data["block_tables"], data["context_lens"], problem.scale,
                           longest, partition)
        got = torch.full_like(data["q"], float("nan"))
        _noalloc(got, data, problem, longest, partition)
        torch.cuda.synchronize()
        device_clean()
        assert same_bits(got, expect), (seed, num_seqs, max_len, partition)
        assert_close(got, oracle_decode(data, problem))
    assert chunked >= 2                            # the chunked merge ran through the scratch


def test_noalloc_rejects_batches_beyond_the_scratch():
    # 64 sequences x 32 heads x 128 partitions of 512 tokens needs ~134 MB
    fake = ctypes.c_void_p(256)
    status = _native.lib().pa_decode_split_noalloc(
        fake, fake, fake, fake, fake, 4096, fake, 64, 32, 8, 128, 16, 1 << 20, 0.1,
        _native.PA_DTYPE_BF16, 65536, 512, None)
    assert status == 2
    assert b"scratch" in _native.lib().pa_last_error()
