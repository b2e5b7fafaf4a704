"""pa_decode_split_noalloc: the split decode for callers that cannot allocate
device memory (a plugin whose host framework owns all device memory, a
serving process with a fixed budget and no allocation after start-up).  It
must give what pa_decode_split gives with a caller workspace, call after
call, although every call reuses the library's one built-in scratch array.

This file is collected last, so a stop-at-first-failure run has already run
every other test; it also passes on its own in a fresh process."""

import ctypes

import numpy as np
import pytest
import torch

import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import _native
from gpu_common import assert_close, device_clean

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("seeds", [(41, 42)])
def test_noalloc_matches_caller_workspace_two_calls_in_a_row(seeds):
    for call, seed in enumerate(seeds):
        problem = pa_inputs.random_small(seed, num_seqs=5, max_len=2500 + 700 * call,
                                         num_heads=32, num_kv_heads=8, head_dim=128,
                                         block_size=16, dtype="bf16", fixed={0: 1})
        data = pa_inputs.materialize(problem, "cuda")
        max_len = int(problem.context_lens.max())
        partition = 256
        need = pa.pa_decode_split_workspace_bytes(5, 32, 128, max_len, partition)
        assert need <= 16 * 1024 * 1024            # fits the built-in scratch
        expect = torch.empty_like(data["q"])
        pa.pa_decode_split(expect, data["q"], data["k_cache"], data["v_cache"],
                           data["block_tables"], data["context_lens"], problem.scale,
                           max_len, partition)
        got = torch.full_like(data["q"], float("nan"))
        _noalloc(got, data, problem, max_len, partition)
        torch.cuda.synchronize()
        assert_close(got, expect.double().cpu())
        device_clean()


def test_noalloc_rejects_batches_beyond_the_scratch():
    # 64 sequences x 32 heads x 128 partitions of 512 tokens needs ~134 MB
    fake = ctypes.c_void_p(256)
    status = _native.lib().pa_decode_split_noalloc(
        fake, fake, fake, fake, fake, 4096, fake, 64, 32, 8, 128, 16, 1 << 20, 0.1,
        _native.PA_DTYPE_BF16, 65536, 512, None)
    assert status == 2
    assert b"scratch" in _native.lib().pa_last_error()
