"""Host validation mode and the kernels' own bounds checks turn bad indices
into errors (statuses or device error bits) instead of faults."""

import numpy as np
import pytest
import torch

import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import device_clean

pytestmark = pytest.mark.gpu


def _small():
    problem = pa_inputs.random_small(900, num_seqs=3, max_len=60, num_heads=8, num_kv_heads=2,
                                     head_dim=128, block_size=16, dtype="bf16")
    return problem, pa_inputs.materialize(problem, "cuda")


def test_validate_mode_rejects_bad_block_id():
    problem, data = _small()
    data["block_tables"][1, 0] = problem.num_blocks + 3
    out = torch.empty_like(data["q"])
    pa.pa_set_option("validate", 1)
    try:
        with pytest.raises(pa.PagedAttnError) as e:
            pa.pa_decode(out, data["q"], data["k_cache"], data["v_cache"], data["block_tables"],
                         data["context_lens"], problem.scale)
        assert e.value.status == 4
    finally:
        pa.pa_set_option("validate", 0)


def test_kernel_flags_bad_block_id_and_long_context():
    problem, data = _small()
    data["block_tables"][1, 0] = -5
    data["context_lens"][2] = data["block_tables"].shape[1] * 16 + 100
    out = torch.empty_like(data["q"])
    pa.pa_decode(out, data["q"], data["k_cache"], data["v_cache"], data["block_tables"],
                 data["context_lens"], problem.scale)
    flags = pa.pa_device_error(clear=True)
    assert flags & 1 and flags & 2
    device_clean()


def test_validate_mode_rejects_duplicate_copy_destination():
    problem, data = _small()
    pa.pa_set_option("validate", 1)
    try:
        with pytest.raises(pa.PagedAttnError):
            pa.pa_copy_blocks(data["k_cache"], data["v_cache"],
                              torch.tensor([[0, 1], [2, 1]], dtype=torch.int64, device="cuda"))
    finally:
        pa.pa_set_option("validate", 0)


def test_split_workspace_too_small_is_rejected():
    problem, data = _small()
    out = torch.empty_like(data["q"])
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PagedAttnError):
        pa.pa_decode_split(out, data["q"], data["k_cache"], data["v_cache"],
                           data["block_tables"], data["context_lens"], problem.scale,
                           max_context_len=60, partition_size=16, workspace=ws)


def test_binding_rejects_wrong_dtypes_and_shapes_before_the_library():
    problem, data = _small()
    out = torch.empty_like(data["q"])
    args = [out, data["q"], data["k_cache"], data["v_cache"], data["block_tables"],
            data["context_lens"], problem.scale]
    bad = [
        (4, data["block_tables"].long()),                        # int64 tables
        (5, data["context_lens"].long()),                        # int64 lengths
        (3, data["v_cache"][:-1].contiguous()),                  # pools of different sizes
        (0, out.float()),                                        # out in another dtype
        (1, data["q"][:, :4].contiguous()),                      # q and out shapes differ
    ]
    for i, t in bad:
        call = list(args)
        call[i] = t
        with pytest.raises(ValueError):
            pa.pa_decode(*call)
    with pytest.raises(ValueError):
        pa.pa_copy_blocks(data["k_cache"], data["v_cache"],
                          torch.tensor([0, 1], dtype=torch.int64, device="cuda"))
    device_clean()
