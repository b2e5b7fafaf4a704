"""GPU parity for pa_decode and pa_decode_split against the fp64 oracle:
every built (dtype, head_dim, block_size, group) combination on small ragged
batches, the workload shapes at full size on sampled sequences, permutation
invariance, cluster splits, and poisoned rows."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import (assert_close, device_clean, oracle_decode, run_decode, same_bits,
                        tables_via_oracle_allocator)

pytestmark = pytest.mark.gpu


def test_tiny_decode_append_decode():
    """3 sequences (5, 16, 37 tokens), fp32: decode, append one token per
    sequence through the allocator and reshape_and_cache, decode again."""
    problem = pa_inputs.tiny()
    data = pa_inputs.materialize(problem, "cuda")
    assert_close(run_decode(data, problem), oracle_decode(data, problem))
    device_clean()

    alloc, tables, lengths = tables_via_oracle_allocator(problem)
    assert all(list(problem.block_tables[i, :len(t)]) == t for i, t in enumerate(tables))
    slots, cows = oracle.append_slots(alloc, tables, lengths)
    new = pa_inputs.step_tokens(3, 4, 4, 64, "f32", problem.seed, 0, "cuda")
    k_ref, v_ref = oracle.reshape_and_cache(new["key"].cpu(), new["value"].cpu(),
                                            data["k_cache"].cpu(), data["v_cache"].cpu(), slots)
    pa.pa_reshape_and_cache(new["key"], new["value"], data["k_cache"], data["v_cache"],
                            torch.tensor(slots, dtype=torch.int64, device="cuda"))
    problem.context_lens = np.array(lengths, dtype=np.int32)
    for i, t in enumerate(tables):
        problem.block_tables[i, :len(t)] = t
    data["block_tables"] = torch.from_numpy(problem.block_tables).cuda()
    data["context_lens"] = torch.from_numpy(problem.context_lens).cuda()
    data["q"] = new["q"]
    got = run_decode(data, problem)
    ref = oracle.paged_decode(new["q"].cpu(), k_ref, v_ref, problem.block_tables,
                              problem.context_lens, problem.scale)
    assert_close(got, ref)
    device_clean()


COMBOS = [(dt, d, bs, g) for dt in ("bf16", "f32") for d in (64, 128, 256)
          for bs in (8, 16, 32, 64, 128) for g in (1, 2, 4, 8)]


@pytest.mark.parametrize("dtype,d,bs,g", COMBOS)
def test_decode_all_instances_small(dtype, d, bs, g):
    hk = 2
    # a single token, an empty sequence, exactly one full block, two ragged
    problem = pa_inputs.random_small(COMBOS.index((dtype, d, bs, g)), num_seqs=5, max_len=150,
                                     num_heads=hk * g, num_kv_heads=hk, head_dim=d,
                                     block_size=bs, dtype=dtype, zero_len=True,
                                     fixed={0: 1, 1: 0, 2: bs})
    data = pa_inputs.materialize(problem, "cuda")
    ref = oracle_decode(data, problem)
    assert_close(run_decode(data, problem), ref)
    assert_close(run_decode(data, problem, split=True, partition=2 * bs), ref)
    device_clean()


@pytest.mark.parametrize("ctas", [1, 2, 4, 8])
def test_cluster_split_agrees(ctas):
    problem = pa_inputs.random_small(77, num_seqs=6, max_len=900, num_heads=16, num_kv_heads=4,
                                     head_dim=128, block_size=16, dtype="bf16", fixed={0: 3})
    data = pa_inputs.materialize(problem, "cuda")
    ref = oracle_decode(data, problem)
    pa.pa_set_option("decode_split_ctas", ctas)
    try:
        assert_close(run_decode(data, problem), ref)
    finally:
        pa.pa_set_option("decode_split_ctas", 0)
    device_clean()


def test_permutation_invariance_bitwise():
    """The same logical tokens under three physical placements give the same
    bits: the kernel's arithmetic depends on logical order only."""
    rng = np.random.default_rng(5)
    length, hk, d, bs, hq = 333, 8, 128, 16, 32
    n = -(-length // bs)
    key = torch.randn((n * bs, hk, d), device="cuda").to(torch.bfloat16)
    val = torch.randn((n * bs, hk, d), device="cuda").to(torch.bfloat16)
    q = torch.randn((1, hq, d), device="cuda").to(torch.bfloat16)
    outs = []
    for trial in range(3):
        nb = n + 50
        perm = rng.permutation(nb)[:n]
        kc = torch.full((nb, bs, hk, d), float("nan"), device="cuda", dtype=torch.bfloat16)
        vc = kc.clone()
        kc[torch.from_numpy(perm).cuda()] = key.view(n, bs, hk, d)
        vc[torch.from_numpy(perm).cuda()] = val.view(n, bs, hk, d)
        table = torch.from_numpy(perm.astype(np.int32)[None]).cuda()
        out = torch.empty_like(q)
        pa.pa_decode(out, q, kc, vc, table, torch.tensor([length], dtype=torch.int32,
                                                         device="cuda"), d ** -0.5)
        outs.append(out)
    torch.cuda.synchronize()
    assert same_bits(outs[0], outs[1]) and same_bits(outs[0], outs[2])
    device_clean()


def test_mha_workload_sampled():
    """Batch 64, 32 q = 32 kv heads, lengths U[128, 2048], 8192-block pool."""
    problem = pa_inputs.mha()
    data = pa_inputs.materialize(problem, "cuda")
    got = run_decode(data, problem)
    seqs = [0, 1, 17, 40, 63, int(np.argmax(problem.context_lens))]
    ref = oracle_decode(data, problem, seqs=seqs)
    assert_close(got[seqs], ref[seqs])
    device_clean()


def test_gqa_workload_sampled():
    """Batch 256, 32 q / 8 kv heads, lognormal lengths, pool 110 % of use."""
    problem = pa_inputs.gqa()
    data = pa_inputs.materialize(problem, "cuda")
    got = run_decode(data, problem)
    lens = problem.context_lens
    seqs = sorted({0, 5, 99, 255, int(np.argmax(lens)), int(np.argmin(lens))})
    ref = oracle_decode(data, problem, seqs=seqs)
    assert_close(got[seqs], ref[seqs])
    got_split = run_decode(data, problem, split=True, partition=512)
    assert_close(got_split[seqs], ref[seqs])
    assert not torch.isnan(got).any()
    device_clean()


def test_split_partition_sizes():
    problem = pa_inputs.random_small(3, num_seqs=7, max_len=3000, num_heads=32, num_kv_heads=8,
                                     head_dim=128, block_size=16, dtype="bf16")
    data = pa_inputs.materialize(problem, "cuda")
    ref = oracle_decode(data, problem)
    for part in (16, 64, 512, 4096):
        assert_close(run_decode(data, problem, split=True, partition=part), ref)
    device_clean()


def test_long_context_split():
    """Sequences of 262144 and 1048576 tokens, 32 q / 8 kv heads, 512-token
    partitions merged by log-sum-exp; every output against the oracle."""
    problem = pa_inputs.long_context()
    data = pa_inputs.materialize(problem, "cuda")
    got = run_decode(data, problem, split=True, partition=512)
    got1 = run_decode(data, problem, split=False)       # single pass (cluster split)
    kc, vc, q = data["k_cache"].cpu(), data["v_cache"].cpu(), data["q"].cpu()
    del data
    for s in range(problem.num_seqs):
        ref = oracle.paged_decode(q[s:s + 1], kc, vc, problem.block_tables[s:s + 1],
                                  problem.context_lens[s:s + 1], problem.scale)
        assert_close(got[s:s + 1], ref)
        assert_close(got1[s:s + 1], ref)
    device_clean()


@pytest.mark.parametrize("hq,hk", [(8, 2), (4, 4)])
def test_large_batch_beyond_the_sorted_range(hq, hk):
    """1100 short sequences: more than the kernel sorts in shared memory,
    so items run in natural order; still every output is checked."""
    problem = pa_inputs.random_small(500 + hq, num_seqs=1100, max_len=40, num_heads=hq,
                                     num_kv_heads=hk, head_dim=64, block_size=16, dtype="bf16",
                                     zero_len=True)
    data = pa_inputs.materialize(problem, "cuda")
    assert_close(run_decode(data, problem), oracle_decode(data, problem))
    device_clean()


def test_longest_first_order_with_length_ties():
    """The longest-first grid on a ragged GQA batch whose lengths repeat
    (duplicated lengths exercise the index tie-break of the rank search)."""
    problem = pa_inputs.random_small(808, num_seqs=96, max_len=700, num_heads=32,
                                     num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                                     fixed={i: 333 for i in range(0, 96, 7)})
    data = pa_inputs.materialize(problem, "cuda")
    assert_close(run_decode(data, problem), oracle_decode(data, problem))
    device_clean()


@pytest.mark.parametrize("num_seqs", [255, 256, 257, 600, 1024])
def test_longest_first_order_around_the_register_and_shared_ranges(num_seqs):
    """The rank search holds up to 256 lengths in registers and stages up to
    1024 in shared memory: batches on both sides of each limit, with repeated
    lengths, decode every sequence exactly once."""
    fixed = {i: 41 for i in range(0, num_seqs, 5)}
    problem = pa_inputs.random_small(900 + num_seqs, num_seqs=num_seqs, max_len=120,
                                     num_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                                     dtype="bf16", zero_len=True, fixed=fixed)
    data = pa_inputs.materialize(problem, "cuda")
    out = torch.full_like(data["q"], float("nan"))
    assert_close(run_decode(data, problem, out=out), oracle_decode(data, problem))
    device_clean()


@pytest.mark.parametrize("hk,g,bs", [(1, 4, 16), (3, 2, 16), (1, 8, 8), (3, 1, 32), (4, 4, 16)])
def test_head_dim_64_with_odd_and_even_kv_heads(hk, g, bs):
    """bf16 head_dim 64 with odd and even kv head counts, through the
    longest-first, split and cluster launches."""
    problem = pa_inputs.random_small(700 + 10 * hk + g, num_seqs=7, max_len=400,
                                     num_heads=hk * g, num_kv_heads=hk, head_dim=64,
                                     block_size=bs, dtype="bf16", zero_len=True,
                                     fixed={0: 1, 1: 0, 2: bs})
    data = pa_inputs.materialize(problem, "cuda")
    ref = oracle_decode(data, problem)
    assert_close(run_decode(data, problem), ref)
    assert_close(run_decode(data, problem, split=True, partition=64), ref)
    pa.pa_set_option("decode_split_ctas", 2)
    try:
        assert_close(run_decode(data, problem), ref)
    finally:
        pa.pa_set_option("decode_split_ctas", 0)
    device_clean()


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 256)])
def test_split_merge_in_chunks_with_a_reused_workspace(dtype, d):
    """Few (sequence, head) pairs with many partitions: the merge splits each
    pair's partitions into chunks over several CTAs (some chunks empty for
    short sequences) and the last to arrive adds them.  Three calls reuse one
    workspace, so stale arrival counts would show; every call matches the
    oracle and the calls agree bit for bit."""
    problem = pa_inputs.random_small(4040 + d, num_seqs=5, max_len=4096, num_heads=8,
                                     num_kv_heads=2, head_dim=d, block_size=16, dtype=dtype,
                                     fixed={0: 64, 1: 65, 2: 1100, 3: 4096, 4: 3000})
    data = pa_inputs.materialize(problem, "cuda")
    ref = oracle_decode(data, problem)
    need = pa.pa_decode_split_workspace_bytes(5, 8, d, 4096, 64)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")   # garbage counts
    outs = []
    for _ in range(3):
        out = torch.empty_like(data["q"])
        pa.pa_decode_split(out, data["q"], data["k_cache"], data["v_cache"],
                           data["block_tables"], data["context_lens"], problem.scale,
                           max_context_len=4096, partition_size=64, workspace=ws)
        torch.cuda.synchronize()
        assert_close(out, ref)
        outs.append(out)
    assert same_bits(outs[0], outs[1]) and same_bits(outs[1], outs[2])
    device_clean()
