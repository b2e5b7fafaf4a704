"""Pins for the oracle's decode attention and its split/log-sum-exp merge.

Each pin ties the oracle to something other than itself: pure-Python brute
force with ``math.exp``, ``torch.nn.functional.scaled_dot_product_attention``
in fp64 (a library routine, which also fixes the GQA head grouping), closed
forms, and the invariance of the result under the physical placement of
blocks.  ``tests/test_oracle_mutations.py`` plants plausible mistakes in the
oracle and checks that one of these pins fails.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import pa_inputs
from test_oracle_paging import _scatter_contiguous


def brute_force_decode(q, keys, values, scale):
    """Nested Python loops over lists of floats; q [Hq][D], keys [L][Hk][D]."""
    hq, d = len(q), len(q[0])
    length = len(keys)
    hk = len(keys[0]) if length else 1
    group = hq // hk
    out = [[0.0] * d for _ in range(hq)]
    if length == 0:
        return out
    for h in range(hq):
        kv = h // group
        scores = []
        for t in range(length):
            acc = 0.0
            for j in range(d):
                acc += q[h][j] * keys[t][kv][j]
            scores.append(acc * scale)
        top = max(scores)
        weights = [math.exp(s - top) for s in scores]
        total = sum(weights)
        for j in range(d):
            acc = 0.0
            for t in range(length):
                acc += weights[t] * values[t][kv][j]
            out[h][j] = acc / total
    return out


def max_err_vs_brute_force(problem):
    data = pa_inputs.materialize(problem)
    got = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"],
                              problem.block_tables, problem.context_lens, problem.scale)
    worst = 0.0
    bs = problem.block_size
    for i, length in enumerate(problem.context_lens):
        # gather by explicit (block, row) indexing, token by token
        table = problem.block_tables[i]
        keys = [[[float(x) for x in data["k_cache"][table[t // bs], t % bs, h]]
                 for h in range(problem.num_kv_heads)] for t in range(length)]
        values = [[[float(x) for x in data["v_cache"][table[t // bs], t % bs, h]]
                   for h in range(problem.num_kv_heads)] for t in range(length)]
        q = [[float(x) for x in row] for row in data["q"][i]]
        ref = torch.tensor(brute_force_decode(q, keys, values, problem.scale),
                           dtype=torch.float64)
        worst = max(worst, float((got[i] - ref).abs().max()))
    return worst


def test_tiny_matches_brute_force():
    assert max_err_vs_brute_force(pa_inputs.tiny()) < 1e-12


def test_gqa_tiny_matches_brute_force():
    p = pa_inputs.random_small(7, num_seqs=3, max_len=23, num_heads=8, num_kv_heads=2,
                               head_dim=6, block_size=8, dtype="f32")
    assert max_err_vs_brute_force(p) < 1e-12


def max_err_vs_sdpa(problem, seqs=None):
    """Contiguous-cache attention from the library routine (fp64), which puts
    query head h on kv head h // (Hq/Hk)."""
    data = pa_inputs.materialize(problem)
    got = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"],
                              problem.block_tables, problem.context_lens, problem.scale,
                              seqs=seqs)
    worst = 0.0
    bs = problem.block_size
    flat_k = data["k_cache"].reshape(-1, problem.num_kv_heads, problem.head_dim)
    flat_v = data["v_cache"].reshape(-1, problem.num_kv_heads, problem.head_dim)
    for i in (range(problem.num_seqs) if seqs is None else seqs):
        length = int(problem.context_lens[i])
        n = -(-length // bs)
        # whole blocks in table order, then cut to the sequence length
        rows = torch.cat([torch.arange(b * bs, (b + 1) * bs) for b in problem.block_tables[i, :n]])
        keys = flat_k[rows][:length].to(torch.float64)      # [L, Hk, D]
        values = flat_v[rows][:length].to(torch.float64)
        q = data["q"][i].to(torch.float64)                   # [Hq, D]
        ref = F.scaled_dot_product_attention(
            q[:, None, :], keys.transpose(0, 1), values.transpose(0, 1),
            scale=problem.scale, enable_gqa=True)[:, 0, :]
        worst = max(worst, float((got[i] - ref).abs().max()))
    return worst


@pytest.mark.parametrize("hq,hk", [(4, 4), (8, 2), (32, 8), (6, 1)])
def test_matches_sdpa_random(hq, hk):
    p = pa_inputs.random_small(hq * 10 + hk, num_seqs=4, max_len=70, num_heads=hq,
                               num_kv_heads=hk, head_dim=16, block_size=16, dtype="bf16")
    assert max_err_vs_sdpa(p) < 1e-12


def test_matches_sdpa_gqa_workload_shape():
    """The GQA workload's geometry (32 q / 8 kv heads, head_dim 128, block 16,
    lognormal lengths) on a 4-sequence batch."""
    p = pa_inputs.gqa(num_seqs=4)
    assert max_err_vs_sdpa(p) < 1e-12


def _contig_problem(rng, length, hq, hk, d, bs):
    q = torch.from_numpy(rng.standard_normal((hq, d)))
    k = torch.from_numpy(rng.standard_normal((length, hk, d)))
    v = torch.from_numpy(rng.standard_normal((length, hk, d)))
    return q, k, v


def test_closed_form_single_token():
    """L = 1: the only weight is 1, so out = v_0 exactly."""
    rng = np.random.default_rng(1)
    q, k, v = _contig_problem(rng, 1, 4, 2, 8, 16)
    out = oracle.attention(q, k, v, 0.3)
    for h in range(4):
        assert torch.equal(out[h], v[0, h // 2])


def test_closed_form_zero_query_is_mean():
    """q = 0: all scores equal, out = mean of the values."""
    rng = np.random.default_rng(2)
    q, k, v = _contig_problem(rng, 37, 4, 4, 8, 16)
    out = oracle.attention(torch.zeros_like(q), k, v, 0.5)
    assert torch.allclose(out, v.mean(dim=0), rtol=0, atol=1e-14)


def test_closed_form_constant_values():
    rng = np.random.default_rng(3)
    q, k, _ = _contig_problem(rng, 29, 2, 2, 8, 16)
    v = torch.full((29, 2, 8), 1.75, dtype=torch.float64)
    out = oracle.attention(q, k, v, 0.25)
    assert torch.allclose(out, torch.full_like(out, 1.75), rtol=0, atol=1e-14)


def test_closed_form_two_tokens_sigmoid():
    """Two tokens: out = sigma(s0 - s1) v0 + (1 - sigma(s0 - s1)) v1."""
    rng = np.random.default_rng(4)
    q, k, v = _contig_problem(rng, 2, 3, 3, 5, 16)
    scale = 0.7
    out = oracle.attention(q, k, v, scale)
    for h in range(3):
        s0 = scale * float(q[h] @ k[0, h])
        s1 = scale * float(q[h] @ k[1, h])
        a = 1.0 / (1.0 + math.exp(-(s0 - s1)))
        expect = a * v[0, h] + (1 - a) * v[1, h]
        assert torch.allclose(out[h], expect, rtol=0, atol=1e-14)


def test_empty_sequence_is_zero():
    q = torch.ones((4, 8))
    out = oracle.attention(q, torch.zeros((0, 2, 8)), torch.zeros((0, 2, 8)), 1.0)
    assert torch.equal(out, torch.zeros((4, 8), dtype=torch.float64))


@pytest.mark.parametrize("length,bs", [(37, 16), (64, 16), (5, 8), (100, 32)])
def test_permutation_invariance_bitwise(length, bs):
    """Logically contiguous, physically scattered: the result does not depend
    on where the blocks sit, bit for bit."""
    rng = np.random.default_rng(length + bs)
    hq, hk, d = 8, 2, 16
    q = torch.from_numpy(rng.standard_normal((1, hq, d))).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((length, hk, d))).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((length, hk, d))).to(torch.bfloat16)
    n = -(-length // bs)
    outs = []
    for trial in range(4):
        nb = n + 7
        perm = rng.permutation(nb)
        kc = _scatter_contiguous(k, perm, bs, nb)
        vc = _scatter_contiguous(v, perm, bs, nb)
        table = np.full((1, n + 2), -1, dtype=np.int32)
        table[0, :n] = perm[:n]
        outs.append(oracle.paged_decode(q, kc, vc, table, [length], 0.25))
    contiguous = oracle.attention(q[0], k, v, 0.25)
    for o in outs:
        assert torch.equal(o[0], contiguous)
        assert not torch.isnan(o).any()


def test_poisoned_rows_never_reach_the_result():
    p = pa_inputs.tiny()
    data = pa_inputs.materialize(p)
    assert torch.isnan(data["k_cache"]).any()        # poison present
    out = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"],
                              p.block_tables, p.context_lens, p.scale)
    assert not torch.isnan(out).any()


@pytest.mark.parametrize("partition", [16, 32, 48, 512])
def test_split_equals_single_pass(partition):
    p = pa_inputs.random_small(11, num_seqs=5, max_len=200, num_heads=8, num_kv_heads=2,
                               head_dim=16, block_size=16, dtype="bf16", zero_len=True)
    data = pa_inputs.materialize(p)
    args = (data["q"], data["k_cache"], data["v_cache"], p.block_tables, p.context_lens, p.scale)
    single = oracle.paged_decode(*args)
    split = oracle.paged_decode_split(*args, partition=partition)
    assert float((single - split).abs().max()) < 1e-12


def test_lse_merge_single_partition_is_identity_and_order_free():
    rng = np.random.default_rng(5)
    q, k, v = _contig_problem(rng, 90, 4, 2, 8, 16)
    m, l, o = oracle.split_partials(q, k, v, 0.4, 90)
    assert m.shape[1] == 1
    assert torch.allclose(oracle.lse_merge(m, l, o), oracle.attention(q, k, v, 0.4),
                          rtol=0, atol=1e-14)
    m, l, o = oracle.split_partials(q, k, v, 0.4, 16)
    perm = torch.randperm(m.shape[1], generator=torch.Generator().manual_seed(0))
    a = oracle.lse_merge(m, l, o)
    b = oracle.lse_merge(m[:, perm], l[:, perm], o[:, perm])
    assert torch.allclose(a, b, rtol=0, atol=1e-14)


def test_split_partial_statistics_brute_force():
    """m_p, l_p and o_p of one partition from the definitions, in Python."""
    rng = np.random.default_rng(6)
    q, k, v = _contig_problem(rng, 40, 2, 1, 4, 16)
    scale = 0.6
    m, l, o = oracle.split_partials(q, k, v, scale, 16)
    for p, (t0, t1) in enumerate([(0, 16), (16, 32), (32, 40)]):
        for h in range(2):
            s = [scale * sum(float(q[h, j]) * float(k[t, 0, j]) for j in range(4))
                 for t in range(t0, t1)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            assert abs(float(m[h, p]) - mx) < 1e-13
            assert abs(float(l[h, p]) - sum(e)) < 1e-12
            for j in range(4):
                ref = sum(e[i] * float(v[t0 + i, 0, j]) for i in range(t1 - t0)) / sum(e)
                assert abs(float(o[h, p, j]) - ref) < 1e-13
