"""Decode attention over a paged KV cache (oracle; test infrastructure only).

For each sequence, each query head attends over all of the sequence's
cached tokens: scores are the scaled dot products of the query with every
key, the weights are the softmax of the scores, and the output is the
weighted sum of the values ([course] ch.2 §2.5 steps 3-4: scores of the
query against every key of the block, then the weighted sum of the value
block, repeated over all blocks).  Every head addresses the same pages
([csdn-QA] §三 item 9); with fewer kv heads than query heads, query head h
reads kv head h // (num_heads / num_kv_heads) (contiguous groups -- the
grouping convention of ``torch.nn.functional.scaled_dot_product_attention``
with ``enable_gqa``).

[tech] §3.1 sketches a three-phase kernel whose last phase applies a
softmax *after* accumulating per-block partial outputs.  Read literally
that is not softmax attention; the reading taken is the exact definition
below, which the block-wise GPU kernels reach through an online softmax.

The split ("V2, block-wise computation", [csdn-QA] §四 last paragraph)
cuts a sequence into fixed partitions, computes per partition the running
max m_p, the sum of exponentials l_p and the partition-normalised output
o_p, and merges them with log-sum-exp weights.  That reaches the same
result exactly (up to rounding), which the tests check in fp64.

All arithmetic is fp64.  context_len = 0 gives a zero output row (the pages
are silent on empty sequences).
"""

from __future__ import annotations

import math

import torch

from .paging import gather_sequence


def _kv_head(h: int, num_heads: int, num_kv_heads: int) -> int:
    group = num_heads // num_kv_heads
    return h // group


def attention(q: torch.Tensor, keys: torch.Tensor, values: torch.Tensor,
              scale: float) -> torch.Tensor:
    """Softmax attention of one sequence's query heads over its tokens.

    q [Hq, D], keys/values [L, Hk, D] -> out [Hq, D], all fp64.
    s_t = scale * <q_h, k_t>; w = exp(s - max s) / sum exp(s - max s);
    out_h = sum_t w_t v_t.
    """
    q = q.to(torch.float64)
    keys = keys.to(torch.float64)
    values = values.to(torch.float64)
    num_heads, d = q.shape
    length, num_kv_heads, _ = keys.shape
    if num_heads % num_kv_heads != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    out = torch.zeros((num_heads, d), dtype=torch.float64)
    if length == 0:
        return out
    for h in range(num_heads):
        kv = _kv_head(h, num_heads, num_kv_heads)
        s = scale * (keys[:, kv, :] @ q[h])          # [L]
        e = torch.exp(s - s.max())
        w = e / e.sum()
        out[h] = w @ values[:, kv, :]
    return out


def paged_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 block_tables, context_lens, scale: float,
                 seqs=None) -> torch.Tensor:
    """Decode output [S, Hq, D] (fp64) for every sequence (or the listed ``seqs``).

    Gathers each sequence's keys and values through its block table, then
    applies ``attention``."""
    num_seqs, num_heads, d = q.shape
    bs = k_cache.shape[1]
    out = torch.zeros((num_seqs, num_heads, d), dtype=torch.float64)
    for i in (range(num_seqs) if seqs is None else seqs):
        length = int(context_lens[i])
        keys = gather_sequence(k_cache, block_tables[i], length, bs)
        values = gather_sequence(v_cache, block_tables[i], length, bs)
        out[i] = attention(q[i], keys, values, scale)
    return out


def split_partials(q: torch.Tensor, keys: torch.Tensor, values: torch.Tensor,
                   scale: float, partition: int):
    """Per-partition statistics of one sequence.

    Partition p covers tokens [p*P, min((p+1)*P, L)).  Returns m [Hq, n_p]
    (max score), l [Hq, n_p] (sum of exp(s - m_p)) and o [Hq, n_p, D]
    (sum of exp(s - m_p) v / l_p), all fp64."""
    q = q.to(torch.float64)
    keys = keys.to(torch.float64)
    values = values.to(torch.float64)
    num_heads, d = q.shape
    length, num_kv_heads, _ = keys.shape
    n_p = -(-length // partition)
    m = torch.full((num_heads, n_p), -math.inf, dtype=torch.float64)
    l = torch.zeros((num_heads, n_p), dtype=torch.float64)
    o = torch.zeros((num_heads, n_p, d), dtype=torch.float64)
    for p in range(n_p):
        t0, t1 = p * partition, min((p + 1) * partition, length)
        for h in range(num_heads):
            kv = _kv_head(h, num_heads, num_kv_heads)
            s = scale * (keys[t0:t1, kv, :] @ q[h])
            m[h, p] = s.max()
            e = torch.exp(s - m[h, p])
            l[h, p] = e.sum()
            o[h, p] = (e @ values[t0:t1, kv, :]) / l[h, p]
    return m, l, o


def lse_merge(m: torch.Tensor, l: torch.Tensor, o: torch.Tensor) -> torch.Tensor:
    """Merge partition statistics: M = max_p m_p, w_p = l_p exp(m_p - M),
    out = sum_p w_p o_p / sum_p w_p.  m, l [Hq, n_p]; o [Hq, n_p, D]."""
    num_heads, n_p, d = o.shape
    if n_p == 0:
        return torch.zeros((num_heads, d), dtype=torch.float64)
    big_m = m.max(dim=1, keepdim=True).values                 # [Hq, 1]
    w = l * torch.exp(m - big_m)                               # [Hq, n_p]
    return (w.unsqueeze(-1) * o).sum(dim=1) / w.sum(dim=1, keepdim=True)


def paged_decode_split(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       block_tables, context_lens, scale: float, partition: int,
                       seqs=None) -> torch.Tensor:
    """Decode output via partitions + log-sum-exp merge, fp64 [S, Hq, D]."""
    num_seqs, num_heads, d = q.shape
    bs = k_cache.shape[1]
    out = torch.zeros((num_seqs, num_heads, d), dtype=torch.float64)
    for i in (range(num_seqs) if seqs is None else seqs):
        length = int(context_lens[i])
        keys = gather_sequence(k_cache, block_tables[i], length, bs)
        values = gather_sequence(v_cache, block_tables[i], length, bs)
        m, l, o = split_partials(q[i], keys, values, scale, partition)
        out[i] = lse_merge(m, l, o)
    return out
