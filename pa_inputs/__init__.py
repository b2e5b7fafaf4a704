"""Seeded synthetic inputs for paged KV-cache decode.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only *creates* inputs: sequence lengths, the order in which a
pool hands out its physical blocks, block tables built from that order, and
random tensor data with NaN poison in every cache row that no sequence owns.
It performs none of the method's arithmetic (no attention, no softmax, no
cache writes, no allocator logic beyond "sequence i takes the next
ceil(L_i / block_size) blocks of the shuffled pool").

Workload recipes (the shapes and distributions the pages describe for a
decode batch over a pooled, block-scattered KV cache):

* ``tiny``     - 3 sequences, lengths {5, 16, 37}, block_size 16, 16 blocks,
                 4 q heads = 4 kv heads, head_dim 64, fp32 N(0, 1).
* ``mha``      - batch 64, 32 q heads = 32 kv heads, head_dim 128,
                 lengths uniform in [128, 2048], pool 8192 blocks, bf16.
* ``gqa``      - batch 256, 32 q / 8 kv heads, head_dim 128, lengths
                 lognormal (median 1024, sigma 0.5, capped at 8192), pool
                 sized to 110 % of the blocks in use, bf16.
* ``long``     - 2 sequences of 262144 and 1048576 tokens, 32 q / 8 kv heads,
                 head_dim 128, the pool holds exactly those tokens, bf16.
* ``prefix``   - 64 sequences forked from one prefix of 2048 - bs/2 tokens
                 (or 2048 for the aligned variant) with tails uniform in
                 [0, 512]; block_size in {8, 16, 32}, head_dim in
                 {64, 128, 256}, 32 q / 8 kv heads, bf16.

Seeds: host-side structure uses ``numpy.random.default_rng(3590 + idx)``;
tensor data uses a ``torch.Generator`` on the target device seeded with the
same number (plus a per-step offset for per-step data).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

SEED_BASE = 3590

_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPES[name]


@dataclasses.dataclass
class PagedProblem:
    """Structure of one decode batch over a paged KV cache (host arrays)."""

    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str                      # "f32" or "bf16"
    context_lens: np.ndarray        # int32 [S]
    free_order: np.ndarray          # int32 [num_blocks], a permutation
    block_tables: np.ndarray        # int32 [S, max_blocks_per_seq], -1 padded
    seed: int
    scale: float

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def blocks_for(length: int, block_size: int) -> int:
    return -(-int(length) // int(block_size))


def shuffled_pool(rng: np.random.Generator, num_blocks: int) -> np.ndarray:
    """A seeded random permutation of 0..num_blocks-1 (the pool's hand-out order)."""
    return rng.permutation(num_blocks).astype(np.int32)


def tables_from_order(lengths: np.ndarray, free_order: np.ndarray,
                      block_size: int, max_blocks: int) -> np.ndarray:
    """Sequence i takes the next ceil(L_i/block_size) entries of ``free_order``."""
    tables = np.full((len(lengths), max_blocks), -1, dtype=np.int32)
    pos = 0
    for i, length in enumerate(lengths):
        n = blocks_for(length, block_size)
        if n > max_blocks:
            raise ValueError("sequence needs more blocks than the table holds")
        if pos + n > len(free_order):
            raise ValueError("pool too small for the requested lengths")
        tables[i, :n] = free_order[pos:pos + n]
        pos += n
    return tables


def _problem(name, lengths, hq, hk, d, bs, nb, dtype, seed, max_blocks, rng):
    order = shuffled_pool(rng, nb)
    tables = tables_from_order(lengths, order, bs, max_blocks)
    return PagedProblem(name=name, num_heads=hq, num_kv_heads=hk, head_dim=d,
                        block_size=bs, num_blocks=nb, dtype=dtype,
                        context_lens=np.asarray(lengths, dtype=np.int32),
                        free_order=order, block_tables=tables, seed=seed,
                        scale=1.0 / math.sqrt(d))


# --------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------

def tiny() -> PagedProblem:
    seed = SEED_BASE + 0
    rng = np.random.default_rng(seed)
    lengths = np.array([5, 16, 37], dtype=np.int32)
    return _problem("tiny", lengths, 4, 4, 64, 16, 16, "f32", seed, 4, rng)


def mha(num_seqs: int = 64, max_len: int = 2048, num_blocks: int = 8192) -> PagedProblem:
    seed = SEED_BASE + 1
    rng = np.random.default_rng(seed)
    lengths = rng.integers(128, max_len + 1, size=num_seqs).astype(np.int32)
    return _problem("mha", lengths, 32, 32, 128, 16, num_blocks, "bf16", seed,
                    blocks_for(max_len, 16) + 8, rng)


def gqa_lengths(rng: np.random.Generator, num_seqs: int, median: float = 1024.0,
                sigma: float = 0.5, cap: int = 8192) -> np.ndarray:
    raw = np.exp(math.log(median) + sigma * rng.standard_normal(num_seqs))
    return np.clip(np.rint(raw), 1, cap).astype(np.int32)


def gqa(num_seqs: int = 256, extra_tokens: int = 0, cap: int = 8192,
        headroom: float = 1.10, block_size: int = 16, head_dim: int = 128) -> PagedProblem:
    """GQA decode batch.  ``extra_tokens`` reserves pool room for that many
    appended tokens per sequence (a decode loop grows every sequence by one
    token per step); the pool holds ``headroom`` times the blocks in use at
    the end of such a loop.  The lengths do not depend on ``block_size`` or
    ``head_dim`` (the block-size study varies those over one length mix)."""
    seed = SEED_BASE + 2
    rng = np.random.default_rng(seed)
    lengths = gqa_lengths(rng, num_seqs, cap=cap)
    final = lengths.astype(np.int64) + extra_tokens
    in_use = int(sum(blocks_for(x, block_size) for x in final))
    nb = int(math.ceil(headroom * in_use))
    max_blocks = blocks_for(cap + extra_tokens, block_size)
    return _problem("gqa", lengths, 32, 8, head_dim, block_size, nb, "bf16", seed, max_blocks,
                    rng)


def long_context(lengths=(262144, 1048576)) -> PagedProblem:
    seed = SEED_BASE + 3
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int32)
    nb = int(sum(blocks_for(x, 16) for x in lengths))
    return _problem("long", lengths, 32, 8, 128, 16, nb, "bf16", seed,
                    blocks_for(int(lengths.max()), 16), rng)


@dataclasses.dataclass
class PrefixProblem:
    """A shared prefix forked into many sequences, each with its own tail."""

    block_size: int
    head_dim: int
    num_heads: int
    num_kv_heads: int
    num_seqs: int
    prefix_len: int
    tail_lens: np.ndarray        # int32 [num_seqs]
    num_blocks: int
    free_order: np.ndarray       # int32 permutation
    max_blocks_per_seq: int
    dtype: str
    seed: int
    scale: float


def prefix(block_size: int = 16, head_dim: int = 128, aligned: bool = False,
           num_seqs: int = 64, shared: int = 2048, max_tail: int = 512,
           extra_tokens: int = 0) -> PrefixProblem:
    """``extra_tokens`` reserves pool and table room for that many appended
    tokens per sequence (a decode loop over the forked batch)."""
    seed = SEED_BASE + 4 + 100 * block_size + head_dim + (7 if aligned else 0)
    rng = np.random.default_rng(seed)
    plen = shared if aligned else shared - block_size // 2
    tails = rng.integers(0, max_tail + 1, size=num_seqs).astype(np.int32)
    per_seq = blocks_for(plen + max_tail + extra_tokens, block_size) + 1
    nb = blocks_for(plen, block_size) + num_seqs * (blocks_for(max_tail + extra_tokens,
                                                                block_size) + 2)
    order = shuffled_pool(rng, nb)
    return PrefixProblem(block_size=block_size, head_dim=head_dim, num_heads=32,
                         num_kv_heads=8, num_seqs=num_seqs, prefix_len=plen,
                         tail_lens=tails, num_blocks=nb, free_order=order,
                         max_blocks_per_seq=per_seq, dtype="bf16", seed=seed,
                         scale=1.0 / math.sqrt(head_dim))


def random_small(seed: int, num_seqs: int, max_len: int, num_heads: int,
                 num_kv_heads: int, head_dim: int, block_size: int, dtype: str,
                 slack_blocks: int = 3, zero_len: bool = False,
                 fixed: Optional[dict] = None) -> PagedProblem:
    """Small random problems for parity sweeps (ragged lengths, optional L=0).
    ``fixed`` pins chosen sequences' lengths ({index: length}) before the
    tables are built."""
    rng = np.random.default_rng(SEED_BASE + 1000 + seed)
    lo = 0 if zero_len else 1
    lengths = rng.integers(lo, max_len + 1, size=num_seqs).astype(np.int32)
    for i, n in (fixed or {}).items():
        lengths[i] = n
    in_use = int(sum(blocks_for(x, block_size) for x in lengths))
    nb = in_use + slack_blocks
    max_blocks = blocks_for(max_len, block_size) + 1
    return _problem(f"rand{seed}", lengths, num_heads, num_kv_heads, head_dim,
                    block_size, nb, dtype, SEED_BASE + 1000 + seed, max_blocks, rng)


# --------------------------------------------------------------------------
# Tensor data
# --------------------------------------------------------------------------

def generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def owned_rows(block_tables: np.ndarray, context_lens: np.ndarray,
               block_size: int, num_blocks: int) -> np.ndarray:
    """Boolean [num_blocks, block_size]: True where a row holds a token of
    some sequence (logical block j of sequence i covers tokens
    [j*bs, (j+1)*bs) and only its first L_i - j*bs rows are filled)."""
    owned = np.zeros((num_blocks, block_size), dtype=bool)
    rows = np.arange(block_size)
    for i, length in enumerate(context_lens):
        n = blocks_for(length, block_size)
        if n == 0:
            continue
        ids = block_tables[i, :n].astype(np.int64)
        filled = np.minimum(block_size, int(length) - np.arange(n) * block_size)
        owned[ids] |= rows[None, :] < filled[:, None]
    return owned


def randn(shape, dtype: torch.dtype, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def poisoned_pool(num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                  dtype: torch.dtype, gen: torch.Generator, device,
                  owned: Optional[np.ndarray] = None, chunk_blocks: int = 4096) -> torch.Tensor:
    """A [num_blocks, block_size, kv_heads, head_dim] cache filled with N(0,1)
    where ``owned`` is True and NaN elsewhere (any read of a row no sequence
    owns then shows up as NaN)."""
    pool = torch.empty((num_blocks, block_size, num_kv_heads, head_dim),
                       dtype=dtype, device=device)
    for b0 in range(0, num_blocks, chunk_blocks):
        b1 = min(num_blocks, b0 + chunk_blocks)
        pool[b0:b1] = randn((b1 - b0, block_size, num_kv_heads, head_dim), dtype, gen, device)
    if owned is not None and not owned.all():
        mask = torch.from_numpy(~owned).to(device)
        pool[mask] = float("nan")
    return pool


def materialize(problem: PagedProblem, device="cpu") -> dict:
    """q, k_cache, v_cache (NaN-poisoned), block_tables, context_lens on ``device``."""
    dt = torch_dtype(problem.dtype)
    gen = generator(device, problem.seed)
    owned = owned_rows(problem.block_tables, problem.context_lens,
                       problem.block_size, problem.num_blocks)
    k_cache = poisoned_pool(problem.num_blocks, problem.block_size, problem.num_kv_heads,
                            problem.head_dim, dt, gen, device, owned)
    v_cache = poisoned_pool(problem.num_blocks, problem.block_size, problem.num_kv_heads,
                            problem.head_dim, dt, gen, device, owned)
    q = randn((problem.num_seqs, problem.num_heads, problem.head_dim), dt, gen, device)
    return {
        "q": q,
        "k_cache": k_cache,
        "v_cache": v_cache,
        "block_tables": torch.from_numpy(problem.block_tables).to(device),
        "context_lens": torch.from_numpy(problem.context_lens).to(device),
    }


def step_tokens(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                dtype: str, seed: int, step: int, device="cpu") -> dict:
    """Per-step decode inputs: a query and one new key/value row per sequence."""
    dt = torch_dtype(dtype)
    gen = generator(device, seed * 7919 + 17 * step + 1)
    key = randn((num_seqs, num_kv_heads, head_dim), dt, gen, device)
    value = randn((num_seqs, num_kv_heads, head_dim), dt, gen, device)
    q = randn((num_seqs, num_heads, head_dim), dt, gen, device)
    return {"key": key, "value": value, "q": q}


def token_rows(num_tokens: int, num_kv_heads: int, head_dim: int, dtype: str,
               seed: int, device="cpu") -> tuple:
    """``num_tokens`` fresh key and value rows [T, kv_heads, head_dim]."""
    dt = torch_dtype(dtype)
    gen = generator(device, seed)
    key = randn((num_tokens, num_kv_heads, head_dim), dt, gen, device)
    value = randn((num_tokens, num_kv_heads, head_dim), dt, gen, device)
    return key, value
