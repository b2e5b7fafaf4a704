"""Paged KV-cache decode on B200: Python binding of libpagedattn.so.

Every function here only marshals arguments (tensor pointers, sizes, the
current CUDA stream) into the C ABI declared in ``include/pagedattn.h``; all
work on the hot path runs in the library's CUDA kernels.  PyTorch supplies
device memory and streams.  There is no CPU fallback: the calls raise when
the library is missing or a tensor is not on a CUDA device.

Functions carry the C names:

* ``pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping)``
* ``pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale)``
* ``pa_decode_append(out, q, key, value, k_cache, v_cache, slot_mapping, ...)``
* ``pa_decode_step(out, q, key, value, k_cache, v_cache, slot_mapping, block_tables, ...)``
* ``pa_decode_split(out, q, ..., max_context_len, partition_size, workspace)``
* ``pa_decode_split_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_size)``
* ``pa_decode_shared_prefix(out, q, ..., group_starts, prefix_lens, ...)``
* ``pa_decode_shared_prefix_step(out, q, key, value, ..., slot_mapping, block_tables, ...)``
* ``pa_copy_blocks(k_cache, v_cache, block_mapping)``
* ``pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping)``
* ``pa_device_error(clear=True)``, ``pa_set_option(name, value)``

and ``BlockAllocator`` wraps the host allocator (``pa_alloc_*`` / ``pa_seq_*``).
"""

from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._native import (DEVERR_BITS, PA_DTYPE_BF16, PA_DTYPE_F32, PA_OPT_DECODE_SPLIT_CTAS,
                      PA_OPT_PDL, PA_OPT_TEST_UNDERFED_STAGES, PA_OPT_VALIDATE,
                      PA_OPT_WAIT_LIMIT_US, PagedAttnError, check, lib)

__all__ = [
    "pa_reshape_and_cache", "pa_decode", "pa_decode_append", "pa_decode_step", "pa_decode_split",
    "pa_decode_split_workspace_bytes",
    "pa_decode_split_noalloc", "pa_decode_shared_prefix", "pa_decode_shared_prefix_step",
    "pa_update_block_tables",
    "pa_decode_shared_prefix_workspace_bytes", "pa_copy_blocks", "pa_swap_blocks",
    "pa_device_error", "pa_set_option", "pa_get_option", "BlockAllocator",
    "PagedAttnError", "OutOfBlocks", "DEVERR_BITS",
]

_DTYPES = {torch.float32: PA_DTYPE_F32, torch.bfloat16: PA_DTYPE_BF16}
_OPTIONS = {"validate": PA_OPT_VALIDATE, "decode_split_ctas": PA_OPT_DECODE_SPLIT_CTAS,
            "pdl": PA_OPT_PDL, "wait_limit_us": PA_OPT_WAIT_LIMIT_US,
            "test_underfed_stages": PA_OPT_TEST_UNDERFED_STAGES}


class OutOfBlocks(PagedAttnError):
    pass


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise ValueError(f"dtype {t.dtype} not supported (float32, bfloat16)") from None


def _dev(*tensors):
    for t in tensors:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _need(cond: bool, what: str):
    if not cond:
        raise ValueError(what)


def _cache_pair(k_cache, v_cache):
    """[NB, bs, Hk, D] each, same shape and dtype.  Returns (NB, bs, Hk, D)."""
    _need(k_cache.dim() == 4, "caches must be [num_blocks, block_size, kv_heads, head_dim]")
    _need(v_cache.shape == k_cache.shape and v_cache.dtype == k_cache.dtype,
          "k_cache and v_cache must have the same shape and dtype")
    return tuple(k_cache.shape)


def _decode_args(out, q, k_cache, v_cache, block_tables, context_lens):
    """Shapes and dtypes of a decode call.  Returns (S, Hq, D, NB, bs, Hk)."""
    _dev(out, q, k_cache, v_cache, block_tables, context_lens)
    nb, bs, hk, d = _cache_pair(k_cache, v_cache)
    _need(q.dim() == 3 and q.shape[2] == d, "q must be [num_seqs, num_heads, head_dim]")
    _need(out.shape == q.shape, "out must have q's shape")
    _need(q.dtype == k_cache.dtype and out.dtype == q.dtype, "q, out and caches share one dtype")
    s, hq, _ = q.shape
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.shape[0] == s, "block_tables must be int32 [num_seqs, max_blocks]")
    _need(context_lens.dtype == torch.int32 and tuple(context_lens.shape) == (s,),
          "context_lens must be int32 [num_seqs]")
    return s, hq, d, nb, bs, hk


def _new_rows(key, value, num_tokens, hk, d, cache_dtype, slot_mapping):
    _need(key.shape == value.shape and tuple(key.shape) == (num_tokens, hk, d),
          "key and value must be [num_tokens, kv_heads, head_dim]")
    _need(key.dtype == cache_dtype and value.dtype == cache_dtype,
          "key and value must have the caches' dtype")
    _need(slot_mapping.dtype == torch.int64 and tuple(slot_mapping.shape) == (num_tokens,),
          "slot_mapping must be int64 [num_tokens]")


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """key/value [T, Hk, D]; caches [NB, bs, Hk, D]; slot_mapping int64 [T]."""
    _dev(key, value, k_cache, v_cache, slot_mapping)
    nb, bs, hk, d = _cache_pair(k_cache, v_cache)
    _new_rows(key, value, key.shape[0], hk, d, k_cache.dtype, slot_mapping)
    check(lib().pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(slot_mapping), key.shape[0], hk, d, bs, nb,
                                     _dtype(k_cache), _stream(stream)))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, stream=None):
    """out/q [S, Hq, D]; caches [NB, bs, Hk, D]; block_tables int32 [S, maxB];
    context_lens int32 [S].  Writes ``out`` and returns it."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    check(lib().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                          block_tables.shape[1], _ptr(context_lens), s, hq, hk, d, bs, nb,
                          float(scale), _dtype(q), _stream(stream)))
    return out


def pa_decode_append(out, q, key, value, k_cache, v_cache, slot_mapping, block_tables,
                     context_lens, scale, stream=None):
    """pa_reshape_and_cache of one new row per sequence (key/value [S, Hk, D],
    slot_mapping int64 [S], -1 = none) then pa_decode, in one launch."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    _dev(key, value, slot_mapping)
    _new_rows(key, value, s, hk, d, k_cache.dtype, slot_mapping)
    check(lib().pa_decode_append(_ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(slot_mapping), _ptr(block_tables),
                                 block_tables.shape[1], _ptr(context_lens), s, hq, hk, d, bs, nb,
                                 float(scale), _dtype(q), _stream(stream)))
    return out


def pa_decode_step(out, q, key, value, k_cache, v_cache, slot_mapping, block_tables,
                   context_lens, scale, stream=None):
    """One decode step in one launch: each sequence's last table entry is set
    from its new slot (``block_tables`` is updated in place), the new rows
    are stored, then the batch is decoded -- pa_update_block_tables followed
    by pa_decode_append."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    _dev(key, value, slot_mapping)
    _new_rows(key, value, s, hk, d, k_cache.dtype, slot_mapping)
    check(lib().pa_decode_step(_ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache),
                               _ptr(v_cache), _ptr(slot_mapping), _ptr(block_tables),
                               block_tables.shape[1], _ptr(context_lens), s, hq, hk, d, bs, nb,
                               float(scale), _dtype(q), _stream(stream)))
    return out


def pa_decode_split_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                    partition_size) -> int:
    return int(lib().pa_decode_split_workspace_bytes(num_seqs, num_heads, head_dim,
                                                     max_context_len, partition_size))


def pa_decode_split(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                    max_context_len, partition_size=512, workspace=None, stream=None):
    """Split-K decode; ``workspace`` is a CUDA byte tensor of at least
    ``pa_decode_split_workspace_bytes(...)`` bytes (allocated here if None)."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    need = pa_decode_split_workspace_bytes(s, hq, d, max_context_len, partition_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _dev(workspace)
    nbytes = workspace.numel() * workspace.element_size()
    check(lib().pa_decode_split(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), s,
                                hq, hk, d, bs, nb, float(scale), _dtype(q), int(max_context_len),
                                int(partition_size), _ptr(workspace), nbytes, _stream(stream)))
    return out


def pa_decode_split_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            max_context_len, partition_size=512, stream=None):
    """pa_decode_split for callers that cannot allocate device memory: the
    library's built-in 16 MiB scratch replaces the caller workspace.  Calls
    share that scratch, so calls that overlap on the GPU must not be issued."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    check(lib().pa_decode_split_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_tables), block_tables.shape[1],
                                        _ptr(context_lens), s, hq, hk, d, bs, nb, float(scale),
                                        _dtype(q), int(max_context_len), int(partition_size),
                                        _stream(stream)))
    return out


def pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, head_dim,
                                            max_prefix_len) -> int:
    return int(lib().pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, head_dim,
                                                             max_prefix_len))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            group_starts, prefix_lens, max_group_size, max_prefix_len,
                            workspace=None, stream=None):
    """Decode of a batch whose sequences come in groups sharing a prefix:
    group_starts int32 [G+1] (device), prefix_lens int32 [G] (device, whole
    blocks, multiples of 16).  Same result as pa_decode."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    _dev(group_starts, prefix_lens)
    _need(group_starts.dtype == torch.int32 and prefix_lens.dtype == torch.int32 and
          group_starts.dim() == 1 and prefix_lens.dim() == 1 and
          group_starts.shape[0] == prefix_lens.shape[0] + 1,
          "group_starts must be int32 [groups + 1] and prefix_lens int32 [groups]")
    need = pa_decode_shared_prefix_workspace_bytes(s, hq, d, max_prefix_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _dev(workspace)
    check(lib().pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), s, hq, hk, d, bs, nb, float(scale), _dtype(q),
        _ptr(group_starts), _ptr(prefix_lens), prefix_lens.shape[0], int(max_group_size),
        int(max_prefix_len), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_decode_shared_prefix_step(out, q, key, value, k_cache, v_cache, slot_mapping,
                                 block_tables, context_lens, scale, group_starts, prefix_lens,
                                 max_group_size, max_prefix_len, workspace=None, stream=None):
    """pa_decode_shared_prefix as a whole step: the own-token pass also stores
    each sequence's new row (key/value [S, Hk, D] at slot_mapping int64 [S],
    -1 = none) and sets its last table entry from the slot (``block_tables``
    is updated in place)."""
    s, hq, d, nb, bs, hk = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens)
    _dev(group_starts, prefix_lens, key, value, slot_mapping)
    _need(group_starts.dtype == torch.int32 and prefix_lens.dtype == torch.int32 and
          group_starts.dim() == 1 and prefix_lens.dim() == 1 and
          group_starts.shape[0] == prefix_lens.shape[0] + 1,
          "group_starts must be int32 [groups + 1] and prefix_lens int32 [groups]")
    _new_rows(key, value, s, hk, d, k_cache.dtype, slot_mapping)
    need = pa_decode_shared_prefix_workspace_bytes(s, hq, d, max_prefix_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _dev(workspace)
    check(lib().pa_decode_shared_prefix_step(
        _ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(slot_mapping), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), s, hq,
        hk, d, bs, nb, float(scale), _dtype(q), _ptr(group_starts), _ptr(prefix_lens),
        prefix_lens.shape[0], int(max_group_size), int(max_prefix_len), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def pa_update_block_tables(block_tables, context_lens, slot_mapping, block_size, num_blocks,
                           stream=None):
    """Device tables int32 [S, max_blocks] updated in place after one append
    per sequence: entry (context_lens[s] - 1) // block_size becomes
    slot_mapping[s] // block_size (slot -1: unchanged)."""
    _dev(block_tables, context_lens, slot_mapping)
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2,
          "block_tables must be int32 [num_seqs, max_blocks_per_seq]")
    s = block_tables.shape[0]
    _need(context_lens.dtype == torch.int32 and context_lens.shape == (s,),
          "context_lens must be int32 [num_seqs]")
    _need(slot_mapping.dtype == torch.int64 and slot_mapping.shape == (s,),
          "slot_mapping must be int64 [num_seqs]")
    check(lib().pa_update_block_tables(_ptr(block_tables), block_tables.shape[1],
                                       _ptr(context_lens), _ptr(slot_mapping), s,
                                       int(block_size), int(num_blocks), _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None):
    """block_mapping int64 [P, 2] of (src, dst) on the device."""
    _dev(k_cache, v_cache, block_mapping)
    nb, bs, hk, d = _cache_pair(k_cache, v_cache)
    _need(block_mapping.dtype == torch.int64 and block_mapping.dim() == 2 and
          block_mapping.shape[1] == 2, "block_mapping must be int64 [pairs, 2]")
    check(lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping),
                               block_mapping.shape[0], hk, d, bs, nb, _dtype(k_cache),
                               _stream(stream)))


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping, stream=None):
    """Move blocks between pools (device cache <-> pinned host cache):
    block_mapping int64 [P, 2] of (src, dst), device or pinned host."""
    for t in (dst_k, dst_v, src_k, src_v, block_mapping):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError("pools and mapping must be on a CUDA device or in pinned memory")
    _need(block_mapping.dtype == torch.int64 and block_mapping.dim() == 2 and
          block_mapping.shape[1] == 2, "block_mapping must be int64 [pairs, 2]")
    nb_dst, bs, hk, d = _cache_pair(dst_k, dst_v)
    nb_src = _cache_pair(src_k, src_v)[0]
    _need(tuple(src_k.shape[1:]) == (bs, hk, d) and src_k.dtype == dst_k.dtype,
          "both pools must have the same block shape and dtype")
    check(lib().pa_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v),
                               _ptr(block_mapping), block_mapping.shape[0], hk, d, bs, nb_src,
                               nb_dst, _dtype(dst_k), _stream(stream)))


def pa_device_error(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return the device error word (0 = clean)."""
    flags = ctypes.c_uint32(0)
    status = lib().pa_device_error(_stream(stream), ctypes.byref(flags), int(clear))
    if status not in (0, 6):
        check(status)
    return int(flags.value)


def pa_set_option(name: str, value: int) -> None:
    check(lib().pa_set_option(_OPTIONS[name], int(value)))


def pa_get_option(name: str) -> int:
    return int(lib().pa_get_option(_OPTIONS[name]))


# --------------------------------------------------------------------------
# Host allocator
# --------------------------------------------------------------------------

def _i32(a: np.ndarray):
    if a.dtype != np.int32 or not a.flags["C_CONTIGUOUS"]:
        raise ValueError("host tables must be contiguous int32 arrays")
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class BlockAllocator:
    """Ref-counted block pool (``pa_alloc_*``) plus the sequence helpers
    (``pa_seq_*``) on host int32 tables."""

    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        order = None
        if initial_free_order is not None:
            order = np.ascontiguousarray(initial_free_order, dtype=np.int32)
            if order.shape != (num_blocks,):
                raise ValueError("initial_free_order must hold num_blocks entries")
        self._keep = order
        h = lib().pa_alloc_create(num_blocks, block_size, _i32(order) if order is not None else None)
        if not h:
            raise PagedAttnError(1, lib().pa_last_error().decode())
        self._h = ctypes.c_void_p(h)
        # held here so that destruction works during interpreter shutdown,
        # when module globals may already be gone
        self._destroy = lib().pa_alloc_destroy
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    @staticmethod
    def _check(status):
        if status == 3:
            raise OutOfBlocks(3, lib().pa_last_error().decode())
        check(status)

    def allocate(self) -> int:
        out = ctypes.c_int32(0)
        self._check(lib().pa_alloc_allocate(self._h, ctypes.byref(out)))
        return out.value

    def incref(self, block: int) -> None:
        self._check(lib().pa_alloc_incref(self._h, int(block)))

    def decref(self, block: int) -> None:
        self._check(lib().pa_alloc_decref(self._h, int(block)))

    def num_free(self) -> int:
        return int(lib().pa_alloc_num_free(self._h))

    def ref_count(self, block: int) -> int:
        return int(lib().pa_alloc_ref_count(self._h, int(block)))

    def ref_counts(self) -> list:
        return [self.ref_count(b) for b in range(self.num_blocks)]

    def free_order(self) -> list:
        buf = np.zeros(self.num_blocks, dtype=np.int32)
        n = ctypes.c_int(0)
        self._check(lib().pa_alloc_free_order(self._h, _i32(buf), self.num_blocks, ctypes.byref(n)))
        return buf[: n.value].tolist()

    def append_slot(self, table: np.ndarray, length: int):
        """table: int32 array (mutated).  Returns (slot, cow or None, new_length)."""
        ln = ctypes.c_int(length)
        slot = ctypes.c_int64(0)
        src, dst = ctypes.c_int32(-1), ctypes.c_int32(-1)
        self._check(lib().pa_seq_append_slot(self._h, _i32(table), table.shape[0], ctypes.byref(ln),
                                             ctypes.byref(slot), ctypes.byref(src),
                                             ctypes.byref(dst)))
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None), ln.value

    def append_slots(self, tables: np.ndarray, lengths: np.ndarray, slots_out=None,
                     pairs_out=None):
        """tables int32 [S, stride], lengths int32 [S] (both mutated).
        Returns (slots int64 [S], cow_pairs int32 [n, 2]).  With slots_out
        (int64 [S]) and pairs_out (int32 [S, 2]) given, the results are
        written there and views of them returned (nothing is allocated)."""
        s = tables.shape[0]
        if lengths.dtype != np.intc or not lengths.flags["C_CONTIGUOUS"]:
            raise ValueError("lengths must be a contiguous int32 array")
        slots = np.zeros(s, dtype=np.int64) if slots_out is None else slots_out
        pairs = np.zeros((max(s, 1), 2), dtype=np.int32) if pairs_out is None else pairs_out
        if slots.dtype != np.int64 or slots.shape != (s,) or not slots.flags["C_CONTIGUOUS"]:
            raise ValueError("slots_out must be a contiguous int64 [num_seqs] array")
        if pairs.dtype != np.int32 or pairs.shape[0] < max(s, 1) or not pairs.flags["C_CONTIGUOUS"]:
            raise ValueError("pairs_out must be a contiguous int32 [num_seqs, 2] array")
        n = ctypes.c_int(0)
        self._check(lib().pa_seq_append_slots(
            self._h, _i32(tables), tables.shape[1], lengths.ctypes.data, s,
            slots.ctypes.data, pairs.ctypes.data, ctypes.byref(n)))
        return slots, (pairs[: n.value].copy() if pairs_out is None else pairs[: n.value])

    def extend(self, table: np.ndarray, length: int, num_tokens: int, want_slots: bool = True):
        ln = ctypes.c_int(length)
        slots = np.zeros(max(num_tokens, 1), dtype=np.int64) if want_slots else None
        src, dst = ctypes.c_int32(-1), ctypes.c_int32(-1)
        self._check(lib().pa_seq_extend(
            self._h, _i32(table), table.shape[0], ctypes.byref(ln), num_tokens,
            slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if want_slots else None,
            ctypes.byref(src), ctypes.byref(dst)))
        cow = (src.value, dst.value) if src.value >= 0 else None
        return (slots[:num_tokens] if want_slots else None), cow, ln.value

    def fork(self, parent_table: np.ndarray, num_table_blocks: int, child_table: np.ndarray):
        self._check(lib().pa_seq_fork(self._h, _i32(parent_table), num_table_blocks,
                                      _i32(child_table)))

    def free(self, table: np.ndarray, num_table_blocks: int):
        self._check(lib().pa_seq_free(self._h, _i32(table), num_table_blocks))

    def compact(self, target_num_blocks: int) -> np.ndarray:
        """Pack live blocks below the target; returns int32 [n, 2] (src, dst)
        moves (copy them with pa_copy_blocks, rewrite tables with remap)."""
        moves = np.zeros((max(self.num_blocks, 1), 2), dtype=np.int32)
        n = ctypes.c_int(0)
        self._check(lib().pa_alloc_compact(self._h, int(target_num_blocks), _i32(moves),
                                           self.num_blocks, ctypes.byref(n)))
        self.num_blocks = int(target_num_blocks)
        return moves[: n.value].copy()

    @staticmethod
    def remap(table: np.ndarray, num_table_blocks: int, moves: np.ndarray) -> None:
        """Rewrite a host table in place after a compaction."""
        moves = np.ascontiguousarray(moves, dtype=np.int32)
        check(lib().pa_seq_remap(_i32(table), num_table_blocks, _i32(moves), moves.shape[0]))

    @staticmethod
    def remap_batch(tables: np.ndarray, lengths_in_blocks: np.ndarray, moves: np.ndarray) -> None:
        """Rewrite every host table of a batch in place after a compaction:
        tables int32 [S, stride] (C-contiguous), lengths_in_blocks [S]."""
        if tables.dtype != np.int32 or tables.ndim != 2 or not tables.flags.c_contiguous:
            raise ValueError("tables must be a C-contiguous int32 [num_seqs, stride] array")
        n = np.ascontiguousarray(lengths_in_blocks, dtype=np.intc)
        if n.shape != (tables.shape[0],):
            raise ValueError("lengths_in_blocks must hold one count per table row")
        moves = np.ascontiguousarray(moves, dtype=np.int32)
        check(lib().pa_seq_remap_batch(_i32(tables), tables.shape[1],
                                       n.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                       tables.shape[0], _i32(moves), moves.shape[0]))
