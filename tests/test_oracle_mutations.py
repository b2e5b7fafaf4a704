"""Plant plausible mistakes in the oracle (CPU only, via monkeypatch) and
check that at least one pin catches each: a wrong index, a dropped term, a
wrong sign, a transposed operand, a wrong merge weight, a wrong free-pool
order, a missed reference-count update, and compaction that drops counts,
reuses a destination, overwrites a live block or remaps backwards."""

import importlib
import math

import pytest
import torch

import oracle
import pa_inputs
import test_oracle_allocator as alloc_pins
import test_oracle_attention as att_pins
import test_oracle_paging as paging_pins

att_mod = importlib.import_module("oracle.attention")
paging_mod = importlib.import_module("oracle.paging")
alloc_mod = importlib.import_module("oracle.allocator")


def _fails(fn):
    try:
        fn()
    except (AssertionError, IndexError, ValueError, RuntimeError):
        return True
    return False


def test_wrong_gqa_grouping_is_caught(monkeypatch):
    monkeypatch.setattr(att_mod, "_kv_head", lambda h, hq, hk: h % hk)
    assert _fails(lambda: att_pins.test_matches_sdpa_random(8, 2))


def test_dropped_scale_is_caught(monkeypatch):
    orig = att_mod.attention

    def no_scale(q, k, v, scale):
        return orig(q, k, v, 1.0)
    monkeypatch.setattr(att_mod, "attention", no_scale)
    assert _fails(att_pins.test_tiny_matches_brute_force)


def test_wrong_softmax_sign_is_caught(monkeypatch):
    real_exp = torch.exp
    monkeypatch.setattr(att_mod.torch, "exp", lambda x: real_exp(-x))
    try:
        assert _fails(att_pins.test_tiny_matches_brute_force)
    finally:
        monkeypatch.setattr(att_mod.torch, "exp", real_exp)


def test_values_read_from_keys_is_caught(monkeypatch):
    orig = att_mod.attention
    monkeypatch.setattr(att_mod, "attention", lambda q, k, v, s: orig(q, k, k, s))
    assert _fails(att_pins.test_tiny_matches_brute_force)
    monkeypatch.setattr(oracle, "attention", lambda q, k, v, s: orig(q, k, k, s))
    assert _fails(att_pins.test_closed_form_constant_values)


def test_swapped_block_and_row_is_caught(monkeypatch):
    def swapped(table, t, bs):
        return (t % bs) * bs + int(table[t // bs])
    monkeypatch.setattr(paging_mod, "physical_slot", swapped)
    monkeypatch.setattr(oracle, "physical_slot", swapped)
    assert _fails(paging_pins.test_worked_mapping_example)
    assert _fails(lambda: paging_pins.test_gather_inverts_blockwise_scatter(37, 16))


def test_off_by_one_length_is_caught(monkeypatch):
    orig = paging_mod.gather_sequence
    monkeypatch.setattr(att_mod, "gather_sequence",
                        lambda c, t, n, bs: orig(c, t, n + 1 if n % bs else n, bs))
    assert _fails(att_pins.test_poisoned_rows_never_reach_the_result)


def test_merge_without_partition_sums_is_caught(monkeypatch):
    def bad_merge(m, l, o):
        big_m = m.max(dim=1, keepdim=True).values
        w = torch.exp(m - big_m)                      # l_p dropped
        return (w.unsqueeze(-1) * o).sum(dim=1) / w.sum(dim=1, keepdim=True)
    monkeypatch.setattr(att_mod, "lse_merge", bad_merge)
    assert _fails(lambda: att_pins.test_split_equals_single_pass(16))


def test_fifo_free_pool_is_caught(monkeypatch):
    def fifo_decref(self, block):
        self.ref[block] -= 1
        if self.ref[block] == 0:
            self.free.append(block)
    monkeypatch.setattr(alloc_mod.BlockAllocator, "decref", fifo_decref)
    assert _fails(alloc_pins.test_initial_order_and_lifo_reuse)


def test_copy_on_write_without_decref_is_caught(monkeypatch):
    orig_decref = alloc_mod.BlockAllocator.decref
    calls = {"n": 0}

    def skip_first_decref(self, block):
        calls["n"] += 1
        if calls["n"] == 1:
            return
        orig_decref(self, block)
    monkeypatch.setattr(alloc_mod.BlockAllocator, "decref", skip_first_decref)
    assert _fails(alloc_pins.test_copy_on_write_of_a_shared_partial_block)


def _compaction_variant(carry_counts=True, drop_taken=True, only_free=True):
    """oracle.compact with one step of it changed."""
    def compact(alloc, target):
        live_high = [b for b in range(target, alloc.num_blocks) if alloc.ref[b] > 0]
        low = sorted(b for b in alloc.free if b < target) if only_free else list(range(target))
        if len(live_high) > len(low):
            raise oracle.OutOfBlocks()
        moves = list(zip(live_high, low[:len(live_high)]))
        taken = {d for _, d in moves} if drop_taken else set()
        for s, d in moves:
            alloc.ref[d] = alloc.ref[s] if carry_counts else 1
            alloc.ref[s] = 0
        alloc.free = [b for b in alloc.free if b < target and b not in taken]
        alloc.ref = alloc.ref[:target]
        alloc.num_blocks = target
        return moves
    return compact


@pytest.mark.parametrize("mutation", [dict(carry_counts=False), dict(drop_taken=False),
                                      dict(only_free=False)])
def test_compaction_mistakes_are_caught(monkeypatch, mutation):
    monkeypatch.setattr(oracle, "compact", _compaction_variant(**mutation))
    assert any(_fails(lambda s=s: alloc_pins.test_compaction_packs_live_blocks_below_the_target(s))
               for s in range(5))


def test_reversed_remap_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "remap", lambda table, moves: [
        {d: s for s, d in moves}.get(b, b) for b in table])
    assert _fails(lambda: alloc_pins.test_compaction_packs_live_blocks_below_the_target(0))


def test_unmutated_compaction_variant_passes(monkeypatch):
    """The variant builder with nothing changed is the oracle's compaction."""
    monkeypatch.setattr(oracle, "compact", _compaction_variant())
    for s in range(5):
        alloc_pins.test_compaction_packs_live_blocks_below_the_target(s)
