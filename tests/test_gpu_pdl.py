"""Programmatic dependent launch keeps the stream's order: a decode loop of
back-to-back copy-on-write copies, cache writes and decodes (no host sync
between them, forked sequences so the copies run) gives the same output
bits with PA_OPT_PDL on and off, and its last step matches the oracle."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import BlockAllocator
from gpu_common import assert_close, device_clean, same_bits

pytestmark = pytest.mark.gpu

BS, HQ, HK, D, STEPS = 16, 32, 8, 128, 12


def _loop(pdl: bool, split: bool):
    pa.pa_set_option("pdl", 1 if pdl else 0)
    try:
        rng = np.random.default_rng(4242)
        nb, cap = 1200, 64
        alloc = BlockAllocator(nb, BS, rng.permutation(nb).astype(np.int32))
        gen = pa_inputs.generator("cuda", 99)
        kc = pa_inputs.poisoned_pool(nb, BS, HK, D, torch.bfloat16, gen, "cuda")
        vc = pa_inputs.poisoned_pool(nb, BS, HK, D, torch.bfloat16, gen, "cuda")
        tables = np.full((12, cap), -1, dtype=np.int32)
        lens = np.zeros(12, dtype=np.int32)
        for i in range(8):
            _, _, lens[i] = alloc.extend(tables[i], 0, int(rng.integers(40, 700)),
                                         want_slots=False)
        for i in range(8, 12):                       # forks share a partial last block
            alloc.fork(tables[i - 8], -(-int(lens[i - 8]) // BS), tables[i])
            lens[i] = lens[i - 8]
        cpu_k, cpu_v = kc.cpu(), vc.cpu()
        steps = []                      # every input uploaded before the loop
        for st in range(STEPS):
            slots, cows = alloc.append_slots(tables, lens)
            new = pa_inputs.step_tokens(12, HQ, HK, D, "bf16", 7, st, "cuda")
            if len(cows):
                cpu_k, cpu_v = oracle.copy_blocks(cpu_k, cpu_v, cows.tolist())
            cpu_k, cpu_v = oracle.reshape_and_cache(new["key"].cpu(), new["value"].cpu(),
                                                    cpu_k, cpu_v, slots)
            steps.append((torch.from_numpy(cows.astype(np.int64)).cuda() if len(cows) else None,
                          torch.from_numpy(slots).cuda(), new,
                          torch.from_numpy(tables.copy()).cuda(),
                          torch.from_numpy(lens.copy()).cuda(), int(lens.max())))
        outs = [torch.empty_like(steps[0][2]["q"]) for _ in range(STEPS)]
        ws = torch.empty(pa.pa_decode_split_workspace_bytes(12, HQ, D, cap * BS, 64),
                         dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        for (cows_d, slots_d, new, tabs_d, lens_d, max_len), out in zip(steps, outs):
            # only the library's kernels, back to back on the stream
            if cows_d is not None:
                pa.pa_copy_blocks(kc, vc, cows_d)
            pa.pa_reshape_and_cache(new["key"], new["value"], kc, vc, slots_d)
            if split:
                pa.pa_decode_split(out, new["q"], kc, vc, tabs_d, lens_d, D ** -0.5,
                                   max_context_len=max_len, partition_size=64, workspace=ws)
            else:
                pa.pa_decode(out, new["q"], kc, vc, tabs_d, lens_d, D ** -0.5)
        torch.cuda.synchronize()
        assert any(st[0] is not None for st in steps)      # copy-on-write did run
        ref = oracle.paged_decode(steps[-1][2]["q"].cpu(), cpu_k, cpu_v, tables, lens, D ** -0.5)
        return outs, ref
    finally:
        pa.pa_set_option("pdl", 1)


@pytest.mark.parametrize("split", [False, True])
def test_pdl_on_and_off_give_the_same_bits(split):
    on, ref = _loop(True, split)
    off, _ = _loop(False, split)
    assert all(same_bits(a, b) for a, b in zip(on, off))
    assert_close(on[-1], ref)
    device_clean()


def test_pdl_option_round_trip():
    assert pa.pa_get_option("pdl") == 1
    pa.pa_set_option("pdl", 0)
    assert pa.pa_get_option("pdl") == 0
    pa.pa_set_option("pdl", 1)


def _lengths_loop(pdl: bool, problem, data, lens_seq):
    """pa_decode after a torch kernel that rewrites context_lens, back to back
    on one stream with no host synchronisation: the decode grid stages the
    lengths before its dependency wait, which is correct only because a
    caller's kernel completes before a programmatic dependent starts."""
    pa.pa_set_option("pdl", 1 if pdl else 0)
    try:
        lens_d = torch.zeros_like(data["context_lens"])
        zero = torch.zeros_like(lens_d)
        outs = [torch.empty_like(data["q"]) for _ in lens_seq]
        torch.cuda.synchronize()
        for src, out in zip(lens_seq, outs):
            torch.add(src, zero, out=lens_d)              # a kernel right before the decode
            pa.pa_decode(out, data["q"], data["k_cache"], data["v_cache"],
                         data["block_tables"], lens_d, problem.scale)
        torch.cuda.synchronize()
        return outs
    finally:
        pa.pa_set_option("pdl", 1)


def test_lengths_written_by_the_previous_kernel_are_seen():
    # 100 sequences (the longest-first search path); lengths alternate
    # between the full lengths and halves of them, so a decode that read
    # the previous step's lengths would differ from its own
    problem = pa_inputs.random_small(61, num_seqs=100, max_len=700, num_heads=HQ,
                                     num_kv_heads=HK, head_dim=D, block_size=BS, dtype="bf16")
    data = pa_inputs.materialize(problem, "cuda")
    full = data["context_lens"]
    half = torch.div(full, 2, rounding_mode="floor")
    lens_seq = [full if st % 2 == 0 else half for st in range(10)]
    on = _lengths_loop(True, problem, data, lens_seq)
    off = _lengths_loop(False, problem, data, lens_seq)
    assert all(same_bits(a, b) for a, b in zip(on, off))
    assert not same_bits(on[0], on[1])
    cpu = {k: data[k].cpu() for k in ("q", "k_cache", "v_cache")}
    for st in (0, 1):
        ref = oracle.paged_decode(cpu["q"], cpu["k_cache"], cpu["v_cache"], problem.block_tables,
                                  lens_seq[st].cpu().numpy(), problem.scale)
        assert_close(on[st], ref)
        assert_close(on[st + 8], ref)
    device_clean()
