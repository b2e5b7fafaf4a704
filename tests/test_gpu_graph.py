"""The library's calls inside a CUDA graph, as a serving loop runs them: one
decode step (copy-on-write copy, fused append + decode) captured once and
replayed with new inputs copied into the captured buffers gives the same
bits as the same steps run eagerly, and the last step matches the oracle."""

import numpy as np
import pytest
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa
from paged_kv_cache_359_b200 import BlockAllocator
from gpu_common import assert_close, device_clean, same_bits

pytestmark = pytest.mark.gpu

BS, HQ, HK, D, S, STEPS = 16, 32, 8, 128, 16, 6


def _state():
    rng = np.random.default_rng(777)
    nb, cap = 1500, 64
    alloc = BlockAllocator(nb, BS, rng.permutation(nb).astype(np.int32))
    gen = pa_inputs.generator("cuda", 31)
    kc = pa_inputs.poisoned_pool(nb, BS, HK, D, torch.bfloat16, gen, "cuda")
    vc = pa_inputs.poisoned_pool(nb, BS, HK, D, torch.bfloat16, gen, "cuda")
    tables = np.full((S, cap), -1, dtype=np.int32)
    lens = np.zeros(S, dtype=np.int32)
    for i in range(S):
        _, _, lens[i] = alloc.extend(tables[i], 0, int(rng.integers(30, 900)), want_slots=False)
    return alloc, kc, vc, tables, lens


def _host_steps(alloc, tables, lens):
    """Allocator outputs of every step (the same for both runs)."""
    out = []
    for st in range(STEPS):
        slots, cows = alloc.append_slots(tables, lens)
        out.append((slots.copy(), cows.astype(np.int64), tables.copy(), lens.copy()))
    return out


def test_graph_replay_matches_eager_and_the_oracle():
    alloc, kc, vc, tables, lens = _state()
    kc_e, vc_e = kc.clone(), vc.clone()
    cpu_k, cpu_v = kc.cpu(), vc.cpu()
    steps = _host_steps(alloc, tables, lens)
    toks = [pa_inputs.step_tokens(S, HQ, HK, D, "bf16", 5, st, "cuda") for st in range(STEPS)]

    # eager
    eager = []
    for (slots, cows, tabs, ln), t in zip(steps, toks):
        out = torch.empty_like(t["q"])
        pa.pa_decode_append(out, t["q"], t["key"], t["value"], kc_e, vc_e,
                            torch.from_numpy(slots).cuda(), torch.from_numpy(tabs).cuda(),
                            torch.from_numpy(ln).cuda(), D ** -0.5)
        eager.append(out)
    torch.cuda.synchronize()

    # graph: static buffers, one captured step, new inputs copied in before each replay
    q_s = torch.empty_like(toks[0]["q"])
    k_s = torch.empty_like(toks[0]["key"])
    v_s = torch.empty_like(toks[0]["value"])
    slots_s = torch.empty(S, dtype=torch.int64, device="cuda")
    tabs_s = torch.empty(tables.shape, dtype=torch.int32, device="cuda")
    lens_s = torch.empty(S, dtype=torch.int32, device="cuda")
    out_s = torch.empty_like(q_s)

    def load(i):
        slots, _, tabs, ln = steps[i]
        q_s.copy_(toks[i]["q"])
        k_s.copy_(toks[i]["key"])
        v_s.copy_(toks[i]["value"])
        slots_s.copy_(torch.from_numpy(slots))
        tabs_s.copy_(torch.from_numpy(tabs))
        lens_s.copy_(torch.from_numpy(ln))

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        load(0)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            pa.pa_decode_append(out_s, q_s, k_s, v_s, kc, vc, slots_s, tabs_s, lens_s,
                                D ** -0.5, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    got = []
    for i in range(STEPS):
        load(i)
        graph.replay()
        got.append(out_s.clone())
        slots, _, _, _ = steps[i]
        cpu_k, cpu_v = oracle.reshape_and_cache(toks[i]["key"].cpu(), toks[i]["value"].cpu(),
                                                cpu_k, cpu_v, slots)
    torch.cuda.synchronize()
    assert all(same_bits(a, b) for a, b in zip(got, eager))
    assert same_bits(kc, kc_e) and same_bits(vc, vc_e)
    _, _, tabs, ln = steps[-1]
    ref = oracle.paged_decode(toks[-1]["q"].cpu(), cpu_k, cpu_v, tabs, ln, D ** -0.5)
    assert_close(got[-1], ref)
    del graph
    device_clean()
