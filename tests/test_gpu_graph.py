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


def _forked_batch(d=128, prefix=768, members=24, seed=91):
    """`members` sequences forked from one `prefix`-token prompt, own tails of
    up to 300 tokens, 32 q / 8 kv heads, block 16, bf16."""
    rng = np.random.default_rng(seed)
    hq, hk, bs = 32, 8, 16
    tails = rng.integers(1, 300, size=members)
    lens = (prefix + tails).astype(np.int32)
    nb = prefix // bs + int(sum(-(-int(t) // bs) for t in tails)) + 8
    order = rng.permutation(nb).astype(np.int32)
    cap = -(-int(lens.max()) // bs) + 1
    tables = np.full((members, cap), -1, dtype=np.int32)
    tables[:, : prefix // bs] = order[: prefix // bs]
    nxt = prefix // bs
    for i, t in enumerate(tails):
        k = -(-int(t) // bs)
        tables[i, prefix // bs: prefix // bs + k] = order[nxt: nxt + k]
        nxt += k
    problem = pa_inputs.PagedProblem(
        name="fork", num_heads=hq, num_kv_heads=hk, head_dim=d, block_size=bs, num_blocks=nb,
        dtype="bf16", context_lens=lens, free_order=order, block_tables=tables, seed=seed,
        scale=1.0 / np.sqrt(d))
    return problem, pa_inputs.materialize(problem, "cuda")


def _replay_equals_eager(call, out_shape_like):
    """call(out) launches the library's kernels on the current stream."""
    eager = torch.empty_like(out_shape_like)
    call(eager)
    torch.cuda.synchronize()
    out = torch.full_like(out_shape_like, float("nan"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(out)                               # warm-up outside the capture
        torch.cuda.synchronize()
        out.fill_(float("nan"))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            call(out)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    del graph
    return eager, out


@pytest.mark.parametrize("d", [64, 128, 256])
def test_shared_prefix_decode_replays_from_a_graph(d):
    # the shared pass (tcgen05) and the own-token pass, which streams before
    # it waits for the shared pass, captured with programmatic dependent launch
    problem, data = _forked_batch(d=d)
    s, prefix = problem.num_seqs, 768
    starts = torch.tensor([0, s], dtype=torch.int32, device="cuda")
    plen = torch.tensor([prefix], dtype=torch.int32, device="cuda")
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(s, 32, d, prefix),
                     dtype=torch.uint8, device="cuda")

    def call(out):
        pa.pa_decode_shared_prefix(out, data["q"], data["k_cache"], data["v_cache"],
                                   data["block_tables"], data["context_lens"], problem.scale,
                                   starts, plen, s, prefix, ws)

    eager, got = _replay_equals_eager(call, data["q"])
    assert same_bits(got, eager)
    ref = oracle.paged_decode(data["q"].cpu(), data["k_cache"].cpu(), data["v_cache"].cpu(),
                              problem.block_tables, problem.context_lens, problem.scale)
    assert_close(got, ref)
    device_clean()


def test_split_decode_replays_from_a_graph():
    # partitions merged in chunks (arrival counts zeroed by the first kernel)
    problem, data = _forked_batch(prefix=4096, members=3, seed=92)
    longest = int(problem.context_lens.max())
    ws = torch.empty(pa.pa_decode_split_workspace_bytes(3, 32, 128, longest, 128),
                     dtype=torch.uint8, device="cuda")

    def call(out):
        pa.pa_decode_split(out, data["q"], data["k_cache"], data["v_cache"],
                           data["block_tables"], data["context_lens"], problem.scale,
                           longest, 128, ws)

    eager, got = _replay_equals_eager(call, data["q"])
    assert same_bits(got, eager)
    device_clean()
