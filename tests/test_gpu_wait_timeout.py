"""The bounded-wait give-up path of the decode kernels, driven without a lost
load: with the test-only option PA_OPT_TEST_UNDERFED_STAGES every stage's
barrier is armed for 16 bytes more than its TMA loads deliver.  Every load
still lands in the CTA's own shared memory, so nothing is in flight when a
CTA leaves, but no stage ever completes and every wait runs out after the
(short) wait limit.  The call must return, the device error word must hold
PA_DEVERR_WAIT_TIMEOUT and nothing else, and the next normal call on the
same context must be clean and match the oracle."""

import numpy as np
import pytest
import torch

import pa_inputs
import paged_kv_cache_359_b200 as pa
from gpu_common import assert_close, device_clean, oracle_decode, run_decode

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT = 4
LIMIT_US = 2000


class underfed:
    """Short wait limit and underfed stages for the body of a `with`."""

    def __enter__(self):
        device_clean()
        self.limit = pa.pa_get_option("wait_limit_us")
        pa.pa_set_option("wait_limit_us", LIMIT_US)
        pa.pa_set_option("test_underfed_stages", 1)
        return self

    def __exit__(self, *exc):
        pa.pa_set_option("test_underfed_stages", 0)
        pa.pa_set_option("wait_limit_us", self.limit)


def _problem(seed, dtype, head_dim=128, block_size=16, num_seqs=4, max_len=700):
    problem = pa_inputs.random_small(seed, num_seqs=num_seqs, max_len=max_len, num_heads=16,
                                     num_kv_heads=4, head_dim=head_dim, block_size=block_size,
                                     dtype=dtype)
    return problem, pa_inputs.materialize(problem, "cuda")


def _expect_timeout_only():
    flags = pa.pa_device_error(clear=True)
    assert flags == WAIT_TIMEOUT, f"device error word 0x{flags:x}"


def test_options_round_trip_and_reject_out_of_range():
    limit = pa.pa_get_option("wait_limit_us")
    assert limit == 2_000_000
    with pytest.raises(pa.PagedAttnError):
        pa.pa_set_option("wait_limit_us", 5)
    assert pa.pa_get_option("wait_limit_us") == limit
    assert pa.pa_get_option("test_underfed_stages") == 0


@pytest.mark.parametrize("dtype,head_dim,block_size", [("bf16", 128, 16), ("bf16", 64, 8),
                                                       ("f32", 128, 16), ("bf16", 256, 32)])
def test_decode_gives_up_then_recovers(dtype, head_dim, block_size):
    problem, data = _problem(71, dtype, head_dim, block_size)
    out = torch.full_like(data["q"], float("nan"))
    with underfed():
        run_decode(data, problem, out=out)
        _expect_timeout_only()
    got = run_decode(data, problem)
    device_clean()
    assert_close(got, oracle_decode(data, problem))


def test_cluster_decode_gives_up_then_recovers():
    problem, data = _problem(72, "bf16", num_seqs=2, max_len=3000)
    pa.pa_set_option("decode_split_ctas", 4)
    try:
        with underfed():
            run_decode(data, problem)
            _expect_timeout_only()
        got = run_decode(data, problem)
    finally:
        pa.pa_set_option("decode_split_ctas", 0)
    device_clean()
    assert_close(got, oracle_decode(data, problem))


def test_split_decode_gives_up_then_recovers():
    problem, data = _problem(73, "bf16", num_seqs=3, max_len=2500)
    with underfed():
        run_decode(data, problem, split=True, partition=512)
        _expect_timeout_only()
    got = run_decode(data, problem, split=True, partition=512)
    device_clean()
    assert_close(got, oracle_decode(data, problem))


def test_fused_append_decode_gives_up_then_recovers():
    problem, data = _problem(74, "bf16")
    s, hk, d = problem.num_seqs, problem.num_kv_heads, problem.head_dim
    # the newest token of every sequence is written by the launch itself
    lens = problem.context_lens
    slots = np.array([problem.block_tables[i, (n - 1) // 16] * 16 + (n - 1) % 16
                      for i, n in enumerate(lens)], dtype=np.int64)
    rows = pa_inputs.token_rows(s, hk, d, "bf16", 99, "cuda")
    slots_d = torch.from_numpy(slots).cuda()
    out = torch.empty_like(data["q"])
    with underfed():
        pa.pa_decode_append(out, data["q"], rows[0], rows[1], data["k_cache"], data["v_cache"],
                            slots_d, data["block_tables"], data["context_lens"], problem.scale)
        _expect_timeout_only()
    pa.pa_decode_append(out, data["q"], rows[0], rows[1], data["k_cache"], data["v_cache"],
                        slots_d, data["block_tables"], data["context_lens"], problem.scale)
    torch.cuda.synchronize()
    device_clean()
    assert_close(out, oracle_decode(data, problem))


def test_shared_prefix_decode_gives_up_then_recovers():
    # 6 sequences forked from a 512-token prefix, own tails of up to 200 tokens
    rng = np.random.default_rng(75)
    bs, hq, hk, d, prefix = 16, 16, 4, 128, 512
    tails = rng.integers(0, 200, size=6)
    lens = (prefix + tails).astype(np.int32)
    nb = prefix // bs + int(sum(-(-t // bs) for t in tails)) + 4
    order = rng.permutation(nb).astype(np.int32)
    cap = -(-int(lens.max()) // bs) + 1
    tables = np.full((6, cap), -1, dtype=np.int32)
    tables[:, : prefix // bs] = order[: prefix // bs]
    nxt = prefix // bs
    for i, t in enumerate(tails):
        k = -(-int(t) // bs)
        tables[i, prefix // bs: prefix // bs + k] = order[nxt: nxt + k]
        nxt += k
    problem = pa_inputs.PagedProblem(
        name="fork", num_heads=hq, num_kv_heads=hk, head_dim=d, block_size=bs, num_blocks=nb,
        dtype="bf16", context_lens=lens, free_order=order, block_tables=tables, seed=75,
        scale=1.0 / np.sqrt(d))
    data = pa_inputs.materialize(problem, "cuda")
    starts = torch.tensor([0, 6], dtype=torch.int32, device="cuda")
    plen = torch.tensor([prefix], dtype=torch.int32, device="cuda")
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(6, hq, d, prefix),
                     dtype=torch.uint8, device="cuda")

    def call(out):
        pa.pa_decode_shared_prefix(out, data["q"], data["k_cache"], data["v_cache"],
                                   data["block_tables"], data["context_lens"], problem.scale,
                                   starts, plen, 6, prefix, ws)
        torch.cuda.synchronize()

    out = torch.empty_like(data["q"])
    with underfed():
        call(out)
        _expect_timeout_only()
    call(out)
    device_clean()
    assert_close(out, oracle_decode(data, problem))
