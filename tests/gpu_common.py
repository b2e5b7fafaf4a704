"""Helpers for the GPU parity tests (CUDA path through the C ABI vs the oracle)."""

import numpy as np
import torch

import oracle
import pa_inputs
import paged_kv_cache_359_b200 as pa

# Attention tolerance: bf16 (or fp32) inputs, fp32 accumulation, output in
# the input dtype.  Pass iff max|gpu - ref| <= 1e-2 and
# max|gpu - ref| / max|ref| <= 1e-2.
ATOL = 1e-2
RTOL = 1e-2


def max_errors(got: torch.Tensor, ref: torch.Tensor):
    got = got.detach().to("cpu", torch.float64)
    ref = ref.to(torch.float64)
    assert got.shape == ref.shape
    assert not torch.isnan(got).any(), "NaN in the GPU result"
    err = float((got - ref).abs().max()) if got.numel() else 0.0
    scale = float(ref.abs().max()) if ref.numel() else 0.0
    return err, (err / scale if scale > 0 else err)


def assert_close(got, ref, atol=ATOL, rtol=RTOL):
    err, rel = max_errors(got, ref)
    assert err <= atol and rel <= rtol, f"max abs err {err:.3e}, normwise rel {rel:.3e}"
    return err, rel


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    a = a.detach().cpu().contiguous()
    b = b.detach().cpu().contiguous()
    if a.dtype != b.dtype or a.shape != b.shape:
        return False
    view = torch.int16 if a.element_size() == 2 else torch.int32
    return torch.equal(a.view(view), b.view(view))


def device_clean():
    flags = pa.pa_device_error(clear=True)
    assert flags == 0, f"device error word 0x{flags:x}"


def run_decode(data, problem, split=False, partition=512, out=None):
    q = data["q"]
    out = torch.empty_like(q) if out is None else out
    if split:
        pa.pa_decode_split(out, q, data["k_cache"], data["v_cache"], data["block_tables"],
                           data["context_lens"], problem.scale,
                           max_context_len=int(np.max(problem.context_lens, initial=0)),
                           partition_size=partition)
    else:
        pa.pa_decode(out, q, data["k_cache"], data["v_cache"], data["block_tables"],
                     data["context_lens"], problem.scale)
    torch.cuda.synchronize()
    return out


def oracle_decode(data, problem, seqs=None):
    return oracle.paged_decode(data["q"].cpu(), data["k_cache"].cpu(), data["v_cache"].cpu(),
                               problem.block_tables, problem.context_lens, problem.scale,
                               seqs=seqs)


def tables_via_oracle_allocator(problem):
    """Replay the pool's hand-out order through the oracle allocator; the
    resulting tables must equal the generator's."""
    alloc = oracle.BlockAllocator(problem.num_blocks, problem.block_size, problem.free_order)
    tables, lengths = [], []
    for length in problem.context_lens:
        t = []
        _, _, ln = oracle.extend(alloc, t, 0, int(length))
        tables.append(t)
        lengths.append(ln)
    return alloc, tables, lengths
