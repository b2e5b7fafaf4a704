"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/pagedattn.h declares, and rejects bad arguments on the host before
any CUDA call (no compute call is made here)."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_359_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary_calls():
    names = declared_symbols()
    for required in ["pa_reshape_and_cache", "pa_decode", "pa_decode_split",
                     "pa_decode_split_workspace_bytes", "pa_copy_blocks", "pa_alloc_create",
                     "pa_seq_append_slot", "pa_seq_fork", "pa_seq_free"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _native.lib()
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing
    assert set(declared_symbols()) == set(_native.SIGNATURES)


def test_status_strings_and_options():
    lib = _native.lib()
    assert lib.pa_version() >= 1
    assert lib.pa_status_string(0) == b"ok"
    assert lib.pa_set_option(_native.PA_OPT_DECODE_SPLIT_CTAS, 3) == 1
    assert lib.pa_set_option(_native.PA_OPT_DECODE_SPLIT_CTAS, 0) == 0


def _decode(**over):
    a = dict(out=16, q=16, kc=16, vc=16, tables=16, maxb=4, lens=16, s=2, hq=8, hk=2, d=128,
             bs=16, nb=10, scale=0.1, dt=_native.PA_DTYPE_BF16)
    a.update(over)
    vp = ctypes.c_void_p
    return _native.lib().pa_decode(vp(a["out"]), vp(a["q"]), vp(a["kc"]), vp(a["vc"]),
                                   vp(a["tables"]), a["maxb"], vp(a["lens"]), a["s"], a["hq"],
                                   a["hk"], a["d"], a["bs"], a["nb"], a["scale"], a["dt"], None)


@pytest.mark.parametrize("over,status", [
    (dict(hq=6, hk=4), 1),          # heads not a multiple of kv heads
    (dict(d=96), 2),                # head_dim not built
    (dict(bs=24), 2),               # block size not built
    (dict(hq=48, hk=2), 2),         # group size 24 not built
    (dict(out=0), 1),               # null pointer
    (dict(q=8), 1),                 # misaligned
    (dict(s=-1), 1),
    (dict(s=0), 0),                 # empty batch: nothing to launch
    (dict(dt=7), 2),
])
def test_decode_argument_checks(over, status):
    assert _decode(**over) == status
    if status:
        assert _native.lib().pa_last_error()


def test_split_workspace_size():
    lib = _native.lib()
    def a256(x):
        return (x + 255) // 256 * 256
    # 2 sequences x 32 heads x ceil(1048576 / 512) partitions: m, l, o, then
    # the reduce's 10 chunks per head (ceil(600 / 64)) of D + 4 floats and counts
    rows = 2 * 32 * 2048
    n = lib.pa_decode_split_workspace_bytes(2, 32, 128, 1048576, 512)
    assert n == 2 * a256(rows * 4) + a256(rows * 128 * 4) + a256(64 * 10 * 132 * 4) + a256(64 * 4)
    # a large batch: one chunk per head, no extra
    rows = 256 * 32 * 2
    n = lib.pa_decode_split_workspace_bytes(256, 32, 128, 1024, 512)
    assert n == 2 * a256(rows * 4) + a256(rows * 128 * 4)
    assert lib.pa_decode_split_workspace_bytes(0, 32, 128, 10, 512) == 0


def test_copy_and_cache_argument_checks():
    lib = _native.lib()
    vp = ctypes.c_void_p
    assert lib.pa_copy_blocks(vp(16), vp(16), vp(16), 0, 8, 128, 16, 4, 1, None) == 0
    assert lib.pa_copy_blocks(vp(16), vp(16), vp(16), 1, 8, 100, 16, 4, 1, None) == 2
    assert lib.pa_reshape_and_cache(vp(16), vp(16), vp(16), vp(16), vp(16), 0, 8, 128, 16, 4,
                                    1, None) == 0
    assert lib.pa_reshape_and_cache(vp(0), vp(16), vp(16), vp(16), vp(16), 3, 8, 128, 16, 4,
                                    1, None) == 1
