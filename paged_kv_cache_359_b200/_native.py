"""ctypes loader for libpagedattn.so (argument marshalling only).

The library is built in-tree by ``paged_kv_cache_359_b200.build``.  There is
no fallback: if the shared library is missing, loading raises.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")

PA_OK = 0
STATUS_NAMES = {
    0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_OUT_OF_BLOCKS",
    4: "PA_ERR_BAD_BLOCK_ID", 5: "PA_ERR_CUDA", 6: "PA_ERR_DEVICE_CHECK",
}
PA_DTYPE_F32, PA_DTYPE_BF16 = 0, 1
PA_OPT_VALIDATE, PA_OPT_DECODE_SPLIT_CTAS, PA_OPT_PDL = 0, 1, 2
PA_OPT_WAIT_LIMIT_US, PA_OPT_TEST_UNDERFED_STAGES = 3, 4

DEVERR_BITS = {
    1: "PA_DEVERR_BLOCK_ID", 2: "PA_DEVERR_CONTEXT_LEN", 4: "PA_DEVERR_WAIT_TIMEOUT",
    8: "PA_DEVERR_SLOT", 16: "PA_DEVERR_COPY_ID", 32: "PA_DEVERR_WORKSPACE",
}

_c_int, _c_size, _c_float, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_intp = ctypes.POINTER(ctypes.c_int)
_u32p = ctypes.POINTER(ctypes.c_uint32)

# name -> (restype, argtypes); every symbol include/pagedattn.h declares
SIGNATURES = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_status_string": (ctypes.c_char_p, [_c_int]),
    "pa_version": (_c_int, []),
    "pa_set_option": (_c_int, [_c_int, _c_int]),
    "pa_get_option": (_c_int, [_c_int]),
    "pa_device_error": (_c_int, [_vp, _u32p, _c_int]),
    "pa_reshape_and_cache": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                      _c_int, _c_int, _vp]),
    "pa_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _c_int,
                           _c_int, _c_int, _c_float, _c_int, _vp]),
    "pa_decode_append": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int,
                                  _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "pa_decode_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int,
                                _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "pa_decode_split_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "pa_decode_split": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _vp,
                                 _c_size, _vp]),
    "pa_decode_split_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int,
                                         _c_int, _vp]),
    "pa_decode_shared_prefix_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "pa_decode_shared_prefix": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp,
                                         _vp, _c_int, _c_int, _c_int, _vp, _c_size, _vp]),
    "pa_decode_shared_prefix_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                                              _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                              _c_int, _c_float, _c_int, _vp, _vp, _c_int, _c_int,
                                              _c_int, _vp, _c_size, _vp]),
    "pa_update_block_tables": (_c_int, [_vp, _c_int, _vp, _vp, _c_int, _c_int, _c_int, _vp]),
    "pa_copy_blocks": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _vp]),
    "pa_swap_blocks": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _c_int, _c_int, _vp]),
    "pa_alloc_create": (_vp, [_c_int, _c_int, _i32p]),
    "pa_alloc_destroy": (None, [_vp]),
    "pa_alloc_allocate": (_c_int, [_vp, _i32p]),
    "pa_alloc_incref": (_c_int, [_vp, ctypes.c_int32]),
    "pa_alloc_decref": (_c_int, [_vp, ctypes.c_int32]),
    "pa_alloc_num_free": (_c_int, [_vp]),
    "pa_alloc_num_blocks": (_c_int, [_vp]),
    "pa_alloc_block_size": (_c_int, [_vp]),
    "pa_alloc_ref_count": (_c_int, [_vp, ctypes.c_int32]),
    "pa_alloc_free_order": (_c_int, [_vp, _i32p, _c_int, _intp]),
    "pa_seq_append_slot": (_c_int, [_vp, _i32p, _c_int, _intp, _i64p, _i32p, _i32p]),
    "pa_seq_append_slots": (_c_int, [_vp, _i32p, _c_int, _vp, _c_int, _vp, _vp, _intp]),
    "pa_seq_extend": (_c_int, [_vp, _i32p, _c_int, _intp, _c_int, _i64p, _i32p, _i32p]),
    "pa_seq_fork": (_c_int, [_vp, _i32p, _c_int, _i32p]),
    "pa_seq_free": (_c_int, [_vp, _i32p, _c_int]),
    "pa_alloc_compact": (_c_int, [_vp, _c_int, _i32p, _c_int, _intp]),
    "pa_seq_remap": (_c_int, [_i32p, _c_int, _i32p, _c_int]),
    "pa_seq_remap_batch": (_c_int, [_i32p, _c_int, _intp, _c_int, _i32p, _c_int]),
}


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status
        self.message = message


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m paged_kv_cache_359_b200.build` (there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int) -> None:
    if status != PA_OK:
        msg = lib().pa_last_error()
        raise PagedAttnError(status, msg.decode() if msg else "")
