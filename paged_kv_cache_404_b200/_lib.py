"""ctypes loader for libpagedkv.so (the C ABI in include/pagedkv.h).

There is no fallback: if the library has not been built, every call raises.
Build it with ``python -m paged_kv_cache_404_b200.build``.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedkv.so")

PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED, PKV_ECUDA, PKV_ENOMEM, PKV_ENOENT, PKV_ESWAPPED = range(7)
PKV_F32, PKV_BF16, PKV_FP8_E4M3 = 0, 1, 2

# Every exported symbol of include/pagedkv.h with (restype, argtypes).
_p, _i, _f, _z = C.c_void_p, C.c_int, C.c_float, C.c_size_t
SIGNATURES = {
    "pkv_status_string": (C.c_char_p, [_i]),
    "pkv_version": (_i, []),
    "pkv_paged_kv_write": (_i, [_p, _p, _i, _p, _i, _p, _p, _i, _i, _i, _i, _i, _f, _f, _p, _p]),
    "pkv_decode_workspace_bytes": (_z, [_i, _i, _i, _i, _i]),
    "pkv_paged_attention_decode": (_i, [_p, _p, _i, _p, _p, _i, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                        _f, _f, _f, _i, _p, _z, _p, _p]),
    "pkv_paged_attention_decode_noalloc": (_i, [_p, _p, _i, _p, _p, _i, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                                _f, _f, _f, _i, _p, _p]),
    "pkv_decode_workspace_bytes_shared": (_z, [_i, _i, _i, _i, _i]),
    "pkv_paged_attention_decode_shared": (_i, [_p, _p, _i, _p, _p, _i, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                               _f, _f, _f, _i, _p, _p, _i, _p, _i, _p, _z, _p, _p]),
    "pkv_paged_attention_prefill": (_i, [_p, _p, _i, _p, _p, _i, _p, _i, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                         _i, _f, _f, _f, _p, _p]),
    "pkv_copy_blocks": (_i, [_p, _p, _z, _p, _i, _i, _p, _p]),
    "pkv_swap_blocks": (_i, [_p, _p, _i, _p, _p, _i, _z, _p, _i, _p, _p]),
    "pkv_bm_create": (_i, [_i, _i, _p, _i, C.POINTER(_p)]),
    "pkv_bm_destroy": (None, [_p]),
    "pkv_bm_alloc_seq": (_i, [_p, _i, _p]),
    "pkv_bm_fork": (_i, [_p, C.c_int32, _p]),
    "pkv_bm_fork_many": (_i, [_p, _p, _i, _p]),
    "pkv_bm_free_many": (_i, [_p, _p, _i]),
    "pkv_bm_append_tokens": (_i, [_p, _p, _i, _p, _p, _p, _p]),
    "pkv_bm_free_seq": (_i, [_p, C.c_int32]),
    "pkv_bm_num_free": (_i, [_p]),
    "pkv_bm_seq_len": (_i, [_p, C.c_int32, _p]),
    "pkv_bm_refcount": (_i, [_p, C.c_int32, _p]),
    "pkv_bm_block_table": (_i, [_p, C.c_int32, _p, _i, _p]),
    "pkv_bm_slots": (_i, [_p, C.c_int32, _i, _i, _p]),
    "pkv_bm_tables": (_i, [_p, _p, _i, _p, _i, C.c_int32, _p]),
    "pkv_bm_free_list": (_i, [_p, _p, _i, _p]),
    "pkv_bm_prefix_groups": (_i, [_p, _p, _i, _p, _p, _p, _p]),
    "pkv_bm_set_prefix_cache": (_i, [_p, _i]),
    "pkv_bm_alloc_seq_tokens": (_i, [_p, _p, _i, _p, _p]),
    "pkv_bm_num_cached_blocks": (_i, [_p]),
    "pkv_bm_set_host_pool": (_i, [_p, _i]),
    "pkv_bm_swap_out": (_i, [_p, C.c_int32, _p, _i, _p]),
    "pkv_bm_swap_in": (_i, [_p, C.c_int32, _p, _i, _p]),
    "pkv_bm_is_swapped": (_i, [_p, C.c_int32, _p]),
    "pkv_bm_num_free_host": (_i, [_p]),
}

_lib = None


class PagedKVError(RuntimeError):
    """A non-zero pkv_status from the library."""

    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def lib():
    """The loaded library; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libpagedkv.so is not built (%s); run `python -m paged_kv_cache_404_b200.build`"
                               % LIB_PATH)
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status):
    return lib().pkv_status_string(int(status)).decode()


def check(fn, status):
    if status != PKV_OK:
        raise PagedKVError(fn, status)
