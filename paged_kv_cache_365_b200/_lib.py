"""ctypes loader for libpkv.so and the prototypes of the C ABI (include/pkv.h).

Importing this module loads the in-tree library and fails loudly if it is
missing: there is no fallback implementation.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpkv.so")

c_int, c_int32, c_int64, c_float, c_size_t, c_void_p, c_uint32 = (
    ctypes.c_int, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
    ctypes.c_void_p, ctypes.c_uint32)
P = ctypes.POINTER

PKV_OK, PKV_EINVAL, PKV_ENOMEM, PKV_ECUDA = 0, 1, 2, 3

ERR_BLOCK_RANGE = 0x1
ERR_CONTEXT_RANGE = 0x2
ERR_SLOT_RANGE = 0x4
ERR_COPY_RANGE = 0x8
ERR_TIMEOUT = 0x10

STATIC_WORKSPACE_BYTES = 16 << 20  # PKV_STATIC_WORKSPACE_BYTES

# pkv_op: which call's partition rule pkv_partition_tokens applies
OP_DECODE, OP_DECODE_FP8, OP_MULTI, OP_DECODE_PREFIX, OP_MULTI_FP8 = 0, 1, 2, 3, 4

# name -> (restype, argtypes); the same list as include/pkv.h
PROTOTYPES = {
    "pkv_status_string": (ctypes.c_char_p, [c_int]),
    "pkv_abi_version": (c_int, []),
    "pkv_kv_append": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                              c_int, c_int, c_int, c_int, c_int, c_void_p]),
    "pkv_copy_blocks": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                c_void_p]),
    "pkv_copy_blocks_check": (c_int, [P(c_int32), c_int, c_int]),
    "pkv_kv_append_copy": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int, c_int,
                                   c_int, c_int, c_int, c_void_p]),
    "pkv_swap_blocks": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_int, c_int,
                                c_int, c_int, c_void_p]),
    "pkv_swap_blocks_check": (c_int, [P(c_int32), c_int, c_int, c_int]),
    "pkv_decode_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_decode": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                           c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                           c_float, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pkv_decode_prefix_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_decode_prefix": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                                  c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                  c_int, c_float, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pkv_paged_attention_decode_prefix_phase": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                                        c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int,
                                                        c_int, c_int, c_float, c_int, c_int, c_void_p, c_size_t,
                                                        c_int, c_void_p]),
    "pkv_paged_attention_decode_static_ws": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                                     c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                     c_float, c_int, c_int, c_void_p]),
    "pkv_selftest_bounded_wait": (c_int, [ctypes.c_longlong, c_void_p]),
    "pkv_kv_append_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                  c_int, c_float, c_float, c_void_p]),
    "pkv_paged_attention_decode_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                               c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_float, c_float,
                                               c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pkv_multi_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_multi": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int,
                                          c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int,
                                          c_int, c_void_p, c_size_t, c_void_p]),
    "pkv_paged_attention_multi_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                              c_int, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                              c_float, c_float, c_float, c_int, c_int, c_void_p, c_size_t,
                                              c_void_p]),
    "pkv_get_error": (c_int, [P(c_uint32), c_void_p]),
    "pkv_partition_tokens": (c_int, [c_int, c_int, c_int, c_int]),
    "pkv_decode_prefix_fp8_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_decode_prefix_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                                      c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                      c_int, c_float, c_float, c_float, c_int, c_int, c_void_p,
                                                      c_size_t, c_void_p]),
    "pkv_decode_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_int, c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int,
                                c_int, c_int, c_float, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pkv_decode_step_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_int, c_int,
                                    c_int, c_int, c_int, c_float, c_float, c_float, c_int, c_int, c_void_p, c_size_t,
                                    c_void_p]),
    "pkv_cow_copy_rows": (c_int, [P(c_int32), c_int, P(c_int64), c_int, P(c_int32)]),
    "pkv_common_prefix_pages": (c_int, [P(c_int32), c_int, c_int, P(c_int32), P(c_int)]),
    "pkv_cascade_prefix_pages": (c_int, [P(c_int32), c_int, c_int, P(c_int32), c_int, P(c_int)]),
    "pkv_alloc_step_copies": (c_int, [c_void_p, P(c_int64), c_int, P(c_int64), P(c_int32), P(c_int)]),
    "pkv_alloc_create": (c_int, [c_int, P(c_int32), P(c_void_p)]),
    "pkv_alloc_destroy": (None, [c_void_p]),
    "pkv_alloc_add_seq": (c_int, [c_void_p, c_int64]),
    "pkv_alloc_fork": (c_int, [c_void_p, c_int64, c_int64]),
    "pkv_alloc_free_seq": (c_int, [c_void_p, c_int64]),
    "pkv_alloc_append_slot": (c_int, [c_void_p, c_int64, P(c_int64), P(c_int32), P(c_int32)]),
    "pkv_alloc_append_tokens": (c_int, [c_void_p, c_int64, c_int, P(c_int64), P(c_int32), P(c_int)]),
    "pkv_alloc_step": (c_int, [c_void_p, P(c_int64), c_int, P(c_int64), P(c_int32), P(c_int)]),
    "pkv_alloc_block_table": (c_int, [c_void_p, c_int64, P(c_int32), c_int, P(c_int), P(c_int64)]),
    "pkv_alloc_block_tables": (c_int, [c_void_p, P(c_int64), c_int, P(c_int32), c_int, c_int32,
                                       P(c_int32)]),
    "pkv_alloc_state": (c_int, [c_void_p, P(c_int32), P(c_int), P(c_int32)]),
    "pkv_alloc_num_free": (c_int, [c_void_p]),
    "pkv_alloc_num_blocks": (c_int, [c_void_p]),
    "pkv_alloc_num_seqs": (c_int, [c_void_p]),
    "pkv_alloc_set_host_pool": (c_int, [c_void_p, c_int]),
    "pkv_alloc_swap_out": (c_int, [c_void_p, P(c_int64), c_int, P(c_int32), c_int, P(c_int)]),
    "pkv_alloc_swap_in": (c_int, [c_void_p, P(c_int64), c_int, P(c_int32), c_int, P(c_int)]),
    "pkv_alloc_host_state": (c_int, [c_void_p, P(c_int32), P(c_int), P(c_int32)]),
    "pkv_alloc_swapped_table": (c_int, [c_void_p, c_int64, P(c_int32), c_int, P(c_int), P(c_int64)]),
    "pkv_alloc_num_swapped": (c_int, [c_void_p]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libpkv.so not found at {LIB_PATH}: build it first "
            "(python -m paged_kv_cache_365_b200._build, or __graft_entry__.build()); "
            "there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib.pkv_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})")
        self.status = status


def check(status: int, what: str) -> None:
    if status != PKV_OK:
        raise PkvError(status, what)
