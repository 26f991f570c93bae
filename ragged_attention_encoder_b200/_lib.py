"""ctypes declarations of the C ABI in include/rae.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librae.so")
TEST_LIB_PATH = os.path.join(_HERE, "librae_test.so")

RAE_OK = 0
RAE_ERR_INVALID_ARG = 1
RAE_ERR_UNSUPPORTED = 2
RAE_ERR_CAPACITY = 3
RAE_ERR_CUDA = 4
RAE_ERR_DEVICE_TIMEOUT = 5

STATUS_NAMES = {
    RAE_OK: "RAE_OK",
    RAE_ERR_INVALID_ARG: "RAE_ERR_INVALID_ARG",
    RAE_ERR_UNSUPPORTED: "RAE_ERR_UNSUPPORTED",
    RAE_ERR_CAPACITY: "RAE_ERR_CAPACITY",
    RAE_ERR_CUDA: "RAE_ERR_CUDA",
    RAE_ERR_DEVICE_TIMEOUT: "RAE_ERR_DEVICE_TIMEOUT",
}

i32 = ctypes.c_int32
i64 = ctypes.c_int64
P32 = ctypes.POINTER(ctypes.c_int32)
vp = ctypes.c_void_p
sz = ctypes.c_size_t


class RaeConfig(ctypes.Structure):
    _fields_ = [
        ("num_qo_heads", i32),
        ("num_kv_heads", i32),
        ("head_dim", i32),
        ("page_size", i32),
        ("max_batch", i32),
        ("max_q_tokens", i32),
        ("max_kv_pages", i32),
        ("max_tiles", i32),
        ("max_partial_rows", i32),
        ("num_sms", i32),
    ]


class RaePlan(ctypes.Structure):
    _fields_ = [
        ("kind", i32),
        ("slot", i32),
        ("num_tiles", i32),
        ("num_ctas", i32),
        ("num_merge_rows", i32),
        ("batch", i32),
        ("total_q", i32),
        ("rows_max", i32),
        ("block_size", i32),
        ("image_words", i32),
        ("generation", i64),
        ("off_cta_ptr", i32),
        ("off_tiles", i32),
        ("off_merge", i32),
        ("off_a", i32),
        ("off_b", i32),
        ("off_c", i32),
        ("off_d", i32),
        ("kv_extent", i32),
    ]


# name -> (restype, argtypes); every symbol that include/rae.h declares.
SIGNATURES = {
    "rae_create": (ctypes.c_int, [ctypes.POINTER(vp), ctypes.POINTER(RaeConfig)]),
    "rae_destroy": (ctypes.c_int, [vp]),
    "rae_last_error": (ctypes.c_char_p, [vp]),
    "rae_workspace_bytes": (sz, [vp]),
    "rae_plan_image_bytes": (sz, [vp]),
    "rae_write_context": (ctypes.c_int, [vp, vp, vp, P32, P32, P32, i32, vp, vp, i32, vp, vp]),
    "rae_plan_paged": (ctypes.c_int, [vp, i32, P32, P32, P32, P32, i32, i32, vp, vp,
                                      ctypes.POINTER(RaePlan)]),
    "rae_plan_ragged": (ctypes.c_int, [vp, i32, P32, P32, i32, i32, vp, vp,
                                       ctypes.POINTER(RaePlan)]),
    "rae_plan_paged_causal": (ctypes.c_int, [vp, i32, P32, P32, P32, P32, i32, i32, vp, vp,
                                             ctypes.POINTER(RaePlan)]),
    "rae_append_kv": (ctypes.c_int, [vp, vp, vp, P32, P32, P32, P32, i32, vp, vp, i32, vp, vp]),
    "rae_o_proj_partial": (ctypes.c_int, [vp, vp, i32, i32, vp, i32, vp, vp, vp, vp]),
    "rae_project_write_context": (ctypes.c_int, [vp, vp, i32, vp, vp, vp, vp, P32, P32, P32, i32,
                                                 vp, vp, i32, vp, vp]),
    "rae_run_paged": (ctypes.c_int, [vp, ctypes.POINTER(RaePlan), vp, vp, vp, i32, vp,
                                     ctypes.c_float, vp, vp]),
    "rae_run_ragged": (ctypes.c_int, [vp, ctypes.POINTER(RaePlan), vp, vp, vp, i32, vp,
                                      ctypes.c_float, vp, vp]),
    "rae_check_device_status": (ctypes.c_int, [vp, vp, vp]),
    "rae_set_wait_timeout_ns": (ctypes.c_int, [vp, i64]),
    "rae_plan_paged_host": (ctypes.c_int, [ctypes.POINTER(RaeConfig), P32, P32, P32, P32, i32,
                                           i32, vp, sz, ctypes.POINTER(RaePlan),
                                           ctypes.c_char_p, sz]),
    "rae_plan_ragged_host": (ctypes.c_int, [ctypes.POINTER(RaeConfig), P32, P32, i32, i32, vp,
                                            sz, ctypes.POINTER(RaePlan), ctypes.c_char_p, sz]),
    "rae_plan_paged_causal_host": (ctypes.c_int, [ctypes.POINTER(RaeConfig), P32, P32, P32, P32,
                                                  i32, i32, vp, sz, ctypes.POINTER(RaePlan),
                                                  ctypes.c_char_p, sz]),
    "rae_plan_image_bytes_for": (sz, [ctypes.POINTER(RaeConfig)]),
    "rae_write_context_noalloc": (ctypes.c_int, [vp, vp, P32, P32, P32, i32, vp, vp, i32, i32,
                                                 i32, i32, vp]),
    "rae_enable_kernel_timing": (ctypes.c_int, [vp, i32]),
    "rae_read_kernel_timing": (ctypes.c_int, [vp, ctypes.POINTER(ctypes.c_float),
                                              ctypes.POINTER(ctypes.c_float), i32,
                                              ctypes.POINTER(i32)]),
}

# Entry points of include/rae_test_hooks.h, exported by librae_test.so only.
TEST_SIGNATURES = {
    "rae_test_silence_producer": (ctypes.c_int, [i32]),
}

_lib = None
_test_lib = None


def _open(path: str, signatures) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing; build it with `python -m ragged_attention_encoder_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in signatures.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load() -> ctypes.CDLL:
    """Loads librae.so.  Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is None:
        _lib = _open(LIB_PATH, SIGNATURES)
    return _lib


def load_test() -> ctypes.CDLL:
    """Loads librae_test.so (the library plus its fault-injection hooks), for tests only."""
    global _test_lib
    if _test_lib is None:
        _test_lib = _open(TEST_LIB_PATH, {**SIGNATURES, **TEST_SIGNATURES})
    return _test_lib
