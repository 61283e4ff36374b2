"""ctypes declarations of the C ABI in ``include/bfa.h``.

Loading fails loudly: there is no fallback implementation of any entry point.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# BFA_LIBRARY=checked selects the bounds-checked build (libbfa_checked.so: the
# same kernels with every plan-indexed access checked and guard bytes around
# plan arrays, reported by bfa_plan_device_status); the default is libbfa.so.
LIB_PATH = os.path.join(_HERE, "libbfa_checked.so" if os.environ.get("BFA_LIBRARY") == "checked" else "libbfa.so")

c_i32p = ctypes.POINTER(ctypes.c_int32)
c_i64p = ctypes.POINTER(ctypes.c_int64)
c_u8p = ctypes.POINTER(ctypes.c_uint8)
c_u32p = ctypes.POINTER(ctypes.c_uint32)
c_void = ctypes.c_void_p

STATUS = {
    0: "BFA_OK", -1: "BFA_ERR_INVALID_ARG", -2: "BFA_ERR_UNSUPPORTED", -3: "BFA_ERR_NOT_DEVICE",
    -4: "BFA_ERR_NONCANONICAL_BSR", -5: "BFA_ERR_CAPACITY", -6: "BFA_ERR_CUDA", -7: "BFA_ERR_TIMEOUT",
    -8: "BFA_ERR_BOUNDS",
}

# every entry point declared in include/bfa.h: name -> (restype, argtypes)
SIGNATURES = {
    "bfa_version": (ctypes.c_char_p, []),
    "bfa_last_error": (ctypes.c_char_p, []),
    "bfa_is_available": (ctypes.c_int, []),
    "bfa_make_block_ids": (ctypes.c_int, [c_void, c_void, ctypes.c_int, ctypes.c_int, ctypes.c_int, c_void,
                                          c_void, c_void, c_void, c_void, c_void]),
    "bfa_plan_dense": (ctypes.c_int, [c_void, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      ctypes.POINTER(c_void), c_void]),
    "bfa_plan_blockids": (ctypes.c_int, [c_void, c_void, c_void, c_void, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, c_void, c_void, c_void, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.POINTER(c_void), c_void]),
    "bfa_plan_predicate": (ctypes.c_int, [c_void, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, c_void,
                                          c_void, c_void, ctypes.c_int, ctypes.c_int, ctypes.POINTER(c_void), c_void]),
    "bfa_plan_bsr": (ctypes.c_int, [c_void, c_void, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, c_void,
                                    ctypes.POINTER(c_void), c_void]),
    "bfa_plan_bsr_packed": (ctypes.c_int, [c_void, c_void, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           c_void, ctypes.POINTER(c_void), c_void]),
    "bfa_plan_block_bits": (ctypes.c_int, [c_void, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, c_void,
                                           ctypes.POINTER(c_void), c_void]),
    "bfa_fwd": (ctypes.c_int, [c_void, c_void, c_void, c_void, c_i64p, c_i64p, c_i64p, ctypes.c_int,
                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, c_void, c_i64p,
                               c_void, c_void]),
    "bfa_bwd": (ctypes.c_int, [c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_i64p, c_i64p, c_i64p,
                               c_i64p, c_i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                               c_void, c_void, c_void, c_i64p, c_i64p, c_i64p, c_void]),
    "bfa_fwd_approx": (ctypes.c_int, [c_void, c_void, c_void, c_void, c_i64p, c_i64p, c_i64p, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                      c_void, c_i64p, c_void, c_void]),
    "bfa_fwd_paged": (ctypes.c_int, [c_void, c_void, c_i64p, c_void, c_void, c_i64p, ctypes.c_int64, ctypes.c_int,
                                     c_void, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_float, c_void, c_i64p, c_void, c_void]),
    "bfa_plan_get_info": (ctypes.c_int, [c_void, c_void]),
    "bfa_plan_stats": (ctypes.c_int, [c_void, c_i64p, c_i64p, c_i64p, c_void]),
    "bfa_plan_export": (ctypes.c_int, [c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_void]),
    "bfa_plan_export_pairs": (ctypes.c_int, [c_void, c_void, c_void, c_void]),
    "bfa_plan_export_cols": (ctypes.c_int, [c_void, c_void, c_void, c_void, c_void, c_void]),
    "bfa_plan_device_status": (ctypes.c_int, [c_void, c_void]),
    "bfa_plan_destroy": (None, [c_void]),
    "bfa_set_wait_timeout_ns": (None, [ctypes.c_uint64]),
    "bfa_set_bwd_deterministic": (None, [ctypes.c_int]),
    "bfa_selftest_wait_timeout": (ctypes.c_int, [c_void]),
    "bfa_plan_dense_noalloc": (ctypes.c_int, [c_void, ctypes.c_int64, ctypes.c_int, ctypes.c_int, c_void, c_void,
                                              c_void, c_void, c_void, c_void, c_void]),
}


class PlanInfo(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("varlen", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("n_rows", ctypes.c_int32), ("grid_tiles", ctypes.c_int64), ("batch", ctypes.c_int32),
                ("hkv", ctypes.c_int32), ("sq", ctypes.c_int32), ("sk", ctypes.c_int32),
                ("max_kv_tiles", ctypes.c_int32), ("window_left", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("n_pairs", ctypes.c_int32), ("packed_fine", ctypes.c_int32), ("n_cols", ctypes.c_int32),
                ("heads_per_kv", ctypes.c_int32)]


class MaskTerm(ctypes.Structure):
    _fields_ = [("diag_lo", ctypes.c_int32), ("diag_hi", ctypes.c_int32), ("q_lo", ctypes.c_int32),
                ("q_hi", ctypes.c_int32), ("k_lo", ctypes.c_int32), ("k_hi", ctypes.c_int32)]


class BfaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_lib = None


def load():
    """Load ``libbfa.so`` (built by ``mask_skipping_flashattention_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbfa.so not found at {LIB_PATH}; build it with "
                          "`python mask_skipping_flashattention_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(code):
    if code != 0:
        msg = load().bfa_last_error().decode(errors="replace")
        raise BfaError(code, msg)
