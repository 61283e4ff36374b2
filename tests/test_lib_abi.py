"""The C-ABI library loads and exports every entry point ``include/bfa.h`` declares (CPU only)."""

import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bfa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bfa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_plan_and_forward_calls():
    names = _declared()
    for n in ("bfa_plan_dense", "bfa_plan_blockids", "bfa_plan_bsr", "bfa_fwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from mask_skipping_flashattention_b200 import _lib
    lib = ctypes.CDLL(_lib.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) == set(_lib.SIGNATURES), "binding signatures out of sync with bfa.h"


def test_checked_library_exports_the_same_symbols():
    """The bounds-checked build (libbfa_checked.so) is a drop-in twin of libbfa.so."""
    from mask_skipping_flashattention_b200 import _lib
    path = os.path.join(os.path.dirname(_lib.LIB_PATH), "libbfa_checked.so")
    lib = ctypes.CDLL(path)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    lib.bfa_version.restype = ctypes.c_char_p
    assert b"checked" in lib.bfa_version()


def test_library_reports_no_device_without_a_gpu():
    import torch
    import mask_skipping_flashattention_b200 as bfa
    assert bfa._L.bfa_version().startswith(b"bfa")
    if not torch.cuda.is_available():
        assert not bfa.is_available()
        assert bfa.load_error()


def test_cpu_tensors_are_rejected_before_any_launch():
    import pytest
    import torch
    import mask_skipping_flashattention_b200 as bfa
    if torch.cuda.is_available():
        pytest.skip("checked in the GPU suite")
    with pytest.raises(bfa.BfaError) as e:
        bfa.plan_dense(torch.ones(4, 4, dtype=torch.bool), stream=0)
    assert e.value.status in ("BFA_ERR_NOT_DEVICE",)
